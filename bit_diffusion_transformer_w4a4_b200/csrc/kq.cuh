// Kernel 1 of the layer: activation smoothing, per-token group quantisation
// to 4 bits with packing, and the rank-r down projection T = X' L1 computed
// from the same shared-memory tiles on the tensor cores.
//
// Method: "Problemas do Nunchaku Qwen e como corrigi-los em 2025"
// (apatero.com), section "O que e Nunchaku e como acelera modelos Qwen" --
// the down projection is fused with the quantisation kernel so both branches
// share the activations; "Nunchaku Lite ... integrated into Diffusers"
// (axbrief.com), section "The Mechanics of 4-Bit Efficiency and SVDQuant" --
// activation outliers are divided out (moved into the weights) before the
// 4-bit quantisation.
//
// CTA tile: 128 tokens x (K / ksplit) input channels.  The K range of a row
// block is split over `ksplit` CTAs so that a 4608-token layer still fills
// the 148 SMs in one wave.  Their partial T tiles are added into T with
// fp32 vector reductions (split 0 clears the row block's T at its start and
// raises a per-launch flag that the others check before adding), or -- for
// the entry point
// that allocates nothing and keeps T deterministic -- go to a scratch buffer
// that the last CTA of the row block to finish sums in split order, with a
// per-block arrival counter that it resets.
//
// Warp roles (576 threads):
//   warps 0-15 quantisers, one token row per thread; warp w covers rows
//              32*(w%4).. and every fourth 64-column chunk (group w/4)
//   warp 16    TMA producer (X chunk [128 x 64] bf16, L1^T chunk [r x 64],
//              1/lambda of the chunk)
//   warp 17    tcgen05 MMA issuer and tensor-memory owner
#pragma once

#include "ptx.cuh"

namespace svdq {

constexpr int KQ_QWARPS = 16;  // quantiser warps: 4 chunk groups x 4 row quarters
constexpr int KQ_THREADS = (KQ_QWARPS + 2) * 32;
constexpr int KQ_CHUNK = 64;  // columns per pipeline stage

// Correctly rounded x / s for s > 0 finite: one correction step of
// Markstein's division method (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 1990):
// with y = RN(1/s), q0 = RN(x*y), the residual r = x - s*q0 is exact in one
// fma and q1 = RN(q0 + r*y) is the correctly rounded quotient.  The kernels
// only divide bf16 values by bf16 / E4M3 scales; the library's self-test
// compares this routine against IEEE division over all such operand pairs.
// The correction step can turn -0 into +0; the quotient's sign is x's sign
// (s > 0), so it is put back explicitly.  The residual x - s*q0 must not
// underflow and 1/s must be a normal number: the caller divides groups whose
// scale lies outside [2^-90, 2^126) exactly instead.
__device__ __forceinline__ float div_by_scale(float x, float s, float y) {
  const float q0 = __fmul_rn(x, y);
  const float r = __fmaf_rn(-q0, s, x);
  const float q1 = __fmaf_rn(r, y, q0);
  return __uint_as_float(__float_as_uint(q1) | (__float_as_uint(x) & 0x80000000u));
}
constexpr float kMinFastScale = 8.07793567e-28f;     // 2^-90: smallest scale of the fast path
constexpr float kMaxFastScale = 8.50705917e+37f;  // 2^126: above it 1/s is subnormal

// x / s as the quantiser computes it: the one-step method for normal s,
// IEEE division when s is subnormal (its reciprocal would overflow).
__device__ __forceinline__ float quant_div(float x, float s, float y) {
  return (s >= kMinFastScale && s < kMaxFastScale) ? div_by_scale(x, s, y) : __fdiv_rn(x, s);
}

// E4M3 (satfinite, RN) of a non-negative fp32, and its exact value.
__device__ __forceinline__ uint32_t e4m3_rn(float v) {
  uint16_t h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(v));
  return h & 0xFFu;
}
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  uint32_t h2;
  const uint16_t c = static_cast<uint16_t>(code);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}
// Eight fp32 -> eight E2M1 codes (RN, satfinite), element 0 in the low nibble.
__device__ __forceinline__ uint32_t e2m1x8(const float* v) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}
// Largest magnitude of the 2n bf16 values held in n packed words, as fp32:
// pairwise magnitude maxima on bf16x2 (max.xorsign.abs keeps the larger
// |value|; its sign is not used), then the larger of the two halves.  Exact:
// only comparisons.
template <int NW>
__device__ __forceinline__ float bf16_amax(const uint32_t* w) {
  uint32_t m[NW];
#pragma unroll
  for (int i = 0; i < NW; ++i) m[i] = w[i];
#pragma unroll
  for (int step = 1; step < NW; step *= 2)
#pragma unroll
    for (int i = 0; i + step < NW; i += 2 * step)
      asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m[i]) : "r"(m[i]), "r"(m[i + step]));
  return fmaxf(fabsf(bf16lo(m[0])), fabsf(bf16hi(m[0])));
}

// Round half to even to an integer in [-8, 7], two's complement nibble.
__device__ __forceinline__ uint32_t int4_rn(float v) {
  v = fminf(fmaxf(v, -8.0f), 7.0f);
  // adding 1.5 * 2^23 leaves the rounded integer in the low mantissa bits
  return __float_as_uint(__fadd_rn(v, 12582912.0f)) & 0xFu;
}

struct KQParams {
  const float* inv_lam;  // [K]
  uint8_t* codes;        // [M x K/2]
  void* scales;          // INT4: bf16 [M x K/64]; NVFP4: tiled E4M3
  float* t;              // [M x R]
  float* tpart;          // scratch: partial T tiles [ksplit x num_m x 128 x R] (ksplit > 1)
  int* counters;         // scratch: arrivals per 128-row block, zero between launches
  int t_accumulate;      // ksplit > 1: add the partial tiles into T with fp32
                         // reductions instead of the scratch pass; split 0 of a row
                         // block zeroes its rows of T first and publishes
                         // tflags[row block] = epoch, which the other splits await
  unsigned int* tflags;  // [row blocks]
  unsigned int epoch;    // nonzero, new for every launch on the same flags
  int M, K, ksplit, chunks;  // chunks of 64 columns per CTA
  int* err;
  uint32_t debug_mask;
  uint64_t timeout_ns;
};

template <int VARIANT, int R>
struct KQSmem {
  static constexpr int X_BYTES = 128 * KQ_CHUNK * 2;  // 16 KB
  static constexpr int L_BYTES = R * KQ_CHUNK * 2;    // r x 128 B
  static constexpr int IL_BYTES = KQ_CHUNK * 4;       // 1/lambda for the chunk
  // a stage holds the X and L1^T tiles (1 KB multiples, so every stage keeps
  // the 128-byte swizzle's alignment); the chunk's 1/lambda sits in a ring
  // of its own.  As many stages as shared memory holds (static shared
  // memory -- the E4M3 table and the reduction flag -- takes up to 2 KB once
  // the 1 KB-aligned dynamic region follows it): a CTA's chunks are mostly in
  // flight at once.
  static constexpr int STAGE = X_BYTES + L_BYTES;
  static constexpr int FREE = 232448 - 2048 - 512 - 1024;
  static constexpr int STAGES = FREE / (STAGE + IL_BYTES) < 16 ? FREE / (STAGE + IL_BYTES) : 16;
  static constexpr int IL_OFF = STAGES * STAGE;
  static constexpr int BAR_OFF = IL_OFF + STAGES * IL_BYTES;
  static constexpr int TOTAL = BAR_OFF + 512 + 1024;  // barriers + slack for 1 KB alignment
  static_assert(TOTAL + 2048 <= 232448, "shared memory per CTA");
  static_assert(STAGES * 3 + 2 <= 64, "barriers");
};

// 1/6 and 1/7 rounded to nearest: scale = amax / 6 (NVFP4) or amax / 7 (INT4)
// is computed with the same one-step division as the codes.
constexpr float kRcp6 = 0.16666667163372039794921875f;
constexpr float kRcp7 = 0.14285714924335479736328125f;

// VARIANT 0 = INT4 (G 64, bf16 scale, amax/7); 1 = NVFP4 (G 16, E4M3 scale, amax/6)
template <int VARIANT, int R>
__global__ void __launch_bounds__(KQ_THREADS, 1)
    kq_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1t,
              KQParams p) {
  using S = KQSmem<VARIANT, R>;
  constexpr int NST = S::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR_OFF);
  const uint32_t bar_full = smem_u32(bars + 0);          // [NST]
  const uint32_t bar_ready = smem_u32(bars + NST);       // [NST] X' written
  const uint32_t bar_empty = smem_u32(bars + 2 * NST);   // [NST]
  const uint32_t bar_tfull = smem_u32(bars + 3 * NST);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * NST + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ks = blockIdx.x;            // K-split index
  const int m0 = blockIdx.y * 128;
  const int kbase = ks * p.chunks * KQ_CHUNK;
  const Guard guard{p.err, abort_flag, p.timeout_ns};
  constexpr uint32_t TMEM_COLS = R <= 32 ? 32 : R;
  constexpr int PRODUCER = KQ_QWARPS;      // warp index of the TMA producer
  constexpr int MMA = KQ_QWARPS + 1;       // warp index of the MMA issuer

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_ready + 8 * s, 128);              // the 128 quantiser threads of a chunk
      mbar_init(bar_empty + 8 * s, R > 0 ? 1 : 128);
    }
    mbar_init(bar_tfull, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (R > 0 && warp == MMA) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  // E4M3 scale code -> (value, RN(1 / value)) for the NVFP4 quantiser (the
  // codes of non-negative satfinite scales are 0..126)
  __shared__ float2 e4lut[128];
  if (VARIANT == 1 && threadIdx.x < 128) {
    const float v = e4m3_value(threadIdx.x);
    e4lut[threadIdx.x] = make_float2(v, v > 0.0f && threadIdx.x < 127 ? __frcp_rn(v) : 0.0f);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = R > 0 ? *tmem_slot : 0;
  // X may still be being written by the previous kernel of the stream, and
  // the outputs may still be read by it: see griddep_wait()
  griddep_wait();
  griddep_launch_dependents();
  if (R > 0 && p.t_accumulate && ks == 0 && warp == MMA) {
    // split 0 clears the row block's T (read by the previous kernel of the
    // stream until griddep_wait) before any split adds into it: the MMA
    // warp, idle until the first chunk is quantised, does it
    const int rows = min(128, p.M - m0);
    float4* dst = reinterpret_cast<float4*>(p.t + static_cast<size_t>(m0) * R);
    for (int i = lane; i < rows * (R / 4); i += 32) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    __threadfence();
    __syncwarp();
    if (lane == 0) st_release_gpu(p.tflags + blockIdx.y, p.epoch);
  }

  if (warp == PRODUCER) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      if (R > 0) tma_prefetch_desc(&tm_l1t);
      uint32_t issued = 0, issued_par = 0;  // per-stage outstanding loads
      for (int c = 0; c < p.chunks; ++c) {
        const int s = c % NST;
        const uint32_t ph = (c / NST) & 1;
        if (!wait_bounded(bar_empty + 8 * s, ph ^ 1, guard, 0x101)) break;
        issued &= ~(1u << s);
        if ((p.debug_mask & 2u) && c == 1) continue;  // test hook: never fill this stage
        const uint32_t st = sbase + s * S::STAGE;
        const int k0 = kbase + c * KQ_CHUNK;
        mbar_expect_tx(bar_full + 8 * s, S::X_BYTES + S::L_BYTES + S::IL_BYTES);
        tma_load_2d(st, &tm_x, bar_full + 8 * s, k0, m0);
        if (R > 0) tma_load_2d(st + S::X_BYTES, &tm_l1t, bar_full + 8 * s, k0, 0);
        bulk_load(sbase + S::IL_OFF + s * S::IL_BYTES, p.inv_lam + k0, S::IL_BYTES, bar_full + 8 * s);
        issued |= 1u << s;
        issued_par = (issued_par & ~(1u << s)) | (ph << s);
      }
      if (*abort_flag) {  // let copies still in flight land before the CTA exits
        for (int s = 0; s < NST; ++s)
          if (issued & (1u << s)) {
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar_full + 8 * s, (issued_par >> s) & 1) &&
                   global_timer_ns() - t0 < p.timeout_ns) {
            }
          }
      }
    }
  } else if (warp == MMA) {
    // --------------------------------------------------------------- MMA issue
    if (R > 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, R);
      bool ok = true;
      for (int c = 0; c < p.chunks && ok; ++c) {
        const int s = c % NST;
        const uint32_t ph = (c / NST) & 1;
        ok = wait_bounded(bar_full + 8 * s, ph, guard, 0x102) &&
             wait_bounded(bar_ready + 8 * s, ph, guard, 0x103);
        if (!ok) break;
        tc_fence_after();
        const uint32_t st = sbase + s * S::STAGE;
#pragma unroll
        for (int kk = 0; kk < KQ_CHUNK / 16; ++kk) {
          const uint64_t a = smem_desc(st + kk * 32, 16, 1024, SWZ_128B);
          const uint64_t b = smem_desc(st + S::X_BYTES + kk * 32, 16, 1024, SWZ_128B);
          mma_bf16(tmem, a, b, idesc, (c | kk) != 0);
        }
        tc_commit(bar_empty + 8 * s);
      }
      tc_commit(bar_tfull);  // also serves as the drain point on the abort path
      if (!ok) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bar_tfull, 0) && global_timer_ns() - t0 < p.timeout_ns) {
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- quantise
    const int q = warp & 3;
    const int grp = warp >> 2;              // chunk group: chunks c with c % 4 == grp
    const int row = q * 32 + lane;
    const int grow = m0 + row;
    const bool live = grow < p.M;
    const int kh = p.K / 2;
    for (int c = grp; c < p.chunks; c += KQ_QWARPS / 4) {
      const int s = c % NST;
      const uint32_t ph = (c / NST) & 1;
      if (!wait_bounded(bar_full + 8 * s, ph, guard, 0x104)) break;
      uint8_t* xt = smem + s * S::STAGE;
      const float4* il = reinterpret_cast<const float4*>(smem + S::IL_OFF + s * S::IL_BYTES);
      const int k0 = kbase + c * KQ_CHUNK;
      // 64 bf16 of this row (de-swizzled), smoothed: x' = bf16(x * inv_lambda)
      uint32_t w[32];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 v = *reinterpret_cast<const uint4*>(xt + swz_off(row, j, 128));
        const float4 f0 = il[2 * j], f1 = il[2 * j + 1];
        // two round-to-nearest fp32 products per instruction, then bf16 RN
        const uint64_t p0 = f2_mul(f2_pack(bf16lo(v.x), bf16hi(v.x)), f2_pack(f0.x, f0.y));
        const uint64_t p1 = f2_mul(f2_pack(bf16lo(v.y), bf16hi(v.y)), f2_pack(f0.z, f0.w));
        const uint64_t p2 = f2_mul(f2_pack(bf16lo(v.z), bf16hi(v.z)), f2_pack(f1.x, f1.y));
        const uint64_t p3 = f2_mul(f2_pack(bf16lo(v.w), bf16hi(v.w)), f2_pack(f1.z, f1.w));
        w[4 * j] = pack_bf16x2(f2_lo(p0), f2_hi(p0));
        w[4 * j + 1] = pack_bf16x2(f2_lo(p1), f2_hi(p1));
        w[4 * j + 2] = pack_bf16x2(f2_lo(p2), f2_hi(p2));
        w[4 * j + 3] = pack_bf16x2(f2_lo(p3), f2_hi(p3));
      }
      // Each thread orders its own shared-memory accesses of this stage before
      // the async proxy (tensor core or the TMA refill) touches it again, and
      // arrives itself.
      if (R > 0) {
        // X' replaces X in place: it is the A operand of the down projection
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(xt + swz_off(row, j, 128)) =
              make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        fence_proxy_async_smem();
        mbar_arrive(bar_ready + 8 * s);
      } else {
        fence_proxy_async_smem();
        mbar_arrive(bar_empty + 8 * s);
      }
      // group quantisation (all in registers)
      uint32_t packed[8];
      if (VARIANT == 1) {
        uint32_t sc = 0;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float a = bf16_amax<8>(w + 8 * g);
          const uint32_t code = e4m3_rn(div_by_scale(a, 6.0f, kRcp6));
          const float2 sy = e4lut[code];  // the scale's value and RN(1 / value)
          const float s_ = sy.x;
          sc |= code << (8 * g);
          if (s_ > 0.0f) {           // E4M3 scales are >= 2^-9: 1/s is finite
            // div_by_scale on two values per instruction: q0 = x y,
            // r = fma(q0, -s, x) (= fma(-q0, s, x) exactly), q1 = fma(r, y, q0),
            // then x's sign put back
            const uint64_t y2 = f2_pack(sy.y, sy.y), ns2 = f2_pack(-s_, -s_);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              float v[8];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const uint32_t ww = w[8 * g + 4 * h + e];
                const uint64_t x2 = f2_pack(bf16lo(ww), bf16hi(ww));
                const uint64_t q0 = f2_mul(x2, y2);
                const uint64_t q1 = f2_fma(f2_fma(q0, ns2, x2), y2, q0);
                v[2 * e] = __uint_as_float(__float_as_uint(f2_lo(q1)) | ((ww << 16) & 0x80000000u));
                v[2 * e + 1] = __uint_as_float(__float_as_uint(f2_hi(q1)) | (ww & 0x80000000u));
              }
              packed[2 * g + h] = e2m1x8(v);
            }
          } else {
            packed[2 * g] = 0u;
            packed[2 * g + 1] = 0u;
          }
        }
        if (live) {
          // tiled scale layout: 512-byte atom per (128-row block, 64-column block)
          uint8_t* sp = reinterpret_cast<uint8_t*>(p.scales) +
                        (static_cast<size_t>(blockIdx.y) * (p.K / 64) + (k0 / 64)) * 512 +
                        (row & 31) * 16 + (row >> 5) * 4;
          *reinterpret_cast<uint32_t*>(sp) = sc;
        }
      } else {
        const float a = fmaxf(fmaxf(bf16_amax<8>(w), bf16_amax<8>(w + 8)),
                              fmaxf(bf16_amax<8>(w + 16), bf16_amax<8>(w + 24)));
        const __nv_bfloat16 sb = __float2bfloat16_rn(div_by_scale(a, 7.0f, kRcp7));
        const float s_ = __bfloat162float(sb);
        if (s_ >= kMinFastScale && s_ < kMaxFastScale) {
          const float y = __frcp_rn(s_);
          // div_by_scale on two values per instruction (its sign repair is not
          // needed: -0 and +0 give the same INT4 code); then rint by adding
          // 1.5 * 2^23, which leaves the integer in the low mantissa bits.
          // The clamp to [-8, 7] is not needed here: s = bf16(amax / 7) is at
          // least (amax / 7)(1 - 2^-9), so |x / s| <= 7.014 and rint is in
          // [-7, 7].
          const uint64_t y2 = f2_pack(y, y), ns2 = f2_pack(-s_, -s_);
          const uint64_t mg2 = f2_pack(12582912.0f, 12582912.0f);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint32_t pk = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t ww = w[4 * j + e];
              const uint64_t x2 = f2_pack(bf16lo(ww), bf16hi(ww));
              const uint64_t q0 = f2_mul(x2, y2);
              const uint64_t r2 = f2_add(f2_fma(f2_fma(q0, ns2, x2), y2, q0), mg2);
              pk |= (__float_as_uint(f2_lo(r2)) & 0xFu) << (8 * e);
              pk |= (__float_as_uint(f2_hi(r2)) & 0xFu) << (8 * e + 4);
            }
            packed[j] = pk;
          }
        } else if (s_ > 0.0f) {  // scale outside the fast path's range: exact division
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint32_t pk = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t ww = w[4 * j + e];
              pk |= int4_rn(__fdiv_rn(bf16lo(ww), s_)) << (8 * e);
              pk |= int4_rn(__fdiv_rn(bf16hi(ww), s_)) << (8 * e + 4);
            }
            packed[j] = pk;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) packed[j] = 0u;
        }
        if (live)
          reinterpret_cast<__nv_bfloat16*>(p.scales)[static_cast<size_t>(grow) * (p.K / 64) +
                                                     k0 / 64] = sb;
      }
      if (live) {
        uint4* cp = reinterpret_cast<uint4*>(p.codes + static_cast<size_t>(grow) * kh + k0 / 2);
        cp[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        cp[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
      }
    }
  }

  // ------------------------------------------------------- T = X' L1 epilogue
  if constexpr (R > 0) {
    // partial tile of this K range: straight to T when the row block is not
    // split, else to the scratch slot of this split
    const int num_m = gridDim.y;
    if (warp < 4) {  // one warp per 32-lane group of tensor memory
      const int row = warp * 32 + lane;
      const int grow = m0 + row;
      bool ok = wait_bounded(bar_tfull, 0, guard, 0x105);
      if (ok) tc_fence_after();
      if (p.ksplit > 1 && p.t_accumulate && ks != 0) {
        // split 0 has cleared this row block's T (long ago, in practice)
        bool seen = true;
        if (lane == 0) {
          const uint64_t t0 = global_timer_ns();
          while (ld_acquire_gpu(p.tflags + blockIdx.y) != p.epoch) {
            if (*abort_flag || global_timer_ns() - t0 > p.timeout_ns) {
              if (!*abort_flag) {
                *abort_flag = 1;
                atomicCAS(p.err, 0, 0x106);
              }
              seen = false;
              break;
            }
          }
        }
        ok = ok && __shfl_sync(0xffffffffu, seen, 0);
      }
      const uint32_t ta = tmem + (static_cast<uint32_t>(warp * 32) << 16);
      // stream the row's R fp32 values out of tensor memory 16 or 32 columns at a time
      constexpr int CW = R < 32 ? R : 32;
#pragma unroll 1
      for (int c0 = 0; c0 < R; c0 += CW) {
        uint32_t v[CW];
        if (ok) {
          if constexpr (CW == 16) tmem_ld_x16(ta + c0, v);
          else tmem_ld_x32(ta + c0, v);
          tmem_ld_wait();
        }
        if (ok && grow < p.M) {
          if (p.ksplit > 1 && p.t_accumulate) {
            // the split partials meet in T itself (fire-and-forget vector
            // reductions; their order across the splits is not fixed)
            float4* dst = reinterpret_cast<float4*>(p.t + static_cast<size_t>(grow) * R + c0);
#pragma unroll
            for (int j = 0; j < CW / 4; ++j)
              atomicAdd(dst + j, make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                             __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])));
          } else {
            float* drow = p.ksplit == 1
                              ? p.t + static_cast<size_t>(grow) * R
                              : p.tpart + ((static_cast<size_t>(ks) * num_m + blockIdx.y) * 128 + row) * R;
            float4* dst = reinterpret_cast<float4*>(drow + c0);
#pragma unroll
            for (int j = 0; j < CW / 4; ++j)
              dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                   __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
          }
        }
      }
    }
    if (p.ksplit > 1 && !p.t_accumulate) {
      // The last split CTA of this row block to arrive sums the partial tiles
      // in split order (deterministic) and resets the block's counter.
      __shared__ int last;
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) last = atomicAdd(p.counters + blockIdx.y, 1) == p.ksplit - 1;
      __syncthreads();
      if (last) {
        __threadfence();
        const int rows = min(128, p.M - m0);
        for (int it = threadIdx.x; it < rows * (R / 4); it += KQ_THREADS) {
          const int rr = it / (R / 4), j = it % (R / 4);
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int src = 0; src < p.ksplit; ++src) {
            const float4 f = __ldcg(reinterpret_cast<const float4*>(
                p.tpart + ((static_cast<size_t>(src) * num_m + blockIdx.y) * 128 + rr) * R) + j);
            acc.x += f.x; acc.y += f.y; acc.z += f.z; acc.w += f.w;
          }
          if (!*abort_flag)
            reinterpret_cast<float4*>(p.t + static_cast<size_t>(m0 + rr) * R)[j] = acc;
        }
        if (threadIdx.x == 0) p.counters[blockIdx.y] = 0;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (R > 0 && warp == MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace svdq
