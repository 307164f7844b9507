// Pieces shared by the two GEMM kernels (NVFP4 and INT4): parameters, the
// low-rank operand preparation and the output epilogue.
//
// The low-rank up projection T L2 ("Problemas do Nunchaku Qwen...",
// apatero.com, section "O que e Nunchaku e como acelera modelos Qwen": the
// up projection is fused into the 4-bit compute kernel) runs on the tensor
// cores as extra bf16 k-steps into the same fp32 accumulator.  T arrives in
// fp32; it is split into T_hi = bf16(T) and T_lo = bf16(T - T_hi) so that
//   T L2 = [T_hi | T_lo] . [L2 ; L2]
// keeps 16 significant bits of T (bf16 x bf16 products are exact in fp32).
#pragma once

#include "ptx.cuh"

namespace svdq {

constexpr int KG_THREADS = 640;  // 4 control warps + 16 epilogue warps
constexpr int KG_EPI_WARPS = 16;
constexpr int KG_BM = 128;
constexpr int KG_BN = 256;

struct KGParams {
  const uint8_t* sfa;   // NVFP4: tiled activation scales; INT4: bf16 [M x K/64]
  const uint8_t* sfb;   // NVFP4: tiled weight scales; INT4: bf16 [K/64 x Npad]
  const float* t;       // [M x R] fp32 (unused when R == 0)
  const uint16_t* bias; // bf16 [N] or null
  uint16_t* y;          // bf16 [M x N]
  int M, N, K;
  int num_m, num_n;
  int gelu;
  // NVFP4 weights with a per-tensor scale 2^e: the accumulator is multiplied
  // by out_scale = 2^e before bias / GELU and T by t_scale = 2^-e before the
  // low-rank MMAs (both exact powers of two; 1 otherwise)
  float out_scale, t_scale;
  // fused QKV epilogue (qkv_hd > 0): columns [Q | K | V] of qkv_hd each; Q
  // and K heads (128 features) RMS-normalised (times gq / gk, bf16 [128]) and
  // rotated pairwise by rope: the row-blocked table of rope_block_kernel
  // (float4 [rows / 32][32 two-pair chunks][32 rows] of cos, sin, cos, sin)
  int qkv_hd;
  float norm_eps;
  const uint16_t* gq;
  const uint16_t* gk;
  const float* rope;
  int* err;
  uint32_t debug_mask;
  uint64_t timeout_ns;
};

// GELU, tanh form, of two values with paired fp32 arithmetic:
//   0.5 x (1 + tanh(u)) = x / (1 + exp(-2u)) = x / (1 + 2^a),
//   u = sqrt(2/pi) (x + 0.044715 x^3),  a = x (c1 + c2 x^2),
//   c1 = -2 log2(e) sqrt(2/pi),  c2 = 0.044715 c1,
// with the hardware's approximate base-2 exponential and reciprocal (both
// within a few fp32 ulps; x / (1 + 2^a) -> -0 or 0 as 2^a overflows).
__device__ __forceinline__ uint64_t gelu_tanh2(uint64_t x) {
  const uint64_t t = f2_fma(f2_mul(x, x), f2_pack(-0.10294324160f, -0.10294324160f),
                            f2_pack(-2.3022081852f, -2.3022081852f));
  const uint64_t a = f2_mul(x, t);
  float e0, e1, r0, r1;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e0) : "f"(f2_lo(a)));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(f2_hi(a)));
  const uint64_t d = f2_add(f2_pack(e0, e1), f2_pack(1.0f, 1.0f));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(f2_lo(d)));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r1) : "f"(f2_hi(d)));
  return f2_mul(x, f2_pack(r0, r1));
}
// In place on 2n values.
template <int N2>
__device__ __forceinline__ void gelu_tanh_pairs(float* v) {
#pragma unroll
  for (int e = 0; e < 2 * N2; e += 2) {
    const uint64_t g = gelu_tanh2(f2_pack(v[e], v[e + 1]));
    v[e] = f2_lo(g);
    v[e + 1] = f2_hi(g);
  }
}

// v[0..7] (columns n..n+7) <- v * out_scale (+ bias), in pairs.
__device__ __forceinline__ void scale_bias_pairs(const KGParams& p, int n, float* v) {
  uint64_t x[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] = f2_pack(v[2 * e], v[2 * e + 1]);
  if (p.out_scale != 1.0f) {  // 2^e, only with an NVFP4 per-tensor weight scale (x 1 is exact)
    const uint64_t os2 = f2_pack(p.out_scale, p.out_scale);
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = f2_mul(x[e], os2);
  }
  if (p.bias != nullptr && n < p.N) {
    const uint4 bb = __ldg(reinterpret_cast<const uint4*>(p.bias + n));
    const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = f2_add(x[e], f2_pack(bf16lo(bw[e]), bf16hi(bw[e])));
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    v[2 * e] = f2_lo(x[e]);
    v[2 * e + 1] = f2_hi(x[e]);
  }
}

// Write [T_hi | T_lo] of rows m0..m0+127 into the A operand buffer of the
// low-rank k-steps: 128 rows x (64 bf16 = 128 B) chunks, 128B swizzle.
// Called by NT epilogue threads (etid = 0..NT-1).
template <int R, int NT = KG_EPI_WARPS * 32>
__device__ __forceinline__ void prep_lowrank_a(uint8_t* alr, const float* __restrict__ t, int m0,
                                               int M, int etid, float tsc = 1.0f) {
  constexpr int SEG = R / 8;  // 8 values of T per item
  for (int it = etid; it < 128 * SEG; it += NT) {
    const int row = it / SEG;
    const int seg = it % SEG;
    const int gm = m0 + row;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (gm < M) {
      const float4* src = reinterpret_cast<const float4*>(t + static_cast<size_t>(gm) * R + seg * 8);
      a = __ldg(src);
      b = __ldg(src + 1);
    }
    const float v[8] = {__fmul_rn(a.x, tsc), __fmul_rn(a.y, tsc), __fmul_rn(a.z, tsc), __fmul_rn(a.w, tsc),
                        __fmul_rn(b.x, tsc), __fmul_rn(b.y, tsc), __fmul_rn(b.z, tsc), __fmul_rn(b.w, tsc)};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
      const float h0 = __low2float(h), h1 = __high2float(h);
      const __nv_bfloat162 l = __floats2bfloat162_rn(__fsub_rn(v[2 * j], h0), __fsub_rn(v[2 * j + 1], h1));
      hi[j] = *reinterpret_cast<const uint32_t*>(&h);
      lo[j] = *reinterpret_cast<const uint32_t*>(&l);
    }
    const int chi = seg * 8;      // logical bf16 column of T_hi
    const int clo = R + seg * 8;  // logical bf16 column of T_lo
    *reinterpret_cast<uint4*>(alr + (chi / 64) * 16384 + swz_off(row, (chi % 64) / 8, 128)) =
        make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(alr + (clo / 64) * 16384 + swz_off(row, (clo % 64) / 8, 128)) =
        make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// Epilogue store, warp-cooperative with full-line stores.  Lane l holds
// 64 accumulator columns [n_base, n_base + 64) of row row0 + l: + bias,
// GELU, bf16.  After bias,
// GELU and bf16 packing each lane has eight 16-byte chunks of its row; an 8x8
// transpose of those chunks inside each group of 8 lanes (three butterfly
// stages of shfl.xor, stage b swapping bit b of the lane and chunk indices)
// leaves lane 8g+c with chunk c of the rows of lanes 8g..8g+7.  Store k then
// writes, per 8-lane group, one contiguous 128-byte row segment, instead of
// 32 scattered 16-byte pieces.  All 32 lanes must call it.
// With FINAL the 64 values are already the outputs (no scale, bias or GELU).
template <bool FINAL = false>
__device__ __forceinline__ void store_rows64_coalesced(const KGParams& p, int row0, int n_base,
                                                       const float* acc, int lane) {
  uint32_t w[32];
#pragma unroll
  for (int j8 = 0; j8 < 8; ++j8) {
    const int n = n_base + 8 * j8;
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = acc[8 * j8 + e];
    if (!FINAL) {
      scale_bias_pairs(p, n, v);
      if (p.gelu) gelu_tanh_pairs<4>(v);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) w[4 * j8 + e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
  }
#pragma unroll
  for (int b = 1; b < 8; b <<= 1) {
    const bool up = (lane & b) != 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (c & b) continue;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t send = up ? w[4 * c + e] : w[4 * (c | b) + e];
        const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, b);
        if (up) w[4 * c + e] = recv;
        else w[4 * (c | b) + e] = recv;
      }
    }
  }
  const int n = n_base + 8 * (lane & 7);
  if (n >= p.N) return;
  const int rg = row0 + (lane & ~7);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int gm = rg + k;
    if (gm < p.M)
      *reinterpret_cast<uint4*>(p.y + static_cast<size_t>(gm) * p.N + n) =
          make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
  }
}

// The same for 32 columns per lane: four 16-byte chunks, a 4 x 4 transpose
// inside each group of 4 lanes (shfl.xor 1, 2), then each store writes, per
// 4-lane group, a contiguous 64-byte row segment.  All 32 lanes must call it.
__device__ __forceinline__ void store_rows32_coalesced(const KGParams& p, int row0, int n_base,
                                                       const float* acc, int lane) {
  uint32_t w[16];
#pragma unroll
  for (int j8 = 0; j8 < 4; ++j8) {
    const int n = n_base + 8 * j8;
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = acc[8 * j8 + e];
    scale_bias_pairs(p, n, v);
    if (p.gelu) gelu_tanh_pairs<4>(v);
#pragma unroll
    for (int e = 0; e < 4; ++e) w[4 * j8 + e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
  }
#pragma unroll
  for (int b = 1; b < 4; b <<= 1) {
    const bool up = (lane & b) != 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (c & b) continue;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t send = up ? w[4 * c + e] : w[4 * (c | b) + e];
        const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, b);
        if (up) w[4 * c + e] = recv;
        else w[4 * (c | b) + e] = recv;
      }
    }
  }
  const int n = n_base + 8 * (lane & 3);
  if (n >= p.N) return;
  const int rg = row0 + (lane & ~3);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int gm = rg + k;
    if (gm < p.M)
      *reinterpret_cast<uint4*>(p.y + static_cast<size_t>(gm) * p.N + n) =
          make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
  }
}

// Fused QKV epilogue for one epilogue warp's 32 rows x 64 columns
// [n_base, n_base + 64) (row = row0 + lane), then the coalesced store.
// "Nunchaku Lite ..." (axbrief.com), section "The Trade-off Between Fused
// Kernels and Generality": the QKV projection, the Q/K normalisation and the
// rotary embedding in one kernel.  Per value: v = acc * out_scale (+ bias);
// for Q and K columns, per 128-feature head: v <- v / sqrt(mean(v^2) + eps)
// * g, then pairs (2i, 2i+1) rotated by token row's (cos, sin) of pair i
// (read from the row-blocked copy of the caller's table).
// A head spans two warps (slices cs and cs ^ 1 of the same lane quarter q).
// Each publishes its rows' partial sums of squares in red ([4][4][32]
// floats) and the pair exchanges them through mbarrier xbar[q + 4 (cs/2)]
// (64 arrivals a phase): phase 2k when both have written, 2k + 1 when both
// have read, so the next tile's write cannot overtake the partner's read.
// The two partials are added in slice order (both warps use the same sum).
// Waits are bounded; false means the CTA is aborting.
__device__ __forceinline__ bool epilogue_qkv64(const KGParams& p, int row0, int n_base, const float* acc,
                                               int lane, int q, int cs, float* red, uint32_t xbar,
                                               uint32_t& xph, const Guard& guard) {
  float v[64];
#pragma unroll
  for (int c = 0; c < 64; ++c) v[c] = __fmul_rn(acc[c], p.out_scale);
  if (p.bias != nullptr && n_base < p.N) {
#pragma unroll
    for (int c8 = 0; c8 < 8; ++c8) {
      const uint4 bb = __ldg(reinterpret_cast<const uint4*>(p.bias + n_base + 8 * c8));
      const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[8 * c8 + 2 * e] = __fadd_rn(v[8 * c8 + 2 * e], bf16lo(bw[e]));
        v[8 * c8 + 2 * e + 1] = __fadd_rn(v[8 * c8 + 2 * e + 1], bf16hi(bw[e]));
      }
    }
  }
  if (n_base < 2 * p.qkv_hd && n_base < p.N) {
    const uint16_t* g = n_base < p.qkv_hd ? p.gq : p.gk;
    const int d0 = n_base % 128;  // first feature of this slice within its head
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 64; ++c) ss = __fmaf_rn(v[c], v[c], ss);
    const uint32_t xb = xbar + 8 * (q + 4 * (cs >> 1));
    red[(q * 4 + cs) * 32 + lane] = ss;
    mbar_arrive(xb);
    if (!__all_sync(0xffffffffu, wait_bounded(xb, xph & 1, guard, 0x240))) return false;
    const float tot = __fadd_rn(red[(q * 4 + (cs & ~1)) * 32 + lane], red[(q * 4 + (cs | 1)) * 32 + lane]);
    mbar_arrive(xb);
    if (!__all_sync(0xffffffffu, wait_bounded(xb, (xph + 1) & 1, guard, 0x241))) return false;
    xph += 2;
    const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot, 128.0f), p.norm_eps)));
#pragma unroll
    for (int c8 = 0; c8 < 8; ++c8) {
      const uint4 gg = __ldg(reinterpret_cast<const uint4*>(g + d0 + 8 * c8));
      const uint32_t gw[4] = {gg.x, gg.y, gg.z, gg.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[8 * c8 + 2 * e] = __fmul_rn(__fmul_rn(v[8 * c8 + 2 * e], inv), bf16lo(gw[e]));
        v[8 * c8 + 2 * e + 1] = __fmul_rn(__fmul_rn(v[8 * c8 + 2 * e + 1], inv), bf16hi(gw[e]));
      }
    }
    // row0 is a multiple of 32 and the blocked table covers every row of
    // every tile (rows past M hold the identity rotation): each load reads
    // the 32 rows' chunk d0 / 4 + i2, 512 contiguous bytes
    const float4* cs4 = reinterpret_cast<const float4*>(p.rope) +
                        (static_cast<size_t>(row0 / 32) * 32 + d0 / 4) * 32 + lane;
#pragma unroll
    for (int i2 = 0; i2 < 16; ++i2) {  // two pairs per 16-byte load: (cos, sin, cos, sin)
      const float4 t = __ldg(cs4 + 32 * i2);
      const float a0 = v[4 * i2], b0 = v[4 * i2 + 1], a1 = v[4 * i2 + 2], b1 = v[4 * i2 + 3];
      v[4 * i2] = __fsub_rn(__fmul_rn(a0, t.x), __fmul_rn(b0, t.y));
      v[4 * i2 + 1] = __fadd_rn(__fmul_rn(a0, t.y), __fmul_rn(b0, t.x));
      v[4 * i2 + 2] = __fsub_rn(__fmul_rn(a1, t.z), __fmul_rn(b1, t.w));
      v[4 * i2 + 3] = __fadd_rn(__fmul_rn(a1, t.w), __fmul_rn(b1, t.z));
    }
  }
  store_rows64_coalesced<true>(p, row0, n_base, v, lane);
  return true;
}

// Wait for the producer's outstanding loads before the CTA exits (abort path).
__device__ __forceinline__ void drain_loads(uint32_t bar_full, uint32_t issued, uint32_t issued_par,
                                            int stages, uint64_t limit_ns) {
  for (int s = 0; s < stages; ++s)
    if (issued & (1u << s)) {
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(bar_full + 8 * s, (issued_par >> s) & 1) &&
             global_timer_ns() - t0 < limit_ns) {
      }
    }
}

}  // namespace svdq
