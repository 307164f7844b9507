// Kernel 2, INT4 variant on 16-bit tensor cores (opt-in: SVDQ_INT4_F16):
// the same product as kg_int4_kernel,
//   acc[m,n] = sum_g s_x[m,g] s_w[n,g] sum_{k in g} q_x[m,k] q_w[n,k],
// computed as one fp16 GEMM of the dequantised operands
//   A[m,k] = s_x[m,g(k)] q_x[m,k],   B[n,k] = s_w[n,g(k)] q_w[n,k].
// Both are exact in fp16 while the scales stay in fp16's range: a bf16 scale
// has 8 significant bits and |q| <= 8 has at most 3, so the product has at
// most 11 -- fp16's precision -- and every A*B product is exact in the fp32
// accumulator.  Only the summation order differs from the per-group form.
// The per-group rescale of the int8 kernel (M N K/64 conversions and
// multiply-adds, latency-bound per group) disappears: one epilogue per tile.
//
// Method: "Nunchaku 1.3.0 for Python3.14.x & alpha" (note.com), section
// "SVDQ-FP4 on Blackwell", part "1. INT4" (INT4 -8..+7, W ~ int4 * scale);
// "Nunchaku Lite ... integrated into Diffusers" (axbrief.com), section "The
// Mechanics of 4-Bit Efficiency and SVDQuant" (W4A4 residual + 16-bit
// low-rank branch).
//
// Weights arrive dequantised (fp16 [N x K], prepared at load, exactness
// checked there); activations are dequantised per stage in shared memory.
// Both operands hold K in the same order, permuted inside every block of 8
// as (0,4,1,5,2,6,3,7): the order in which four lop3 operations lay out the
// eight nibbles of a 32-bit word as fp16 pairs.  A dot product does not
// depend on the order of its terms.
// Persistent CTAs, one per SM, tile 128 x 256, one 64-group per stage, two
// 128 x 256 fp32 accumulators in tensor memory (all 512 columns: no scale
// factors live there), so the MMAs of tile j+1 run while tile j drains.
// Warp roles (576 threads):
//   warp 0      TMA producer: packed activation codes (32B swizzle), fp16
//               weight tile (128B swizzle)
//   warp 1      MMA issuer (kind::f16, fp16 x fp16, four k-steps of 16 per
//               stage; low-rank bf16 k-steps), tensor-memory owner
//   warps 2-9   dequantise the activation codes: q (from the nibble) times
//               s_x, written as fp16 in the MMA's 128B-swizzled layout; one
//               group of two warps per ring slot, two rows per thread
//   warps 10-17 epilogue: drain an accumulator, next tile's low-rank
//               operand, bias + GELU + bf16 stores
#pragma once

#include <cuda_fp16.h>

#include "kg_common.cuh"

namespace svdq {

// Largest activation scale whose products with |q| <= 7 stay finite in fp16
// (7 * s <= 65504).  Larger scales are reported as a device error.
constexpr float kInt4F16MaxScale = 9357.0f;

constexpr int KGI4H_DQ_WARPS = 8;
constexpr int KGI4H_EPI_WARPS = 8;
constexpr int KGI4H_THREADS = (2 + KGI4H_DQ_WARPS + KGI4H_EPI_WARPS) * 32;

// K order inside each block of 8 (both operands): position p holds element
// kInt4F16Perm[p] of the block.
constexpr int kInt4F16Perm[8] = {0, 4, 1, 5, 2, 6, 3, 7};

template <int R>
struct KGI4HSmem {
  static constexpr int STAGES = R >= 64 ? 3 : 4;  // one dequantising group (2 warps) per slot
  static constexpr int APK_BYTES = KG_BM * 32;   // 128 rows x 32 B packed (64 codes)
  static constexpr int AH_BYTES = KG_BM * 128;   // 128 rows x 64 fp16
  static constexpr int B_BYTES = KG_BN * 128;    // 256 rows x 64 fp16
  static constexpr int STAGE = APK_BYTES + AH_BYTES + B_BYTES;
  static constexpr int LR_CHUNKS = R > 0 ? (2 * R + 63) / 64 : 0;
  static constexpr int LR_STEPS = R / 8;                      // bf16 k-steps of 16 over [T_hi | T_lo]
  static constexpr int LR_STAGES = (LR_STEPS + 3) / 4;        // a 128-byte B row holds 4 k-steps
  static constexpr int ALR_OFF = STAGES * STAGE;
  static constexpr int BAR_OFF = ALR_OFF + LR_CHUNKS * 16384;
  static constexpr int TOTAL = BAR_OFF + 256 + 1024;  // barriers, tensor-memory slot, alignment
  static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
  static_assert(TOTAL <= 232448, "shared memory per CTA");
  static_assert(2 * STAGES <= KGI4H_DQ_WARPS, "two dequantising warps per ring slot");
};

// kind::f16 with fp16 A and B, fp32 accumulate, K-major both.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Eight INT4 codes (two's complement nibbles, element 0 lowest) times the
// scale pair s2, as four fp16x2 words holding the elements (0,4) (1,5) (2,6)
// (3,7).  lop3 with table 0x6A computes mask ? (w ^ c) : c: it keeps the
// masked nibbles, flips their sign bit (q + 8 = q xor 8 for a 4-bit code) and
// fills the rest with the fp16 exponent of 1024, so a nibble in bits 0-3 of a
// half reads 1024 + (q + 8) and one in bits 4-7 reads 1024 + 16 (q + 8).
// Subtracting 1032, or scaling by 1/16 and subtracting 72, gives q exactly;
// the product with s (8 significant bits) is exact while it stays in range.
__device__ __forceinline__ void dequant8_f16(uint32_t w, uint32_t s2, uint32_t* out) {
  const uint32_t w8 = w >> 8;
  uint32_t t[4];
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t[0]) : "r"(w), "r"(0x000F000Fu), "r"(0x64086408u));
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t[1]) : "r"(w), "r"(0x00F000F0u), "r"(0x64806480u));
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t[2]) : "r"(w8), "r"(0x000F000Fu), "r"(0x64086408u));
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t[3]) : "r"(w8), "r"(0x00F000F0u), "r"(0x64806480u));
#pragma unroll
  for (int j = 0; j < 4; j += 2) {
    uint32_t q0, q1;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(q0) : "r"(t[j]), "r"(0x64086408u));
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(q1) : "r"(t[j + 1]), "r"(0x2C002C00u), "r"(0xD480D480u));
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out[j]) : "r"(q0), "r"(s2));
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out[j + 1]) : "r"(q1), "r"(s2));
  }
}

template <int R>
__global__ void __launch_bounds__(KGI4H_THREADS, 1)
    kg_int4h_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_blr, KGParams p) {
  using S = KGI4HSmem<R>;
  constexpr int NST = S::STAGES;
  constexpr int NEPI = KGI4H_EPI_WARPS * 32;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR_OFF);
  const uint32_t bar_full = smem_u32(bars);
  const uint32_t bar_ready = smem_u32(bars + NST);       // dequantised A written
  const uint32_t bar_empty = smem_u32(bars + 2 * NST);
  const uint32_t bar_acc_full = smem_u32(bars + 3 * NST);       // two, one per accumulator
  const uint32_t bar_acc_empty = smem_u32(bars + 3 * NST + 2);  // two
  const uint32_t bar_lr_full = smem_u32(bars + 3 * NST + 4);
  const uint32_t bar_drain = smem_u32(bars + 3 * NST + 5);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * NST + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Guard guard{p.err, abort_flag, p.timeout_ns};
  const int num_tiles = p.num_m * p.num_n;
  const int ng = p.K / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_ready + 8 * s, 64);  // one group of dequantising threads
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_acc_full + 8 * b, 1);
      mbar_init(bar_acc_empty + 8 * b, KGI4H_EPI_WARPS);
    }
    mbar_init(bar_lr_full, NEPI);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // inputs written by the activation kernel: see griddep_wait()
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      if (R > 0) tma_prefetch_desc(&tm_blr);
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x, j = 0; tile < num_tiles && ok; tile += gridDim.x, ++j) {
        const int mb = tile % p.num_m, nb = tile / p.num_m;
        for (int g = 0; g < ng; ++g) {
          if (!(ok = wait_bounded(bar_empty + 8 * s, ph ^ 1, guard, 0x341))) break;
          issued &= ~(1u << s);
          if (!((p.debug_mask & 1u) && j == 0 && g == 1)) {  // test hook: leave one stage empty
            const uint32_t st = sbase + s * S::STAGE;
            const uint32_t fb = bar_full + 8 * s;
            mbar_expect_tx(fb, S::APK_BYTES + S::B_BYTES);
            tma_load_2d(st, &tm_a, fb, g * 32, mb * KG_BM);
            tma_load_2d(st + S::APK_BYTES + S::AH_BYTES, &tm_b, fb, g * 64, nb * KG_BN);
            issued |= 1u << s;
            issued_par = (issued_par & ~(1u << s)) | (ph << s);
          }
          if (++s == NST) { s = 0; ph ^= 1; }
        }
        for (int l = 0; l < S::LR_STAGES && ok; ++l) {
          if (!(ok = wait_bounded(bar_empty + 8 * s, ph ^ 1, guard, 0x342))) break;
          issued &= ~(1u << s);
          const uint32_t fb = bar_full + 8 * s;
          mbar_expect_tx(fb, S::B_BYTES);
          tma_load_2d(sbase + s * S::STAGE + S::APK_BYTES + S::AH_BYTES, &tm_blr, fb, l * 64, nb * KG_BN);
          issued |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == NST) { s = 0; ph ^= 1; }
        }
      }
      if (*abort_flag) drain_loads(bar_full, issued, issued_par, NST, p.timeout_ns);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t id_h = idesc_f16_f32(KG_BM, KG_BN);
      constexpr uint32_t id_bf = idesc_bf16_f32(KG_BM, KG_BN);
      const uint64_t dA0 = smem_desc(sbase + S::APK_BYTES, 16, 1024, SWZ_128B);
      const uint64_t dB0 = smem_desc(sbase + S::APK_BYTES + S::AH_BYTES, 16, 1024, SWZ_128B);
      const uint64_t dLRA0 = smem_desc(sbase + S::ALR_OFF, 16, 1024, SWZ_128B);
      constexpr uint64_t kStage = S::STAGE >> 4;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = blockIdx.x, j = 0; tile < num_tiles && ok; tile += gridDim.x, ++j) {
        const int b = j & 1;
        const uint32_t acc = tmem + b * KG_BN;
        if (j >= 2 && !(ok = wait_bounded(bar_acc_empty + 8 * b, ((j >> 1) - 1) & 1, guard, 0x343))) break;
        tc_fence_after();
        for (int g = 0; g < ng; ++g) {
          if (!(ok = wait_bounded(bar_ready + 8 * s, ph, guard, 0x344))) break;
          tc_fence_after();
          const uint64_t so = kStage * s;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(acc, dA0 + so + 2 * kk, dB0 + so + 2 * kk, id_h, (g | kk) != 0);
          tc_commit(bar_empty + 8 * s);
          if (++s == NST) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        if (R > 0) {
          if (!(ok = wait_bounded(bar_lr_full, j & 1, guard, 0x345))) break;
          tc_fence_after();
          for (int l = 0; l < S::LR_STAGES; ++l) {
            if (!(ok = wait_bounded(bar_ready + 8 * s, ph, guard, 0x346))) break;
            tc_fence_after();
            const uint64_t so = kStage * s;
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) {
              const int kk = 4 * l + k2;  // k-step over [T_hi | T_lo]
              if (kk < S::LR_STEPS)
                mma_bf16(acc, dLRA0 + (kk / 4) * 1024 + (kk % 4) * 2, dB0 + so + 2 * k2, id_bf, 1);
            }
            tc_commit(bar_empty + 8 * s);
            if (++s == NST) { s = 0; ph ^= 1; }
          }
          if (!ok) break;
        }
        tc_commit(bar_acc_full + 8 * b);
      }
      // drain: every MMA issued so far has completed before tensor memory is freed
      tc_commit(bar_drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(bar_drain, 0) && global_timer_ns() - t0 < p.timeout_ns) {
      }
    }
  } else if (warp < 2 + KGI4H_DQ_WARPS) {
    // ------------------------------------------------ dequantise activations
    // NST groups of two warps (one group per ring slot) take every NST-th
    // stage use, two rows per thread, so each thread has NST MMA stages' time
    // for its share and every slot is dequantised by one group.  A group's
    // previous use of a slot is then always its own, so its parity wait on the
    // slot is unambiguous.  With three slots, warps 8 and 9 stay idle.
    const int grp = (warp - 2) >> 1;                 // takes the uses u with u % NST == grp
    const int t = ((warp - 2) & 1) * 32 + lane;      // rows t and t + 64 of the tile
    const __nv_bfloat16* sx_all = reinterpret_cast<const __nv_bfloat16*>(p.sfa);
    int s = 0;
    uint32_t ph = 0, u = 0;
    bool ok = grp < NST;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      int gm[2];
      const __nv_bfloat16* sxr[2];
      float nx[2];
      // this thread's first group in the tile; its rows' scales are loaded
      // one use ahead (rows past M: 0)
      const int g0 = (grp - static_cast<int>(u % NST) + NST) % NST;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        gm[h] = (tile % p.num_m) * KG_BM + t + 64 * h;
        sxr[h] = sx_all + static_cast<size_t>(gm[h] < p.M ? gm[h] : 0) * ng;
        nx[h] = (gm[h] < p.M && g0 < ng) ? __bfloat162float(sxr[h][g0]) : 0.0f;
      }
      for (int g = 0; g < ng; ++g, ++u) {
        if (static_cast<int>(u % NST) == grp) {
          float sx[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            sx[h] = nx[h];
            if (g + NST < ng && gm[h] < p.M) nx[h] = __bfloat162float(sxr[h][g + NST]);
          }
          if (!(ok = wait_bounded(bar_full + 8 * s, ph, guard, 0x349))) break;
          const uint8_t* apk = smem + s * S::STAGE;
          uint8_t* ah = smem + s * S::STAGE + S::APK_BYTES;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int row = t + 64 * h;
            if (sx[h] > kInt4F16MaxScale) atomicCAS(p.err, 0, 0x34f);  // fp16 would overflow
            const __half2 s2h = __float2half2_rn(sx[h]);
            const uint32_t s2 = *reinterpret_cast<const uint32_t*>(&s2h);
            const uint4 v0 = *reinterpret_cast<const uint4*>(apk + swz_off(row, 0, 32));
            const uint4 v1 = *reinterpret_cast<const uint4*>(apk + swz_off(row, 1, 32));
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            // 64 codes = 8 chunks of 8 fp16 (16 bytes) of the 128-byte row
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint32_t o[4];
              dequant8_f16(w[c], s2, o);
              *reinterpret_cast<uint4*>(ah + swz_off(row, c, 128)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(bar_ready + 8 * s);
        }
        if (++s == NST) { s = 0; ph ^= 1; }
      }
      // low-rank stages carry only the B operand; still pass each one through
      // the ready barrier so its phase stays in step with the stage ring
      for (int l = 0; l < S::LR_STAGES && ok; ++l, ++u) {
        if (static_cast<int>(u % NST) == grp) {
          if (!(ok = wait_bounded(bar_full + 8 * s, ph, guard, 0x34c))) break;
          mbar_arrive(bar_ready + 8 * s);
        }
        if (++s == NST) { s = 0; ph ^= 1; }
      }
    }
  } else {
    // ----------------------------------------------------------------- epilogue
    const int e = warp - 2 - KGI4H_DQ_WARPS;  // 0..7
    const int q = warp & 3;                   // tensor-memory lane group of this warp
    const int cs = e >> 2;                    // 128-column half of the tile
    const int etid = e * 32 + lane;
    uint8_t* alr = smem + S::ALR_OFF;
    if constexpr (R > 0) {
      if (static_cast<int>(blockIdx.x) < num_tiles) {
        prep_lowrank_a<R, NEPI>(alr, p.t, (blockIdx.x % p.num_m) * KG_BM, p.M, etid);
        fence_proxy_async_smem();
        mbar_arrive(bar_lr_full);
      }
    }
    for (int tile = blockIdx.x, j = 0; tile < num_tiles; tile += gridDim.x, ++j) {
      const int mb = tile % p.num_m, nb = tile / p.num_m;
      const int b = j & 1;
      if (!__all_sync(0xffffffffu, wait_bounded(bar_acc_full + 8 * b, (j >> 1) & 1, guard, 0x347, 128))) break;
      tc_fence_after();
      if constexpr (R > 0) {
        // the accumulator is complete, so the low-rank MMAs have read the
        // operand buffer: prepare the next tile's
        const int next = tile + gridDim.x;
        if (next < num_tiles) {
          prep_lowrank_a<R, NEPI>(alr, p.t, (next % p.num_m) * KG_BM, p.M, etid);
          fence_proxy_async_smem();
          mbar_arrive(bar_lr_full);
        }
      }
      const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + b * KG_BN + cs * 128;
      uint32_t v[64];
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        tmem_ld_x32(ta + 64 * h, v);
        tmem_ld_x32(ta + 64 * h + 32, v + 32);
        tmem_ld_wait();
        if (h == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_acc_empty + 8 * b);
        }
        store_rows64_coalesced(p, mb * KG_BM + q * 32, nb * KG_BN + cs * 128 + 64 * h,
                               reinterpret_cast<const float*>(v), lane);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace svdq
