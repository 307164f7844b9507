// Kernel 2 of one NVFP4 layer (fc1: 4-bit GEMM, low-rank up projection, bias,
// GELU) with the NEXT layer's activation side fused into its epilogue (fc2:
// smoothing, NVFP4 group quantisation and packing, and the rank-r2 down
// projection T2 = X2' L1_2), so the layer's output never makes the round trip
// through HBM that fc2's activation kernel would otherwise need.
//
// Method: "Problemas do Nunchaku Qwen..." (apatero.com), section "O que e
// Nunchaku e como acelera modelos Qwen" -- the down projection fused with
// the quantisation and the up projection with the 4-bit compute, the
// branches sharing the activations and halving the kernel calls; "Nunchaku
// Lite ..." (axbrief.com), section "The Trade-off Between Fused Kernels and
// Generality" -- fused paths bundle consecutive operations to cut memory
// traffic.  Here the fusion spans two layers: fc1's tile is fc2's input tile.
//
// Per output value of fc1 (row m, column n = fc2's input channel):
//   y1 = bf16(GELU?(acc + bias))                  (fc1's output, optionally stored)
//   x2 = bf16(fp32(y1) * inv_lambda2[n])           (fc2's smoothing)
//   per 16 consecutive n: s = e4m3(amax / 6), q = e2m1(x2 / s)   (fc2's codes)
//   T2[m, :] += x2 . L1_2[n, :]                    (fc2's down projection)
// exactly the arithmetic of the activation kernel on fc1's bf16 output, so
// fc2's codes and scales are the same bits as the two-kernel path's.
//
// Structure: the single-SM 128 x 256 tile GEMM (see kg_nvfp4.cuh) with an
// extended epilogue.  Each CTA takes a contiguous range of tiles in
// row-block-major order, so consecutive tiles share the 128-row block and T2
// accumulates in tensor memory (r2 columns beside the scale factors) over the
// tile range's N-blocks; when the row block changes (or the range ends) the 4
// warps of the first column slice drain it and add it into T2 in global
// memory with fp32 atomics (T2 is zeroed before the launch; several CTAs may
// share a row block, so the sum order across CTAs is not fixed).  The T2
// products run on the tensor cores: the four 64-column slices of a tile take
// turns writing their X2' values (bf16, 128-byte swizzle, K-major) into one
// 16 KB shared buffer; after each turn one thread (warp 4, lane 0) issues
// four bf16 MMAs (M 128, N r2, K 16) with L1_2's slice rows as B, staged per
// tile by TMA, and commits the buffer to the NEXT slice's barrier.  Each
// slice has its own "buffer free" barrier that completes once per tile, so
// no waiter is ever more than one phase behind the barrier it polls (with
// one shared barrier, slices two turns ahead would read the parity of a
// phase that has not begun as complete).  Every wait is bounded.
#pragma once

#include "kg_nvfp4.cuh"
#include "kq.cuh"

namespace svdq {

struct KGChainParams {
  const float* inv_lam2;   // fc2's 1/lambda [N1]
  uint8_t* codes2;         // fc2's activation codes [M x N1/2]
  uint8_t* scales2;        // fc2's activation scales, tiled (see svdq_quantize_act_lowrank_down)
  float* t2;               // fc2's T [M x R2], zeroed before the launch
  int store_y;             // also store fc1's output y (bf16 [M x N1])
};

template <int R, int R2>
struct KGChainSmem {
  using B = KGF4Smem<R>;
  static constexpr int X2_OFF = B::XBAR_OFF + 64 + 192;       // 1 KB aligned below
  static constexpr int X2_OFF_A = (X2_OFF + 1023) / 1024 * 1024;
  static constexpr int X2_BYTES = 128 * 128;                  // 128 rows x 64 bf16
  static constexpr int L1_OFF = X2_OFF_A + X2_BYTES;
  static constexpr int L1_BYTES = 4 * R2 * 128;               // 4 slices x R2 rows x 64 bf16
  static constexpr int CBAR_OFF = L1_OFF + L1_BYTES;          // chain barriers (8 x 8 bytes)
  static constexpr int LUT_OFF = CBAR_OFF + 64;               // E4M3 code -> (value, 1/value)
  static constexpr int TOTAL = LUT_OFF + 128 * 8 + 1024;
  static constexpr int T2_COL = (B::SFB_COL + 8 * B::KB * B::STAGES + 31) / 32 * 32;  // after the scale factors
  static_assert(T2_COL + R2 <= 512, "tensor memory columns");
  static_assert(TOTAL <= 232448, "shared memory per CTA");
  static_assert(R2 == 16 || R2 == 32, "T2 MMA width");
};

template <int R, int R2>
__global__ void __launch_bounds__(KG_THREADS, 1)
    kg_nvfp4_chain_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                          const __grid_constant__ CUtensorMap tm_blr,
                          const __grid_constant__ CUtensorMap tm_l1t2, KGParams p, KGChainParams c) {
  using S = KGF4Smem<R>;
  using C = KGChainSmem<R, R2>;
  constexpr int NST = S::STAGES;
  constexpr int KB = S::KB;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR_OFF);
  const uint32_t bar_full = smem_u32(bars);
  const uint32_t bar_empty = smem_u32(bars + NST);
  const uint32_t bar_acc_full = smem_u32(bars + 2 * NST);
  const uint32_t bar_acc_empty = smem_u32(bars + 2 * NST + 1);
  const uint32_t bar_lr_full = smem_u32(bars + 2 * NST + 2);
  const uint32_t bar_drain = smem_u32(bars + 2 * NST + 3);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NST + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t bar_sfa = smem_u32(bars + 2 * NST + 5);
  const uint32_t bar_sfb = smem_u32(bars + 3 * NST + 5);
  const uint32_t bar_sf_drain = smem_u32(bars + 4 * NST + 5);  // two barriers
  // chain barriers
  const uint32_t cbar = sbase + C::CBAR_OFF;
  const uint32_t bar_x2_full = cbar;          // a slice's X2' written (128 arrivals)
  // bar_x2_free + 8 t: slice t may write the buffer (commit after the MMAs of
  // the turn before it: slice t - 1's, or the previous tile's slice 3 for t = 0)
  const uint32_t bar_x2_free = cbar + 8;
  const uint32_t bar_l1_full = cbar + 40;     // the tile's L1_2 rows landed (TMA)
  const uint32_t bar_t2_drained = cbar + 48;  // T2 accumulator drained (128 arrivals)
  const uint32_t bar_t2_final = cbar + 56;    // every T2 MMA completed (commit)
  float2* e4lut = reinterpret_cast<float2*>(smem + C::LUT_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Guard guard{p.err, abort_flag, p.timeout_ns};
  const int num_tiles = p.num_m * p.num_n;
  const int kblk = p.K / 64;
  const int nks = (kblk + KB - 1) / KB;
  // contiguous tile range of this CTA, row-block-major (tile t: mb = t / num_n)
  const int per = (num_tiles + gridDim.x - 1) / gridDim.x;
  const int t_begin = min(num_tiles, static_cast<int>(blockIdx.x) * per);
  const int t_end = min(num_tiles, t_begin + per);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_acc_full, 1);
    mbar_init(bar_acc_empty, KG_EPI_WARPS);
    mbar_init(bar_lr_full, KG_EPI_WARPS * 32);
    mbar_init(bar_drain, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_sfa + 8 * s, 1);
      mbar_init(bar_sfb + 8 * s, 1);
    }
    mbar_init(bar_sf_drain, 1);
    mbar_init(bar_sf_drain + 8, 1);
    mbar_init(bar_x2_full, 128);
    for (int t = 0; t < 4; ++t) mbar_init(bar_x2_free + 8 * t, 1);
    mbar_init(bar_l1_full, 1);
    mbar_init(bar_t2_drained, 128);
    mbar_init(bar_t2_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 128) {
    const float v = e4m3_value(threadIdx.x);
    e4lut[threadIdx.x] = make_float2(v, v > 0.0f && threadIdx.x < 127 ? __frcp_rn(v) : 0.0f);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
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
      for (int tile = t_begin; tile < t_end && ok; ++tile) {
        const int mb = tile / p.num_n, nb = tile % p.num_n;
        for (int ks = 0; ks < nks; ++ks) {
          if (!(ok = wait_bounded(bar_empty + 8 * s, ph ^ 1, guard, 0x251))) break;
          issued &= ~(1u << s);
          const uint32_t st = sbase + s * S::STAGE;
          const uint32_t fb = bar_full + 8 * s;
          const uint32_t kv = min(KB, kblk - KB * ks);
          mbar_expect_tx(fb, S::A_BYTES + S::B_BYTES + 3 * kv * 512);
          tma_load_2d(st, &tm_a, fb, ks * S::ROWB, mb * KG_BM);
          tma_load_2d(st + S::A_BYTES, &tm_b, fb, ks * S::ROWB, nb * KG_BN);
          bulk_load(st + S::A_BYTES + S::B_BYTES, p.sfa + (static_cast<size_t>(mb) * kblk + KB * ks) * 512,
                    kv * 512, fb);
          const uint8_t* sfb0 = p.sfb + (static_cast<size_t>(2 * nb) * kblk + KB * ks) * 512;
          bulk_load(st + S::A_BYTES + S::B_BYTES + S::SFA_BYTES, sfb0, kv * 512, fb);
          bulk_load(st + S::A_BYTES + S::B_BYTES + S::SFA_BYTES + KB * 512, sfb0 + static_cast<size_t>(kblk) * 512,
                    kv * 512, fb);
          issued |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == NST) { s = 0; ph ^= 1; }
        }
        for (int l = 0; l < S::LR_STAGES && ok; ++l) {
          if (!(ok = wait_bounded(bar_empty + 8 * s, ph ^ 1, guard, 0x252))) break;
          issued &= ~(1u << s);
          const uint32_t fb = bar_full + 8 * s;
          mbar_expect_tx(fb, S::B_BYTES);
          tma_load_2d(sbase + s * S::STAGE + S::A_BYTES, &tm_blr, fb, l * (S::ROWB / 2), nb * KG_BN);
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
      constexpr uint32_t id_f4 = idesc_nvf4(KG_BM, KG_BN);
      constexpr uint32_t id_bf = idesc_bf16_f32(KG_BM, KG_BN);
      const uint64_t dA0 = smem_desc(sbase, 16, S::SBO, S::SWZ);
      const uint64_t dB0 = smem_desc(sbase + S::A_BYTES, 16, S::SBO, S::SWZ);
      const uint64_t dLRA0 = smem_desc(sbase + S::ALR_OFF, 16, 1024, SWZ_128B);
      constexpr uint64_t kStage = S::STAGE >> 4;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = t_begin, j = 0; tile < t_end && ok; ++tile, ++j) {
        if (j > 0 && !(ok = wait_bounded(bar_acc_empty, (j - 1) & 1, guard, 0x253))) break;
        tc_fence_after();
        for (int ks = 0; ks < nks; ++ks) {
          const uint64_t so = kStage * s;
          const int kv = min(KB, kblk - KB * ks);
          const uint32_t ca = tmem + S::SFA_COL + KB * 4 * s;
          const uint32_t cb = tmem + S::SFB_COL + KB * 8 * s;
          // the first half of the k-blocks once warp 2's copies are in, the
          // second half once warp 3's are
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            if (kb == 0 || kb == KB / 2) {
              if (!(ok = wait_bounded(kb == 0 ? bar_sfa + 8 * s : bar_sfb + 8 * s, ph, guard,
                                      kb == 0 ? 0x254 : 0x255)))
                break;
              tc_fence_after();
            }
            if (kb < kv)
              mma_nvf4(tmem, dA0 + so + 2 * kb, dB0 + so + 2 * kb, id_f4, ca + 4 * kb, cb + 8 * kb, (ks | kb) != 0);
          }
          if (!ok) break;
          tc_commit(bar_empty + 8 * s);
          if (++s == NST) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        if (R > 0) {
          if (!(ok = wait_bounded(bar_lr_full, j & 1, guard, 0x256))) break;
          tc_fence_after();
          for (int l = 0; l < S::LR_STAGES; ++l) {
            if (!(ok = wait_bounded(bar_sfa + 8 * s, ph, guard, 0x257) &&
                       wait_bounded(bar_sfb + 8 * s, ph, guard, 0x258)))
              break;
            tc_fence_after();
            const uint64_t so = kStage * s;
#pragma unroll
            for (int k2 = 0; k2 < KB; ++k2) {
              const int kk = KB * l + k2;
              if (kk < S::LR_STEPS)
                mma_bf16(tmem, dLRA0 + (kk / 4) * 1024 + (kk % 4) * 2, dB0 + so + 2 * k2, id_bf, 1);
            }
            tc_commit(bar_empty + 8 * s);
            if (++s == NST) { s = 0; ph ^= 1; }
          }
          if (!ok) break;
        }
        tc_commit(bar_acc_full);
      }
      tc_commit(bar_drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(bar_drain, 0) && global_timer_ns() - t0 < p.timeout_ns) {
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------- scale-factor copies
    // Warp 2 copies the scale atoms (A's and both of B's) of the first half
    // of each stage's k-blocks, warp 3 those of the second half, so the two
    // warps issue equal shares.  Every stage (k-blocks or low-rank) completes
    // each warp's barrier once, after its data has landed, so the MMA warp
    // keeps one ring parity for all.
    if (lane == 0) {
      const int h = warp - 2;
      const uint32_t ready = h == 0 ? bar_sfa : bar_sfb;
      const uint64_t dA = smem_desc(sbase + S::A_BYTES + S::B_BYTES, 0, 128, SWZ_NONE);
      const uint64_t dB = smem_desc(sbase + S::A_BYTES + S::B_BYTES + S::SFA_BYTES, 0, 128, SWZ_NONE);
      constexpr uint64_t kStage = S::STAGE >> 4;
      constexpr int KH = KB / 2;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = t_begin; tile < t_end && ok; ++tile) {
        for (int ks = 0; ks < nks; ++ks) {
          if (!(ok = wait_bounded(bar_full + 8 * s, ph, guard, h == 0 ? 0x259 : 0x25a))) break;
          tc_fence_after();
          const int kv = min(KB, kblk - KB * ks);
          const uint32_t ca = tmem + S::SFA_COL + KB * 4 * s;
          const uint32_t cb = tmem + S::SFB_COL + KB * 8 * s;
#pragma unroll
          for (int i = 0; i < KH; ++i) {
            const int kb = h * KH + i;
            if (kb < kv) {
              tmem_cp_32x128b_warpx4(ca + 4 * kb, dA + kStage * s + 32 * kb);
              tmem_cp_32x128b_warpx4(cb + 8 * kb, dB + kStage * s + 32 * kb);
              tmem_cp_32x128b_warpx4(cb + 8 * kb + 4, dB + kStage * s + 32 * (KB + kb));
            }
          }
          tc_commit(ready + 8 * s);
          if (++s == NST) { s = 0; ph ^= 1; }
        }
        for (int l = 0; l < S::LR_STAGES && ok; ++l) {
          if (!(ok = wait_bounded(bar_full + 8 * s, ph, guard, 0x25b))) break;
          tc_commit(ready + 8 * s);
          if (++s == NST) { s = 0; ph ^= 1; }
        }
      }
      // this warp's copies have completed before tensor memory is freed
      const uint32_t drain = bar_sf_drain + 8 * h;
      tc_commit(drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < p.timeout_ns) {
      }
    }
  } else {
    // ----------------------------------------------------------------- epilogue
    const int e = warp - 4;
    const int q = warp & 3;        // tensor-memory lane group of this warp
    const int cs = e >> 2;         // 64-column slice
    const int etid = threadIdx.x - 128;
    const int row = q * 32 + lane;
    uint8_t* alr = smem + S::ALR_OFF;
    uint8_t* x2s = smem + C::X2_OFF_A;
    const bool issuer = warp == 4 && lane == 0;
    const uint32_t l1base = sbase + C::L1_OFF;
    constexpr uint32_t id_t2 = idesc_bf16_f32(KG_BM, R2);
    const uint64_t dX2 = smem_desc(sbase + C::X2_OFF_A, 16, 1024, SWZ_128B);
    const uint64_t dL1 = smem_desc(l1base, 16, 1024, SWZ_128B);
    const uint32_t t2col = tmem + C::T2_COL;
    // the first tile's L1_2 rows
    if (issuer && t_begin < t_end) {
      tma_prefetch_desc(&tm_l1t2);
      mbar_expect_tx(bar_l1_full, C::L1_BYTES);
      const int nb0 = t_begin % p.num_n;
      for (int i = 0; i < 4; ++i)
        tma_load_2d(l1base + i * R2 * 128, &tm_l1t2, bar_l1_full, nb0 * KG_BN + 64 * i, 0);
    }
    if constexpr (R > 0) {
      if (t_begin < t_end) {
        prep_lowrank_a<R>(alr, p.t, (t_begin / p.num_n) * KG_BM, p.M, etid, p.t_scale);
        fence_proxy_async_smem();
        mbar_arrive(bar_lr_full);
      }
    }
    uint32_t turn = 0;    // slice turns so far (4 per tile)
    uint32_t seg = 0;     // finished row-block segments (T2 drains)
    bool fresh = true;    // the next T2 MMA starts a new accumulation
    bool ok = true;
    for (int tile = t_begin, j = 0; tile < t_end && ok; ++tile, ++j) {
      const int mb = tile / p.num_n, nb = tile % p.num_n;
      const bool seg_end = tile + 1 == t_end || (tile + 1) / p.num_n != mb;
      if (!(ok = __all_sync(0xffffffffu, wait_bounded(bar_acc_full, j & 1, guard, 0x25c, 128)))) break;
      tc_fence_after();
      uint32_t v[64];
      const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + cs * 64;
      tmem_ld_x32(ta, v);
      tmem_ld_x32(ta + 32, v + 32);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_acc_empty);
      if constexpr (R > 0) {
        if (tile + 1 < t_end) {
          prep_lowrank_a<R>(alr, p.t, ((tile + 1) / p.num_n) * KG_BM, p.M, etid, p.t_scale);
          fence_proxy_async_smem();
          mbar_arrive(bar_lr_full);
        }
      }
      const int n_base = nb * KG_BN + cs * 64;
      const int gm = mb * KG_BM + row;
      // fc1's output values (bias, GELU, bf16), as fc2's activation kernel would read them
      float* f = reinterpret_cast<float*>(v);
      if (c.store_y) store_rows64_coalesced(p, mb * KG_BM + q * 32, n_base, f, lane);
      uint32_t w[32];  // x2 = bf16(fp32(y1) * inv_lambda2), packed pairs
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        float y[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) y[t] = f[8 * c8 + t];
        scale_bias_pairs(p, n_base + 8 * c8, y);
        if (p.gelu) gelu_tanh_pairs<4>(y);
        const float4 i0 = __ldg(reinterpret_cast<const float4*>(c.inv_lam2 + n_base + 8 * c8));
        const float4 i1 = __ldg(reinterpret_cast<const float4*>(c.inv_lam2 + n_base + 8 * c8 + 4));
        const float il[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const uint32_t y1 = pack_bf16x2(y[2 * t], y[2 * t + 1]);  // fc1's bf16 output
          const uint64_t x2 = f2_mul(f2_pack(bf16lo(y1), bf16hi(y1)), f2_pack(il[2 * t], il[2 * t + 1]));
          w[4 * c8 + t] = pack_bf16x2(f2_lo(x2), f2_hi(x2));
        }
      }
      // fc2's NVFP4 group quantisation of the 64 values (4 groups of 16),
      // the activation kernel's arithmetic
      uint32_t packed[8];
      uint32_t sc = 0;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float a = bf16_amax<8>(w + 8 * g);
        const uint32_t code = e4m3_rn(div_by_scale(a, 6.0f, kRcp6));
        const float2 sy = e4lut[code];
        sc |= code << (8 * g);
        if (sy.x > 0.0f) {
          const uint64_t y2 = f2_pack(sy.y, sy.y), ns2 = f2_pack(-sy.x, -sy.x);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float qv[8];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const uint32_t ww = w[8 * g + 4 * h + t];
              const uint64_t x2 = f2_pack(bf16lo(ww), bf16hi(ww));
              const uint64_t q0 = f2_mul(x2, y2);
              const uint64_t q1 = f2_fma(f2_fma(q0, ns2, x2), y2, q0);
              qv[2 * t] = __uint_as_float(__float_as_uint(f2_lo(q1)) | ((ww << 16) & 0x80000000u));
              qv[2 * t + 1] = __uint_as_float(__float_as_uint(f2_hi(q1)) | (ww & 0x80000000u));
            }
            packed[2 * g + h] = e2m1x8(qv);
          }
        } else {
          packed[2 * g] = 0u;
          packed[2 * g + 1] = 0u;
        }
      }
      if (gm < p.M) {
        const int n2 = p.N;  // fc2's K
        uint4* cp = reinterpret_cast<uint4*>(c.codes2 + static_cast<size_t>(gm) * (n2 / 2) + n_base / 2);
        cp[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        cp[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        uint8_t* sp = c.scales2 + (static_cast<size_t>(mb) * (n2 / 64) + n_base / 64) * 512 + (row & 31) * 16 +
                      (row >> 5) * 4;
        *reinterpret_cast<uint32_t*>(sp) = sc;
      }
      // T2 += X2' . L1_2 over this tile's 256 columns: the slices take turns
      // in the shared buffer (turn t is slice t of this tile).  Slice t's
      // barrier completes once per tile: for t > 0 this tile's phase j, for
      // t = 0 the previous tile's (phase j - 1; at j = 0 the preceding phase
      // of a fresh barrier counts as complete).
      for (int t = 0; t < 4; ++t, ++turn) {
        if (cs == t) {
          const uint32_t par = t == 0 ? ((j & 1) ^ 1) : (j & 1);
          ok = __all_sync(0xffffffffu, wait_bounded(bar_x2_free + 8 * t, par, guard, 0x25d));
          if (ok) {
#pragma unroll
            for (int j8 = 0; j8 < 8; ++j8)
              *reinterpret_cast<uint4*>(x2s + swz_off(row, j8, 128)) =
                  make_uint4(w[4 * j8], w[4 * j8 + 1], w[4 * j8 + 2], w[4 * j8 + 3]);
            fence_proxy_async_smem();
            mbar_arrive(bar_x2_full);
          }
        }
        if (issuer && ok) {
          ok = (t != 0 || wait_bounded(bar_l1_full, j & 1, guard, 0x25e)) &&
               (t != 0 || !fresh || seg == 0 || wait_bounded(bar_t2_drained, (seg - 1) & 1, guard, 0x25f)) &&
               wait_bounded(bar_x2_full, turn & 1, guard, 0x260);
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(t2col, dX2 + 2 * kk, dL1 + (t * R2 * 128 >> 4) + 2 * kk, id_t2,
                       (fresh && kk == 0) ? 0u : 1u);
            fresh = false;
            tc_commit(bar_x2_free + 8 * ((t + 1) & 3));
          }
        }
        __syncwarp();
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      if (!ok) break;
      fresh = __shfl_sync(0xffffffffu, fresh, 0);  // the issuer's view (lane 0 of warp 4)
      if (issuer && tile + 1 < t_end) {
        // L1_2 rows of the next tile, once this tile's T2 MMAs have read them
        // (slice 3's commit is slice 0's barrier, phase j)
        ok = wait_bounded(bar_x2_free, j & 1, guard, 0x261);
        if (ok) {
          mbar_expect_tx(bar_l1_full, C::L1_BYTES);
          const int nb1 = (tile + 1) % p.num_n;
          for (int i = 0; i < 4; ++i)
            tma_load_2d(l1base + i * R2 * 128, &tm_l1t2, bar_l1_full, nb1 * KG_BN + 64 * i, 0);
        }
      }
      __syncwarp();
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      if (seg_end) {
        // the row block's T2 accumulation is complete: drain and add into T2
        if (cs == 0) {
          if (!(ok = __all_sync(0xffffffffu, wait_bounded(bar_x2_free, j & 1, guard, 0x262)))) break;
          tc_fence_after();
          uint32_t tv[R2];
          if constexpr (R2 == 16) tmem_ld_x16(t2col + (static_cast<uint32_t>(q * 32) << 16), tv);
          else tmem_ld_x32(t2col + (static_cast<uint32_t>(q * 32) << 16), tv);
          tmem_ld_wait();
          tc_fence_before();
          if (gm < p.M) {
            float4* dst = reinterpret_cast<float4*>(c.t2 + static_cast<size_t>(gm) * R2);
#pragma unroll
            for (int i = 0; i < R2 / 4; ++i)
              atomicAdd(dst + i, make_float4(__uint_as_float(tv[4 * i]), __uint_as_float(tv[4 * i + 1]),
                                             __uint_as_float(tv[4 * i + 2]), __uint_as_float(tv[4 * i + 3])));
          }
          mbar_arrive(bar_t2_drained);
        }
        ++seg;
        fresh = true;
      }
    }
    // every T2 MMA this CTA issued has completed before tensor memory is freed
    if (issuer) {
      tc_commit(bar_t2_final);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(bar_t2_final, 0) && global_timer_ns() - t0 < p.timeout_ns) {
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
