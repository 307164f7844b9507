// Kernel 2, NVFP4 variant: the 4-bit GEMM on the packed residual,
//   acc[m,n] = sum_g s_x[m,g] s_w[n,g] sum_{k in g} q_x[m,k] q_w[n,k]
// on tcgen05 block-scaled MMA (kind::mxf4nvf4, E2M1 operands, one UE4M3 scale
// per 16 elements), followed in the same tile by the low-rank up projection
// (bf16 MMA into the same fp32 tensor-memory accumulator) and an epilogue
// that adds the bias, applies GELU and stores bf16.
//
// Method: "Nunchaku Lite ... integrated into Diffusers" (axbrief.com),
// section "The Mechanics of 4-Bit Efficiency and SVDQuant" (4-bit residual
// branch with 4-bit activations, W4A4) and section "Hardware Specialization
// and the Compression Workflow" (NVFP4 on Blackwell); "Problemas do Nunchaku
// Qwen..." (apatero.com), section "O que e Nunchaku..." (up projection fused
// into the 4-bit kernel).
//
// Persistent CTAs, one per SM, tile 128 x 256.  A pipeline stage holds KB
// k-blocks of 64 elements: KB = 4 (128-byte rows, 128B swizzle) when shared
// memory allows, KB = 2 (64-byte rows, 64B swizzle) for rank 128, whose
// low-rank operand is larger.  Warp roles (640 threads):
//   warp 0      TMA producer: A/B code tiles (tensor maps) and the matching
//               scale-factor atoms (bulk copies)
//   warp 1      MMA issuer: block-scaled MMAs, then the low-rank bf16 MMAs;
//               owns tensor memory
//   warps 2, 3  scale-factor copies shared -> tensor memory (A's and B's),
//               each stage ahead of the MMAs that read it.  Issued by other
//               threads than the MMAs, the copies overlap the MMA stream
//               instead of queueing in front of it (measured on fc1: 152 ->
//               127 us for this kernel).
//   warps 4-19  epilogue: drain the accumulator, prepare the next tile's
//               low-rank operand, bias + GELU + bf16 stores
#pragma once

#include "kg_common.cuh"

namespace svdq {

template <int R>
struct KGF4Smem {
  static constexpr int KB = R >= 128 ? 2 : 4;           // 64-element k-blocks per stage
  static constexpr int ROWB = 32 * KB;                  // bytes per operand row per stage
  static constexpr uint32_t SWZ = KB == 4 ? SWZ_128B : SWZ_64B;
  static constexpr uint32_t SBO = 8 * ROWB;             // 8-row core-matrix group stride
  static constexpr int STAGES = KB == 4 ? 3 : 5;
  static constexpr int A_BYTES = KG_BM * ROWB;
  static constexpr int B_BYTES = KG_BN * ROWB;
  static constexpr int SFA_BYTES = KB * 512;            // one 128-row atom per k-block
  static constexpr int SFB_BYTES = 2 * KB * 512;        // two atoms (256 rows) per k-block
  static constexpr int STAGE = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int LR_CHUNKS = R > 0 ? (2 * R + 63) / 64 : 0;
  static constexpr int LR_STEPS = R / 8;                // bf16 k-steps of 16 over [T_hi | T_lo]
  static constexpr int LR_STAGES = (LR_STEPS + KB - 1) / KB;  // a stage row holds KB k-steps
  static constexpr int ALR_OFF = STAGES * STAGE;
  static constexpr int BAR_OFF = ALR_OFF + LR_CHUNKS * 16384;
  static constexpr int RED_OFF = BAR_OFF + 256;      // QKV epilogue: [4][4][32] partial sums
  static constexpr int XBAR_OFF = RED_OFF + 2048;    // QKV epilogue: 8 exchange mbarriers
  static constexpr int TOTAL = XBAR_OFF + 64 + 1024;
  // tensor memory columns: accumulator [0, 256), then scale factors
  static constexpr int SFA_COL = 256;
  static constexpr int SFB_COL = 256 + 4 * KB * STAGES;
  static_assert(SFB_COL + 8 * KB * STAGES <= 512, "tensor memory columns");
};

template <int R>
__global__ void __launch_bounds__(KG_THREADS, 1)
    kg_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_blr, KGParams p) {
  using S = KGF4Smem<R>;
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
  // per stage: the scale factors of the first / second half of the stage's
  // k-blocks are in tensor memory (and the stage's data has landed); per
  // copy warp: its copies have drained
  const uint32_t bar_sfa = smem_u32(bars + 2 * NST + 5);
  const uint32_t bar_sfb = smem_u32(bars + 3 * NST + 5);
  const uint32_t bar_sf_drain = smem_u32(bars + 4 * NST + 5);  // two barriers

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Guard guard{p.err, abort_flag, p.timeout_ns};
  const int num_tiles = p.num_m * p.num_n;
  const int kblk = p.K / 64;                // 64-element k-blocks (scale atoms) along K
  const int nks = (kblk + KB - 1) / KB;     // pipeline stages per tile; the last may be partial

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
    for (int i = 0; i < 8; ++i) mbar_init(smem_u32(smem + S::XBAR_OFF) + 8 * i, 64);
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
        for (int ks = 0; ks < nks; ++ks) {
          if (!(ok = wait_bounded(bar_empty + 8 * s, ph ^ 1, guard, 0x201))) break;
          issued &= ~(1u << s);
          if (!((p.debug_mask & 1u) && j == 0 && ks == 1)) {  // test hook: leave one stage empty
            const uint32_t st = sbase + s * S::STAGE;
            const uint32_t fb = bar_full + 8 * s;
            // k-blocks present in this stage; code columns past K are zero-filled
            const uint32_t kv = min(KB, kblk - KB * ks);
            mbar_expect_tx(fb, S::A_BYTES + S::B_BYTES + 3 * kv * 512);
            tma_load_2d(st, &tm_a, fb, ks * S::ROWB, mb * KG_BM);
            tma_load_2d(st + S::A_BYTES, &tm_b, fb, ks * S::ROWB, nb * KG_BN);
            bulk_load(st + S::A_BYTES + S::B_BYTES,
                      p.sfa + (static_cast<size_t>(mb) * kblk + KB * ks) * 512, kv * 512, fb);
            const uint8_t* sfb0 = p.sfb + (static_cast<size_t>(2 * nb) * kblk + KB * ks) * 512;
            bulk_load(st + S::A_BYTES + S::B_BYTES + S::SFA_BYTES, sfb0, kv * 512, fb);
            bulk_load(st + S::A_BYTES + S::B_BYTES + S::SFA_BYTES + KB * 512,
                      sfb0 + static_cast<size_t>(kblk) * 512, kv * 512, fb);
            issued |= 1u << s;
            issued_par = (issued_par & ~(1u << s)) | (ph << s);
          }
          if (++s == NST) { s = 0; ph ^= 1; }
        }
        for (int l = 0; l < S::LR_STAGES && ok; ++l) {
          if (!(ok = wait_bounded(bar_empty + 8 * s, ph ^ 1, guard, 0x202))) break;
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
      // Descriptors are built once; a start address moves in 16-byte units in
      // the low bits, so per-stage / per-k-block offsets are plain additions.
      const uint64_t dA0 = smem_desc(sbase, 16, S::SBO, S::SWZ);
      const uint64_t dB0 = smem_desc(sbase + S::A_BYTES, 16, S::SBO, S::SWZ);
      const uint64_t dLRA0 = smem_desc(sbase + S::ALR_OFF, 16, 1024, SWZ_128B);
      constexpr uint64_t kStage = S::STAGE >> 4;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = blockIdx.x, j = 0; tile < num_tiles && ok; tile += gridDim.x, ++j) {
        if (j > 0 && !(ok = wait_bounded(bar_acc_empty, (j - 1) & 1, guard, 0x203))) break;
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
                                      kb == 0 ? 0x204 : 0x20a)))
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
          if (!(ok = wait_bounded(bar_lr_full, j & 1, guard, 0x205))) break;
          tc_fence_after();
          for (int l = 0; l < S::LR_STAGES; ++l) {
            if (!(ok = wait_bounded(bar_sfa + 8 * s, ph, guard, 0x206) &&
                       wait_bounded(bar_sfb + 8 * s, ph, guard, 0x20b)))
              break;
            tc_fence_after();
            const uint64_t so = kStage * s;
#pragma unroll
            for (int k2 = 0; k2 < KB; ++k2) {
              const int kk = KB * l + k2;  // k-step over [T_hi | T_lo]
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
      // drain: every MMA issued so far has completed before tensor memory is freed
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
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        for (int ks = 0; ks < nks; ++ks) {
          if (!(ok = wait_bounded(bar_full + 8 * s, ph, guard, h == 0 ? 0x208 : 0x209))) break;
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
          if (!(ok = wait_bounded(bar_full + 8 * s, ph, guard, 0x20c))) break;
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
  } else if (warp >= 4) {
    // ----------------------------------------------------------------- epilogue
    const int e = warp - 4;
    const int q = warp & 3;        // tensor-memory lane group of this warp
    const int cs = e >> 2;         // 64-column slice
    const int etid = threadIdx.x - 128;
    uint8_t* alr = smem + S::ALR_OFF;
    float* red = reinterpret_cast<float*>(smem + S::RED_OFF);  // QKV epilogue partial sums
    const uint32_t xbar = smem_u32(smem + S::XBAR_OFF);
    uint32_t xph = 0;
    if constexpr (R > 0) {
      if (static_cast<int>(blockIdx.x) < num_tiles) {
        prep_lowrank_a<R>(alr, p.t, (blockIdx.x % p.num_m) * KG_BM, p.M, etid, p.t_scale);
        fence_proxy_async_smem();
        mbar_arrive(bar_lr_full);
      }
    }
    for (int tile = blockIdx.x, j = 0; tile < num_tiles; tile += gridDim.x, ++j) {
      const int mb = tile % p.num_m, nb = tile / p.num_m;
      if (!__all_sync(0xffffffffu, wait_bounded(bar_acc_full, j & 1, guard, 0x207, 128))) break;
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
        const int next = tile + gridDim.x;
        if (next < num_tiles) {
          prep_lowrank_a<R>(alr, p.t, (next % p.num_m) * KG_BM, p.M, etid, p.t_scale);
          fence_proxy_async_smem();
          mbar_arrive(bar_lr_full);
        }
      }
      if (p.qkv_hd > 0) {
        if (!epilogue_qkv64(p, mb * KG_BM + q * 32, nb * KG_BN + cs * 64, reinterpret_cast<const float*>(v),
                            lane, q, cs, red, xbar, xph, guard))
          break;
      } else
        store_rows64_coalesced(p, mb * KG_BM + q * 32, nb * KG_BN + cs * 64,
                               reinterpret_cast<const float*>(v), lane);
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
