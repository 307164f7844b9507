// Kernel 2, NVFP4 variant on CTA pairs: the same product as kg_nvfp4_kernel
// (4-bit block-scaled GEMM on the packed residual, low-rank up projection into
// the same accumulator, bias + GELU + bf16 epilogue), with the tile computed
// by the two SMs of a TPC together.
//
// Method: "Nunchaku Lite ... integrated into Diffusers" (axbrief.com),
// section "The Mechanics of 4-Bit Efficiency and SVDQuant" (W4A4 residual
// branch) and section "Hardware Specialization and the Compression Workflow"
// (NVFP4 on Blackwell); "Problemas do Nunchaku Qwen..." (apatero.com),
// section "O que e Nunchaku..." (up projection fused into the 4-bit kernel).
//
// A cluster of two CTAs owns a 256 x 256 output tile.  CTA rank r loads rows
// [128 r, 128 r + 128) of the tile's A rows and of its B rows (weight rows
// n), its own A scale atoms and all 256 B rows' scale atoms; the leader
// (rank 0) issues one tcgen05 MMA of M = 256 for the pair, whose tensor cores
// read A from their own SM and B from both, and each SM accumulates its 128
// rows x 256 columns in its own tensor memory.  Per SM this halves the B
// bytes staged per output and the MMA instructions issued per output
// compared with the one-SM kernel.
//
// Warp roles (640 threads per CTA):
//   warp 0      TMA producer (both CTAs): transaction bytes of both CTAs are
//               counted on the leader's full barrier
//   warp 1      leader: MMAs for the pair; both CTAs: tensor-memory
//               allocation (cta_group::2, same warp in both)
//   warps 2, 3  leader: scale-factor copies for the pair (first and second
//               half of each stage's k-blocks), a stage ahead of the MMAs,
//               from threads other than the MMA issuer
//   warps 4-19  epilogue (both CTAs): drain this SM's accumulator half,
//               prepare the next tile's low-rank operand rows, store
// Cross-CTA signals: MMA completion is committed to the barrier at the same
// offset in both CTAs (empty stages, accumulator full); the epilogue warps of
// both CTAs arrive on the leader's accumulator-empty and low-rank-ready
// barriers (release / acquire at cluster scope).  Neither CTA exits before a
// final cluster barrier, so no remote arrive or load targets an exited CTA.
#pragma once

#include "kg_common.cuh"

namespace svdq {

template <int R>
struct KGF4PairSmem {
  static constexpr int KB = 4;                          // 64-element k-blocks per stage
  static constexpr int ROWB = 32 * KB;                  // 128-byte operand rows, 128B swizzle
  static constexpr uint32_t SBO = 8 * ROWB;
  static constexpr int STAGES = R >= 128 ? 4 : 5;
  static constexpr int A_BYTES = 128 * ROWB;            // this CTA's 128 A rows
  static constexpr int B_BYTES = 128 * ROWB;            // this CTA's 128 B rows
  static constexpr int SFA_BYTES = KB * 512;            // one 128-row atom per k-block
  static constexpr int SFB_BYTES = 2 * KB * 512;        // both 128-row atoms of the 256 B rows
  static constexpr int STAGE = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr uint32_t TX = 2 * STAGE;             // bytes of both CTAs per stage
  static constexpr uint32_t LR_TX = 2 * B_BYTES;
  static constexpr int LR_CHUNKS = R > 0 ? (2 * R + 63) / 64 : 0;
  static constexpr int LR_STEPS = R / 8;
  static constexpr int LR_STAGES = (LR_STEPS + KB - 1) / KB;
  static constexpr int ALR_OFF = STAGES * STAGE;
  static constexpr int BAR_OFF = ALR_OFF + LR_CHUNKS * 16384;
  static constexpr int RED_OFF = BAR_OFF + 256;      // QKV epilogue: [4][4][32] partial sums
  static constexpr int XBAR_OFF = RED_OFF + 2048;    // QKV epilogue: 8 exchange mbarriers
  static constexpr int TOTAL = XBAR_OFF + 64 + 1024;
  static constexpr int SFA_COL = 256;
  static constexpr int SFB_COL = 256 + 4 * KB * STAGES;
  static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
  static_assert(SFB_COL + 8 * KB * STAGES <= 512, "tensor memory columns");
  static_assert(TOTAL <= 232448, "shared memory per CTA");
};

template <int R>
__global__ void __launch_bounds__(KG_THREADS, 1)
    kg_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                         const __grid_constant__ CUtensorMap tm_blr,
                         const __grid_constant__ CUtensorMap tm_sfa,
                         const __grid_constant__ CUtensorMap tm_sfb, KGParams p) {
  using S = KGF4PairSmem<R>;
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
  const uint32_t bar_sfa = smem_u32(bars + 2 * NST + 5);        // leader: k-blocks 0-1 scales copied
  const uint32_t bar_sfb = smem_u32(bars + 3 * NST + 5);        // leader: k-blocks 2-3 scales copied
  const uint32_t bar_sf_drain = smem_u32(bars + 4 * NST + 5);   // two barriers

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cid = static_cast<int>(blockIdx.x >> 1);
  const int nclu = static_cast<int>(gridDim.x >> 1);
  const Guard guard{p.err, abort_flag, p.timeout_ns};
  const int num_tiles = p.num_m * p.num_n;  // p.num_m counts 256-row blocks
  const int kblk = p.K / 64;
  const int nks = (kblk + KB - 1) / KB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_acc_full, 1);
    mbar_init(bar_acc_empty, 2 * KG_EPI_WARPS);
    mbar_init(bar_lr_full, 2 * KG_EPI_WARPS);
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
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The activation codes, scales and T come from the previous kernel of the
  // stream (see griddep_wait()); the producer first issues the weight halves
  // of the first stages, which do not depend on it.
  if (!(warp == 0 && lane == 0)) griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      tma_prefetch_desc(&tm_sfa);
      tma_prefetch_desc(&tm_sfb);
      if (R > 0) tma_prefetch_desc(&tm_blr);
      const uint32_t full0 = mapa_shared(bar_full, 0);  // the leader's full barriers
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      // Weight half (B codes, B scale atoms) of the first tile's first stages,
      // issued before the dependency wait: the stage's full barrier completes
      // only when its activation half has landed too.
      const int pre = (cid < num_tiles && !(p.debug_mask & 1u)) ? min(NST, nks) : 0;
      if (pre > 0) {
        const int nb = cid / p.num_m;
        const int brow = nb * 256 + static_cast<int>(rank) * 128;
        for (int ks = 0; ks < pre; ++ks) {  // fresh ring: every slot is free
          const uint32_t st = sbase + ks * S::STAGE;
          const uint32_t fb = full0 + 8 * ks;
          if (rank == 0) mbar_expect_tx(bar_full + 8 * ks, S::TX);
          tma_load_2d_pair(st + S::A_BYTES, &tm_b, fb, ks * S::ROWB, brow);
          tma_load_2d_pair(st + S::A_BYTES + S::B_BYTES + S::SFA_BYTES, &tm_sfb, fb, 0,
                           2 * nb * kblk + KB * ks);
          tma_load_2d_pair(st + S::A_BYTES + S::B_BYTES + S::SFA_BYTES + KB * 512, &tm_sfb, fb, 0,
                           (2 * nb + 1) * kblk + KB * ks);
          issued |= 1u << ks;
        }
      }
      griddep_wait();
      for (int tile = cid, j = 0; tile < num_tiles && ok; tile += nclu, ++j) {
        const int mb = tile % p.num_m, nb = tile / p.num_m;
        const int arow = mb * 256 + static_cast<int>(rank) * 128;   // this CTA's A rows
        const int brow = nb * 256 + static_cast<int>(rank) * 128;   // this CTA's B rows
        const int sfa_atom = (2 * mb + static_cast<int>(rank)) * kblk;
        for (int ks = 0; ks < nks; ++ks) {
          const uint32_t st = sbase + s * S::STAGE;
          const uint32_t fb = full0 + 8 * s;
          if (j == 0 && ks < pre) {  // weight half already in flight: the activation half
            tma_load_2d_pair(st, &tm_a, fb, ks * S::ROWB, arow);
            tma_load_2d_pair(st + S::A_BYTES + S::B_BYTES, &tm_sfa, fb, 0, sfa_atom + KB * ks);
            if (++s == NST) { s = 0; ph ^= 1; }
            continue;
          }
          if (!(ok = wait_bounded(bar_empty + 8 * s, ph ^ 1, guard, 0x221))) break;
          issued &= ~(1u << s);
          if (!((p.debug_mask & 1u) && j == 0 && ks == 1)) {  // test hook: leave one stage empty
            if (rank == 0) mbar_expect_tx(bar_full + 8 * s, S::TX);
            // whole boxes always: rows past M, N or the last k-block are zero-filled
            tma_load_2d_pair(st, &tm_a, fb, ks * S::ROWB, arow);
            tma_load_2d_pair(st + S::A_BYTES, &tm_b, fb, ks * S::ROWB, brow);
            tma_load_2d_pair(st + S::A_BYTES + S::B_BYTES, &tm_sfa, fb, 0, sfa_atom + KB * ks);
            tma_load_2d_pair(st + S::A_BYTES + S::B_BYTES + S::SFA_BYTES, &tm_sfb, fb, 0,
                             2 * nb * kblk + KB * ks);
            tma_load_2d_pair(st + S::A_BYTES + S::B_BYTES + S::SFA_BYTES + KB * 512, &tm_sfb, fb, 0,
                             (2 * nb + 1) * kblk + KB * ks);
            issued |= 1u << s;
            issued_par = (issued_par & ~(1u << s)) | (ph << s);
          }
          if (++s == NST) { s = 0; ph ^= 1; }
        }
        for (int l = 0; l < S::LR_STAGES && ok; ++l) {
          if (!(ok = wait_bounded(bar_empty + 8 * s, ph ^ 1, guard, 0x222))) break;
          issued &= ~(1u << s);
          if (rank == 0) mbar_expect_tx(bar_full + 8 * s, S::LR_TX);
          tma_load_2d_pair(sbase + s * S::STAGE + S::A_BYTES, &tm_blr, full0 + 8 * s,
                           l * (S::ROWB / 2), brow);
          issued |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == NST) { s = 0; ph ^= 1; }
        }
      }
      // The leader's full barriers count both CTAs' bytes: waiting on them
      // drains the pair's loads in flight.
      if (*abort_flag && rank == 0) drain_loads(bar_full, issued, issued_par, NST, p.timeout_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issue (leader)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t id_f4 = idesc_nvf4(256, 256);
      constexpr uint32_t id_bf = idesc_bf16_f32(256, 256);
      const uint64_t dA0 = smem_desc(sbase, 16, S::SBO, SWZ_128B);
      const uint64_t dB0 = smem_desc(sbase + S::A_BYTES, 16, S::SBO, SWZ_128B);
      const uint64_t dLRA0 = smem_desc(sbase + S::ALR_OFF, 16, 1024, SWZ_128B);
      constexpr uint64_t kStage = S::STAGE >> 4;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = cid, j = 0; tile < num_tiles && ok; tile += nclu, ++j) {
        if (j > 0 && !(ok = wait_bounded_cl(bar_acc_empty, (j - 1) & 1, guard, 0x223))) break;
        tc_fence_after();
        for (int ks = 0; ks < nks; ++ks) {
          const uint64_t so = kStage * s;
          const int kv = min(KB, kblk - KB * ks);
          const uint32_t ca = tmem + S::SFA_COL + KB * 4 * s;
          const uint32_t cb = tmem + S::SFB_COL + KB * 8 * s;
          // first half of the k-blocks once warp 2's copies are in, the second
          // half once warp 3's are
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            if (kb == 0 || kb == KB / 2) {
              if (!(ok = wait_bounded(kb == 0 ? bar_sfa + 8 * s : bar_sfb + 8 * s, ph, guard,
                                      kb == 0 ? 0x224 : 0x228)))
                break;
              tc_fence_after();
            }
            if (kb < kv)
              mma_nvf4_pair(tmem, dA0 + so + 2 * kb, dB0 + so + 2 * kb, id_f4, ca + 4 * kb, cb + 8 * kb,
                            (ks | kb) != 0);
          }
          if (!ok) break;
          tc_commit_pair(bar_empty + 8 * s, 0x3);
          if (++s == NST) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        if (R > 0) {
          if (!(ok = wait_bounded_cl(bar_lr_full, j & 1, guard, 0x225))) break;
          tc_fence_after();
          for (int l = 0; l < S::LR_STAGES; ++l) {
            if (!(ok = wait_bounded(bar_sfa + 8 * s, ph, guard, 0x226) &&
                       wait_bounded(bar_sfb + 8 * s, ph, guard, 0x229)))
              break;
            tc_fence_after();
            const uint64_t so = kStage * s;
#pragma unroll
            for (int k2 = 0; k2 < KB; ++k2) {
              const int kk = KB * l + k2;
              if (kk < S::LR_STEPS)
                mma_bf16_pair(tmem, dLRA0 + (kk / 4) * 1024 + (kk % 4) * 2, dB0 + so + 2 * k2, id_bf, 1);
            }
            tc_commit_pair(bar_empty + 8 * s, 0x3);
            if (++s == NST) { s = 0; ph ^= 1; }
          }
          if (!ok) break;
        }
        tc_commit_pair(bar_acc_full, 0x3);
      }
      // every MMA of the pair has completed before either CTA frees tensor memory
      tc_commit_pair(bar_drain, 0x1);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(bar_drain, 0) && global_timer_ns() - t0 < p.timeout_ns) {
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------ scale-factor copies (leader)
    // Each copy lands in both CTAs' tensor memory, from each CTA's own stage;
    // every stage completes the leader's ready barrier once, after the
    // pair's data has landed (the leader's full barrier counts both CTAs).
    // Warp 2 copies the scale atoms of the stage's first half of k-blocks
    // (A's and both of B's), warp 3 those of the second half: six copies per
    // warp and stage, which one warp issues in less time than the stage's
    // four MMAs take.
    if (lane == 0 && rank == 0) {
      const int h = warp - 2;
      const uint32_t ready = h == 0 ? bar_sfa : bar_sfb;
      const uint64_t dA = smem_desc(sbase + S::A_BYTES + S::B_BYTES, 0, 128, SWZ_NONE);
      const uint64_t dB = smem_desc(sbase + S::A_BYTES + S::B_BYTES + S::SFA_BYTES, 0, 128, SWZ_NONE);
      constexpr uint64_t kStage = S::STAGE >> 4;
      constexpr int KH = KB / 2;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += nclu) {
        for (int ks = 0; ks < nks; ++ks) {
          if (!(ok = wait_bounded(bar_full + 8 * s, ph, guard, h == 0 ? 0x22a : 0x22b))) break;
          tc_fence_after();
          const int kv = min(KB, kblk - KB * ks);
          const uint32_t ca = tmem + S::SFA_COL + KB * 4 * s;
          const uint32_t cb = tmem + S::SFB_COL + KB * 8 * s;
#pragma unroll
          for (int i = 0; i < KH; ++i) {
            const int kb = h * KH + i;
            if (kb < kv) {
              tmem_cp_32x128b_warpx4_pair(ca + 4 * kb, dA + kStage * s + 32 * kb);
              tmem_cp_32x128b_warpx4_pair(cb + 8 * kb, dB + kStage * s + 32 * kb);
              tmem_cp_32x128b_warpx4_pair(cb + 8 * kb + 4, dB + kStage * s + 32 * (KB + kb));
            }
          }
          tc_commit_pair(ready + 8 * s, 0x1);
          if (++s == NST) { s = 0; ph ^= 1; }
        }
        for (int l = 0; l < S::LR_STAGES && ok; ++l) {
          if (!(ok = wait_bounded(bar_full + 8 * s, ph, guard, 0x22c))) break;
          tc_commit_pair(ready + 8 * s, 0x1);
          if (++s == NST) { s = 0; ph ^= 1; }
        }
      }
      // this warp's copies have completed before tensor memory is freed
      const uint32_t drain = bar_sf_drain + 8 * h;
      tc_commit_pair(drain, 0x1);
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
    const uint32_t acc_empty0 = mapa_shared(bar_acc_empty, 0);
    const uint32_t lr_full0 = mapa_shared(bar_lr_full, 0);
    if constexpr (R > 0) {
      if (cid < num_tiles) {
        prep_lowrank_a<R>(alr, p.t, (cid % p.num_m) * 256 + static_cast<int>(rank) * 128, p.M, etid, p.t_scale);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(lr_full0);
      }
    }
    for (int tile = cid, j = 0; tile < num_tiles; tile += nclu, ++j) {
      const int mb = tile % p.num_m, nb = tile / p.num_m;
      if (!__all_sync(0xffffffffu, wait_bounded(bar_acc_full, j & 1, guard, 0x227, 128))) break;
      tc_fence_after();
      uint32_t v[64];
      const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + cs * 64;
      tmem_ld_x32(ta, v);
      tmem_ld_x32(ta + 32, v + 32);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0);
      if constexpr (R > 0) {
        const int next = tile + nclu;
        if (next < num_tiles) {
          prep_lowrank_a<R>(alr, p.t, (next % p.num_m) * 256 + static_cast<int>(rank) * 128, p.M, etid, p.t_scale);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(lr_full0);
        }
      }
      if (p.qkv_hd > 0) {
        if (!epilogue_qkv64(p, mb * 256 + static_cast<int>(rank) * 128 + q * 32, nb * KG_BN + cs * 64, reinterpret_cast<const float*>(v),
                            lane, q, cs, red, xbar, xph, guard))
          break;
      } else
        store_rows64_coalesced(p, mb * 256 + static_cast<int>(rank) * 128 + q * 32, nb * KG_BN + cs * 64,
                               reinterpret_cast<const float*>(v), lane);
    }
  }

  tc_fence_before();
  cluster_sync();  // the pair's MMAs, loads and remote arrivals are all done
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace svdq
