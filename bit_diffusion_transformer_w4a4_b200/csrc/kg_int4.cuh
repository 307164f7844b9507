// Kernel 2, INT4 variant: the 4-bit GEMM on the packed residual with bf16
// group scales (group 64 along K),
//   acc[m,n] = sum_g s_x[m,g] s_w[n,g] P_g[m,n],  P_g = sum_{k in g} q_x q_w,
// with P_g exact on the int8 tensor cores (tcgen05 kind::i8, s32 accumulate)
// and the scale product applied per group in fp32 by the epilogue warps.
// The low-rank up projection runs as bf16 MMAs into one more accumulator
// buffer that the epilogue adds with weight 1.
//
// Method: "Nunchaku 1.3.0 for Python3.14.x & alpha" (note.com), section
// "SVDQ-FP4 on Blackwell", part "1. INT4" (INT4 -8..+7, W ~ int4 * scale);
// "Nunchaku Lite ... integrated into Diffusers" (axbrief.com), section "The
// Mechanics of 4-Bit Efficiency and SVDQuant" (W4A4 residual + 16-bit
// low-rank branch).
//
// Tile 128 x 128: tensor memory holds four 128-column s32 accumulators, so
// the MMAs run up to three groups ahead of the epilogue's rescale, and each
// epilogue thread keeps 32 fp32 sums (one 32-column tensor-memory load and
// paired fp32 arithmetic per group).  The rescale -- a convert, a multiply
// and an add per output and group, M N K/64 of them -- is the bound of this
// variant; the int8 MMAs take a fraction of it.
//
// Warp roles (640 threads):
//   warp 0      TMA producer: packed activation codes (32B swizzle) and int8
//               weight codes (64B swizzle) for one 64-group per stage
//   warp 1      MMA issuer (two k-steps of 32 per group), tensor-memory owner
//   warps 2-3   unpack activation nibbles to int8 (16 x the code) in the MMA
//               operand layout
//   warps 4-19  epilogue: per-group rescale into fp32 registers, low-rank
//               add, next tile's low-rank operand, bias + GELU + bf16 stores
#pragma once

#include "kg_common.cuh"

namespace svdq {

constexpr int KGI4_BN = 128;   // tile columns (output features)
constexpr int KGI4_BUFS = 4;   // s32 accumulators of 128 columns in tensor memory

constexpr int KGI4_GC = 16;    // groups per staged chunk of scales

template <int R>
struct KGI4Smem {
  static constexpr int STAGES = R >= 128 ? 6 : (R >= 64 ? 8 : 9);
  static constexpr int APK_BYTES = KG_BM * 32;    // 128 rows x 32 B packed (64 codes)
  static constexpr int A8_BYTES = KG_BM * 64;     // 128 rows x 64 int8
  static constexpr int B_BYTES = KGI4_BN * 64;    // 128 rows x 64 int8
  static constexpr int STAGE = APK_BYTES + A8_BYTES + B_BYTES;
  static constexpr int LR_CHUNKS = R > 0 ? (2 * R + 63) / 64 : 0;
  static constexpr int ALR_OFF = STAGES * STAGE;
  // scale chunks, two buffers: the tile's weight scales [GC][128] fp32 and
  // activation scales [128 rows][GC] bf16 at a 36-byte row pitch (9 words:
  // the 32 rows a warp reads fall in 32 distinct banks)
  static constexpr int SW_BYTES = KGI4_GC * KGI4_BN * 4;
  static constexpr int SX_PITCH = KGI4_GC * 2 + 4;
  static constexpr int SC_BUF = SW_BYTES + KG_BM * SX_PITCH;
  static constexpr int SC_OFF = ALR_OFF + LR_CHUNKS * 16384;
  static constexpr int BAR_OFF = SC_OFF + 2 * SC_BUF;
  static constexpr int TOTAL = BAR_OFF + 512 + 1024;
  static_assert(STAGE % 1024 == 0, "stages keep the swizzle alignment");
  static_assert(TOTAL <= 232448, "shared memory per CTA");
};

// 8 two's-complement nibbles (element 0 in the low nibble) -> 8 int8 bytes
// holding 16 x each value: the nibble moves to the byte's high half, so its
// sign bit is the byte's and no sign extension is needed.  The group products
// come out as 16 P; the weight-scale table holds s_w / 16 (exact: a power of
// two), so the rescale below is unchanged.
__device__ __forceinline__ uint2 unpack_s4x8_x16(uint32_t w) {
  const uint32_t lo = (w << 4) & 0xF0F0F0F0u;  // elements 0, 2, 4, 6
  const uint32_t hi = w & 0xF0F0F0F0u;         // elements 1, 3, 5, 7
  uint2 r;
  r.x = __byte_perm(lo, hi, 0x5140);
  r.y = __byte_perm(lo, hi, 0x7362);
  return r;
}

template <int R>
__global__ void __launch_bounds__(KG_THREADS, 1)
    kg_int4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_blr, KGParams p) {
  using S = KGI4Smem<R>;
  constexpr int NST = S::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR_OFF);
  const uint32_t bar_full = smem_u32(bars);
  const uint32_t bar_ready = smem_u32(bars + NST);
  const uint32_t bar_empty = smem_u32(bars + 2 * NST);
  const uint32_t bar_gfull = smem_u32(bars + 3 * NST);                  // [KGI4_BUFS]
  const uint32_t bar_gempty = smem_u32(bars + 3 * NST + KGI4_BUFS);     // [KGI4_BUFS]
  const uint32_t bar_lr_full = smem_u32(bars + 3 * NST + 2 * KGI4_BUFS);
  const uint32_t bar_drain = smem_u32(bars + 3 * NST + 2 * KGI4_BUFS + 1);
  const uint32_t bar_sc_full = smem_u32(bars + 3 * NST + 2 * KGI4_BUFS + 2);  // [2]
  const uint32_t bar_sc_free = smem_u32(bars + 3 * NST + 2 * KGI4_BUFS + 4);  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * NST + 2 * KGI4_BUFS + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Guard guard{p.err, abort_flag, p.timeout_ns};
  const int num_tiles = p.num_m * p.num_n;
  const int ng = p.K / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_ready + 8 * s, 64);   // the 64 transform threads
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < KGI4_BUFS; ++b) {
      mbar_init(bar_gfull + 8 * b, 1);
      mbar_init(bar_gempty + 8 * b, KG_EPI_WARPS);
    }
    mbar_init(bar_lr_full, KG_EPI_WARPS * 32);
    mbar_init(bar_drain, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_sc_full + 8 * b, KG_EPI_WARPS * 32);  // one cp.async arrival per epilogue thread
      mbar_init(bar_sc_free + 8 * b, KG_EPI_WARPS);
    }
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
          if (!(ok = wait_bounded(bar_empty + 8 * s, ph ^ 1, guard, 0x301))) break;
          issued &= ~(1u << s);
          if (!((p.debug_mask & 1u) && j == 0 && g == 1)) {  // test hook: leave one stage empty
            const uint32_t st = sbase + s * S::STAGE;
            const uint32_t fb = bar_full + 8 * s;
            mbar_expect_tx(fb, S::APK_BYTES + S::B_BYTES);
            tma_load_2d(st, &tm_a, fb, g * 32, mb * KG_BM);
            tma_load_2d(st + S::APK_BYTES + S::A8_BYTES, &tm_b, fb, g * 64, nb * KGI4_BN);
            issued |= 1u << s;
            issued_par = (issued_par & ~(1u << s)) | (ph << s);
          }
          if (++s == NST) { s = 0; ph ^= 1; }
        }
        for (int l = 0; l < R / 16 && ok; ++l) {
          if (!(ok = wait_bounded(bar_empty + 8 * s, ph ^ 1, guard, 0x302))) break;
          issued &= ~(1u << s);
          const uint32_t fb = bar_full + 8 * s;
          mbar_expect_tx(fb, KGI4_BN * 64);
          tma_load_2d(sbase + s * S::STAGE + S::APK_BYTES + S::A8_BYTES, &tm_blr, fb, l * 32,
                      nb * KGI4_BN);
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
      constexpr uint32_t id_s8 = idesc_s8_s32(KG_BM, KGI4_BN);
      constexpr uint32_t id_bf = idesc_bf16_f32(KG_BM, KGI4_BN);
      const uint32_t alr = sbase + S::ALR_OFF;
      int s = 0;
      uint32_t ph = 0, gc = 0;
      bool ok = true;
      for (int tile = blockIdx.x, j = 0; tile < num_tiles && ok; tile += gridDim.x, ++j) {
        for (int g = 0; g < ng; ++g, ++gc) {
          const uint32_t b = gc % KGI4_BUFS, use = gc / KGI4_BUFS;
          if (!(ok = wait_bounded(bar_gempty + 8 * b, (use & 1) ^ 1, guard, 0x303))) break;
          if (!(ok = wait_bounded(bar_ready + 8 * s, ph, guard, 0x304))) break;
          if (!(ok = wait_bounded(bar_full + 8 * s, ph, guard, 0x305))) break;
          tc_fence_after();
          const uint32_t st = sbase + s * S::STAGE;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint64_t a = smem_desc(st + S::APK_BYTES + kk * 32, 16, 512, SWZ_64B);
            const uint64_t bd = smem_desc(st + S::APK_BYTES + S::A8_BYTES + kk * 32, 16, 512, SWZ_64B);
            mma_s8(tmem + b * KGI4_BN, a, bd, id_s8, kk);
          }
          tc_commit(bar_empty + 8 * s);
          tc_commit(bar_gfull + 8 * b);
          if (++s == NST) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        if (R > 0) {
          const uint32_t b = gc % KGI4_BUFS, use = gc / KGI4_BUFS;
          if (!(ok = wait_bounded(bar_gempty + 8 * b, (use & 1) ^ 1, guard, 0x306))) break;
          if (!(ok = wait_bounded(bar_lr_full, j & 1, guard, 0x307))) break;
          tc_fence_after();
          for (int l = 0; l < R / 16; ++l) {
            if (!(ok = wait_bounded(bar_full + 8 * s, ph, guard, 0x308))) break;
            if (!(ok = wait_bounded(bar_ready + 8 * s, ph, guard, 0x30d))) break;
            tc_fence_after();
            const uint32_t bst = sbase + s * S::STAGE + S::APK_BYTES + S::A8_BYTES;
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
              const int kk = 2 * l + k2;
              const uint64_t a = smem_desc(alr + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024, SWZ_128B);
              const uint64_t bd = smem_desc(bst + k2 * 32, 16, 512, SWZ_64B);
              mma_bf16(tmem + b * KGI4_BN, a, bd, id_bf, kk != 0);
            }
            tc_commit(bar_empty + 8 * s);
            if (++s == NST) { s = 0; ph ^= 1; }
          }
          if (!ok) break;
          tc_commit(bar_gfull + 8 * b);
          ++gc;
        }
      }
      tc_commit(bar_drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(bar_drain, 0) && global_timer_ns() - t0 < p.timeout_ns) {
      }
    }
  } else if (warp < 4) {
    // --------------------------------------------- nibble -> int8 transform
    const int tt = threadIdx.x - 64;  // 0..63: rows tt and tt + 64
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int g = 0; g < ng; ++g) {
        if (!(ok = wait_bounded(bar_full + 8 * s, ph, guard, 0x309))) break;
        const uint8_t* apk = smem + s * S::STAGE;
        uint8_t* a8 = smem + s * S::STAGE + S::APK_BYTES;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = tt + 64 * h;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(apk + swz_off(row, c, 32));
            const uint2 o0 = unpack_s4x8_x16(v.x), o1 = unpack_s4x8_x16(v.y);
            const uint2 o2 = unpack_s4x8_x16(v.z), o3 = unpack_s4x8_x16(v.w);
            *reinterpret_cast<uint4*>(a8 + swz_off(row, 2 * c, 64)) = make_uint4(o0.x, o0.y, o1.x, o1.y);
            *reinterpret_cast<uint4*>(a8 + swz_off(row, 2 * c + 1, 64)) = make_uint4(o2.x, o2.y, o3.x, o3.y);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar_ready + 8 * s);
        if (++s == NST) { s = 0; ph ^= 1; }
      }
      // low-rank stages carry only the B operand; still pass each one through
      // the ready barrier so its phase stays in step with the stage ring
      for (int l = 0; l < R / 16 && ok; ++l) {
        if (!(ok = wait_bounded(bar_full + 8 * s, ph, guard, 0x30c))) break;
        mbar_arrive(bar_ready + 8 * s);
        if (++s == NST) { s = 0; ph ^= 1; }
      }
    }
  } else {
    // ----------------------------------------------------------------- epilogue
    const int e = warp - 4;
    const int q = warp & 3;
    const int cs = e >> 2;
    const int row = q * 32 + lane;
    const int etid = threadIdx.x - 128;
    uint8_t* alr = smem + S::ALR_OFF;
    const __nv_bfloat16* sx_all = reinterpret_cast<const __nv_bfloat16*>(p.sfa);
    const float* sw_all = reinterpret_cast<const float*>(p.sfb);
    const int npad = (p.N + 255) / 256 * 256;  // row stride of the weight-scale table
    const int nchunk = (ng + KGI4_GC - 1) / KGI4_GC;
    // Scales of a tile come in chunks of GC groups, staged by all epilogue
    // threads with cp.async one chunk ahead of their use: chunk u goes to
    // buffer u & 1 once the 16 warps have released that buffer's previous
    // chunk (u - 2), and its barrier completes when every thread's copies
    // have landed.  Zero fill past M and past the last group.
    auto stage = [&](int tile, int c, uint32_t u) -> bool {
      const uint32_t b = u & 1, k = u >> 1;
      if (!__all_sync(0xffffffffu, wait_bounded(bar_sc_free + 8 * b, (k & 1) ^ 1, guard, 0x30e))) return false;
      const uint32_t buf = sbase + S::SC_OFF + b * S::SC_BUF;
      const int mb = tile % p.num_m, nb = tile / p.num_m;
      const int g0 = c * KGI4_GC;
      {  // weight scales: GC rows of 512 contiguous bytes, one 16-byte piece per thread
        const int gi = etid >> 5, c4 = etid & 31;
        const bool in = g0 + gi < ng;
        const float* src = sw_all + static_cast<size_t>(in ? g0 + gi : 0) * npad + nb * KGI4_BN + 4 * c4;
        cp_async_16(buf + gi * (KGI4_BN * 4) + 16 * c4, src, in ? 16u : 0u);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // activation scales: 128 rows x GC/2 words, two per thread
        const int it = etid + 512 * h;
        const int r = it >> 3, w = it & 7;
        const int gm = mb * KG_BM + r;
        const bool in = gm < p.M && g0 + 2 * w < ng;  // ng is even: a word is both groups or neither
        const __nv_bfloat16* src = sx_all + (in ? static_cast<size_t>(gm) * ng + g0 + 2 * w : 0);
        cp_async_4(buf + S::SW_BYTES + r * S::SX_PITCH + 4 * w, src, in ? 4u : 0u);
      }
      cp_async_mbar_arrive(bar_sc_full + 8 * b);
      return true;
    };
    if constexpr (R > 0) {
      if (static_cast<int>(blockIdx.x) < num_tiles) {
        prep_lowrank_a<R>(alr, p.t, (blockIdx.x % p.num_m) * KG_BM, p.M, etid);
        fence_proxy_async_smem();
        mbar_arrive(bar_lr_full);
      }
    }
    uint32_t gc = 0;
    uint32_t u = 0;  // scale chunks consumed so far
    bool ok = static_cast<int>(blockIdx.x) >= num_tiles || stage(blockIdx.x, 0, 0);
    for (int tile = blockIdx.x, j = 0; tile < num_tiles && ok; tile += gridDim.x, ++j) {
      const int mb = tile % p.num_m, nb = tile / p.num_m;
      const int n_base = nb * KGI4_BN + cs * 32;
      uint64_t acc[16];  // 32 fp32 sums, in pairs
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = 0ull;
      const uint32_t tq = tmem + (static_cast<uint32_t>(q * 32) << 16) + cs * 32;
      // float(P) for the s32 group product P (16 x a sum of 64 products of
      // 4-bit codes, |P| <= 65536 < 2^24): the hardware conversion, exact.
      // (The magic-number form, bits(P + bits(1.5 * 2^23)) - 1.5 * 2^23 in an
      // integer add and a paired fp32 add, measured 612 against 547 us for
      // qkv's kernel 2.)
      const uint8_t* scb = nullptr;
      for (int g = 0; g < ng; ++g, ++gc) {
        const int gi = g % KGI4_GC;
        if (gi == 0) {
          // the next chunk (this tile's, or the next tile's first) into the other buffer
          const int c = g / KGI4_GC;
          if (c + 1 < nchunk) ok = stage(tile, c + 1, u + 1);
          else if (tile + static_cast<int>(gridDim.x) < num_tiles) ok = stage(tile + gridDim.x, 0, u + 1);
          if (!ok) break;
          if (!(ok = __all_sync(0xffffffffu, wait_bounded(bar_sc_full + 8 * (u & 1), (u >> 1) & 1, guard, 0x30f))))
            break;
          scb = smem + S::SC_OFF + (u & 1) * S::SC_BUF;
        }
        const uint32_t b = gc % KGI4_BUFS, use = gc / KGI4_BUFS;
        const float sx = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(scb + S::SW_BYTES + row * S::SX_PITCH + 2 * gi));
        const uint64_t sx2 = f2_pack(sx, sx);
        const float4* swr = reinterpret_cast<const float4*>(scb + gi * (KGI4_BN * 4) + cs * 128);
        if (!(ok = __all_sync(0xffffffffu, wait_bounded(bar_gfull + 8 * b, use & 1, guard, 0x30a)))) break;
        tc_fence_after();
        uint32_t v[32];
        tmem_ld_x32(tq + b * KGI4_BN, v);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_gempty + 8 * b);
        // acc += (s_x * s_w[n]) * P[n], two columns per instruction
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 w = swr[i4];
          const uint64_t s01 = f2_mul(sx2, f2_pack(w.x, w.y));
          const uint64_t s23 = f2_mul(sx2, f2_pack(w.z, w.w));
          const uint64_t p01 = f2_pack(__int2float_rn(static_cast<int>(v[4 * i4])),
                                       __int2float_rn(static_cast<int>(v[4 * i4 + 1])));
          const uint64_t p23 = f2_pack(__int2float_rn(static_cast<int>(v[4 * i4 + 2])),
                                       __int2float_rn(static_cast<int>(v[4 * i4 + 3])));
          acc[2 * i4] = f2_fma(p01, s01, acc[2 * i4]);
          acc[2 * i4 + 1] = f2_fma(p23, s23, acc[2 * i4 + 1]);
        }
        if (gi == KGI4_GC - 1 || g == ng - 1) {
          // this warp is done with the chunk's buffer
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_sc_free + 8 * (u & 1));
          ++u;
        }
      }
      if (!ok) break;
      if constexpr (R > 0) {
        const uint32_t b = gc % KGI4_BUFS, use = gc / KGI4_BUFS;
        if (!(ok = __all_sync(0xffffffffu, wait_bounded(bar_gfull + 8 * b, use & 1, guard, 0x30b)))) break;
        tc_fence_after();
        uint32_t v[32];
        tmem_ld_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + b * KGI4_BN + cs * 32, v);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_gempty + 8 * b);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          acc[i] = f2_pack(__fadd_rn(f2_lo(acc[i]), __uint_as_float(v[2 * i])),
                           __fadd_rn(f2_hi(acc[i]), __uint_as_float(v[2 * i + 1])));
        ++gc;
        const int next = tile + gridDim.x;
        if (next < num_tiles) {
          // the low-rank MMAs of this tile have completed: reuse the operand buffer
          prep_lowrank_a<R>(alr, p.t, (next % p.num_m) * KG_BM, p.M, etid);
          fence_proxy_async_smem();
          mbar_arrive(bar_lr_full);
        }
      }
      float out[32];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        out[2 * i] = f2_lo(acc[i]);
        out[2 * i + 1] = f2_hi(acc[i]);
      }
      store_rows32_coalesced(p, mb * KG_BM + q * 32, n_base, out, lane);
    }
    cp_async_wait_all();  // no copy into this CTA's shared memory outlives it
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace svdq
