// AWQ W4A16 linear layer: 4-bit weights with group scales and integer zero
// points, 16-bit activations, y = (x / a) . W_deq^T (+ bias).
//
// Method: "Nunchaku Lite ... integrated into Diffusers" (axbrief.com),
// section "The Mechanics of 4-Bit Efficiency and SVDQuant" (AWQW4A16Linear:
// 4-bit weights, 16-bit activations) and section "The Trade-off Between Fused
// Kernels and Generality" (the scanner gives modulation linear layers AWQ
// W4A16).  Modulation layers take one token per image (M = batch), so the
// layer is a matrix-vector product bound by the HBM stream of the 4-bit
// weights: it runs on the CUDA cores, not the tensor cores.
//
// Per element: x' = fp32(x) *_RN fp32(1/a_k) (fp32, not rounded further);
// for each group g of 64 along K: part = sum_{k in g} x'_k (q_k - z_g) in
// fp32 (q - z is an exact small integer), y += s_g * part.
//
// Layout: codes [N x K/2] bytes (element 2j in the low nibble), group
// parameters [N x K/64] 32-bit words (bf16 scale in the high half, zero
// point in the low byte), 1/a fp32 [K], bias bf16 [N] or null.
//
// Work split: a persistent grid (one or two CTAs per SM) in which each CTA stages
// x' of up to MT tokens once in shared memory (one 32-element chunk per 36
// floats, so the lanes' 16-byte reads of their own chunks hit distinct
// banks), then each warp takes RW weight rows at a time; lane l reads the
// 16-byte code chunks l, l+32, ... of each row (a warp reads 512 contiguous
// bytes per load), CB chunks of every row loaded before any is decoded;
// decoding turns eight codes per word with byte permutes into fp32 2^23 + q,
// subtracts 2^23 + z and accumulates x' (q - z) with packed fp32x2 FMAs; the
// row's partial sums meet in a warp shuffle reduction.
#pragma once

#include "ptx.cuh"

namespace svdq {

constexpr int AWQ_THREADS = 256;
constexpr int AWQ_G = 64;
// Per tokens-per-pass MT: weight rows per warp and item (each x' value read
// from shared memory serves all of them), 16-byte code chunks per lane and
// row per item, and resident CTAs per SM.  Two items' codes are held in
// registers (the next one loads while the current one is decoded), so the
// registers grow with rows x chunks and with the tokens' partial sums.
template <int MT> constexpr int awq_rw() { return MT <= 4 ? 2 : 1; }
template <int MT> constexpr int awq_cb() { return MT <= 2 ? 3 : 2; }
template <int MT> constexpr int awq_ctas() { return MT <= 4 ? 2 : 1; }

// byte `sel` of a, as the fp32 bit pattern 0x4B0000bb (= 2^23 + byte)
template <int SEL>
__device__ __forceinline__ uint32_t byte_as_magic(uint32_t a) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(0x4B000000u), "n"(0x7440 + SEL));
  return d;
}

struct AWQParams {
  const uint8_t* codes;   // [N x K/2]
  const uint32_t* gp;     // [N x K/64]: (bf16 scale << 16) | zero
  const float* inv_a;     // [K]
  const uint16_t* x;      // bf16 [M x K]
  const uint16_t* bias;   // bf16 [N] or null
  uint16_t* y;            // bf16 [M x N]
  int M, K, N;
};

template <int MT>
struct AWQSmem {
  static size_t bytes(int K) { return static_cast<size_t>(MT) * (K / 32) * 36 * 4; }
};

template <int MT>
__global__ void __launch_bounds__(AWQ_THREADS, awq_ctas<MT>())
    kawq_kernel(AWQParams p) {
  constexpr int CB = awq_cb<MT>();
  constexpr int RW = awq_rw<MT>();
  extern __shared__ __align__(16) float xs[];  // [MT][K/32][36]
  const int nck = p.K / 32;                    // 16-byte code chunks per row
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpb = AWQ_THREADS / 32;
  // A warp's work is a list of items: rows n0 .. n0 + RW - 1 (n0 = n_first +
  // i gstride) x chunks cb .. cb + 32 CB - 1 of them (lane l takes chunks
  // cb + l, cb + 32 + l, ...); a row's items are consecutive.
  const int gstride = gridDim.x * wpb * RW;
  const int n_first = (blockIdx.x * wpb + warp) * RW;
  const int ncb = (nck + 32 * CB - 1) / (32 * CB);  // items per row group
  const int nit = n_first < p.N ? (p.N - n_first + gstride - 1) / gstride * ncb : 0;

  uint4 cwa[CB][RW], cwb[CB][RW];
  uint32_t gwa[CB][RW], gwb[CB][RW];
  auto load = [&](uint4 (&cw)[CB][RW], uint32_t (&gw)[CB][RW], int it) {
    const int n0 = n_first + (it / ncb) * gstride;
    const int cb = (it % ncb) * 32 * CB;
#pragma unroll
    for (int c = 0; c < CB; ++c) {
      const int ci = cb + 32 * c + lane;
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        const int n = min(n0 + r, p.N - 1);  // rows past N recompute row N-1, never stored
        if (ci < nck) {
          cw[c][r] = __ldcs(reinterpret_cast<const uint4*>(p.codes + static_cast<size_t>(n) * (p.K / 2)) + ci);
          gw[c][r] = __ldg(p.gp + static_cast<size_t>(n) * (p.K / AWQ_G) + ci / 2);
        } else {
          cw[c][r] = make_uint4(0u, 0u, 0u, 0u);
          gw[c][r] = 0u;                    // scale 0: contributes nothing
        }
      }
    }
  };

  float acc[RW][MT];
  int m0 = 0, mt = 0;
  // decode one item into acc; after a row group's last item, reduce across
  // the warp, store and clear
  auto compute = [&](const uint4 (&cw)[CB][RW], const uint32_t (&gw)[CB][RW], int it) {
    const int cb = (it % ncb) * 32 * CB;
#pragma unroll
    for (int c = 0; c < CB; ++c) {
      const int ci = min(cb + 32 * c + lane, nck - 1);
      const float* xc = xs + ci * 36;
      uint64_t part[RW][MT];
#pragma unroll
      for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) part[r][m] = 0ull;
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
        // x' of these eight positions, once for all the item's rows
        uint64_t xv[MT][4];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const float4 xa = *reinterpret_cast<const float4*>(xc + m * nck * 36 + 8 * wi);
          const float4 xb = *reinterpret_cast<const float4*>(xc + m * nck * 36 + 8 * wi + 4);
          xv[m][0] = f2_pack(xa.x, xa.y);
          xv[m][1] = f2_pack(xa.z, xa.w);
          xv[m][2] = f2_pack(xb.x, xb.y);
          xv[m][3] = f2_pack(xb.z, xb.w);
        }
#pragma unroll
        for (int r = 0; r < RW; ++r) {
          const float nz = -(8388608.0f + static_cast<float>(gw[c][r] & 0xFFu));
          const uint64_t nzz = f2_pack(nz, nz);
          const uint32_t word = wi == 0 ? cw[c][r].x : wi == 1 ? cw[c][r].y : wi == 2 ? cw[c][r].z : cw[c][r].w;
          const uint32_t lo = word & 0x0F0F0F0Fu;         // codes 8wi + 2b
          const uint32_t hi = (word >> 4) & 0x0F0F0F0Fu;  // codes 8wi + 2b + 1
          uint64_t q[4];
          q[0] = f2_add(f2_pack(__uint_as_float(byte_as_magic<0>(lo)), __uint_as_float(byte_as_magic<0>(hi))), nzz);
          q[1] = f2_add(f2_pack(__uint_as_float(byte_as_magic<1>(lo)), __uint_as_float(byte_as_magic<1>(hi))), nzz);
          q[2] = f2_add(f2_pack(__uint_as_float(byte_as_magic<2>(lo)), __uint_as_float(byte_as_magic<2>(hi))), nzz);
          q[3] = f2_add(f2_pack(__uint_as_float(byte_as_magic<3>(lo)), __uint_as_float(byte_as_magic<3>(hi))), nzz);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            part[r][m] = f2_fma(xv[m][0], q[0], part[r][m]);
            part[r][m] = f2_fma(xv[m][1], q[1], part[r][m]);
            part[r][m] = f2_fma(xv[m][2], q[2], part[r][m]);
            part[r][m] = f2_fma(xv[m][3], q[3], part[r][m]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        const float sc = __uint_as_float(gw[c][r] & 0xFFFF0000u);
#pragma unroll
        for (int m = 0; m < MT; ++m)
          acc[r][m] = __fmaf_rn(sc, __fadd_rn(f2_lo(part[r][m]), f2_hi(part[r][m])), acc[r][m]);
      }
    }
    if (it % ncb == ncb - 1) {
      const int n0 = n_first + (it / ncb) * gstride;
#pragma unroll
      for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          float v = acc[r][m];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          acc[r][m] = v;
        }
      // lane r*MT + m stores output (m, n0 + r)
#pragma unroll
      for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (lane == r * MT + m && m < mt && n0 + r < p.N) {
            float v = acc[r][m];
            if (p.bias) v = __fadd_rn(v, bf16lo(p.bias[n0 + r]));
            const __nv_bfloat16 b = __float2bfloat16_rn(v);
            p.y[static_cast<size_t>(m0 + m) * p.N + n0 + r] = *reinterpret_cast<const uint16_t*>(&b);
          }
          acc[r][m] = 0.f;
        }
    }
  };

  // the weights are constant: the first item is in flight while the
  // previous kernel of the stream finishes and while x' is staged
  if (nit > 0) load(cwa, gwa, 0);
  // x may still be written by the previous kernel of the stream
  griddep_wait();
  griddep_launch_dependents();
  for (m0 = 0; m0 < p.M; m0 += MT) {
    mt = min(MT, p.M - m0);
    __syncthreads();
    // x' = fp32(x) * (1/a) for MT tokens, eight elements per item
    for (int i = threadIdx.x; i < MT * (p.K / 8); i += AWQ_THREADS) {
      const int m = i / (p.K / 8), k = 8 * (i % (p.K / 8));
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (m < mt) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(m0 + m) * p.K + k));
        const float4 a0 = __ldg(reinterpret_cast<const float4*>(p.inv_a + k));
        const float4 a1 = __ldg(reinterpret_cast<const float4*>(p.inv_a + k + 4));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
        const float ia[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[2 * e] = __fmul_rn(bf16lo(ww[e]), ia[2 * e]);
          v[2 * e + 1] = __fmul_rn(bf16hi(ww[e]), ia[2 * e + 1]);
        }
      }
      float* dst = xs + (m * nck + k / 32) * 36 + (k % 32);
      *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4*>(dst + 4) = make_float4(v[4], v[5], v[6], v[7]);
    }
    __syncthreads();
    if (m0 > 0 && nit > 0) load(cwa, gwa, 0);
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = 0.f;
    // two items per trip: the next item's loads are issued before the
    // current one is decoded
    for (int it = 0; it < nit; it += 2) {
      if (it + 1 < nit) load(cwb, gwb, it + 1);
      compute(cwa, gwa, it);
      if (it + 1 >= nit) break;
      if (it + 2 < nit) load(cwa, gwa, it + 2);
      compute(cwb, gwb, it + 1);
    }
  }
}

}  // namespace svdq
