// Host side of libsvdq: argument validation, weight re-tiling at load,
// TMA tensor maps, kernel launches and device-status reporting.
// The C declarations and their documentation live in include/svdq.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/svdq.h"
#include "kawq.cuh"
#include "kprep.cuh"
#include "kg_int4.cuh"
#include "kg_int4h.cuh"
#include "kg_nvfp4.cuh"
#include "kg_nvfp4_chain.cuh"
#include "kg_nvfp4_pair.cuh"
#include "kq.cuh"
#include "krope.cuh"

using namespace svdq;

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per bounded wait

#define SVDQ_TRY(expr)                                              \
  do {                                                              \
    cudaError_t e_ = (expr);                                        \
    if (e_ != cudaSuccess) return e_ == cudaErrorMemoryAllocation   \
                               ? SVDQ_ERR_OOM : SVDQ_ERR_CUDA;      \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// fp16 bits of v if v is exactly an fp16 value (finite, normal or subnormal).
bool fp16_exact(float v, uint16_t* out) {
  uint32_t b;
  std::memcpy(&b, &v, 4);
  const uint16_t sign = static_cast<uint16_t>((b >> 16) & 0x8000u);
  const float a = std::fabs(v);
  if (a == 0.0f) { *out = sign; return true; }
  if (!(a <= 65504.0f)) return false;
  if (a >= 6.103515625e-05f) {  // normal: 2^-14 .. 65504, 10 stored fraction bits
    const uint32_t e = ((b >> 23) & 0xFFu) - 127u + 15u;
    if (b & 0x1FFFu) return false;  // fraction bits below fp16's
    *out = static_cast<uint16_t>(sign | (e << 10) | ((b >> 13) & 0x3FFu));
    return true;
  }
  const float m = a * 16777216.0f;  // multiples of 2^-24
  if (m != std::floor(m)) return false;
  *out = static_cast<uint16_t>(sign | static_cast<uint16_t>(m));
  return true;
}

svdq_status check_device(int* dev_out, int* sms_out) {
  int dev = 0, n = 0;
  if (cudaGetDeviceCount(&n) != cudaSuccess || n == 0) {
    cudaGetLastError();
    return SVDQ_ERR_UNSUPPORTED_DEVICE;
  }
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  int major = 0, minor = 0, sms = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // the 4-bit tensor-core kernels are built for sm_100a only
  if (major != 10 || minor != 0) return SVDQ_ERR_UNSUPPORTED_DEVICE;
  if (dev_out) *dev_out = dev;
  if (sms_out) *sms_out = sms;
  return SVDQ_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D tiled tensor map over a row-major [rows x cols] matrix.
svdq_status make_tmap(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int elem_bytes,
                      uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
                      CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return SVDQ_ERR_CUDA;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem_bytes)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SVDQ_OK : SVDQ_ERR_CUDA;
}

template <class K>
svdq_status set_smem(K kernel, int bytes) {
  SVDQ_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  return SVDQ_OK;
}

// The dynamic shared-memory opt-in of kernel `Kern` on the current device.
// The attribute belongs to the device's context, so it is set once per
// device ordinal (bit `dev` of a per-kernel mask); two threads that race on a
// first call both set it, which is harmless.
template <auto Kern>
svdq_status ensure_smem(int bytes) {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SVDQ_ERR_CUDA;
  const uint64_t bit = 1ull << dev;
  if (done.load(std::memory_order_acquire) & bit) return SVDQ_OK;
  svdq_status s = set_smem(Kern, bytes);
  if (s == SVDQ_OK) done.fetch_or(bit, std::memory_order_release);
  return s;
}

// Launch configuration with programmatic stream serialisation: the kernel may
// start (prologue: barrier set-up, tensor-memory allocation, tensor-map
// prefetch, weight loads) while the previous kernel of the stream finishes;
// every kernel of the library waits for that kernel (griddepcontrol.wait)
// before it reads or writes global memory the previous kernel may touch.
// `cluster` > 1 adds a cluster dimension.
struct LaunchCfg {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  LaunchCfg(dim3 grid, dim3 block, int smem, cudaStream_t st, int cluster = 1) {
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int n = 1;
    if (cluster > 1) {
      attr[1].id = cudaLaunchAttributeClusterDimension;
      attr[1].val.clusterDim.x = cluster;
      attr[1].val.clusterDim.y = 1;
      attr[1].val.clusterDim.z = 1;
      n = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
  }
};

}  // namespace

struct svdq_weights {
  svdq_variant variant;
  int64_t K, N, r, max_M, npad;
  int64_t lr_cols = 0;          // columns of the [L2^T | L2^T] operand (multiple of 64)
  uint32_t stage_row_bytes = 64;  // bytes per operand row in one GEMM pipeline stage
  uint32_t flags;
  int device, sms;
  float out_scale = 1.0f, t_scale = 1.0f;  // 2^e and 2^-e of the NVFP4 per-tensor scale
  // fused QKV epilogue (SVDQ_EPI_QKV_NORM_ROPE): norm weights, epsilon, the
  // row-blocked rotary table (library-owned, cdiv(max_M, 256) * 256 rows of
  // 512 bytes, rewritten by every call), and the table of the call being
  // launched (rope_blk while the GEMM is launched, else null)
  uint16_t* gq = nullptr;
  uint16_t* gk = nullptr;
  float norm_eps = 0.f;
  float* rope_blk = nullptr;
  const float* rope = nullptr;
  // device weights (library-owned)
  float* inv_lam = nullptr;
  uint16_t* l1t = nullptr;     // [r x K]
  uint16_t* l2dup = nullptr;   // [N x 2r]
  uint8_t* wcodes = nullptr;   // NVFP4 [N x K/2] packed; INT4 [N x K] int8
  uint8_t* wscales = nullptr;  // NVFP4 tiled E4M3; INT4 fp32 [K/64 x npad]
  uint16_t* wh = nullptr;      // INT4 with SVDQ_INT4_F16: fp16 s_w q_w [N x K]
  uint16_t* bias = nullptr;
  // bit-reproducible T (svdq_set_deterministic): split partial T tiles and
  // their per-row-block arrival counters (zero between launches)
  int deterministic = 0;
  float* kq_tpart = nullptr;
  int* kq_counters = nullptr;
  // split partials added into T: per-row-block flags (zeroed at load) and
  // the launch counter whose value split 0 publishes in them
  unsigned int* kq_flags = nullptr;
  unsigned int kq_epoch = 0;
  // forward workspace (sized for max_M)
  uint8_t* ws_codes = nullptr;
  uint8_t* ws_scales = nullptr;
  float* ws_t = nullptr;
  // host-call staging
  void* x_dev = nullptr;
  void* y_dev = nullptr;
  // svdq_linear_forward_host: copy streams (in, out) and per-chunk events,
  // created on first use; the K split its row chunks share (0 = automatic)
  cudaStream_t host_in = nullptr, host_out = nullptr;
  cudaEvent_t host_ev[2 * 8 + 1] = {};
  int kq_ksplit_force = 0;
  int* err = nullptr;
  uint32_t debug_mask = 0;
  uint64_t timeout_ns = kDefaultTimeoutNs;
  CUtensorMap tm_b, tm_blr, tm_l1t;
  // NVFP4 CTA-pair GEMM: 128-row boxes of codes and L2, scale atoms as rows
  // of 128 32-bit words
  CUtensorMap tm_b2, tm_blr2, tm_sfb2;
  // INT4 fp16 GEMM: dequantised weights and L2, 128-byte rows, 256-row boxes
  CUtensorMap tm_bh, tm_blrh;
  // per-call maps, cached by (pointer, M)
  CUtensorMap tm_x, tm_a, tm_a2, tm_sfa2;
  const void* tm_x_ptr = nullptr;
  const void* tm_a_ptr = nullptr;
  const void* tm_a2_ptr = nullptr;
  const void* tm_sfa2_ptr = nullptr;
  int64_t tm_x_M = -1, tm_a_M = -1, tm_a2_M = -1, tm_sfa2_M = -1;
};

namespace {

int group_of(svdq_variant v) { return v == SVDQ_INT4_G64_BF16 ? 64 : 16; }

size_t act_scale_bytes(const svdq_weights* h, int64_t M) {
  if (h->variant == SVDQ_INT4_G64_BF16) return static_cast<size_t>(M) * (h->K / 64) * 2;
  return static_cast<size_t>(cdiv(M, 128) * 128) * (h->K / 16);
}

void free_all(svdq_weights* h) {
  void* ptrs[] = {h->inv_lam, h->l1t, h->l2dup, h->wcodes, h->wscales, h->wh, h->bias, h->ws_codes,
                  h->ws_scales, h->ws_t, h->x_dev, h->y_dev, h->err, h->gq, h->gk, h->rope_blk,
                  h->kq_tpart, h->kq_counters, h->kq_flags};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  for (cudaEvent_t e : h->host_ev)
    if (e) cudaEventDestroy(e);
  if (h->host_in) cudaStreamDestroy(h->host_in);
  if (h->host_out) cudaStreamDestroy(h->host_out);
}

// ------------------------------------------------------------------ launches
// K splits of the activation kernel for M rows: the most (up to 8, dividing
// the K / 64 chunks) that keep the grid within one wave of the SMs.
int kq_auto_ksplit(const svdq_weights* h, int64_t M) {
  const int num_m = static_cast<int>(cdiv(M, 128));
  const int kch = static_cast<int>(h->K / 64);
  int ksplit = 1;
  while (ksplit < 8 && num_m * ksplit * 2 <= h->sms && kch % (ksplit * 2) == 0) ksplit *= 2;
  return ksplit;
}

template <int V, int R>
svdq_status launch_kq_t(svdq_weights* h, const CUtensorMap& tmx, int64_t M, uint8_t* codes,
                        void* scales, float* t, cudaStream_t st) {
  using S = KQSmem<V, R>;
  if (svdq_status s = ensure_smem<kq_kernel<V, R>>(S::TOTAL); s != SVDQ_OK) return s;
  const int num_m = static_cast<int>(cdiv(M, 128));
  const int kch = static_cast<int>(h->K / 64);
  // split the K range so that the grid fills the SMs in one wave (or as the
  // host-buffer entry point fixes it for its row chunks)
  const int ksplit = h->kq_ksplit_force > 0 ? h->kq_ksplit_force : kq_auto_ksplit(h, M);
  // split partials are added into T (split 0 clears it first, see kq.cuh);
  // in deterministic mode they go through the scratch and are summed in
  // split order
  const bool accumulate = R > 0 && ksplit > 1 && !h->deterministic;
  KQParams p;
  p.tflags = h->kq_flags;
  if (accumulate && ++h->kq_epoch == 0) h->kq_epoch = 1;  // 0 is the flags' initial value
  p.epoch = h->kq_epoch;
  p.inv_lam = h->inv_lam;
  p.codes = codes;
  p.scales = scales;
  p.t = t;
  p.tpart = h->kq_tpart;
  p.counters = h->kq_counters;
  p.t_accumulate = accumulate ? 1 : 0;
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(h->K);
  p.ksplit = ksplit;
  p.chunks = kch / ksplit;
  p.err = h->err;
  p.debug_mask = h->debug_mask;
  p.timeout_ns = h->timeout_ns;
  LaunchCfg lc(dim3(ksplit, num_m, 1), dim3(KQ_THREADS, 1, 1), S::TOTAL, st);
  SVDQ_TRY(cudaLaunchKernelEx(&lc.cfg, kq_kernel<V, R>, tmx, h->tm_l1t, p));
  return SVDQ_OK;
}

template <int V>
svdq_status launch_kq_v(svdq_weights* h, const CUtensorMap& tmx, int64_t M, uint8_t* codes,
                        void* scales, float* t, cudaStream_t st) {
  switch (h->r) {
    case 0: return launch_kq_t<V, 0>(h, tmx, M, codes, scales, t, st);
    case 16: return launch_kq_t<V, 16>(h, tmx, M, codes, scales, t, st);
    case 32: return launch_kq_t<V, 32>(h, tmx, M, codes, scales, t, st);
    case 64: return launch_kq_t<V, 64>(h, tmx, M, codes, scales, t, st);
    case 128: return launch_kq_t<V, 128>(h, tmx, M, codes, scales, t, st);
  }
  return SVDQ_ERR_SHAPE;
}

template <int R>
svdq_status launch_kg_int4h_t(svdq_weights* h, const CUtensorMap& tma, int64_t M, const uint8_t* sfa,
                              const float* t, void* y, cudaStream_t st) {
  using S = KGI4HSmem<R>;
  if (svdq_status s = ensure_smem<kg_int4h_kernel<R>>(S::TOTAL); s != SVDQ_OK) return s;
  KGParams p;
  p.sfa = sfa;
  p.sfb = h->wscales;
  p.t = t;
  p.bias = h->bias;
  p.y = static_cast<uint16_t*>(y);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(h->N);
  p.K = static_cast<int>(h->K);
  p.num_m = static_cast<int>(cdiv(M, KG_BM));
  p.num_n = static_cast<int>(cdiv(h->N, KG_BN));
  p.gelu = (h->flags & SVDQ_EPI_GELU) ? 1 : 0;
  p.out_scale = h->out_scale;
  p.t_scale = h->t_scale;
  p.qkv_hd = (h->flags & SVDQ_EPI_QKV_NORM_ROPE) ? static_cast<int>(h->N / 3) : 0;
  p.norm_eps = h->norm_eps;
  p.gq = h->gq;
  p.gk = h->gk;
  p.rope = h->rope;
  p.err = h->err;
  p.debug_mask = h->debug_mask;
  p.timeout_ns = h->timeout_ns;
  const int tiles = p.num_m * p.num_n;
  const int grid = tiles < h->sms ? tiles : h->sms;
  LaunchCfg lc(dim3(grid), dim3(KGI4H_THREADS), S::TOTAL, st);
  SVDQ_TRY(cudaLaunchKernelEx(&lc.cfg, kg_int4h_kernel<R>, tma, h->tm_bh, h->tm_blrh, p));
  return SVDQ_OK;
}

template <int V, int R>
svdq_status launch_kg_t(svdq_weights* h, const CUtensorMap& tma, int64_t M, const uint8_t* sfa,
                        const float* t, void* y, cudaStream_t st) {
  if constexpr (V == 0) {
    if (h->wh) return launch_kg_int4h_t<R>(h, tma, M, sfa, t, y, st);
  }
  const int smem = V == 1 ? KGF4Smem<R>::TOTAL : KGI4Smem<R>::TOTAL;
  auto kern = V == 1 ? kg_nvfp4_kernel<R> : kg_int4_kernel<R>;
  if (svdq_status s = V == 1 ? ensure_smem<kg_nvfp4_kernel<R>>(smem) : ensure_smem<kg_int4_kernel<R>>(smem);
      s != SVDQ_OK)
    return s;
  KGParams p;
  p.sfa = sfa;
  p.sfb = h->wscales;
  p.t = t;
  p.bias = h->bias;
  p.y = static_cast<uint16_t*>(y);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(h->N);
  p.K = static_cast<int>(h->K);
  p.num_m = static_cast<int>(cdiv(M, KG_BM));
  p.num_n = static_cast<int>(cdiv(h->N, V == 1 ? KG_BN : KGI4_BN));
  p.gelu = (h->flags & SVDQ_EPI_GELU) ? 1 : 0;
  p.out_scale = h->out_scale;
  p.t_scale = h->t_scale;
  p.qkv_hd = (h->flags & SVDQ_EPI_QKV_NORM_ROPE) ? static_cast<int>(h->N / 3) : 0;
  p.norm_eps = h->norm_eps;
  p.gq = h->gq;
  p.gk = h->gk;
  p.rope = h->rope;
  p.err = h->err;
  p.debug_mask = h->debug_mask;
  p.timeout_ns = h->timeout_ns;
  const int tiles = p.num_m * p.num_n;
  const int grid = tiles < h->sms ? tiles : h->sms;
  LaunchCfg lc(dim3(grid), dim3(KG_THREADS), smem, st);
  SVDQ_TRY(cudaLaunchKernelEx(&lc.cfg, kern, tma, h->tm_b, h->tm_blr, p));
  return SVDQ_OK;
}

// Clusters of two CTAs that fit on the handle's device at once for this
// kernel (0 if the pair kernel cannot be resident), cached per device
// ordinal (stored + 1, so 0 means not yet known).
template <int R>
int pair_clusters(svdq_weights* h) {
  using S = KGF4PairSmem<R>;
  static std::atomic<int> cache[64];
  if (h->device < 0 || h->device >= 64) return 0;
  const int known = cache[h->device].load(std::memory_order_acquire);
  if (known > 0) return known - 1;
  if (ensure_smem<kg_nvfp4_pair_kernel<R>>(S::TOTAL) != SVDQ_OK) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (h->sms / 2));
  cfg.blockDim = dim3(KG_THREADS);
  cfg.dynamicSmemBytes = S::TOTAL;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kg_nvfp4_pair_kernel<R>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;  // not cached: the next call asks again
  }
  cache[h->device].store(n + 1, std::memory_order_release);
  return n;
}

template <int R>
svdq_status launch_kg_pair_t(svdq_weights* h, int64_t M, const uint8_t* sfa, const float* t,
                             void* y, int clusters, cudaStream_t st) {
  using S = KGF4PairSmem<R>;
  KGParams p;
  p.sfa = sfa;
  p.sfb = h->wscales;
  p.t = t;
  p.bias = h->bias;
  p.y = static_cast<uint16_t*>(y);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(h->N);
  p.K = static_cast<int>(h->K);
  p.num_m = static_cast<int>(cdiv(M, 256));
  p.num_n = static_cast<int>(cdiv(h->N, KG_BN));
  p.gelu = (h->flags & SVDQ_EPI_GELU) ? 1 : 0;
  p.out_scale = h->out_scale;
  p.t_scale = h->t_scale;
  p.qkv_hd = (h->flags & SVDQ_EPI_QKV_NORM_ROPE) ? static_cast<int>(h->N / 3) : 0;
  p.norm_eps = h->norm_eps;
  p.gq = h->gq;
  p.gk = h->gk;
  p.rope = h->rope;
  p.err = h->err;
  p.debug_mask = h->debug_mask;
  p.timeout_ns = h->timeout_ns;
  const int tiles = p.num_m * p.num_n;
  const int n = tiles < clusters ? tiles : clusters;
  LaunchCfg lc(dim3(2 * n), dim3(KG_THREADS), S::TOTAL, st, 2);
  SVDQ_TRY(cudaLaunchKernelEx(&lc.cfg, kg_nvfp4_pair_kernel<R>, h->tm_a2, h->tm_b2, h->tm_blr2,
                              h->tm_sfa2, h->tm_sfb2, p));
  return SVDQ_OK;
}

// Per-call maps of the pair kernel over this call's codes and scales.
svdq_status get_tm_pair(svdq_weights* h, const void* codes, const void* scales, int64_t M) {
  if (h->tm_a2_ptr != codes || h->tm_a2_M != M) {
    svdq_status s = make_tmap(&h->tm_a2, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, h->K / 2, M, 128,
                              128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != SVDQ_OK) return s;
    h->tm_a2_ptr = codes;
    h->tm_a2_M = M;
  }
  if (h->tm_sfa2_ptr != scales || h->tm_sfa2_M != M) {
    svdq_status s = make_tmap(&h->tm_sfa2, scales, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, 128,
                              cdiv(M, 128) * (h->K / 64), 128, 4, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (s != SVDQ_OK) return s;
    h->tm_sfa2_ptr = scales;
    h->tm_sfa2_M = M;
  }
  return SVDQ_OK;
}

template <int V>
svdq_status launch_kg_v(svdq_weights* h, const CUtensorMap& tma, const uint8_t* codes, int64_t M,
                        const uint8_t* sfa, const float* t, void* y, cudaStream_t st) {
  if (V == 1 && M > 128 && !(h->flags & SVDQ_GEMM_SINGLE_SM)) {
    int clusters = 0;
    switch (h->r) {
      case 0: clusters = pair_clusters<0>(h); break;
      case 16: clusters = pair_clusters<16>(h); break;
      case 32: clusters = pair_clusters<32>(h); break;
      case 64: clusters = pair_clusters<64>(h); break;
      case 128: clusters = pair_clusters<128>(h); break;
      default: return SVDQ_ERR_SHAPE;
    }
    if (clusters > 0) {
      svdq_status s = get_tm_pair(h, codes, sfa, M);
      if (s != SVDQ_OK) return s;
      switch (h->r) {
        case 0: return launch_kg_pair_t<0>(h, M, sfa, t, y, clusters, st);
        case 16: return launch_kg_pair_t<16>(h, M, sfa, t, y, clusters, st);
        case 32: return launch_kg_pair_t<32>(h, M, sfa, t, y, clusters, st);
        case 64: return launch_kg_pair_t<64>(h, M, sfa, t, y, clusters, st);
        case 128: return launch_kg_pair_t<128>(h, M, sfa, t, y, clusters, st);
      }
    }
  }
  switch (h->r) {
    case 0: return launch_kg_t<V, 0>(h, tma, M, sfa, t, y, st);
    case 16: return launch_kg_t<V, 16>(h, tma, M, sfa, t, y, st);
    case 32: return launch_kg_t<V, 32>(h, tma, M, sfa, t, y, st);
    case 64: return launch_kg_t<V, 64>(h, tma, M, sfa, t, y, st);
    case 128: return launch_kg_t<V, 128>(h, tma, M, sfa, t, y, st);
  }
  return SVDQ_ERR_SHAPE;
}


// fc1's kernel 2 with fc2's activation side fused into the epilogue.
template <int R, int R2>
svdq_status launch_chain_t(svdq_weights* h1, svdq_weights* h2, const CUtensorMap& tma, int64_t M,
                           const uint8_t* sfa, const float* t, void* y1, uint8_t* codes2, uint8_t* scales2,
                           float* t2, cudaStream_t st) {
  using C = KGChainSmem<R, R2>;
  if (svdq_status s = ensure_smem<kg_nvfp4_chain_kernel<R, R2>>(C::TOTAL); s != SVDQ_OK) return s;
  KGParams p;
  p.sfa = sfa;
  p.sfb = h1->wscales;
  p.t = t;
  p.bias = h1->bias;
  p.y = static_cast<uint16_t*>(y1);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(h1->N);
  p.K = static_cast<int>(h1->K);
  p.num_m = static_cast<int>(cdiv(M, KG_BM));
  p.num_n = static_cast<int>(cdiv(h1->N, KG_BN));
  p.gelu = (h1->flags & SVDQ_EPI_GELU) ? 1 : 0;
  p.out_scale = h1->out_scale;
  p.t_scale = h1->t_scale;
  p.qkv_hd = 0;
  p.norm_eps = 0.f;
  p.gq = p.gk = nullptr;
  p.rope = nullptr;
  p.err = h1->err;
  p.debug_mask = 0;
  p.timeout_ns = h1->timeout_ns;
  KGChainParams c;
  c.inv_lam2 = h2->inv_lam;
  c.codes2 = codes2;
  c.scales2 = scales2;
  c.t2 = t2;
  c.store_y = y1 != nullptr ? 1 : 0;
  const int tiles = p.num_m * p.num_n;
  const int grid = tiles < h1->sms ? tiles : h1->sms;
  LaunchCfg lc(dim3(grid), dim3(KG_THREADS), C::TOTAL, st);
  SVDQ_TRY(cudaLaunchKernelEx(&lc.cfg, kg_nvfp4_chain_kernel<R, R2>, tma, h1->tm_b, h1->tm_blr, h2->tm_l1t, p, c));
  return SVDQ_OK;
}


svdq_status get_tm_x(svdq_weights* h, const void* x, int64_t M) {
  if (h->tm_x_ptr == x && h->tm_x_M == M) return SVDQ_OK;
  svdq_status s = make_tmap(&h->tm_x, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, h->K, M, 64, 128,
                            CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != SVDQ_OK) return s;
  h->tm_x_ptr = x;
  h->tm_x_M = M;
  return SVDQ_OK;
}

svdq_status get_tm_a(svdq_weights* h, const void* codes, int64_t M) {
  if (h->tm_a_ptr == codes && h->tm_a_M == M) return SVDQ_OK;
  svdq_status s =
      h->variant == SVDQ_NVFP4_G16_E4M3
          ? make_tmap(&h->tm_a, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, h->K / 2, M,
                      h->stage_row_bytes, 128,
                      h->stage_row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B)
          : make_tmap(&h->tm_a, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, h->K / 2, M, 32, 128,
                      CU_TENSOR_MAP_SWIZZLE_32B);
  if (s != SVDQ_OK) return s;
  h->tm_a_ptr = codes;
  h->tm_a_M = M;
  return SVDQ_OK;
}

svdq_status check_call(svdq_weights* h, int64_t M) {
  if (!h) return SVDQ_ERR_INVALID_ARG;
  if (M < 1 || M > h->max_M || M > (1ll << 30)) return SVDQ_ERR_SHAPE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (dev != h->device) return SVDQ_ERR_INVALID_ARG;
  return SVDQ_OK;
}

svdq_status check_chain(svdq_weights* h1, svdq_weights* h2, int64_t M) {
  if (!h1 || !h2) return SVDQ_ERR_INVALID_ARG;
  if (h1->variant != SVDQ_NVFP4_G16_E4M3 || h2->variant != SVDQ_NVFP4_G16_E4M3) return SVDQ_ERR_INVALID_ARG;
  if ((h1->flags | h2->flags) & SVDQ_EPI_QKV_NORM_ROPE) return SVDQ_ERR_INVALID_ARG;
  if (h1->N != h2->K || h1->N % 256 != 0) return SVDQ_ERR_SHAPE;
  if (!(h1->r == 0 || h1->r == 32) || !(h2->r == 16 || h2->r == 32)) return SVDQ_ERR_SHAPE;
  if (h1->device != h2->device) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = check_call(h1, M);
  if (s != SVDQ_OK) return s;
  return check_call(h2, M);
}

// ------------------------------------------------------------- self-test
// Exhaustive check of the quantiser's division routine against IEEE division
// over every bf16 dividend and every positive finite scale of the variant
// (E4M3: 126 values; bf16: 32639 values), restricted to the quantiser's
// domain |x / s| <= 8 (a group's values never exceed ~7.02 scales).
//   bad[0]: pairs whose 4-bit codes differ (the kernels rely on 0)
//   bad[1]: pairs whose quotients differ while |IEEE quotient| >= 2^-24
//           (far below the smallest nonzero code threshold, 0.25), plus
//           the scale divisions amax/6 and amax/7 over all finite bf16 amax
__global__ void selftest_div_kernel(int variant, unsigned long long* bad) {
  const uint32_t sidx = blockIdx.x + 1;  // 1 .. number of positive finite scales
  float s;
  if (variant == 1) s = e4m3_value(sidx);
  else s = __uint_as_float(sidx << 16);
  const float y = (s >= kMinFastScale && s < kMaxFastScale) ? __frcp_rn(s) : 0.0f;
  unsigned long long bad_code = 0, bad_quot = 0;
  for (uint32_t xb = threadIdx.x; xb < 65536u; xb += blockDim.x) {
    const float x = __uint_as_float(xb << 16);
    if (!isfinite(x)) continue;
    const float b = __fdiv_rn(x, s);
    if (!(fabsf(b) <= 8.0f)) continue;
    const float a = quant_div(x, s, y);
    uint32_t ca, cb;
    if (variant == 1) {
      float va[8] = {a, 0, 0, 0, 0, 0, 0, 0}, vb[8] = {b, 0, 0, 0, 0, 0, 0, 0};
      ca = e2m1x8(va) & 0xFu;
      cb = e2m1x8(vb) & 0xFu;
    } else {
      ca = int4_rn(a);
      cb = int4_rn(b);
    }
    if (ca != cb) ++bad_code;
    if (fabsf(b) >= 5.9604644775390625e-08f && __float_as_uint(a) != __float_as_uint(b)) ++bad_quot;
  }
  if (blockIdx.x == 0) {
    // the group scale divisions amax / 6 and amax / 7 over every finite bf16 amax
    for (uint32_t xb = threadIdx.x; xb < 65536u; xb += blockDim.x) {
      const float x = __uint_as_float(xb << 16);
      if (!isfinite(x)) continue;
      if (__float_as_uint(div_by_scale(x, 6.0f, kRcp6)) != __float_as_uint(__fdiv_rn(x, 6.0f))) ++bad_quot;
      if (__float_as_uint(div_by_scale(x, 7.0f, kRcp7)) != __float_as_uint(__fdiv_rn(x, 7.0f))) ++bad_quot;
    }
  }
  if (bad_code) atomicAdd(bad, bad_code);
  if (bad_quot) atomicAdd(bad + 1, bad_quot);
}

// ------------------------------------------------- allocation-free variant
// Scratch of svdq_quantize_act_lowrank_down_static, in the library's own
// static device memory (every GPU that loads the library holds it until the
// process exits): split partial T tiles, then one arrival counter per
// 128-row block, then a fallback error word.
constexpr size_t kStaticTpartBytes = 10u << 20;   // 10 MiB of partial T tiles
constexpr int kStaticMaxRowBlocks = 4096;          // M <= 4096 * 128 tokens
constexpr size_t kStaticScratchBytes = kStaticTpartBytes + kStaticMaxRowBlocks * 4 + 256;
static __device__ __align__(256) unsigned char g_kq_static_scratch[kStaticScratchBytes];

std::mutex g_static_mu;
void* g_static_ptr[64] = {};  // device address of the scratch, per device ordinal

// Once per device, with that device current: the scratch's device address.
svdq_status static_scratch(int dev, unsigned char** out) {
  if (dev < 0 || dev >= 64) return SVDQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_kq_static_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return SVDQ_ERR_CUDA;
    }
    g_static_ptr[dev] = ptr;
  }
  *out = static_cast<unsigned char*>(g_static_ptr[dev]);
  return SVDQ_OK;
}

template <int V, int R>
svdq_status launch_kq_static(const CUtensorMap& tmx, const CUtensorMap& tml, const float* inv_lam,
                             int64_t M, int64_t K, int sms, uint8_t* codes, void* scales, float* t,
                             unsigned char* scratch, int* err, cudaStream_t st) {
  using S = KQSmem<V, R>;
  if (svdq_status s = ensure_smem<kq_kernel<V, R>>(S::TOTAL); s != SVDQ_OK) return s;
  const int num_m = static_cast<int>(cdiv(M, 128));
  const int kch = static_cast<int>(K / 64);
  int ksplit = 1;  // same split rule as the handle-based entry point
  while (ksplit < 8 && num_m * ksplit * 2 <= sms && kch % (ksplit * 2) == 0) ksplit *= 2;
  if (R > 0 && ksplit > 1 &&
      static_cast<size_t>(ksplit) * num_m * 128 * R * 4 > kStaticTpartBytes)
    return SVDQ_ERR_SHAPE;
  int* counters = reinterpret_cast<int*>(scratch + kStaticTpartBytes);
  if (R > 0 && ksplit > 1)  // arrival counters must start at zero
    SVDQ_TRY(cudaMemsetAsync(counters, 0, static_cast<size_t>(num_m) * 4, st));
  KQParams p;
  p.inv_lam = inv_lam;
  p.codes = codes;
  p.scales = scales;
  p.t = t;
  p.tpart = reinterpret_cast<float*>(scratch);
  p.counters = counters;
  p.t_accumulate = 0;  // deterministic split-order sum through the static scratch
  p.tflags = nullptr;
  p.epoch = 0;
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(K);
  p.ksplit = ksplit;
  p.chunks = kch / ksplit;
  p.err = err;
  p.debug_mask = 0;
  p.timeout_ns = kDefaultTimeoutNs;
  kq_kernel<V, R><<<dim3(ksplit, num_m, 1), KQ_THREADS, S::TOTAL, st>>>(tmx, tml, p);
  SVDQ_TRY(cudaGetLastError());
  return SVDQ_OK;
}

template <int V>
svdq_status launch_kq_static_v(int64_t r, const CUtensorMap& tmx, const CUtensorMap& tml,
                               const float* inv_lam, int64_t M, int64_t K, int sms, uint8_t* codes,
                               void* scales, float* t, unsigned char* scratch, int* err,
                               cudaStream_t st) {
  switch (r) {
    case 0: return launch_kq_static<V, 0>(tmx, tml, inv_lam, M, K, sms, codes, scales, t, scratch, err, st);
    case 16: return launch_kq_static<V, 16>(tmx, tml, inv_lam, M, K, sms, codes, scales, t, scratch, err, st);
    case 32: return launch_kq_static<V, 32>(tmx, tml, inv_lam, M, K, sms, codes, scales, t, scratch, err, st);
    case 64: return launch_kq_static<V, 64>(tmx, tml, inv_lam, M, K, sms, codes, scales, t, scratch, err, st);
    case 128: return launch_kq_static<V, 128>(tmx, tml, inv_lam, M, K, sms, codes, scales, t, scratch, err, st);
  }
  return SVDQ_ERR_SHAPE;
}

}  // namespace

struct svdq_awq {
  int64_t K, N, max_M;
  int device, sms;
  uint8_t* codes = nullptr;   // [N x K/2]
  uint32_t* gp = nullptr;     // [N x K/64]: (bf16 scale << 16) | zero point
  float* inv_a = nullptr;     // [K]
  uint16_t* bias = nullptr;   // [N] or null
};

namespace {

void awq_free_all(svdq_awq* h) {
  void* ptrs[] = {h->codes, h->gp, h->inv_a, h->bias};
  for (void* q : ptrs)
    if (q) cudaFree(q);
}

constexpr int kAwqSmemCap = 100 * 1024;  // staged tokens per pass are chosen to fit

template <int MT>
svdq_status launch_awq(svdq_awq* h, const void* x, void* y, int64_t M, cudaStream_t st) {
  const size_t smem = AWQSmem<MT>::bytes(static_cast<int>(h->K));
  // the opt-in is the largest size any K can ask for (the cap below), so the
  // per-device cache stays valid for every later call
  if (svdq_status s = ensure_smem<kawq_kernel<MT>>(kAwqSmemCap); s != SVDQ_OK) return s;
  AWQParams p;
  p.codes = h->codes;
  p.gp = h->gp;
  p.inv_a = h->inv_a;
  p.x = static_cast<const uint16_t*>(x);
  p.bias = h->bias;
  p.y = static_cast<uint16_t*>(y);
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(h->K);
  p.N = static_cast<int>(h->N);
  // persistent: up to three CTAs per SM (x' is staged once per CTA)
  const int64_t rows_per_cta = (AWQ_THREADS / 32) * awq_rw<MT>();
  const int64_t want = cdiv(h->N, rows_per_cta);
  const int64_t resident = static_cast<int64_t>(awq_ctas<MT>()) * h->sms;
  const int grid = static_cast<int>(want < resident ? want : resident);
  LaunchCfg lc(dim3(grid), dim3(AWQ_THREADS), static_cast<int>(smem), st);
  SVDQ_TRY(cudaLaunchKernelEx(&lc.cfg, kawq_kernel<MT>, p));
  return SVDQ_OK;
}

}  // namespace


// ------------------------------------------------------------ weight prep
namespace {

// fp64 -> bf16 bits, round to nearest even (values in bf16's normal range
// or zero; the prep only rounds factor entries of moderate magnitude).
uint16_t bf16_bits_rn(double v) {
  if (v == 0.0) return std::signbit(v) ? 0x8000u : 0u;
  int ex;
  std::frexp(v, &ex);
  const int lead = std::max(ex - 1, -126);
  const int ue = lead - 7;
  const double q = std::ldexp(std::nearbyint(std::ldexp(v, -ue)), ue);  // default rounding mode: to nearest even
  const float f = static_cast<float>(q);                                  // exact
  uint32_t b;
  std::memcpy(&b, &f, 4);
  return static_cast<uint16_t>(b >> 16);
}

// Upper-triangular R with R^T R = G (G symmetric positive definite, l x l,
// row-major) and its inverse; false if G is not numerically positive.
bool cholesky_inv(const std::vector<double>& G, int l, std::vector<double>& Rinv) {
  std::vector<double> R(static_cast<size_t>(l) * l, 0.0);
  for (int i = 0; i < l; ++i) {
    double d = G[i * l + i];
    for (int k = 0; k < i; ++k) d -= R[k * l + i] * R[k * l + i];
    if (!(d > 0.0)) return false;
    R[i * l + i] = std::sqrt(d);
    for (int j = i + 1; j < l; ++j) {
      double v = G[i * l + j];
      for (int k = 0; k < i; ++k) v -= R[k * l + i] * R[k * l + j];
      R[i * l + j] = v / R[i * l + i];
    }
  }
  Rinv.assign(static_cast<size_t>(l) * l, 0.0);
  for (int j = 0; j < l; ++j) {  // solve R x = e_j by back substitution
    for (int i = l - 1; i >= 0; --i) {
      double v = (i == j) ? 1.0 : 0.0;
      for (int k = i + 1; k < l; ++k) v -= R[i * l + k] * Rinv[k * l + j];
      Rinv[i * l + j] = v / R[i * l + i];
    }
  }
  return true;
}

// Eigen-decomposition of a symmetric l x l matrix by cyclic Jacobi rotations:
// A = V diag(ev) V^T, eigenvalues in descending order, V's columns the vectors.
void jacobi_eig(std::vector<double> A, int l, std::vector<double>& ev, std::vector<double>& V) {
  V.assign(static_cast<size_t>(l) * l, 0.0);
  for (int i = 0; i < l; ++i) V[i * l + i] = 1.0;
  for (int sweep = 0; sweep < 100; ++sweep) {
    double off = 0.0, tot = 0.0;
    for (int i = 0; i < l; ++i)
      for (int j = 0; j < l; ++j) {
        tot += A[i * l + j] * A[i * l + j];
        if (i != j) off += A[i * l + j] * A[i * l + j];
      }
    if (off <= 1e-30 * tot) break;
    for (int p = 0; p < l - 1; ++p)
      for (int q = p + 1; q < l; ++q) {
        const double apq = A[p * l + q];
        if (apq == 0.0) continue;
        const double theta = (A[q * l + q] - A[p * l + p]) / (2.0 * apq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        const double c = 1.0 / std::sqrt(t * t + 1.0), sn = t * c;
        for (int k = 0; k < l; ++k) {  // A = J^T A J
          const double akp = A[k * l + p], akq = A[k * l + q];
          A[k * l + p] = c * akp - sn * akq;
          A[k * l + q] = sn * akp + c * akq;
        }
        for (int k = 0; k < l; ++k) {
          const double apk = A[p * l + k], aqk = A[q * l + k];
          A[p * l + k] = c * apk - sn * aqk;
          A[q * l + k] = sn * apk + c * aqk;
        }
        for (int k = 0; k < l; ++k) {
          const double vkp = V[k * l + p], vkq = V[k * l + q];
          V[k * l + p] = c * vkp - sn * vkq;
          V[k * l + q] = sn * vkp + c * vkq;
        }
      }
  }
  std::vector<int> idx(l);
  for (int i = 0; i < l; ++i) idx[i] = i;
  std::sort(idx.begin(), idx.end(), [&](int a, int b) { return A[a * l + a] > A[b * l + b]; });
  std::vector<double> V2(static_cast<size_t>(l) * l);
  ev.resize(l);
  for (int c = 0; c < l; ++c) {
    ev[c] = A[idx[c] * l + idx[c]];
    for (int k = 0; k < l; ++k) V2[k * l + c] = V[k * l + idx[c]];
  }
  V.swap(V2);
}

struct DevBuf {
  void* p = nullptr;
  ~DevBuf() { if (p) cudaFree(p); }
  bool alloc(size_t bytes) {
    if (cudaMalloc(&p, bytes < 256 ? 256 : bytes) != cudaSuccess) {
      cudaGetLastError();
      p = nullptr;
      return false;
    }
    return true;
  }
  template <class T> T* as() const { return static_cast<T*>(p); }
};

// C = op(A) op(B) (fp32) with split-K over the contraction, C zeroed first.
svdq_status gemm_f32(const float* A, int64_t as0, int64_t as1, const float* B, int64_t bs0, int64_t bs1,
                     float* C, int64_t Mr, int64_t Nc, int64_t Kd, int sms, cudaStream_t st) {
  SVDQ_TRY(cudaMemsetAsync(C, 0, static_cast<size_t>(Mr) * Nc * 4, st));
  const int64_t tiles = cdiv(Mr, 64) * cdiv(Nc, 64);
  int64_t splits = std::max<int64_t>(1, std::min<int64_t>(cdiv(4 * sms, tiles), cdiv(Kd, 256)));
  const int64_t kslice = cdiv(cdiv(Kd, splits), 16) * 16;
  splits = cdiv(Kd, kslice);
  dim3 grid(static_cast<unsigned>(cdiv(Nc, 64)), static_cast<unsigned>(cdiv(Mr, 64)), static_cast<unsigned>(splits));
  prep_gemm_f32_kernel<<<grid, 256, 0, st>>>(A, as0, as1, B, bs0, bs1, C, Nc, Mr, Nc, Kd, kslice);
  SVDQ_TRY(cudaGetLastError());
  return SVDQ_OK;
}

// Y [rows x l] := an orthonormal basis of its column span, by two rounds of
// Cholesky QR (Gram matrix in fp64 on the GPU, its factor on the host).
svdq_status orthonormalize(float* Y, int64_t rows, int l, double* G_dev, cudaStream_t st) {
  DevBuf yo;
  if (!yo.alloc(static_cast<size_t>(rows) * l * 4)) return SVDQ_ERR_OOM;
  for (int round = 0; round < 2; ++round) {
    prep_gram_f64_kernel<<<dim3(l, l), 256, 0, st>>>(Y, rows, l, G_dev);
    SVDQ_TRY(cudaGetLastError());
    std::vector<double> G(static_cast<size_t>(l) * l), Rinv;
    SVDQ_TRY(cudaMemcpyAsync(G.data(), G_dev, G.size() * 8, cudaMemcpyDeviceToHost, st));
    SVDQ_TRY(cudaStreamSynchronize(st));
    if (!cholesky_inv(G, l, Rinv)) return SVDQ_ERR_RANGE;
    SVDQ_TRY(cudaMemcpyAsync(G_dev, Rinv.data(), Rinv.size() * 8, cudaMemcpyHostToDevice, st));
    prep_rmul_small_kernel<<<static_cast<unsigned>(cdiv(rows * l, 256)), 256, 0, st>>>(Y, rows, l, G_dev,
                                                                                      yo.as<float>());
    SVDQ_TRY(cudaGetLastError());
    SVDQ_TRY(cudaMemcpyAsync(Y, yo.p, static_cast<size_t>(rows) * l * 4, cudaMemcpyDeviceToDevice, st));
    SVDQ_TRY(cudaStreamSynchronize(st));  // Rinv (host) outlives the copy
  }
  return SVDQ_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

const char* svdq_status_string(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "SVDQ_OK";
    case SVDQ_ERR_INVALID_ARG: return "SVDQ_ERR_INVALID_ARG";
    case SVDQ_ERR_SHAPE: return "SVDQ_ERR_SHAPE";
    case SVDQ_ERR_ALIGNMENT: return "SVDQ_ERR_ALIGNMENT";
    case SVDQ_ERR_UNSUPPORTED_DEVICE: return "SVDQ_ERR_UNSUPPORTED_DEVICE";
    case SVDQ_ERR_OOM: return "SVDQ_ERR_OOM";
    case SVDQ_ERR_CUDA: return "SVDQ_ERR_CUDA";
    case SVDQ_ERR_DEVICE_TIMEOUT: return "SVDQ_ERR_DEVICE_TIMEOUT";
    case SVDQ_ERR_RANGE: return "SVDQ_ERR_RANGE";
  }
  return "SVDQ_ERR_UNKNOWN";
}

const char* svdq_version(void) { return "svdq 0.2.0 sm_100a"; }

svdq_status svdq_weights_load(const svdq_weight_desc* d, svdq_weights_t* out, void* stream) {
  if (!d || !out) return SVDQ_ERR_INVALID_ARG;
  *out = nullptr;
  if (d->variant != SVDQ_INT4_G64_BF16 && d->variant != SVDQ_NVFP4_G16_E4M3) return SVDQ_ERR_INVALID_ARG;
  if (d->flags & ~(SVDQ_EPI_GELU | SVDQ_GEMM_SINGLE_SM | SVDQ_INT4_F16 | SVDQ_EPI_QKV_NORM_ROPE))
    return SVDQ_ERR_INVALID_ARG;
  if (d->flags & SVDQ_EPI_QKV_NORM_ROPE) {
    if (d->variant != SVDQ_NVFP4_G16_E4M3 || (d->flags & SVDQ_EPI_GELU)) return SVDQ_ERR_INVALID_ARG;
    if (!d->q_norm || !d->k_norm || !(d->norm_eps > 0.0f) || !(d->norm_eps < 1.0f)) return SVDQ_ERR_INVALID_ARG;
    if (d->N % 384 != 0) return SVDQ_ERR_SHAPE;
  }
  const int64_t K = d->K, N = d->N, r = d->r;
  if (K < 128 || K % 128 != 0 || K > (1 << 20)) return SVDQ_ERR_SHAPE;
  if (N < 16 || N % 16 != 0 || N > (1 << 20)) return SVDQ_ERR_SHAPE;
  if (!(r == 0 || r == 16 || r == 32 || r == 64 || r == 128)) return SVDQ_ERR_SHAPE;
  if (d->max_M < 1 || d->max_M > (1ll << 30)) return SVDQ_ERR_SHAPE;
  if (!d->lambda || !d->w_codes || !d->w_scales) return SVDQ_ERR_INVALID_ARG;
  if (d->w_scale_exp != 0 && d->variant != SVDQ_NVFP4_G16_E4M3) return SVDQ_ERR_INVALID_ARG;
  if (d->w_scale_exp < -100 || d->w_scale_exp > 100) return SVDQ_ERR_INVALID_ARG;
  if (r > 0 && (!d->L1 || !d->L2)) return SVDQ_ERR_INVALID_ARG;
  for (int64_t k = 0; k < K; ++k)
    if (!(d->lambda[k] > 0.0f) || !(d->lambda[k] < INFINITY)) return SVDQ_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  svdq_status ds = check_device(&dev, &sms);
  if (ds != SVDQ_OK) return ds;

  svdq_weights* h = new (std::nothrow) svdq_weights();
  if (!h) return SVDQ_ERR_OOM;
  h->variant = d->variant;
  h->K = K;
  h->N = N;
  h->r = r;
  h->max_M = d->max_M;
  h->npad = cdiv(N, 256) * 256;
  h->flags = d->flags;
  h->out_scale = std::ldexp(1.0f, d->w_scale_exp);
  h->t_scale = std::ldexp(1.0f, -d->w_scale_exp);
  h->device = dev;
  h->sms = sms;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G = group_of(d->variant);

  auto fail = [&](svdq_status s) {
    cudaStreamSynchronize(st);
    free_all(h);
    delete h;
    return s;
  };
  auto dmalloc = [&](void** p, size_t bytes) -> bool {
    if (cudaMalloc(p, bytes < 256 ? 256 : bytes) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    return true;
  };

  // ---- host-side re-layout (load time only)
  std::vector<float> inv(K);
  for (int64_t k = 0; k < K; ++k) inv[k] = 1.0f / d->lambda[k];  // IEEE fp32 division
  // [L2^T | L2^T], zero-padded to a multiple of 64 columns (one 128-byte row)
  h->lr_cols = r > 0 ? (2 * r + 63) / 64 * 64 : 0;
  std::vector<uint16_t> l1t(static_cast<size_t>(r) * K), l2dup(static_cast<size_t>(N) * h->lr_cols, 0);
  for (int64_t k = 0; k < K; ++k)
    for (int64_t j = 0; j < r; ++j) l1t[j * K + k] = d->L1[k * r + j];
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < r; ++j) {
      const uint16_t v = d->L2[j * N + n];
      l2dup[n * h->lr_cols + j] = v;
      l2dup[n * h->lr_cols + r + j] = v;
    }
  std::vector<uint8_t> codes, scales;
  std::vector<uint16_t> wh;
  if (d->variant == SVDQ_NVFP4_G16_E4M3) {
    codes.assign(d->w_codes, d->w_codes + static_cast<size_t>(N) * (K / 2));
    scales.assign(static_cast<size_t>(h->npad) * (K / 16), 0);
    const uint8_t* sc = static_cast<const uint8_t*>(d->w_scales);
    for (int64_t n = 0; n < N; ++n)
      for (int64_t b = 0; b < K / 16; ++b) {
        const size_t off = (static_cast<size_t>(n / 128) * (K / 64) + b / 4) * 512 +
                           (n % 32) * 16 + ((n / 32) % 4) * 4 + (b % 4);
        scales[off] = sc[n * (K / 16) + b];
      }
  } else {
    codes.resize(static_cast<size_t>(N) * K);
    for (size_t i = 0; i < static_cast<size_t>(N) * (K / 2); ++i) {
      const uint8_t b = d->w_codes[i];
      codes[2 * i] = static_cast<uint8_t>(static_cast<int8_t>(static_cast<uint8_t>(b << 4)) >> 4);
      codes[2 * i + 1] = static_cast<uint8_t>(static_cast<int8_t>(b) >> 4);
    }
    scales.assign(static_cast<size_t>(K / 64) * h->npad * 4, 0);
    float* sf = reinterpret_cast<float*>(scales.data());
    const uint16_t* sc = static_cast<const uint16_t*>(d->w_scales);
    for (int64_t n = 0; n < N; ++n)
      for (int64_t g = 0; g < K / 64; ++g) {
        const uint32_t bits = static_cast<uint32_t>(sc[n * (K / 64) + g]) << 16;
        float f;
        std::memcpy(&f, &bits, 4);
        sf[g * h->npad + n] = f;
      }
    if (d->flags & SVDQ_INT4_F16) {
      // s_w q_w as fp16, which must be exact (else SVDQ_ERR_RANGE), with K
      // permuted inside each block of 8 in the order the kernel's activation
      // dequantiser produces
      wh.resize(static_cast<size_t>(N) * K);
      for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
          const int64_t ks = (k & ~int64_t(7)) + kInt4F16Perm[k & 7];
          const float v = sf[(ks / 64) * h->npad + n] * static_cast<float>(static_cast<int8_t>(codes[n * K + ks]));
          if (!fp16_exact(v, &wh[n * K + k])) return fail(SVDQ_ERR_RANGE);
        }
    }
  }

  // ---- device allocations and copies
  if (d->variant == SVDQ_INT4_G64_BF16) {
    // the int8 GEMM's activation operand holds 16 x the codes: its weight
    // scales are stored as s_w / 16 (exact), after the host uses above
    float* sf = reinterpret_cast<float*>(scales.data());
    for (size_t i = 0; i < scales.size() / 4; ++i) sf[i] *= 0.0625f;
  }
  if (!dmalloc(reinterpret_cast<void**>(&h->inv_lam), K * 4) ||
      !dmalloc(reinterpret_cast<void**>(&h->wcodes), codes.size()) ||
      !dmalloc(reinterpret_cast<void**>(&h->wscales), scales.size()) ||
      !dmalloc(reinterpret_cast<void**>(&h->err), 256) ||
      !dmalloc(reinterpret_cast<void**>(&h->ws_codes), static_cast<size_t>(h->max_M) * (K / 2)) ||
      !dmalloc(reinterpret_cast<void**>(&h->ws_scales), act_scale_bytes(h, h->max_M)))
    return fail(SVDQ_ERR_OOM);
  if (r > 0 && (!dmalloc(reinterpret_cast<void**>(&h->l1t), l1t.size() * 2) ||
                !dmalloc(reinterpret_cast<void**>(&h->l2dup), l2dup.size() * 2) ||
                !dmalloc(reinterpret_cast<void**>(&h->ws_t), static_cast<size_t>(h->max_M) * r * 4)))
    return fail(SVDQ_ERR_OOM);
  if (d->bias && !dmalloc(reinterpret_cast<void**>(&h->bias), N * 2)) return fail(SVDQ_ERR_OOM);
  if (d->flags & SVDQ_EPI_QKV_NORM_ROPE) {
    if (!dmalloc(reinterpret_cast<void**>(&h->gq), 256) || !dmalloc(reinterpret_cast<void**>(&h->gk), 256) ||
        !dmalloc(reinterpret_cast<void**>(&h->rope_blk), static_cast<size_t>(cdiv(h->max_M, 256)) * 256 * 512))
      return fail(SVDQ_ERR_OOM);
    if (cudaMemcpy(h->gq, d->q_norm, 256, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(h->gk, d->k_norm, 256, cudaMemcpyHostToDevice) != cudaSuccess)
      return fail(SVDQ_ERR_CUDA);
    h->norm_eps = d->norm_eps;
  }
  if (!wh.empty() && !dmalloc(reinterpret_cast<void**>(&h->wh), wh.size() * 2)) return fail(SVDQ_ERR_OOM);
  if (r > 0) {
    const size_t nf = static_cast<size_t>(cdiv(h->max_M, 128)) * 4;
    if (!dmalloc(reinterpret_cast<void**>(&h->kq_flags), nf)) return fail(SVDQ_ERR_OOM);
    if (cudaMemset(h->kq_flags, 0, nf) != cudaSuccess) return fail(SVDQ_ERR_CUDA);
  }

  // synchronous copies: the host vectors go out of scope on return
  if (cudaMemcpy(h->inv_lam, inv.data(), K * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(h->wcodes, codes.data(), codes.size(), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(h->wscales, scales.data(), scales.size(), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemset(h->err, 0, 256) != cudaSuccess)
    return fail(SVDQ_ERR_CUDA);
  if (r > 0 && (cudaMemcpy(h->l1t, l1t.data(), l1t.size() * 2, cudaMemcpyHostToDevice) != cudaSuccess ||
                cudaMemcpy(h->l2dup, l2dup.data(), l2dup.size() * 2, cudaMemcpyHostToDevice) != cudaSuccess))
    return fail(SVDQ_ERR_CUDA);
  if (d->bias && cudaMemcpy(h->bias, d->bias, N * 2, cudaMemcpyHostToDevice) != cudaSuccess)
    return fail(SVDQ_ERR_CUDA);
  if (!wh.empty() && cudaMemcpy(h->wh, wh.data(), wh.size() * 2, cudaMemcpyHostToDevice) != cudaSuccess)
    return fail(SVDQ_ERR_CUDA);

  // ---- weight-side tensor maps
  // NVFP4 stages are 128-byte rows (128B swizzle) except at rank 128 (64-byte
  // rows); the INT4 kernel uses 64-byte rows
  const bool wide = d->variant == SVDQ_NVFP4_G16_E4M3 && r < 128;
  const uint32_t rowb = wide ? 128 : 64;
  const CUtensorMapSwizzle swz = wide ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  h->stage_row_bytes = rowb;
  // B tiles: 256 rows for the NVFP4 single-SM kernel, 128 for the INT4 kernel
  const uint32_t brows = d->variant == SVDQ_NVFP4_G16_E4M3 ? 256 : KGI4_BN;
  svdq_status s = d->variant == SVDQ_NVFP4_G16_E4M3
                      ? make_tmap(&h->tm_b, h->wcodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N,
                                  rowb, brows, swz)
                      : make_tmap(&h->tm_b, h->wcodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N, 64,
                                  brows, CU_TENSOR_MAP_SWIZZLE_64B);
  if (s != SVDQ_OK) return fail(s);
  if (r > 0) {
    if ((s = make_tmap(&h->tm_blr, h->l2dup, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, h->lr_cols, N,
                       rowb / 2, brows, swz)) != SVDQ_OK)
      return fail(s);
    if ((s = make_tmap(&h->tm_l1t, h->l1t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, r, 64,
                       static_cast<uint32_t>(r), CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
      return fail(s);
  } else {
    h->tm_blr = h->tm_b;  // never read when r == 0
    h->tm_l1t = h->tm_b;
  }
  if (h->wh) {
    if ((s = make_tmap(&h->tm_bh, h->wh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, K, N, 64, 256,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
      return fail(s);
    if (r > 0) {
      if ((s = make_tmap(&h->tm_blrh, h->l2dup, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, h->lr_cols, N, 64, 256,
                         CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
        return fail(s);
    } else {
      h->tm_blrh = h->tm_bh;  // never read when r == 0
    }
  }
  if (d->variant == SVDQ_NVFP4_G16_E4M3) {
    if ((s = make_tmap(&h->tm_b2, h->wcodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, 128, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
      return fail(s);
    if ((s = make_tmap(&h->tm_sfb2, h->wscales, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, 128,
                       (h->npad / 128) * (K / 64), 128, 4, CU_TENSOR_MAP_SWIZZLE_NONE)) != SVDQ_OK)
      return fail(s);
    if (r > 0) {
      if ((s = make_tmap(&h->tm_blr2, h->l2dup, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, h->lr_cols, N,
                         64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
        return fail(s);
    } else {
      h->tm_blr2 = h->tm_b2;  // never read when r == 0
    }
  }
  (void)G;
  *out = h;
  return SVDQ_OK;
}

svdq_status svdq_weights_free(svdq_weights_t h) {
  if (!h) return SVDQ_OK;
  cudaDeviceSynchronize();
  free_all(h);
  delete h;
  return SVDQ_OK;
}

svdq_status svdq_act_scales_bytes(svdq_weights_t h, int64_t M, size_t* bytes) {
  if (!h || !bytes || M < 0) return SVDQ_ERR_INVALID_ARG;
  *bytes = act_scale_bytes(h, M);
  return SVDQ_OK;
}

svdq_status svdq_quantize_act_lowrank_down(svdq_weights_t h, const void* x, int64_t M,
                                           uint8_t* act_codes, void* act_scales, float* t,
                                           void* stream) {
  svdq_status s = check_call(h, M);
  if (s != SVDQ_OK) return s;
  if (!x || !act_codes || !act_scales || (h->r > 0 && !t)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(act_codes) || !aligned16(act_scales) || (t && !aligned16(t)))
    return SVDQ_ERR_ALIGNMENT;
  if ((s = get_tm_x(h, x, M)) != SVDQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return h->variant == SVDQ_NVFP4_G16_E4M3
             ? launch_kq_v<1>(h, h->tm_x, M, act_codes, act_scales, t, st)
             : launch_kq_v<0>(h, h->tm_x, M, act_codes, act_scales, t, st);
}

svdq_status svdq_w4a4_gemm_lowrank_up(svdq_weights_t h, const uint8_t* act_codes,
                                      const void* act_scales, const float* t, int64_t M, void* y,
                                      void* stream) {
  svdq_status s = check_call(h, M);
  if (s != SVDQ_OK) return s;
  if ((h->flags & SVDQ_EPI_QKV_NORM_ROPE) && !h->rope) return SVDQ_ERR_INVALID_ARG;  // use the _qkv call
  if (!act_codes || !act_scales || !y || (h->r > 0 && !t)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(act_codes) || !aligned16(act_scales) || !aligned16(y) || (t && !aligned16(t)))
    return SVDQ_ERR_ALIGNMENT;
  if ((s = get_tm_a(h, act_codes, M)) != SVDQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint8_t* sfa = static_cast<const uint8_t*>(act_scales);
  return h->variant == SVDQ_NVFP4_G16_E4M3 ? launch_kg_v<1>(h, h->tm_a, act_codes, M, sfa, t, y, st)
                                           : launch_kg_v<0>(h, h->tm_a, act_codes, M, sfa, t, y, st);
}

svdq_status svdq_linear_forward(svdq_weights_t h, const void* x, void* y, int64_t M, void* stream) {
  svdq_status s = svdq_quantize_act_lowrank_down(h, x, M, h ? h->ws_codes : nullptr,
                                                 h ? h->ws_scales : nullptr, h ? h->ws_t : nullptr,
                                                 stream);
  if (s != SVDQ_OK) return s;
  return svdq_w4a4_gemm_lowrank_up(h, h->ws_codes, h->ws_scales, h->ws_t, M, y, stream);
}

svdq_status svdq_w4a4_gemm_lowrank_up_qkv(svdq_weights_t h, const uint8_t* act_codes,
                                          const void* act_scales, const float* t, int64_t M,
                                          const float* rope, void* y, void* stream) {
  if (!h || !(h->flags & SVDQ_EPI_QKV_NORM_ROPE) || !rope) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = check_call(h, M);
  if (s != SVDQ_OK) return s;
  if (!act_codes || !act_scales || !y || (h->r > 0 && !t)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(rope) || !aligned16(act_codes) || !aligned16(act_scales) || !aligned16(y) ||
      (t && !aligned16(t)))
    return SVDQ_ERR_ALIGNMENT;
  // the row-blocked table for every row of every GEMM tile (256-row tiles on
  // SM pairs, 128 on single SMs), then the GEMM reading it
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LaunchCfg lc(dim3(static_cast<unsigned>(cdiv(M, 256) * 8)), dim3(256), 0, st);
  SVDQ_TRY(cudaLaunchKernelEx(&lc.cfg, rope_block_kernel, reinterpret_cast<const float4*>(rope),
                              static_cast<int>(M), reinterpret_cast<float4*>(h->rope_blk)));
  h->rope = h->rope_blk;
  s = svdq_w4a4_gemm_lowrank_up(h, act_codes, act_scales, t, M, y, stream);
  h->rope = nullptr;
  return s;
}

svdq_status svdq_linear_forward_qkv(svdq_weights_t h, const void* x, const float* rope, void* y, int64_t M,
                                    void* stream) {
  if (!h || !(h->flags & SVDQ_EPI_QKV_NORM_ROPE) || !rope) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = svdq_quantize_act_lowrank_down(h, x, M, h->ws_codes, h->ws_scales, h->ws_t, stream);
  if (s != SVDQ_OK) return s;
  return svdq_w4a4_gemm_lowrank_up_qkv(h, h->ws_codes, h->ws_scales, h->ws_t, M, rope, y, stream);
}

svdq_status svdq_linear_forward_host(svdq_weights_t h, const void* x_host, void* y_host, int64_t M,
                                     void* stream) {
  svdq_status s = check_call(h, M);
  if (s != SVDQ_OK) return s;
  if (!x_host || !y_host) return SVDQ_ERR_INVALID_ARG;
  if (!h->x_dev) {
    if (cudaMalloc(&h->x_dev, static_cast<size_t>(h->max_M) * h->K * 2) != cudaSuccess ||
        cudaMalloc(&h->y_dev, static_cast<size_t>(h->max_M) * h->N * 2) != cudaSuccess) {
      cudaGetLastError();
      return SVDQ_ERR_OOM;
    }
  }
  if (!h->host_in) {
    if (cudaStreamCreateWithFlags(&h->host_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&h->host_out, cudaStreamNonBlocking) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    for (cudaEvent_t& e : h->host_ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return SVDQ_ERR_CUDA;
  }
  // Row chunks of at least 256 rows (at most 8; a last chunk of 128 rows or
  // fewer joins the one before, so every chunk runs on the same GEMM kernel
  // as the whole M would): chunk c's input copy (stream host_in) overlaps
  // the layer on earlier chunks (the caller's stream) and their output copies
  // (host_out), whose two directions run at once.  Each chunk's activation
  // kernel uses the K split of the whole M, so the chunks produce exactly
  // what one call over M would.  The workspace is reused chunk after chunk
  // (the layer's launches are ordered on the caller's stream).
  const int64_t C = std::max<int64_t>(256, cdiv(cdiv(M, 6), 256) * 256);
  int64_t bounds[9];
  int nc = 0;
  for (int64_t r0 = 0; r0 < M && nc < 8; r0 += C) bounds[nc++] = r0;
  if (nc > 1 && M - bounds[nc - 1] <= 128) --nc;
  bounds[nc] = M;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaEvent_t* ev = h->host_ev;  // [0, nc) inputs copied, [8, 8 + nc) chunks computed, [16] entry / exit
  const size_t xrow = static_cast<size_t>(h->K) * 2, yrow = static_cast<size_t>(h->N) * 2;
  // the staging buffers are free once the caller's stream reaches this call
  SVDQ_TRY(cudaEventRecord(ev[16], st));
  SVDQ_TRY(cudaStreamWaitEvent(h->host_in, ev[16], 0));
  SVDQ_TRY(cudaStreamWaitEvent(h->host_out, ev[16], 0));
  h->kq_ksplit_force = kq_auto_ksplit(h, M);
  for (int c = 0; c < nc; ++c) {
    const int64_t r0 = bounds[c], mc = bounds[c + 1] - r0;
    uint8_t* xd = static_cast<uint8_t*>(h->x_dev) + r0 * xrow;
    uint8_t* yd = static_cast<uint8_t*>(h->y_dev) + r0 * yrow;
    if (cudaMemcpyAsync(xd, static_cast<const uint8_t*>(x_host) + r0 * xrow, mc * xrow,
                        cudaMemcpyHostToDevice, h->host_in) != cudaSuccess ||
        cudaEventRecord(ev[c], h->host_in) != cudaSuccess || cudaStreamWaitEvent(st, ev[c], 0) != cudaSuccess) {
      s = SVDQ_ERR_CUDA;
      break;
    }
    if ((s = svdq_linear_forward(h, xd, yd, mc, stream)) != SVDQ_OK) break;
    if (cudaEventRecord(ev[8 + c], st) != cudaSuccess || cudaStreamWaitEvent(h->host_out, ev[8 + c], 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<uint8_t*>(y_host) + r0 * yrow, yd, mc * yrow, cudaMemcpyDeviceToHost,
                        h->host_out) != cudaSuccess) {
      s = SVDQ_ERR_CUDA;
      break;
    }
  }
  h->kq_ksplit_force = 0;
  // the caller's stream completes after the last output copy (also on an
  // error above, after the copies already enqueued)
  if (cudaEventRecord(ev[16], h->host_out) != cudaSuccess || cudaStreamWaitEvent(st, ev[16], 0) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  return s;
}

svdq_status svdq_device_status(svdq_weights_t h, void* stream) {
  if (!h) return SVDQ_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return SVDQ_ERR_CUDA;
  int e = 0;
  if (cudaMemcpy(&e, h->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (e != 0) {
    cudaMemset(h->err, 0, sizeof(int));
    // an aborted launch may leave split arrival counters mid-count
    if (h->kq_counters) cudaMemset(h->kq_counters, 0, cdiv(h->max_M, 128) * 4);
    return e == 0x34f ? SVDQ_ERR_RANGE : SVDQ_ERR_DEVICE_TIMEOUT;
  }
  return SVDQ_OK;
}

svdq_status svdq_set_deterministic(svdq_weights_t h, int on) {
  if (!h || (on != 0 && on != 1)) return SVDQ_ERR_INVALID_ARG;
  if (on && h->r > 0 && !h->kq_tpart) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
    if (dev != h->device) return SVDQ_ERR_INVALID_ARG;
    const size_t nc = static_cast<size_t>(cdiv(h->max_M, 128)) * 4;
    if (cudaMalloc(&h->kq_tpart, static_cast<size_t>(h->sms) * 128 * h->r * 4) != cudaSuccess) {
      cudaGetLastError();
      h->kq_tpart = nullptr;
      return SVDQ_ERR_OOM;
    }
    if (cudaMalloc(&h->kq_counters, nc) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(h->kq_tpart);
      h->kq_tpart = nullptr;
      h->kq_counters = nullptr;
      return SVDQ_ERR_OOM;
    }
    if (cudaMemset(h->kq_counters, 0, nc) != cudaSuccess) return SVDQ_ERR_CUDA;
  }
  h->deterministic = on;
  return SVDQ_OK;
}

svdq_status svdq_device_error_site(svdq_weights_t h, void* stream, int* site) {
  if (!h || !site) return SVDQ_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (cudaMemcpy(site, h->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SVDQ_ERR_CUDA;
  return SVDQ_OK;
}

svdq_status svdq_debug_set_fault(svdq_weights_t h, uint32_t mask, uint32_t timeout_us) {
  if (!h || (mask & ~3u)) return SVDQ_ERR_INVALID_ARG;
  h->debug_mask = mask;
  h->timeout_ns = timeout_us ? static_cast<uint64_t>(timeout_us) * 1000ull : kDefaultTimeoutNs;
  return SVDQ_OK;
}

svdq_status svdq_quantize_act_lowrank_down_static(svdq_variant variant, int64_t K, int64_t r,
                                                  const float* inv_lambda, const uint16_t* l1t,
                                                  const void* x, int64_t M, uint8_t* act_codes,
                                                  void* act_scales, float* t, int* device_error,
                                                  void* stream) {
  if (variant != SVDQ_INT4_G64_BF16 && variant != SVDQ_NVFP4_G16_E4M3) return SVDQ_ERR_INVALID_ARG;
  if (K < 128 || K % 128 != 0 || K > (1 << 20)) return SVDQ_ERR_SHAPE;
  if (!(r == 0 || r == 16 || r == 32 || r == 64 || r == 128)) return SVDQ_ERR_SHAPE;
  if (M < 1 || cdiv(M, 128) > kStaticMaxRowBlocks) return SVDQ_ERR_SHAPE;
  if (!inv_lambda || !x || !act_codes || !act_scales || (r > 0 && (!l1t || !t)))
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(inv_lambda) || !aligned16(x) || !aligned16(act_codes) || !aligned16(act_scales) ||
      (r > 0 && (!aligned16(l1t) || !aligned16(t))))
    return SVDQ_ERR_ALIGNMENT;
  int dev = 0, sms = 0;
  svdq_status s = check_device(&dev, &sms);
  if (s != SVDQ_OK) return s;
  unsigned char* scratch = nullptr;
  if ((s = static_scratch(dev, &scratch)) != SVDQ_OK) return s;
  int* err = device_error ? device_error
                          : reinterpret_cast<int*>(scratch + kStaticTpartBytes + kStaticMaxRowBlocks * 4);
  CUtensorMap tmx, tml;
  if ((s = make_tmap(&tmx, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, M, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
    return s;
  if (r > 0) {
    if ((s = make_tmap(&tml, l1t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, r, 64,
                       static_cast<uint32_t>(r), CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
      return s;
  } else {
    tml = tmx;  // never read when r == 0
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return variant == SVDQ_NVFP4_G16_E4M3
             ? launch_kq_static_v<1>(r, tmx, tml, inv_lambda, M, K, sms, act_codes, act_scales, t, scratch, err, st)
             : launch_kq_static_v<0>(r, tmx, tml, inv_lambda, M, K, sms, act_codes, act_scales, t, scratch, err, st);
}

svdq_status svdq_w4a4_gemm_lowrank_up_chain(svdq_weights_t h1, const uint8_t* act_codes,
                                            const void* act_scales, const float* t, int64_t M, void* y1,
                                            svdq_weights_t h2, uint8_t* act_codes2, void* act_scales2,
                                            float* t2, void* stream) {
  svdq_status s = check_chain(h1, h2, M);
  if (s != SVDQ_OK) return s;
  if (!act_codes || !act_scales || (h1->r > 0 && !t) || !act_codes2 || !act_scales2 || !t2)
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(act_codes) || !aligned16(act_scales) || (t && !aligned16(t)) || (y1 && !aligned16(y1)) ||
      !aligned16(act_codes2) || !aligned16(act_scales2) || !aligned16(t2))
    return SVDQ_ERR_ALIGNMENT;
  if ((s = get_tm_a(h1, act_codes, M)) != SVDQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SVDQ_TRY(cudaMemsetAsync(t2, 0, static_cast<size_t>(M) * h2->r * 4, st));  // T2 is accumulated atomically
  const uint8_t* sfa = static_cast<const uint8_t*>(act_scales);
  uint8_t* sc2 = static_cast<uint8_t*>(act_scales2);
  if (h1->r == 0)
    return h2->r == 16 ? launch_chain_t<0, 16>(h1, h2, h1->tm_a, M, sfa, t, y1, act_codes2, sc2, t2, st)
                       : launch_chain_t<0, 32>(h1, h2, h1->tm_a, M, sfa, t, y1, act_codes2, sc2, t2, st);
  return h2->r == 16 ? launch_chain_t<32, 16>(h1, h2, h1->tm_a, M, sfa, t, y1, act_codes2, sc2, t2, st)
                     : launch_chain_t<32, 32>(h1, h2, h1->tm_a, M, sfa, t, y1, act_codes2, sc2, t2, st);
}

svdq_status svdq_linear_forward_chain(svdq_weights_t h1, svdq_weights_t h2, const void* x, void* y2, int64_t M,
                                      void* stream) {
  svdq_status s = check_chain(h1, h2, M);
  if (s != SVDQ_OK) return s;
  if (!x || !y2) return SVDQ_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // T2 is zeroed first, so the three kernels follow one another with
  // programmatic dependent launch and nothing in between
  SVDQ_TRY(cudaMemsetAsync(h2->ws_t, 0, static_cast<size_t>(M) * h2->r * 4, st));
  if ((s = svdq_quantize_act_lowrank_down(h1, x, M, h1->ws_codes, h1->ws_scales, h1->ws_t, stream)) != SVDQ_OK)
    return s;
  if ((s = get_tm_a(h1, h1->ws_codes, M)) != SVDQ_OK) return s;
  const uint8_t* sfa = h1->ws_scales;
  if (h1->r == 0)
    s = h2->r == 16 ? launch_chain_t<0, 16>(h1, h2, h1->tm_a, M, sfa, h1->ws_t, nullptr, h2->ws_codes, h2->ws_scales, h2->ws_t, st)
                    : launch_chain_t<0, 32>(h1, h2, h1->tm_a, M, sfa, h1->ws_t, nullptr, h2->ws_codes, h2->ws_scales, h2->ws_t, st);
  else
    s = h2->r == 16 ? launch_chain_t<32, 16>(h1, h2, h1->tm_a, M, sfa, h1->ws_t, nullptr, h2->ws_codes, h2->ws_scales, h2->ws_t, st)
                    : launch_chain_t<32, 32>(h1, h2, h1->tm_a, M, sfa, h1->ws_t, nullptr, h2->ws_codes, h2->ws_scales, h2->ws_t, st);
  if (s != SVDQ_OK) return s;
  return svdq_w4a4_gemm_lowrank_up(h2, h2->ws_codes, h2->ws_scales, h2->ws_t, M, y2, stream);
}

svdq_status svdq_awq_load(const svdq_awq_desc* d, svdq_awq_t* out, void* stream) {
  if (!d || !out) return SVDQ_ERR_INVALID_ARG;
  *out = nullptr;
  const int64_t K = d->K, N = d->N;
  if (K < 64 || K % 64 != 0 || K > 16384) return SVDQ_ERR_SHAPE;
  if (N < 1 || N > (1 << 24)) return SVDQ_ERR_SHAPE;
  if (d->max_M < 1 || d->max_M > (1ll << 30)) return SVDQ_ERR_SHAPE;
  if (!d->a || !d->codes || !d->scales || !d->zeros) return SVDQ_ERR_INVALID_ARG;
  for (int64_t k = 0; k < K; ++k)
    if (!(d->a[k] > 0.0f) || !(d->a[k] < INFINITY)) return SVDQ_ERR_INVALID_ARG;
  const int64_t ng = K / 64;
  for (int64_t i = 0; i < N * ng; ++i)
    if (d->zeros[i] > 15) return SVDQ_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  svdq_status ds = check_device(&dev, &sms);
  if (ds != SVDQ_OK) return ds;
  svdq_awq* h = new (std::nothrow) svdq_awq();
  if (!h) return SVDQ_ERR_OOM;
  h->K = K;
  h->N = N;
  h->max_M = d->max_M;
  h->device = dev;
  h->sms = sms;
  auto fail = [&](svdq_status st) {
    cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    awq_free_all(h);
    delete h;
    return st;
  };
  std::vector<float> inv(K);
  for (int64_t k = 0; k < K; ++k) inv[k] = 1.0f / d->a[k];  // IEEE fp32 division
  std::vector<uint32_t> gp(static_cast<size_t>(N) * ng);
  for (size_t i = 0; i < gp.size(); ++i)
    gp[i] = (static_cast<uint32_t>(d->scales[i]) << 16) | d->zeros[i];
  if (cudaMalloc(reinterpret_cast<void**>(&h->codes), static_cast<size_t>(N) * (K / 2)) != cudaSuccess ||
      cudaMalloc(reinterpret_cast<void**>(&h->gp), gp.size() * 4) != cudaSuccess ||
      cudaMalloc(reinterpret_cast<void**>(&h->inv_a), K * 4) != cudaSuccess ||
      (d->bias && cudaMalloc(reinterpret_cast<void**>(&h->bias), N * 2) != cudaSuccess)) {
    cudaGetLastError();
    return fail(SVDQ_ERR_OOM);
  }
  if (cudaMemcpy(h->codes, d->codes, static_cast<size_t>(N) * (K / 2), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(h->gp, gp.data(), gp.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(h->inv_a, inv.data(), K * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
      (d->bias && cudaMemcpy(h->bias, d->bias, N * 2, cudaMemcpyHostToDevice) != cudaSuccess))
    return fail(SVDQ_ERR_CUDA);
  *out = h;
  return SVDQ_OK;
}

svdq_status svdq_awq_free(svdq_awq_t h) {
  if (!h) return SVDQ_OK;
  cudaDeviceSynchronize();
  awq_free_all(h);
  delete h;
  return SVDQ_OK;
}

svdq_status svdq_awq_w4a16_forward(svdq_awq_t h, const void* x, void* y, int64_t M, void* stream) {
  if (!h) return SVDQ_ERR_INVALID_ARG;
  if (M < 1 || M > h->max_M) return SVDQ_ERR_SHAPE;
  if (!x || !y) return SVDQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 3u) || (reinterpret_cast<uintptr_t>(y) & 1u)) return SVDQ_ERR_ALIGNMENT;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (dev != h->device) return SVDQ_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // tokens staged per pass: as many as fit, up to 8
  const size_t cap = kAwqSmemCap;
  if (M >= 5 && AWQSmem<8>::bytes(static_cast<int>(h->K)) <= cap) return launch_awq<8>(h, x, y, M, st);
  if (M >= 3 && AWQSmem<4>::bytes(static_cast<int>(h->K)) <= cap) return launch_awq<4>(h, x, y, M, st);
  if (M >= 2 && AWQSmem<2>::bytes(static_cast<int>(h->K)) <= cap) return launch_awq<2>(h, x, y, M, st);
  return launch_awq<1>(h, x, y, M, st);
}

svdq_status svdq_prep_calibrate(const void* x, int64_t M, const void* w, int64_t K, int64_t N, float alpha,
                                float* lambda, void* stream) {
  if (!x || !w || !lambda) return SVDQ_ERR_INVALID_ARG;
  if (M < 1 || K < 1 || N < 1 || M > (1ll << 31) || K > (1ll << 24) || N > (1ll << 24)) return SVDQ_ERR_SHAPE;
  if (!(alpha >= 0.0f && alpha <= 1.0f)) return SVDQ_ERR_INVALID_ARG;
  svdq_status s = check_device(nullptr, nullptr);
  if (s != SVDQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DevBuf ax, aw;
  if (!ax.alloc(K * 4) || !aw.alloc(K * 4)) return SVDQ_ERR_OOM;
  SVDQ_TRY(cudaMemsetAsync(ax.p, 0, K * 4, st));
  const int rows_per = 256;
  prep_col_amax_kernel<<<dim3(static_cast<unsigned>(cdiv(K, 256)), static_cast<unsigned>(cdiv(M, rows_per))), 256, 0, st>>>(
      static_cast<const uint16_t*>(x), M, K, rows_per, ax.as<unsigned>());
  prep_row_amax_kernel<<<static_cast<unsigned>(K), 256, 0, st>>>(static_cast<const uint16_t*>(w), K, N, aw.as<unsigned>());
  prep_lambda_kernel<<<static_cast<unsigned>(cdiv(K, 256)), 256, 0, st>>>(ax.as<unsigned>(), aw.as<unsigned>(), K,
                                                                           static_cast<double>(alpha), lambda);
  SVDQ_TRY(cudaGetLastError());
  SVDQ_TRY(cudaStreamSynchronize(st));  // the scratch is freed on return
  return SVDQ_OK;
}

svdq_status svdq_prep_lowrank(const void* w, const float* lambda, int64_t K, int64_t N, int64_t r,
                              const float* omega, int64_t l, int power_iters, uint16_t* L1, uint16_t* L2,
                              void* stream) {
  if (!w || !lambda || !omega || !L1 || !L2) return SVDQ_ERR_INVALID_ARG;
  if (K < 1 || N < 1 || K > (1 << 20) || N > (1 << 20)) return SVDQ_ERR_SHAPE;
  if (r < 1 || l < r || l > 192 || l > K || l > N) return SVDQ_ERR_SHAPE;
  if (power_iters < 0 || power_iters > 8) return SVDQ_ERR_INVALID_ARG;
  int sms = 0;
  svdq_status s = check_device(nullptr, &sms);
  if (s != SVDQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int li = static_cast<int>(l);
  DevBuf wh, Y, Z, B, G;
  if (!wh.alloc(static_cast<size_t>(K) * N * 4) || !Y.alloc(static_cast<size_t>(K) * l * 4) ||
      !Z.alloc(static_cast<size_t>(N) * l * 4) || !B.alloc(static_cast<size_t>(l) * N * 4) || !G.alloc(l * l * 8))
    return SVDQ_ERR_OOM;
  float* W = wh.as<float>();
  prep_smooth_kernel<<<static_cast<unsigned>(cdiv(K * N, 256)), 256, 0, st>>>(static_cast<const uint16_t*>(w), lambda,
                                                                               K, N, W);
  SVDQ_TRY(cudaGetLastError());
  // range finder: Y = W_hat Omega, then power iterations Y = W_hat (W_hat^T Y)
  if ((s = gemm_f32(W, N, 1, omega, l, 1, Y.as<float>(), K, l, N, sms, st)) != SVDQ_OK) return s;
  if ((s = orthonormalize(Y.as<float>(), K, li, G.as<double>(), st)) != SVDQ_OK) return s;
  for (int it = 0; it < power_iters; ++it) {
    if ((s = gemm_f32(W, 1, N, Y.as<float>(), l, 1, Z.as<float>(), N, l, K, sms, st)) != SVDQ_OK) return s;
    if ((s = orthonormalize(Z.as<float>(), N, li, G.as<double>(), st)) != SVDQ_OK) return s;
    if ((s = gemm_f32(W, N, 1, Z.as<float>(), l, 1, Y.as<float>(), K, l, N, sms, st)) != SVDQ_OK) return s;
    if ((s = orthonormalize(Y.as<float>(), K, li, G.as<double>(), st)) != SVDQ_OK) return s;
  }
  // B = Q^T W_hat [l x N]
  if ((s = gemm_f32(Y.as<float>(), 1, l, W, N, 1, B.as<float>(), l, N, K, sms, st)) != SVDQ_OK) return s;
  std::vector<float> Bh(static_cast<size_t>(l) * N), Qh(static_cast<size_t>(K) * l);
  SVDQ_TRY(cudaMemcpyAsync(Bh.data(), B.p, Bh.size() * 4, cudaMemcpyDeviceToHost, st));
  SVDQ_TRY(cudaMemcpyAsync(Qh.data(), Y.p, Qh.size() * 4, cudaMemcpyDeviceToHost, st));
  SVDQ_TRY(cudaStreamSynchronize(st));
  // small SVD of B on the host (fp64): B B^T = U diag(sigma^2) U^T, V = B^T U / sigma
  std::vector<double> C(static_cast<size_t>(l) * l, 0.0);
  for (int a = 0; a < li; ++a)
    for (int b = a; b < li; ++b) {
      double t = 0.0;
      for (int64_t n = 0; n < N; ++n) t += static_cast<double>(Bh[a * N + n]) * Bh[b * N + n];
      C[a * l + b] = C[b * l + a] = t;
    }
  std::vector<double> ev, U;
  jacobi_eig(C, li, ev, U);
  std::vector<uint16_t> l1(static_cast<size_t>(K) * r), l2(static_cast<size_t>(r) * N);
  for (int64_t i = 0; i < r; ++i) {
    const double sig = std::sqrt(std::max(ev[i], 0.0));
    const double rs = std::sqrt(sig);
    for (int64_t k = 0; k < K; ++k) {  // L1 = Q U_r sqrt(S)
      double t = 0.0;
      for (int a = 0; a < li; ++a) t += static_cast<double>(Qh[k * l + a]) * U[a * l + i];
      l1[k * r + i] = bf16_bits_rn(t * rs);
    }
    for (int64_t n = 0; n < N; ++n) {  // L2 = sqrt(S) V_r^T, V = B^T U / sigma
      double t = 0.0;
      for (int a = 0; a < li; ++a) t += static_cast<double>(Bh[a * N + n]) * U[a * l + i];
      l2[i * N + n] = bf16_bits_rn(sig > 0.0 ? t / rs : 0.0);
    }
  }
  SVDQ_TRY(cudaMemcpyAsync(L1, l1.data(), l1.size() * 2, cudaMemcpyHostToDevice, st));
  SVDQ_TRY(cudaMemcpyAsync(L2, l2.data(), l2.size() * 2, cudaMemcpyHostToDevice, st));
  SVDQ_TRY(cudaStreamSynchronize(st));
  return SVDQ_OK;
}

svdq_status svdq_prep_residual_quantize(svdq_variant variant, const void* w, const float* lambda,
                                        const uint16_t* L1, const uint16_t* L2, int64_t K, int64_t N, int64_t r,
                                        int tensor_scale, uint8_t* codes, void* scales, int32_t* w_scale_exp,
                                        void* stream) {
  if (variant != SVDQ_INT4_G64_BF16 && variant != SVDQ_NVFP4_G16_E4M3) return SVDQ_ERR_INVALID_ARG;
  if (!w || !lambda || !codes || !scales || !w_scale_exp || (r > 0 && (!L1 || !L2))) return SVDQ_ERR_INVALID_ARG;
  if (tensor_scale && variant != SVDQ_NVFP4_G16_E4M3) return SVDQ_ERR_INVALID_ARG;
  const int G = group_of(variant);
  if (K < G || K % G != 0 || K > (1 << 20) || N < 1 || N > (1 << 20)) return SVDQ_ERR_SHAPE;
  if (r < 0 || r > 128) return SVDQ_ERR_SHAPE;
  svdq_status s = check_device(nullptr, nullptr);
  if (s != SVDQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int ri = static_cast<int>(r);
  const uint16_t* wb = static_cast<const uint16_t*>(w);
  int e = 0;
  if (tensor_scale) {
    DevBuf am;
    if (!am.alloc(8)) return SVDQ_ERR_OOM;
    SVDQ_TRY(cudaMemsetAsync(am.p, 0, 8, st));
    prep_residual_amax_kernel<<<dim3(static_cast<unsigned>(cdiv(N, 128)), static_cast<unsigned>(cdiv(K, 16))), 128, 0, st>>>(
        wb, lambda, L1, L2, K, N, ri, am.as<unsigned long long>());
    SVDQ_TRY(cudaGetLastError());
    double amax = 0.0;
    SVDQ_TRY(cudaMemcpyAsync(&amax, am.p, 8, cudaMemcpyDeviceToHost, st));
    SVDQ_TRY(cudaStreamSynchronize(st));
    if (amax > 0.0) {  // smallest e with amax / 6 <= 448 * 2^e
      int x;
      const double m = std::frexp(amax / 6.0 / 448.0, &x);
      e = (m == 0.5) ? x - 1 : x;
    }
  }
  dim3 grid(static_cast<unsigned>(cdiv(N, 128)), static_cast<unsigned>(K / G));
  if (variant == SVDQ_INT4_G64_BF16)
    prep_residual_quant_kernel<0><<<grid, 128, 0, st>>>(wb, lambda, L1, L2, K, N, ri, 0, codes, scales);
  else
    prep_residual_quant_kernel<1><<<grid, 128, 0, st>>>(wb, lambda, L1, L2, K, N, ri, e, codes, scales);
  SVDQ_TRY(cudaGetLastError());
  *w_scale_exp = e;
  return SVDQ_OK;
}

svdq_status svdq_selftest_division(int variant, unsigned long long* mismatches) {
  if (!mismatches || (variant != 0 && variant != 1)) return SVDQ_ERR_INVALID_ARG;
  svdq_status ds = check_device(nullptr, nullptr);
  if (ds != SVDQ_OK) return ds;
  unsigned long long* d = nullptr;
  SVDQ_TRY(cudaMalloc(&d, 2 * sizeof(unsigned long long)));
  cudaMemset(d, 0, 2 * sizeof(unsigned long long));
  // E4M3: codes 1..126 are the positive finite scales; bf16: 0x0001..0x7F7F
  const int nscales = variant == 1 ? 126 : 0x7F7F;
  selftest_div_kernel<<<nscales, 256>>>(variant, d);
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess)
    e = cudaMemcpy(mismatches, d, 2 * sizeof(unsigned long long), cudaMemcpyDeviceToHost);
  cudaFree(d);
  return e == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

#ifdef SVDQ_WAIT_PROFILE
// Instrumented builds only: read and clear the per-site wait counters.
int svdq_wait_profile(unsigned long long* cycles, unsigned long long* counts) {
  cudaDeviceSynchronize();
  cudaMemcpyFromSymbol(cycles, g_wait_cycles, sizeof(g_wait_cycles));
  cudaMemcpyFromSymbol(counts, g_wait_count, sizeof(g_wait_count));
  static unsigned long long zero[1024] = {};
  cudaMemcpyToSymbol(g_wait_cycles, zero, sizeof(zero));
  cudaMemcpyToSymbol(g_wait_count, zero, sizeof(zero));
  return 0;
}
#endif

}  // extern "C"
