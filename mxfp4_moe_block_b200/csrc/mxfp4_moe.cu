// mxfp4_moe.cu -- the C ABI of include/mxfp4_moe.h: argument checks, kernel
// choice and launches.  Every kernel of the library is compiled into this one
// translation unit (the .cuh files), for sm_100a.
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "route_permute.cuh"
#include "ffn_fma.cuh"
#include "ffn_tc.cuh"
#include "combine.cuh"
#include "accept.cuh"
#include "quantize.cuh"

using namespace moe;

namespace {

constexpr int kMaxDevices = 64;

// One NVTX range per C-ABI call, named after the call, for timeline tools
// (a function-pointer check and nothing more when none is attached).
struct CallRange {
  explicit CallRange(const char *name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange &) = delete;
  CallRange &operator=(const CallRange &) = delete;
};

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  bool greedy_attr = false;   // non-portable cluster size allowed for greedy_kernel
  bool permute_attr = false;  // 33*1024 ints of dynamic shared memory for the permutation
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int current_device(int *dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

const DeviceInfo *device_info() {
  int dev;
  if (current_device(&dev) != MOE_OK) return nullptr;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo &d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return nullptr;
    d.ready = true;
  }
  return &d;
}

// Status of a launch made with cudaLaunchKernelEx (the error is returned,
// and also left in the runtime's last-error slot, which this clears).
int launched(cudaError_t e) {
  if (e != cudaSuccess) {
    fprintf(stderr, "mxfp4_moe: launch failed: %s\n", cudaGetErrorString(e));
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    fprintf(stderr, "mxfp4_moe: launch failed: %s\n", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

inline size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

}  // namespace

extern "C" {

const char *moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or variant";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_WORKSPACE: return "workspace too small or misaligned";
    case MOE_ERR_DEVICE: return "device status word set";
    default: return "unknown status";
  }
}

int moe_version(void) { return 10000; }

// Dynamic shared memory of the one-CTA permutation (33*E ints, E <= 1024),
// set once per device for both kernels that run it.
static int permute_attributes() {
  DeviceInfo *dev = const_cast<DeviceInfo *>(device_info());
  if (!dev) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!dev->permute_attr) {
    const int bytes = 33 * 1024 * (int)sizeof(int);
    if (cudaFuncSetAttribute(permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(route_permute_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess ||
        cudaFuncSetAttribute(route_permute_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess ||
        cudaFuncSetAttribute(route_permute_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess ||
        cudaFuncSetAttribute(route_permute_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess ||
        cudaFuncSetAttribute(route_permute_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess ||
        cudaFuncSetAttribute(route_permute_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess)
      return launch_status();
    dev->permute_attr = true;
  }
  return MOE_OK;
}

// ------------------------------------------------------------------ route --
int moe_route_topk(const float *logits, int T, int E, int k, int32_t *topk_idx,
                   float *topk_w, moe_stream_t stream) {
  const CallRange range("moe_route_topk");
  if (T < 0 || E < 1 || k < 1 || k > E || k > 32) return MOE_ERR_INVALID_ARG;
  if (E > 1024) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!logits || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  const dim3 block(128), grid((unsigned)((T + 3) / 4));
  cudaStream_t s = (cudaStream_t)stream;
  auto kern = E <= 32    ? route_topk_kernel<1>
              : E <= 64  ? route_topk_kernel<2>
              : E <= 128 ? route_topk_kernel<4>
              : E <= 256 ? route_topk_kernel<8>
              : E <= 512 ? route_topk_kernel<16>
                         : route_topk_kernel<32>;
  return launched(launch_pdl(kern, grid, block, 0, s, logits, T, E, k, topk_idx, topk_w));
}

// ---------------------------------------------------------------- permute --
int moe_permute(const int32_t *topk_idx, int T, int k, int E, int32_t *expert_offsets,
                int32_t *sorted_pair, int32_t *pair_row, moe_stream_t stream) {
  const CallRange range("moe_permute");
  if (T < 0 || k < 1 || k > 32 || E < 1) return MOE_ERR_INVALID_ARG;
  if (E > 1024) return MOE_ERR_UNSUPPORTED;
  const long long P = (long long)T * k;
  if (P > (1ll << 24)) return MOE_ERR_UNSUPPORTED;
  if (!expert_offsets) return MOE_ERR_INVALID_ARG;
  if (P > 0 && (!topk_idx || !sorted_pair || !pair_row)) return MOE_ERR_INVALID_ARG;
  const size_t smem = (size_t)33 * E * sizeof(int);
  const int st = permute_attributes();
  if (st != MOE_OK) return st;
  return launched(launch_pdl(permute_kernel, 1, 1024, smem, (cudaStream_t)stream, topk_idx, (int)P,
                             E, expert_offsets, sorted_pair, pair_row));
}

// ---------------------------------------------------- route + permute --
int moe_route_permute(const float *logits, int T, int E, int k, int32_t *topk_idx, float *topk_w,
                      int32_t *expert_offsets, int32_t *sorted_pair, int32_t *pair_row,
                      moe_stream_t stream) {
  const CallRange range("moe_route_permute");
  if (T < 0 || E < 1 || k < 1 || k > E || k > 32) return MOE_ERR_INVALID_ARG;
  if (E > 1024) return MOE_ERR_UNSUPPORTED;
  if ((long long)T * k > (1ll << 24)) return MOE_ERR_UNSUPPORTED;
  if (!expert_offsets) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!logits || !topk_idx || !topk_w || !sorted_pair || !pair_row))
    return MOE_ERR_INVALID_ARG;
  if (T == 0 || T > ROUTE_PERMUTE_MAX_T) {
    const int st = moe_route_topk(logits, T, E, k, topk_idx, topk_w, stream);
    if (st != MOE_OK) return st;
    return moe_permute(topk_idx, T, k, E, expert_offsets, sorted_pair, pair_row, stream);
  }
  const int st = permute_attributes();
  if (st != MOE_OK) return st;
  const size_t smem = (size_t)33 * E * sizeof(int);
  auto kern = E <= 32    ? route_permute_kernel<1>
              : E <= 64  ? route_permute_kernel<2>
              : E <= 128 ? route_permute_kernel<4>
              : E <= 256 ? route_permute_kernel<8>
              : E <= 512 ? route_permute_kernel<16>
                         : route_permute_kernel<32>;
  return launched(launch_pdl(kern, 1, 1024, smem, (cudaStream_t)stream, logits, T, E, k, topk_idx,
                             topk_w, expert_offsets, sorted_pair, pair_row));
}

// -------------------------------------------------------------------- FFN --
// Workspace layout (each part 256-byte aligned): h bf16 [P, I] first (the
// documented accessor), then x as float [T, H], h as float [P, I], then the
// tensor-core variant's operands.
struct WsLayout {
  size_t h, x32, h32, tc, total;
};

static WsLayout ws_layout(int T, int k, int H, int I) {
  const size_t P = (size_t)T * k;
  WsLayout w;
  size_t o = 0;
  w.h = o;   o += align256(P * I * sizeof(uint16_t));
  w.x32 = o; o += align256((size_t)T * H * sizeof(float));
  w.h32 = o; o += align256(P * I * sizeof(float));
  w.tc = o;  o += tc_workspace_bytes(P, H, I);
  w.total = o < 256 ? 256 : o;
  return w;
}

size_t mxfp4_moe_ffn_workspace_bytes(int T, int k, int H, int I) {
  if (T < 0 || k < 1 || H < 0 || I < 0) return 0;
  return ws_layout(T, k, H, I).total;
}

const uint16_t *mxfp4_moe_ffn_workspace_h(const void *workspace) {
  return reinterpret_cast<const uint16_t *>(workspace);
}

int mxfp4_moe_ffn_variant(const uint16_t *x, int T, int H, int I, int E, int k,
                          const uint8_t *w13_codes, const uint8_t *w13_scales,
                          const uint8_t *w2_codes, const uint8_t *w2_scales,
                          const int32_t *expert_offsets, const int32_t *sorted_pair, float *y,
                          void *workspace, size_t workspace_bytes, int variant,
                          moe_stream_t stream) {
  const CallRange range("mxfp4_moe_ffn_variant");
  if (T < 0 || H <= 0 || I <= 0 || E < 1 || k < 1 || k > 32 || k > E) return MOE_ERR_INVALID_ARG;
  if (H % 128 || I % 128) return MOE_ERR_INVALID_ARG;
  if (E > 1024) return MOE_ERR_UNSUPPORTED;
  if (variant < MOE_FFN_AUTO || variant > MOE_FFN_TENSOR_F8_PAIR) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !w13_codes || !w13_scales || !w2_codes || !w2_scales || !expert_offsets ||
      !sorted_pair || !y || !workspace)
    return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < mxfp4_moe_ffn_workspace_bytes(T, k, H, I) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255))
    return MOE_ERR_WORKSPACE;
  const DeviceInfo *dev = device_info();
  if (!dev) return MOE_ERR_CUDA;
  const size_t P = (size_t)T * k;
  if (variant == MOE_FFN_AUTO) variant = tc_prefer(P, E, H) ? MOE_FFN_TENSOR : MOE_FFN_FMA;

  const WsLayout wl = ws_layout(T, k, H, I);
  uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
  FfnArgs a{x, T, H, I, E, k, w13_codes, w13_scales, w2_codes, w2_scales,
            expert_offsets, sorted_pair, reinterpret_cast<uint16_t *>(ws + wl.h), y,
            reinterpret_cast<float *>(ws + wl.x32), reinterpret_cast<float *>(ws + wl.h32)};
  cudaStream_t s = (cudaStream_t)stream;
  if (variant == MOE_FFN_TENSOR) return tc_ffn(a, ws + wl.tc, dev->sms, s, -1);
  if (variant == MOE_FFN_TENSOR_F8) return tc_ffn(a, ws + wl.tc, dev->sms, s, KIND_F8);
  if (variant == MOE_FFN_TENSOR_F4) return tc_ffn(a, ws + wl.tc, dev->sms, s, KIND_F4);
  if (variant == MOE_FFN_TENSOR_FUSED)
    return tc_ffn(a, ws + wl.tc, dev->sms, s, KIND_F4_FUSED);
  if (variant == MOE_FFN_TENSOR_F8_PAIR)
    return tc_ffn(a, ws + wl.tc, dev->sms, s, KIND_F8_PAIR);
  const size_t n8 = (size_t)T * H / 8;
  int st = launched(launch_pdl(x_to_f32_kernel,
                               (unsigned)std::min<size_t>((n8 + 255) / 256, (size_t)dev->sms * 8),
                               256, 0, s, x, n8, a.x32));
  if (st != MOE_OK) return st;
  st = launched(launch_pdl(ffn1_fma_kernel<4>, dev->sms, FMA_THREADS, 0, s, a));
  if (st != MOE_OK) return st;
  return launched(launch_pdl(ffn2_fma_kernel<8>, dev->sms, FMA_THREADS, 0, s, a));
}

int mxfp4_moe_ffn(const uint16_t *x, int T, int H, int I, int E, int k,
                  const uint8_t *w13_codes, const uint8_t *w13_scales,
                  const uint8_t *w2_codes, const uint8_t *w2_scales,
                  const int32_t *expert_offsets, const int32_t *sorted_pair, float *y,
                  void *workspace, size_t workspace_bytes, moe_stream_t stream) {
  const CallRange range("mxfp4_moe_ffn");
  return mxfp4_moe_ffn_variant(x, T, H, I, E, k, w13_codes, w13_scales, w2_codes, w2_scales,
                               expert_offsets, sorted_pair, y, workspace, workspace_bytes,
                               MOE_FFN_AUTO, stream);
}

// -------------------------------------------------------- FFN, no alloc --
// Scratch of mxfp4_moe_ffn_noalloc: a fixed array in the library's own
// device global memory, shared by every call on a device.  Host code must
// not hand the symbol itself to a kernel (on the host it names a host-side
// stand-in); its device address is looked up once per device below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

namespace {
void *g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;
}  // namespace

int mxfp4_moe_ffn_noalloc(const uint16_t *x, int T, int H, int I, int E, int k,
                          const uint8_t *w13_codes, const uint8_t *w13_scales,
                          const uint8_t *w2_codes, const uint8_t *w2_scales,
                          const int32_t *expert_offsets, const int32_t *sorted_pair, float *y,
                          moe_stream_t stream) {
  const CallRange range("mxfp4_moe_ffn_noalloc");
  // the argument checks of mxfp4_moe_ffn_variant first, so that a bad
  // argument is reported as such whatever the problem's scratch need
  if (T < 0 || H <= 0 || I <= 0 || E < 1 || k < 1 || k > 32 || k > E) return MOE_ERR_INVALID_ARG;
  if (H % 128 || I % 128) return MOE_ERR_INVALID_ARG;
  if (E > 1024) return MOE_ERR_UNSUPPORTED;
  if (mxfp4_moe_ffn_workspace_bytes(T, k, H, I) > (size_t)MOE_NOALLOC_SCRATCH_BYTES) {
    fprintf(stderr,
            "mxfp4_moe_ffn_noalloc: T=%d k=%d H=%d I=%d needs %zu scratch bytes, more than the "
            "built-in %u\n",
            T, k, H, I, mxfp4_moe_ffn_workspace_bytes(T, k, H, I),
            (unsigned)MOE_NOALLOC_SCRATCH_BYTES);
    return MOE_ERR_WORKSPACE;
  }
  int dev;
  const int st = current_device(&dev);
  if (st != MOE_OK) return st;
  void *scratch;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
      void *p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
      }
      g_noalloc_ptr[dev] = p;
    }
    scratch = g_noalloc_ptr[dev];
  }
  return mxfp4_moe_ffn_variant(x, T, H, I, E, k, w13_codes, w13_scales, w2_codes, w2_scales,
                               expert_offsets, sorted_pair, y, scratch,
                               (size_t)MOE_NOALLOC_SCRATCH_BYTES, MOE_FFN_AUTO, stream);
}

// ---------------------------------------------------------------- combine --
int moe_combine(const float *y, const int32_t *pair_row, const float *topk_w, int T, int k,
                int H, const uint16_t *residual, uint16_t *out, moe_stream_t stream) {
  const CallRange range("moe_combine");
  if (T < 0 || k < 1 || k > 32 || H <= 0 || H % 8) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!y || !pair_row || !topk_w || !out) return MOE_ERR_INVALID_ARG;
  const dim3 grid((unsigned)T, (unsigned)((H + 1023) / 1024));
  return launched(launch_pdl(combine_kernel, grid, 256, 0, (cudaStream_t)stream, y, pair_row,
                             topk_w, T, k, H, residual, out));
}

int moe_rms_norm(const uint16_t *x, int T, int H, float eps, uint16_t *out,
                 moe_stream_t stream) {
  const CallRange range("moe_rms_norm");
  if (T < 0 || H <= 0 || H % 8 || !(eps >= 0.f)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !out) return MOE_ERR_INVALID_ARG;
  return launched(launch_pdl(rms_norm_kernel, T, 256, 0, (cudaStream_t)stream, x, T, H, eps, out));
}

// ----------------------------------------------------------------- accept --
// Greedy acceptance over R target rows per sequence (R = K, or K + 1 with a
// bonus row).
static int greedy_launch(const float *logits, const int32_t *draft, int S, int K, int V, int R,
                         int32_t *accept_len, int32_t *next_token, moe_stream_t stream) {
  if (S < 0 || K < 1 || K > 32 || V < 1) return MOE_ERR_INVALID_ARG;
  if (S == 0) return MOE_OK;
  if (!logits || !draft || !accept_len || !next_token) return MOE_ERR_INVALID_ARG;
  if (S > 65535 || V > (1 << GREEDY_TOKEN_BITS)) return MOE_ERR_UNSUPPORTED;
  DeviceInfo *dev = const_cast<DeviceInfo *>(device_info());
  if (!dev) return MOE_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!dev->greedy_attr) {
      if (cudaFuncSetAttribute(greedy_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
          cudaSuccess)
        return launch_status();
      dev->greedy_attr = true;
    }
  }
  const cudaStream_t s = (cudaStream_t)stream;
  // Cluster size per row: slices of about 48 KB, at least two CTAs per SM
  // over all rows, at least GREEDY_THREADS elements (or float4 units) each.
  const long long rows = (long long)S * R;
  const long long units = (V & 3) == 0 ? V / 4 : V;
  long long csize = std::max<long long>((4LL * V + 49151) / 49152, (2LL * dev->sms + rows - 1) / rows);
  csize = std::min<long long>(csize, std::max<long long>(1, units / GREEDY_THREADS));
  csize = std::max<long long>(1, std::min<long long>(csize, GREEDY_MAX_CLUSTER));

  int st = launched(launch_pdl(greedy_init_kernel, (unsigned)std::min<long long>((S + 255) / 256, 256),
                               256, 0, s, S, accept_len, next_token));
  if (st != MOE_OK) return st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)csize, (unsigned)R, (unsigned)S);
  cfg.blockDim = dim3(GREEDY_THREADS, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return launched(
      cudaLaunchKernelEx(&cfg, greedy_kernel, logits, draft, S, K, V, R, accept_len, next_token));
}

int block_accept_greedy(const float *logits, const int32_t *draft, int S, int K, int V,
                        int32_t *accept_len, int32_t *next_token, moe_stream_t stream) {
  const CallRange range("block_accept_greedy");
  return greedy_launch(logits, draft, S, K, V, K, accept_len, next_token, stream);
}

int block_accept_greedy_bonus(const float *logits, const int32_t *draft, int S, int K, int V,
                              int32_t *accept_len, int32_t *next_token, moe_stream_t stream) {
  const CallRange range("block_accept_greedy_bonus");
  return greedy_launch(logits, draft, S, K, V, K + 1, accept_len, next_token, stream);
}

static int rejection_launch(const float *p, const float *q, const int32_t *draft,
                            const float *u_accept, const float *u_resample, int S, int K, int V,
                            int R, int32_t *accept_len, int32_t *next_token, moe_stream_t stream) {
  if (S < 0 || K < 1 || K > 32 || V < 1 || V > (1 << 24)) return MOE_ERR_INVALID_ARG;
  if (S == 0) return MOE_OK;
  if (!p || !q || !draft || !u_accept || !u_resample || !accept_len || !next_token)
    return MOE_ERR_INVALID_ARG;
  if (S > (1 << 30)) return MOE_ERR_UNSUPPORTED;
  int threads = ((V + 31) / 32) * 32;
  if (threads > 1024) threads = 1024;
  return launched(launch_pdl(rejection_kernel, S, threads, 0, (cudaStream_t)stream, p, q, draft,
                             u_accept, u_resample, S, K, V, R, accept_len, next_token));
}

int block_accept_rejection(const float *p, const float *q, const int32_t *draft,
                           const float *u_accept, const float *u_resample, int S, int K, int V,
                           int32_t *accept_len, int32_t *next_token, moe_stream_t stream) {
  const CallRange range("block_accept_rejection");
  return rejection_launch(p, q, draft, u_accept, u_resample, S, K, V, K, accept_len, next_token,
                          stream);
}

int block_accept_rejection_bonus(const float *p, const float *q, const int32_t *draft,
                                 const float *u_accept, const float *u_resample, int S, int K,
                                 int V, int32_t *accept_len, int32_t *next_token,
                                 moe_stream_t stream) {
  const CallRange range("block_accept_rejection_bonus");
  return rejection_launch(p, q, draft, u_accept, u_resample, S, K, V, K + 1, accept_len,
                          next_token, stream);
}

// --------------------------------------------------------------- quantise --
int mxfp4_quantize(const uint16_t *w, int64_t R, int K, uint8_t *codes, uint8_t *scales,
                   moe_stream_t stream) {
  const CallRange range("mxfp4_quantize");
  if (R < 0 || K < 32 || K % 32) return MOE_ERR_INVALID_ARG;
  if (R == 0) return MOE_OK;
  if (!w || !codes || !scales) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(w) & 15) || (reinterpret_cast<uintptr_t>(codes) & 3))
    return MOE_ERR_INVALID_ARG;
  if (R > (int64_t(1) << 40) / K) return MOE_ERR_UNSUPPORTED;
  const DeviceInfo *dev = device_info();
  if (!dev) return MOE_ERR_CUDA;
  const size_t n8 = (size_t)R * (size_t)K / 8;
  const size_t blocks = (n8 + (size_t)QUANT_THREADS * QUANT_UNROLL - 1) /
                        ((size_t)QUANT_THREADS * QUANT_UNROLL);
  const unsigned grid = (unsigned)std::min<size_t>(blocks, (size_t)dev->sms * 8);
  return launched(launch_pdl(mxfp4_quantize_kernel, grid, QUANT_THREADS, 0, (cudaStream_t)stream,
                             w, n8, codes, scales));
}

// ----------------------------------------------------------------- status --
int moe_get_device_status(moe_stream_t stream, int *detail) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  if (detail) *detail = v;
  return v ? MOE_ERR_DEVICE : MOE_OK;
}

int moe_set_wait_limit_ns(uint64_t ns, moe_stream_t stream) {
  // the host value is staged by the runtime before the call returns
  const unsigned long long v = ns ? (unsigned long long)ns : 2000000000ull;
  if (cudaMemcpyToSymbolAsync(g_wait_limit_ns, &v, sizeof(v), 0, cudaMemcpyHostToDevice,
                              (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

int moe_clear_device_status(moe_stream_t stream) {
  void *addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_status) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemsetAsync(addr, 0, sizeof(int), (cudaStream_t)stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // extern "C"
