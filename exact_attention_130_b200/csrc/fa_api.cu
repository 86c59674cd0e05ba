// fa_api.cu -- the C ABI of libfa_sm100.so: argument validation, per-device
// state, TMA tensor-map encoding, and dispatch to the kernel launchers.
// Every entry point validates before it touches the GPU and returns a status;
// nothing here aborts or exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "fa_internal.h"

namespace fa {

// One status word per device (each device gets its own copy of this
// variable when the module loads there). Kernels write it when a bounded
// wait gives up; fa_device_status() reads and clears it.
__device__ unsigned int g_status_word;

namespace {

thread_local char t_last_error[512] = "";

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;

struct DeviceState {
  // set (release) after the other fields; read (acquire) before using them,
  // so a thread that sees it set also sees the fields it guards
  std::atomic<bool> ready{false};
  int num_sms = 0;
  int cc_major = 0, cc_minor = 0;
  unsigned int* status_word = nullptr;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mu;
std::atomic<unsigned long long> g_wait_limit_ns{kDefaultWaitLimitNs};
std::atomic<int> g_debug_skip{0};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status invalid(fa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
  return s;
}

// Current device, its SM count and status word; set up once per device.
fa_status device_ctx(cudaStream_t stream, LaunchCtx* ctx) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return invalid(FA_ERR_UNSUPPORTED, "device index %d", dev);
  DeviceState& ds = g_dev[dev];
  if (!ds.ready.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!ds.ready.load(std::memory_order_relaxed)) {
      cudaDeviceProp prop;
      e = cudaGetDeviceProperties(&prop, dev);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
      if (prop.major != 10 || prop.minor != 0)
        return invalid(FA_ERR_UNSUPPORTED,
                       "device %d is sm_%d%d; this library is built for sm_100a (B200)", dev,
                       prop.major, prop.minor);
      void* addr = nullptr;
      e = cudaGetSymbolAddress(&addr, g_status_word);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status word)");
      ds.num_sms = prop.multiProcessorCount;
      ds.cc_major = prop.major;
      ds.cc_minor = prop.minor;
      ds.status_word = static_cast<unsigned int*>(addr);
      ds.ready.store(true, std::memory_order_release);
    }
  }
  ctx->stream = stream;
  ctx->status_word = ds.status_word;
  ctx->wait_limit_ns = g_wait_limit_ns.load();
  ctx->num_sms = ds.num_sms;
  ctx->debug_skip_load = 0;
  return FA_OK;
}

fa_status check_bhnd(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1)
    return invalid(FA_ERR_INVALID_ARG, "B, H, N must be >= 1 (got %d, %d, %d)", B, H, N);
  const long long rows = (long long)B * H * N;
  if (rows > 0x7fffffffLL)
    return invalid(FA_ERR_INVALID_ARG, "B*H*N = %lld exceeds 2^31-1", rows);
  if (d != 64 && d != 128) return invalid(FA_ERR_UNSUPPORTED, "head dim %d (need 64 or 128)", d);
  return FA_OK;
}

fa_status check_scale(float scale) {
  if (!std::isfinite(scale) || !(scale > 0.f))
    return invalid(FA_ERR_INVALID_ARG, "scale must be finite and > 0 (got %g)", (double)scale);
  return FA_OK;
}

fa_status check_ptrs(std::initializer_list<const void*> ptrs, const char* names) {
  int i = 0;
  for (const void* p : ptrs) {
    if (p == nullptr) return invalid(FA_ERR_INVALID_ARG, "null pointer (argument %d of %s)", i, names);
    if (!aligned16(p))
      return invalid(FA_ERR_ALIGNMENT, "pointer %d of %s is not 16-byte aligned", i, names);
    ++i;
  }
  return FA_OK;
}

struct ProfRecord {
  unsigned int kid;
  cudaEvent_t start, stop;
};
std::atomic<bool> g_prof_on{false};
std::mutex g_prof_mu;
std::vector<ProfRecord> g_prof;

}  // namespace

ProfileScope::ProfileScope(unsigned int kernel_id, cudaStream_t stream)
    : kid_(kernel_id), stream_(stream) {
  if (!g_prof_on.load(std::memory_order_relaxed)) return;
  if (cudaEventCreate(&start_) != cudaSuccess) {
    start_ = nullptr;
    return;
  }
  if (cudaEventRecord(start_, stream_) != cudaSuccess) {
    cudaEventDestroy(start_);
    start_ = nullptr;
  }
}

ProfileScope::~ProfileScope() {
  if (!start_) return;
  cudaEvent_t stop = nullptr;
  if (cudaEventCreate(&stop) != cudaSuccess || cudaEventRecord(stop, stream_) != cudaSuccess) {
    if (stop) cudaEventDestroy(stop);
    cudaEventDestroy(start_);
    return;
  }
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof.push_back({kid_, start_, stop});
}

void set_last_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
}

fa_status cuda_fail(cudaError_t e, const char* what) {
  snprintf(t_last_error, sizeof(t_last_error), "%s: %s (%s)", what, cudaGetErrorString(e),
           cudaGetErrorName(e));
  return FA_ERR_CUDA;
}

fa_status current_launch_ctx(cudaStream_t stream, LaunchCtx* ctx) {
  return device_ctx(stream, ctx);
}

fa_status make_tmap_3d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t inner,
                       uint64_t rows, uint64_t outer, uint32_t box_inner, uint32_t box_rows,
                       int swizzle_bytes) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (!g_encode) return invalid(FA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4)
    return invalid(FA_ERR_UNSUPPORTED, "tensor map element size %d", elem_bytes);
  const uint64_t elem = uint64_t(elem_bytes);
  const CUtensorMapDataType dtype = elem_bytes == 1   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                    : elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                      : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  cuuint64_t dims[3] = {inner, rows, outer};
  cuuint64_t strides[2] = {inner * elem, inner * rows * elem};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                        : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                              : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return invalid(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", int(r));
  return FA_OK;
}

}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_ALIGNMENT: return "FA_ERR_ALIGNMENT";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
  }
  return "FA_ERR_UNKNOWN";
}

const char* fa_last_error(void) { return t_last_error; }

int fa_abi_version(void) { return 104; }

void fa_set_wait_limit(unsigned long long ns) {
  g_wait_limit_ns.store(ns ? ns : kDefaultWaitLimitNs);
}

void fa_debug_skip_load(int kernel_id) { g_debug_skip.store(kernel_id > 0 ? kernel_id : 0); }

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, float scale, int causal, cudaStream_t stream) {
  fa_status st;
  if ((st = check_ptrs({q, k, v, o, lse}, "fa_fwd(q,k,v,o,lse)")) != FA_OK) return st;
  if ((st = check_bhnd(B, H, N, d)) != FA_OK) return st;
  if ((st = check_scale(scale)) != FA_OK) return st;
  if (causal != 0 && causal != 1) return invalid(FA_ERR_INVALID_ARG, "causal must be 0 or 1");
  LaunchCtx ctx;
  if ((st = device_ctx(stream, &ctx)) != FA_OK) return st;
  ctx.debug_skip_load = g_debug_skip.exchange(0);
  return launch_fwd_bf16(q, k, v, o, lse, B, H, N, d, scale, causal != 0, ctx);
}

fa_status fa_fwd_pair(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int N, int d, float scale, int causal, cudaStream_t stream) {
  fa_status st;
  if ((st = check_ptrs({q, k, v, o, lse}, "fa_fwd_pair(q,k,v,o,lse)")) != FA_OK) return st;
  if ((st = check_bhnd(B, H, N, d)) != FA_OK) return st;
  if (d != 128) return invalid(FA_ERR_UNSUPPORTED, "fa_fwd_pair: head dim %d (needs 128)", d);
  if ((st = check_scale(scale)) != FA_OK) return st;
  if (causal != 0 && causal != 1) return invalid(FA_ERR_INVALID_ARG, "causal must be 0 or 1");
  LaunchCtx ctx;
  if ((st = device_ctx(stream, &ctx)) != FA_OK) return st;
  return launch_fwd_pair(q, k, v, o, lse, B, H, N, d, scale, causal != 0, ctx);
}

// Validates the bias / dropout options shared by fa_fwd_ex and fa_bwd_ex.
static fa_status make_extras(const void* bias, long long bias_stride_b, long long bias_stride_h,
                             int B, int H, int N, float p_drop, unsigned long long seed,
                             unsigned int offset, FwdExtras* ex) {
  if (bias != nullptr && (reinterpret_cast<uintptr_t>(bias) & 15u) != 0)
    return invalid(FA_ERR_ALIGNMENT, "bias is not 16-byte aligned");
  if (bias_stride_b < 0 || bias_stride_h < 0)
    return invalid(FA_ERR_INVALID_ARG, "bias strides must be >= 0");
  if (bias != nullptr) {
    // the last element read: (B-1) sb + (H-1) sh + N*N - 1 must not overflow
    const long double last = (long double)(B - 1) * bias_stride_b +
                             (long double)(H - 1) * bias_stride_h + (long double)N * N;
    if (last > 9.0e18L) return invalid(FA_ERR_INVALID_ARG, "bias extent overflows");
  }
  if (!(p_drop >= 0.f && p_drop < 1.f))
    return invalid(FA_ERR_INVALID_ARG, "dropout probability must be in [0, 1) (got %g)",
                   (double)p_drop);
  double t = std::nearbyint(256.0 * (1.0 - (double)p_drop));
  if (t < 1.0) t = 1.0;
  if (t > 256.0) t = 256.0;
  ex->bias = bias;
  ex->bias_stride_b = bias_stride_b;
  ex->bias_stride_h = bias_stride_h;
  ex->seed = seed;
  ex->offset = offset;
  ex->keep_t = int(t);
  return FA_OK;
}

int fa_dropout_keep_threshold(float p_drop) {
  FwdExtras ex;
  if (make_extras(nullptr, 0, 0, 1, 1, 1, p_drop, 0, 0, &ex) != FA_OK) return -1;
  return ex.keep_t;
}

fa_status fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int H, int N, int d, float scale, int causal, const void* bias,
                    long long bias_stride_b, long long bias_stride_h, float p_drop,
                    unsigned long long seed, unsigned int offset, cudaStream_t stream) {
  fa_status st;
  if ((st = check_ptrs({q, k, v, o, lse}, "fa_fwd_ex(q,k,v,o,lse)")) != FA_OK) return st;
  if ((st = check_bhnd(B, H, N, d)) != FA_OK) return st;
  if ((st = check_scale(scale)) != FA_OK) return st;
  if (causal != 0 && causal != 1) return invalid(FA_ERR_INVALID_ARG, "causal must be 0 or 1");
  FwdExtras ex;
  if ((st = make_extras(bias, bias_stride_b, bias_stride_h, B, H, N, p_drop, seed, offset,
                        &ex)) != FA_OK)
    return st;
  LaunchCtx ctx;
  if ((st = device_ctx(stream, &ctx)) != FA_OK) return st;
  ctx.debug_skip_load = g_debug_skip.exchange(0);
  return launch_fwd_bf16(q, k, v, o, lse, B, H, N, d, scale, causal != 0, ctx, &ex);
}

fa_status fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B,
                     int H, int N, int d, float scale, int causal, cudaStream_t stream) {
  fa_status st;
  if ((st = check_ptrs({q, k, v, o, lse}, "fa_fwd_f32(q,k,v,o,lse)")) != FA_OK) return st;
  if ((st = check_bhnd(B, H, N, d)) != FA_OK) return st;
  if ((st = check_scale(scale)) != FA_OK) return st;
  if (causal != 0 && causal != 1) return invalid(FA_ERR_INVALID_ARG, "causal must be 0 or 1");
  LaunchCtx ctx;
  if ((st = device_ctx(stream, &ctx)) != FA_OK) return st;
  return launch_fwd_f32(q, k, v, o, lse, B, H, N, d, scale, causal != 0, ctx);
}

fa_status fa_fwd_tf32(const float* q, const float* k, const float* v, float* o, float* lse, int B,
                      int H, int N, int d, float scale, int causal, cudaStream_t stream) {
  fa_status st;
  if ((st = check_ptrs({q, k, v, o, lse}, "fa_fwd_tf32(q,k,v,o,lse)")) != FA_OK) return st;
  if ((st = check_bhnd(B, H, N, d)) != FA_OK) return st;
  if ((st = check_scale(scale)) != FA_OK) return st;
  if (causal != 0 && causal != 1) return invalid(FA_ERR_INVALID_ARG, "causal must be 0 or 1");
  LaunchCtx ctx;
  if ((st = device_ctx(stream, &ctx)) != FA_OK) return st;
  return launch_fwd_tf32(q, k, v, o, lse, B, H, N, d, scale, causal != 0, ctx);
}

int fa_fp8_vt_keys(int N) { return N >= 1 && N <= 0x7ffffff0 ? fp8_vt_keys(N) : 0; }

fa_status fa_fp8_prepare(const void* q, const void* k, const void* v, const float* signs, int B,
                         int H, int N, int d, void* q8, void* k8, void* vt8, float* q_scale,
                         float* k_scale, float* v_amax, cudaStream_t stream) {
  fa_status st;
  if ((st = check_ptrs({q, k, v, q8, k8, vt8, q_scale, k_scale, v_amax},
                       "fa_fp8_prepare(q,k,v,q8,k8,vt8,q_scale,k_scale,v_amax)")) != FA_OK)
    return st;
  if (signs != nullptr && (reinterpret_cast<uintptr_t>(signs) & 3u) != 0)
    return invalid(FA_ERR_ALIGNMENT, "signs is not 4-byte aligned");
  if ((st = check_bhnd(B, H, N, d)) != FA_OK) return st;
  if (d != 128) return invalid(FA_ERR_UNSUPPORTED, "the FP8 path needs d = 128 (got %d)", d);
  if ((long long)B * H > 65535)
    return invalid(FA_ERR_INVALID_ARG, "B*H = %lld exceeds 65535", (long long)B * H);
  if ((long long)B * H * d * fp8_vt_keys(N) > 0x7fffffffffffLL)
    return invalid(FA_ERR_INVALID_ARG, "the transposed V is too large");
  LaunchCtx ctx;
  if ((st = device_ctx(stream, &ctx)) != FA_OK) return st;
  return launch_fp8_prepare(q, k, v, signs, B, H, N, d, q8, k8, vt8, q_scale, k_scale, v_amax,
                            ctx);
}

fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* q_scale,
                     const float* k_scale, const float* v_amax, void* o, float* lse, int B, int H,
                     int N, int d, float scale, int causal, cudaStream_t stream) {
  fa_status st;
  if ((st = check_ptrs({q8, k8, vt8, q_scale, k_scale, v_amax, o, lse},
                       "fa_fwd_fp8(q8,k8,vt8,q_scale,k_scale,v_amax,o,lse)")) != FA_OK)
    return st;
  if ((st = check_bhnd(B, H, N, d)) != FA_OK) return st;
  if (d != 128) return invalid(FA_ERR_UNSUPPORTED, "the FP8 path needs d = 128 (got %d)", d);
  if ((st = check_scale(scale)) != FA_OK) return st;
  if (causal != 0 && causal != 1) return invalid(FA_ERR_INVALID_ARG, "causal must be 0 or 1");
  LaunchCtx ctx;
  if ((st = device_ctx(stream, &ctx)) != FA_OK) return st;
  ctx.debug_skip_load = g_debug_skip.exchange(0);
  return launch_fwd_fp8(q8, k8, vt8, q_scale, k_scale, v_amax, o, lse, B, H, N, d, scale,
                        causal != 0, ctx);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (check_bhnd(B, H, N, d) != FA_OK) return 0;
  return bwd_workspace_bytes(B, H, N, d);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                 float scale, int causal, void* workspace, size_t workspace_bytes,
                 cudaStream_t stream) {
  fa_status st;
  if ((st = check_ptrs({q, k, v, o, lse, dO, dq, dk, dv},
                       "fa_bwd(q,k,v,o,lse,dO,dq,dk,dv)")) != FA_OK)
    return st;
  if ((st = check_bhnd(B, H, N, d)) != FA_OK) return st;
  if ((st = check_scale(scale)) != FA_OK) return st;
  if (causal != 0 && causal != 1) return invalid(FA_ERR_INVALID_ARG, "causal must be 0 or 1");
  const size_t need = bwd_workspace_bytes(B, H, N, d);
  if (workspace == nullptr || workspace_bytes < need)
    return invalid(FA_ERR_WORKSPACE, "fa_bwd needs %zu bytes of workspace (got %zu)", need,
                   workspace ? workspace_bytes : size_t(0));
  if (!aligned16(workspace)) return invalid(FA_ERR_ALIGNMENT, "workspace is not 16-byte aligned");
  LaunchCtx ctx;
  if ((st = device_ctx(stream, &ctx)) != FA_OK) return st;
  ctx.debug_skip_load = g_debug_skip.exchange(0);
  return launch_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal != 0, workspace,
                    ctx);
}

fa_status fa_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                    float scale, int causal, const void* bias, long long bias_stride_b,
                    long long bias_stride_h, float p_drop, unsigned long long seed,
                    unsigned int offset, void* workspace, size_t workspace_bytes,
                    cudaStream_t stream) {
  fa_status st;
  if ((st = check_ptrs({q, k, v, o, lse, dO, dq, dk, dv},
                       "fa_bwd_ex(q,k,v,o,lse,dO,dq,dk,dv)")) != FA_OK)
    return st;
  if ((st = check_bhnd(B, H, N, d)) != FA_OK) return st;
  if ((st = check_scale(scale)) != FA_OK) return st;
  if (causal != 0 && causal != 1) return invalid(FA_ERR_INVALID_ARG, "causal must be 0 or 1");
  FwdExtras ex;
  if ((st = make_extras(bias, bias_stride_b, bias_stride_h, B, H, N, p_drop, seed, offset,
                        &ex)) != FA_OK)
    return st;
  const size_t need = bwd_workspace_bytes(B, H, N, d);
  if (workspace == nullptr || workspace_bytes < need)
    return invalid(FA_ERR_WORKSPACE, "fa_bwd_ex needs %zu bytes of workspace (got %zu)", need,
                   workspace ? workspace_bytes : size_t(0));
  if (!aligned16(workspace)) return invalid(FA_ERR_ALIGNMENT, "workspace is not 16-byte aligned");
  LaunchCtx ctx;
  if ((st = device_ctx(stream, &ctx)) != FA_OK) return st;
  ctx.debug_skip_load = g_debug_skip.exchange(0);
  return launch_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal != 0, workspace,
                    ctx, &ex);
}

size_t fa_decode_workspace_size(int B, int H, int Lmax, int d, int num_splits) {
  if (B < 1 || H < 1 || Lmax < 1 || (d != 64 && d != 128) || num_splits < 0 || num_splits > 1024)
    return 0;
  // the automatic chunk count depends only on the shape (and the SM count,
  // for which the size is taken at its maximum so a buffer sized here fits
  // any device of this family)
  const int chunks = decode_num_chunks(B, H, Lmax, num_splits, 0);
  const size_t by_chunks = decode_workspace_bytes(B, H, d, chunks);
  if (num_splits > 0) return by_chunks;
  // the automatic split of the paged decode may balance tiles over
  // persistent CTAs instead (4 to 8 query heads per KV head), whose partials
  // need at most this much
  const size_t balanced = decode_balanced_workspace_bytes(B, H, d);
  return by_chunks > balanced ? by_chunks : balanced;
}

fa_status fa_decode_splitkv(const void* q, const void* kcache, const void* vcache,
                            const int* seqlens, void* o, float* lse, int B, int H, int Lmax, int d,
                            float scale, int num_splits, void* workspace, size_t workspace_bytes,
                            cudaStream_t stream) {
  fa_status st;
  if ((st = check_ptrs({q, kcache, vcache, o, lse}, "fa_decode_splitkv(q,kcache,vcache,o,lse)")) !=
      FA_OK)
    return st;
  if (seqlens == nullptr || (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return invalid(FA_ERR_INVALID_ARG, "seqlens must be a non-null, 4-byte aligned int32 array");
  if (B < 1 || H < 1 || Lmax < 1)
    return invalid(FA_ERR_INVALID_ARG, "B, H, Lmax must be >= 1 (got %d, %d, %d)", B, H, Lmax);
  if ((long long)B * H * Lmax > 0x7fffffffLL)
    return invalid(FA_ERR_INVALID_ARG, "B*H*Lmax exceeds 2^31-1");
  if (d != 64 && d != 128) return invalid(FA_ERR_UNSUPPORTED, "head dim %d (need 64 or 128)", d);
  if ((st = check_scale(scale)) != FA_OK) return st;
  if (num_splits < 0 || num_splits > 1024)
    return invalid(FA_ERR_INVALID_ARG, "num_splits must be in [0, 1024] (got %d)", num_splits);
  const int chunks = decode_num_chunks(B, H, Lmax, num_splits, 0);
  const size_t need = decode_workspace_bytes(B, H, d, chunks);
  if (workspace == nullptr || workspace_bytes < need)
    return invalid(FA_ERR_WORKSPACE, "fa_decode_splitkv needs %zu bytes of workspace (got %zu)",
                   need, workspace ? workspace_bytes : size_t(0));
  if (!aligned16(workspace)) return invalid(FA_ERR_ALIGNMENT, "workspace is not 16-byte aligned");
  LaunchCtx ctx;
  if ((st = device_ctx(stream, &ctx)) != FA_OK) return st;
  ctx.debug_skip_load = g_debug_skip.exchange(0);
  return launch_decode(q, kcache, vcache, seqlens, o, lse, B, H, Lmax, d, scale, chunks,
                       workspace, ctx);
}

fa_status fa_decode_paged(const void* q, const void* kpages, const void* vpages,
                          const int* block_table, const int* seqlens, void* o, float* lse,
                          int B, int Hq, int Hkv, int num_pages, int page_size, int max_pages,
                          int d, float scale, int num_splits, void* workspace,
                          size_t workspace_bytes, cudaStream_t stream) {
  fa_status st;
  if ((st = check_ptrs({q, kpages, vpages, o, lse}, "fa_decode_paged(q,kpages,vpages,o,lse)")) !=
      FA_OK)
    return st;
  if (seqlens == nullptr || (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return invalid(FA_ERR_INVALID_ARG, "seqlens must be a non-null, 4-byte aligned int32 array");
  if (block_table == nullptr || (reinterpret_cast<uintptr_t>(block_table) & 3u))
    return invalid(FA_ERR_INVALID_ARG, "block_table must be a non-null, 4-byte aligned int32 array");
  if (B < 1 || Hq < 1 || Hkv < 1 || num_pages < 1 || max_pages < 1)
    return invalid(FA_ERR_INVALID_ARG, "B, Hq, Hkv, num_pages, max_pages must be >= 1");
  if (Hq % Hkv != 0)
    return invalid(FA_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  if (!(page_size == 16 || page_size == 32 || (page_size >= 64 && page_size % 64 == 0)))
    return invalid(FA_ERR_UNSUPPORTED, "page_size %d (need 16, 32 or a multiple of 64)", page_size);
  if ((long long)max_pages * page_size > 0x7fffffffLL ||
      (long long)num_pages * Hkv * page_size > 0x7fffffffLL ||
      (long long)B * max_pages > 0x7fffffffLL || (long long)B * Hq > 0x7fffffffLL)
    return invalid(FA_ERR_INVALID_ARG, "sizes exceed 2^31-1");
  if (d != 64 && d != 128) return invalid(FA_ERR_UNSUPPORTED, "head dim %d (need 64 or 128)", d);
  if ((st = check_scale(scale)) != FA_OK) return st;
  if (num_splits < 0 || num_splits > 1024)
    return invalid(FA_ERR_INVALID_ARG, "num_splits must be in [0, 1024] (got %d)", num_splits);
  const int Lmax = max_pages * page_size;
  const int chunks = decode_num_chunks(B, Hq, Lmax, num_splits, 0);
  const size_t need = fa_decode_workspace_size(B, Hq, Lmax, d, num_splits);
  if (workspace == nullptr || workspace_bytes < need)
    return invalid(FA_ERR_WORKSPACE, "fa_decode_paged needs %zu bytes of workspace (got %zu)",
                   need, workspace ? workspace_bytes : size_t(0));
  if (!aligned16(workspace)) return invalid(FA_ERR_ALIGNMENT, "workspace is not 16-byte aligned");
  LaunchCtx ctx;
  if ((st = device_ctx(stream, &ctx)) != FA_OK) return st;
  ctx.debug_skip_load = g_debug_skip.exchange(0);
  return launch_decode_paged(q, kpages, vpages, block_table, seqlens, o, lse, B, Hq, Hkv,
                             num_pages, page_size, max_pages, d, scale, chunks, num_splits == 0,
                             workspace, ctx);
}

void fa_profile_begin(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof) {
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  g_prof.clear();
  g_prof_on.store(true);
}

int fa_profile_end(int* launches, double* total_ms, int capacity) {
  g_prof_on.store(false);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (int k = 0; k < capacity; ++k) {
    if (launches) launches[k] = 0;
    if (total_ms) total_ms[k] = 0.0;
  }
  int rc = 10;
  for (auto& r : g_prof) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess ||
        cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess)
      rc = -1;
    if (int(r.kid) < capacity) {
      if (launches) launches[r.kid] += 1;
      if (total_ms) total_ms[r.kid] += ms;
    }
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  g_prof.clear();
  return rc;
}

fa_status fa_device_status(cudaStream_t stream, unsigned int* detail) {
  if (detail) *detail = 0;
  LaunchCtx ctx;
  fa_status st = device_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int word = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&word, g_status_word, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "read status word");
  if (word) {
    e = cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "clear status word");
  }
  if (detail) *detail = word;
  if (word && (word & 0xffu) == 2u) {
    set_last_error("a kernel found an invalid value in device memory: kernel %u, site %u",
                   word >> 16, (word >> 8) & 0xff);
    return FA_ERR_INVALID_ARG;
  }
  if (word) {
    set_last_error("a device-side wait gave up: kernel %u, site %u", word >> 16, (word >> 8) & 0xff);
    return FA_ERR_TIMEOUT;
  }
  return FA_OK;
}

}  // extern "C"
