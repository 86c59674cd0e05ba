// fa_internal.h -- declarations shared by the host API and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include <utility>

#include "fa.h"

namespace fa {

// Everything a launcher needs besides the tensors.
struct LaunchCtx {
  cudaStream_t stream;
  unsigned int* status_word;      // device address of the status word
  unsigned long long wait_limit_ns;
  int num_sms;
  int debug_skip_load;            // test hook, see fa_debug_skip_load()
};

// Launch `kernel` on the stream as a programmatic dependent of the kernel
// before it: its launch overlaps that kernel's end, and the kernel itself
// waits (grid_dependency_wait) before reading what the first one wrote.
template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Kernel ids recorded in the status word.
enum KernelId : unsigned int {
  KID_FWD = 1,
  KID_FWD_F32 = 2,
  KID_BWD_PRE = 3,
  KID_BWD = 4,      // dK/dV kernel
  KID_BWD_DQ = 5,   // dQ kernel
  KID_DECODE = 6,
  KID_DECODE_MERGE = 7,
  KID_FP8_PREP = 9,  // FP8 rotation and quantisation (no waits)
};

// Brackets one kernel launch with CUDA events when profiling is on
// (fa_profile_begin); no-op otherwise.
class ProfileScope {
 public:
  ProfileScope(unsigned int kernel_id, cudaStream_t stream);
  ~ProfileScope();
  ProfileScope(const ProfileScope&) = delete;
  ProfileScope& operator=(const ProfileScope&) = delete;

 private:
  unsigned int kid_;
  cudaStream_t stream_;
  cudaEvent_t start_ = nullptr;
};

// Launch context of the current device (SM count, status word, wait limit),
// setting the device up on first use.
fa_status current_launch_ctx(cudaStream_t stream, LaunchCtx* ctx);

// Records a message for fa_last_error() on this thread.
void set_last_error(const char* fmt, ...);
fa_status cuda_fail(cudaError_t e, const char* what);

// 3-D tiled tensor map over a [outer, rows, inner] tensor of 1-byte (uint8
// codes), 2-byte (bf16) or 4-byte (fp32) elements (inner contiguous), box =
// box_inner x box_rows x 1, zero fill out of bounds. swizzle_bytes: 128 or
// 32 (box_inner * elem_bytes must then equal it) or 0.
fa_status make_tmap_3d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t inner,
                       uint64_t rows, uint64_t outer, uint32_t box_inner, uint32_t box_rows,
                       int swizzle_bytes);

// Options of the bf16 forward and backward: an additive bias (bf16, rows
// of N keys, element strides over batch and head, 0 = broadcast) and
// dropout on P (keep iff the generator byte < keep_t, 1..256; 256 = off).
struct FwdExtras {
  const void* bias;
  long long bias_stride_b, bias_stride_h;
  unsigned long long seed;
  uint32_t offset;
  int keep_t;
};
fa_status launch_fwd_bf16(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int N, int d, float scale, bool causal,
                          const LaunchCtx& ctx, const FwdExtras* ex = nullptr);
// The same forward on CTA pairs (tcgen05 .cta_group::2), bf16, d = 128.
fa_status launch_fwd_pair(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int N, int d, float scale, bool causal,
                          const LaunchCtx& ctx);
// Keys per row of the transposed FP8 V ([B, H, d, fp8_vt_keys(N)] codes):
// N rounded up to 16, so that every row starts 16-byte aligned.
inline int fp8_vt_keys(int N) { return (N + 15) & ~15; }
fa_status launch_fp8_prepare(const void* q, const void* k, const void* v, const float* signs,
                             int B, int H, int N, int d, void* q8, void* k8, void* vt8,
                             float* q_scale, float* k_scale, float* v_amax, const LaunchCtx& ctx);
fa_status launch_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* q_scale,
                         const float* k_scale, const float* v_amax, void* o, float* lse, int B,
                         int H, int N, int d, float scale, bool causal, const LaunchCtx& ctx);
fa_status launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                         int B, int H, int N, int d, float scale, bool causal,
                         const LaunchCtx& ctx);
fa_status launch_fwd_tf32(const float* q, const float* k, const float* v, float* o, float* lse,
                         int B, int H, int N, int d, float scale, bool causal,
                         const LaunchCtx& ctx);
fa_status launch_bwd(const void* q, const void* k, const void* v, const void* o,
                     const float* lse, const void* dO, void* dq, void* dk, void* dv, int B,
                     int H, int N, int d, float scale, bool causal, void* workspace,
                     const LaunchCtx& ctx, const FwdExtras* ex = nullptr);
size_t bwd_workspace_bytes(int B, int H, int N, int d);
int decode_num_chunks(int B, int H, int Lmax, int num_splits, int num_sms);
size_t decode_workspace_bytes(int B, int H, int d, int chunks);
fa_status launch_decode_paged(const void* q, const void* kpages, const void* vpages,
                              const int* block_table, const int* seqlens, void* o, float* lse,
                              int B, int Hq, int Hkv, int num_pages, int page_size, int max_pages,
                              int d, float scale, int chunks, bool auto_split, void* workspace,
                              const LaunchCtx& ctx);
fa_status launch_decode_paged_tc(const void* q, const void* kpages, const void* vpages,
                                 const int* block_table, const int* seqlens, int B, int Hq,
                                 int Hkv, int num_pages, int page_size, int max_pages, int d,
                                 float scale, int chunks, float* part_o, float* part_lse,
                                 const LaunchCtx& ctx);
fa_status launch_decode_paged_tct(const void* q, const void* kpages, const void* vpages,
                                  const int* block_table, const int* seqlens, int B, int Hq,
                                  int Hkv, int num_pages, int page_size, int max_pages, int d,
                                  float scale, int chunks, float* part_o, float* part_lse,
                                  void* workspace, void* o, float* lse, const LaunchCtx& ctx);
// Bytes of workspace the balanced schedule of the keys-as-rows paged decode
// needs (decode_tct_sm100.cu), for B sequences of H query heads.
size_t decode_balanced_workspace_bytes(int B, int H, int d);
fa_status launch_decode(const void* q, const void* kcache, const void* vcache,
                        const int* seqlens, void* o, float* lse, int B, int H, int Lmax, int d,
                        float scale, int chunks, void* workspace, const LaunchCtx& ctx,
                        const char* caller = "fa_decode_splitkv");

}  // namespace fa
