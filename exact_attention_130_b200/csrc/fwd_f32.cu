// fwd_f32.cu -- attention forward on fp32 tensors, computed in fp32.
//
// Same function and the same one-pass recurrence as the bf16 kernel
// ("Bellek Duvarinin Fizigi", "Online Softmax" and "Forward gecisin
// iskeleti"): K/V tiles stream through shared memory, each query row keeps a
// running maximum m, running sum l and unnormalised output O~, rescaled by
// 2^(m_old - m_new); O = O~ / l at the end.
//
// The tensor cores have no fp32 operand type (tf32 would round every input to
// a 10-bit mantissa), so this small-problem path runs on the CUDA cores:
// one CTA = 32 query rows of one (batch, head); four threads share a row,
// each owning every fourth head-dimension element, so a quad reads four
// consecutive floats of a K or V row (no bank conflicts) and combines its
// partial dot products with two shuffles.
#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kRows = 32;   // query rows per CTA
constexpr int kKeys = 32;   // keys per shared-memory tile
constexpr int kThreads = 128;
constexpr float kLn2 = 0.69314718055994530942f;

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads)
    fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                   const float* __restrict__ v, float* __restrict__ o, float* __restrict__ lse,
                   int N, float scale_log2) {
  constexpr int P = D / 4;  // elements per thread
  __shared__ float ks[kKeys][D];
  __shared__ float vs[kKeys][D];
  const size_t bh = blockIdx.y;
  const int row0 = blockIdx.x * kRows;
  const int tid = threadIdx.x;
  const int part = tid & 3;
  const int row = row0 + (tid >> 2);
  const float* qb = q + bh * size_t(N) * D;
  const float* kb = k + bh * size_t(N) * D;
  const float* vb = v + bh * size_t(N) * D;

  float qr[P], acc[P];
#pragma unroll
  for (int i = 0; i < P; ++i) {
    qr[i] = row < N ? qb[size_t(row) * D + i * 4 + part] : 0.f;
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int kend = CAUSAL ? min(N, row0 + kRows) : N;
  for (int k0 = 0; k0 < kend; k0 += kKeys) {
    __syncthreads();
    for (int idx = tid; idx < kKeys * D; idx += kThreads) {
      const int kk = idx / D, col = idx % D;
      const int key = k0 + kk;
      ks[kk][col] = key < N ? kb[size_t(key) * D + col] : 0.f;
      vs[kk][col] = key < N ? vb[size_t(key) * D + col] : 0.f;
    }
    __syncthreads();
    float s[kKeys];
    float mx = -INFINITY;
#pragma unroll
    for (int kk = 0; kk < kKeys; ++kk) {
      float part_dot = 0.f;
#pragma unroll
      for (int i = 0; i < P; ++i) part_dot = fmaf(qr[i], ks[kk][i * 4 + part], part_dot);
      part_dot += __shfl_xor_sync(0xffffffffu, part_dot, 1);
      part_dot += __shfl_xor_sync(0xffffffffu, part_dot, 2);
      const int key = k0 + kk;
      const bool visible = key < N && (!CAUSAL || key <= row);
      s[kk] = visible ? part_dot * scale_log2 : -INFINITY;
      mx = fmaxf(mx, s[kk]);
    }
    const float m_new = fmaxf(m, mx);
    if (m_new == -INFINITY) continue;  // nothing visible yet for this row
    const float alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - m_new);
    m = m_new;
    float rs = 0.f;
#pragma unroll
    for (int kk = 0; kk < kKeys; ++kk) {
      s[kk] = ex2_approx(s[kk] - m);
      rs += s[kk];
    }
    l = l * alpha + rs;
#pragma unroll
    for (int i = 0; i < P; ++i) {
      float a = acc[i] * alpha;
#pragma unroll
      for (int kk = 0; kk < kKeys; ++kk) a = fmaf(s[kk], vs[kk][i * 4 + part], a);
      acc[i] = a;
    }
  }
  if (row < N) {
    const float inv_l = 1.0f / l;
    float* ob = o + bh * size_t(N) * D + size_t(row) * D;
#pragma unroll
    for (int i = 0; i < P; ++i) ob[i * 4 + part] = acc[i] * inv_l;
    if (part == 0) lse[bh * size_t(N) + row] = (m + lg2_approx(l)) * kLn2;
  }
}

template <int D, bool CAUSAL>
fa_status launch(const float* q, const float* k, const float* v, float* o, float* lse, int BH,
                 int N, float scale, const LaunchCtx& ctx) {
  dim3 grid((N + kRows - 1) / kRows, BH);
  {
    ProfileScope prof(KID_FWD_F32, ctx.stream);
    fwd_f32_kernel<D, CAUSAL><<<grid, kThreads, 0, ctx.stream>>>(q, k, v, o, lse, N,
                                                                  scale * 1.4426950408889634f);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fwd_f32 kernel launch");
  return FA_OK;
}

}  // namespace

fa_status launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                         int B, int H, int N, int d, float scale, bool causal,
                         const LaunchCtx& ctx) {
  const int BH = B * H;
  if (BH > 65535) {
    set_last_error("fa_fwd_f32: B*H = %d exceeds 65535", BH);
    return FA_ERR_UNSUPPORTED;
  }
  if (d == 128)
    return causal ? launch<128, true>(q, k, v, o, lse, BH, N, scale, ctx)
                  : launch<128, false>(q, k, v, o, lse, BH, N, scale, ctx);
  return causal ? launch<64, true>(q, k, v, o, lse, BH, N, scale, ctx)
                : launch<64, false>(q, k, v, o, lse, BH, N, scale, ctx);
}

}  // namespace fa
