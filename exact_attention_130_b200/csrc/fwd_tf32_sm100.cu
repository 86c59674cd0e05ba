// fwd_tf32_sm100.cu -- the fp32 forward with its two products on the tensor
// cores in TF32 ("Bellek Duvarinin Fizigi", "Online Softmax" and "Forward
// gecisin iskeleti": the same one-pass recurrence as every forward here).
//
// tcgen05 has no fp32 operand type; .kind::tf32 multiplies operands with a
// 10-bit mantissa and accumulates in fp32. The hardware would simply drop
// the low 13 bits of an fp32 input, which biases every product toward zero
// (about 2^-10 relative, enough to move the LSE of N(0,1) scores by ~1e-3),
// so the threads round Q, K, V and P to TF32 to nearest (cvt.rna) on their
// way into shared memory; the error is then unbiased, unit roundoff 2^-11.
//
// One CTA = 128 query rows of one (batch, head), 128 threads, thread t =
// query row t = TMEM lane t. Per 64-key tile: the threads load K (K-major)
// and V transposed (V^T, K-major, the B operand of O += P V), thread 0
// issues S = Q K^T (M = 128, N = 64, K = d), the threads run the online
// softmax on their S row, write P (TF32) to shared memory and rescale O in
// TMEM when the running maximum moves, and thread 0 issues O += P V
// (N = d, K = 64). No pipelining: this path is for small problems (the
// fp32 workload is one 128-row tile), where it is latency-bound anyway.
// Every mbarrier wait is bounded in time.
#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kTM = 128;   // query rows per CTA (the MMA's M)
constexpr int kTK = 64;    // keys per tile
constexpr int kTThreads = 128;
constexpr float kLn2T = 0.69314718055994530942f;

// K-major operand tiles in the 128-byte swizzle: [K / 32 chunks][rows][128 B],
// the 16-byte unit u of a row stored at u ^ (row % 8)
template <int D>
struct TLayout {
  static constexpr int kQChunk = kTM * 128;             // bytes per 32-wide K chunk
  static constexpr int kKChunk = kTK * 128;
  static constexpr int kVtChunk = D * 128;              // V^T: D rows, K = keys
  static constexpr int kPChunk = kTM * 128;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + (D / 32) * kQChunk;
  static constexpr int kOffVt = kOffK + (D / 32) * kKChunk;
  static constexpr int kOffP = kOffVt + (kTK / 32) * kVtChunk;
  static constexpr int kOffBar = kOffP + (kTK / 32) * kPChunk;  // S_DONE, PV_DONE
  static constexpr int kOffMisc = kOffBar + 16;                  // TMEM base, abort flag
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory");
  static constexpr uint32_t kColO = kTK;                         // S: columns 0..63
  static constexpr uint32_t kTmemCols = D == 128 ? 256 : 128;
};

__device__ __forceinline__ uint32_t swz(int row, int k) {  // byte of (row, k) in its chunk
  return uint32_t(row) * 128u + (uint32_t(((k & 31) >> 2) ^ (row & 7)) << 4) + uint32_t(k & 3) * 4u;
}
__device__ __forceinline__ float tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}
__device__ __forceinline__ float4 tf32_rna4(float4 v) {
  return make_float4(tf32_rna(v.x), tf32_rna(v.y), tf32_rna(v.z), tf32_rna(v.w));
}
// Instruction descriptor of .kind::tf32: TF32 A and B (format 2), fp32
// accumulator, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t(N) >> 3) << 17) | ((uint32_t(M) >> 4) << 24);
}
__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n"
      "}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kTThreads)
    fwd_tf32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                    const float* __restrict__ v, float* __restrict__ o, float* __restrict__ lse,
                    int N, float scale_log2, unsigned int* status, unsigned long long limit_ns) {
  using L = TLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_s = sbase + L::kOffBar, bar_pv = bar_s + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  const int t = threadIdx.x, warp = t >> 5;
  const size_t bh = blockIdx.y;
  const int row0 = blockIdx.x * kTM;
  const int row = row0 + t;
  const float* qb = q + bh * size_t(N) * D;
  const float* kb = k + bh * size_t(N) * D;
  const float* vb = v + bh * size_t(N) * D;

  if (t == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_pv, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  // Q tile, rounded to TF32 (rows past N zero)
  for (int e = t; e < kTM * (D / 4); e += kTThreads) {
    const int r = e / (D / 4), c = (e % (D / 4)) * 4;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row0 + r < N) x = *reinterpret_cast<const float4*>(qb + size_t(row0 + r) * D + c);
    *reinterpret_cast<float4*>(smem + L::kOffQ + (c >> 5) * L::kQChunk + swz(r, c)) = tf32_rna4(x);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, status, limit_ns, KID_FWD_F32};
  const uint32_t lane_base = uint32_t(warp * 32) << 16;

  float m = -INFINITY, l = 0.f;
  const int kend = CAUSAL ? min(N, row0 + kTM) : N;
  const int n_tiles = (kend + kTK - 1) / kTK;
  bool ok = true;
  for (int j = 0; j < n_tiles; ++j) {
    const int k0 = j * kTK;
    if (j > 0) {
      // P V(j-1) has read P, V^T (and S(j-1) read K): the buffers are free
      ok = wait_bounded(bar_pv, (j - 1) & 1, wc, 1);
      ok = __syncthreads_and(ok);
      if (!ok) break;
      tc_fence_after();
    }
    // K tile (K-major) and V^T (keys along K), rounded to TF32, zero past N
    for (int e = t; e < kTK * (D / 4); e += kTThreads) {
      const int r = e / (D / 4), c = (e % (D / 4)) * 4;
      const int key = k0 + r;
      float4 kx = make_float4(0.f, 0.f, 0.f, 0.f), vx = kx;
      if (key < N) {
        kx = *reinterpret_cast<const float4*>(kb + size_t(key) * D + c);
        vx = *reinterpret_cast<const float4*>(vb + size_t(key) * D + c);
      }
      *reinterpret_cast<float4*>(smem + L::kOffK + (c >> 5) * L::kKChunk + swz(r, c)) = tf32_rna4(kx);
      vx = tf32_rna4(vx);
      uint8_t* vt = smem + L::kOffVt + (r >> 5) * L::kVtChunk;
      *reinterpret_cast<float*>(vt + swz(c + 0, r)) = vx.x;
      *reinterpret_cast<float*>(vt + swz(c + 1, r)) = vx.y;
      *reinterpret_cast<float*>(vt + swz(c + 2, r)) = vx.z;
      *reinterpret_cast<float*>(vt + swz(c + 3, r)) = vx.w;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (t == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_tf32(kTM, kTK);
#pragma unroll
      for (int kk = 0; kk < D / 8; ++kk)
        mma_tf32(tmem,
                 sdesc_sw128(sbase + L::kOffQ + (kk >> 2) * L::kQChunk + (kk & 3) * 32, 16, 1024),
                 sdesc_sw128(sbase + L::kOffK + (kk >> 2) * L::kKChunk + (kk & 3) * 32, 16, 1024),
                 idesc, kk > 0 ? 1u : 0u);
      tc_commit(bar_s);
    }
    ok = wait_bounded(bar_s, j & 1, wc, 2);
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();
    uint32_t sr[64];
    tmem_ld64_wait(tmem + lane_base, sr);
    float s[kTK];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < kTK; ++i) {
      const int key = k0 + i;
      const bool vis = key < N && (!CAUSAL || key <= row);
      s[i] = vis ? __uint_as_float(sr[i]) * scale_log2 : -INFINITY;
      mx = fmaxf(mx, s[i]);
    }
    const float m_new = fmaxf(m, mx);
    // (a row past N, or one with no visible key yet, keeps P = 0)
    const float m_use = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = m == -INFINITY ? 0.f : ex2_approx(m - m_use);
    float rs = 0.f;
#pragma unroll
    for (int i = 0; i < kTK; ++i) {
      s[i] = ex2_approx(s[i] - m_use);
      rs += s[i];
    }
    // (tcgen05.ld/st are warp-wide: a warp rescales if any of its rows must,
    // the others by alpha = 1)
    if (__any_sync(0xffffffffu, j > 0 && alpha != 1.f)) {
      // O~ through tile j-1 (P V(j-1) complete) times alpha
      uint32_t orow[64];
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        tmem_ld64_wait(tmem + lane_base + L::kColO + h * 64, orow);
#pragma unroll
        for (int i = 0; i < 64; ++i) orow[i] = __float_as_uint(__uint_as_float(orow[i]) * alpha);
        tmem_st64(tmem + lane_base + L::kColO + h * 64, orow);
      }
      tmem_st_wait();
    }
    l = l * alpha + rs;
    m = m_new;
    // P (TF32) as the K-major A operand of O += P V
#pragma unroll
    for (int c = 0; c < kTK; c += 4)
      *reinterpret_cast<float4*>(smem + L::kOffP + (c >> 5) * L::kPChunk + swz(t, c)) =
          tf32_rna4(make_float4(s[c], s[c + 1], s[c + 2], s[c + 3]));
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (t == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_tf32(kTM, D);
#pragma unroll
      for (int kk = 0; kk < kTK / 8; ++kk)
        mma_tf32(tmem + L::kColO,
                 sdesc_sw128(sbase + L::kOffP + (kk >> 2) * L::kPChunk + (kk & 3) * 32, 16, 1024),
                 sdesc_sw128(sbase + L::kOffVt + (kk >> 2) * L::kVtChunk + (kk & 3) * 32, 16, 1024),
                 idesc, (j > 0 || kk > 0) ? 1u : 0u);
      tc_commit(bar_pv);
    }
  }
  if (ok && n_tiles > 0) ok = wait_bounded(bar_pv, (n_tiles - 1) & 1, wc, 3);
  ok = __syncthreads_and(ok);
  if (ok) {
    // (every lane loads: tcgen05.ld is warp-wide; rows past N store nothing)
    tc_fence_after();
    const float inv_l = 1.0f / l;
    float* ob = o + bh * size_t(N) * D + size_t(row) * D;
    uint32_t orow[64];
#pragma unroll
    for (int h = 0; h < D / 64; ++h) {
      tmem_ld64_wait(tmem + lane_base + L::kColO + h * 64, orow);
      if (row < N) {
#pragma unroll
        for (int i = 0; i < 64; i += 4)
          *reinterpret_cast<float4*>(ob + h * 64 + i) =
              make_float4(__uint_as_float(orow[i]) * inv_l, __uint_as_float(orow[i + 1]) * inv_l,
                          __uint_as_float(orow[i + 2]) * inv_l, __uint_as_float(orow[i + 3]) * inv_l);
      }
    }
    if (row < N) lse[bh * size_t(N) + row] = (m + lg2_approx(l)) * kLn2T;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

template <int D, bool CAUSAL>
fa_status launch_t(const float* q, const float* k, const float* v, float* o, float* lse, int BH,
                   int N, float scale, const LaunchCtx& ctx) {
  const int smem = TLayout<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(fwd_tf32_kernel<D, CAUSAL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(fwd_tf32)");
  dim3 grid((N + kTM - 1) / kTM, BH);
  {
    ProfileScope prof(KID_FWD_F32, ctx.stream);
    fwd_tf32_kernel<D, CAUSAL><<<grid, kTThreads, smem, ctx.stream>>>(
        q, k, v, o, lse, N, scale * 1.4426950408889634f, ctx.status_word, ctx.wait_limit_ns);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fwd_tf32 kernel launch");
  return FA_OK;
}

}  // namespace

fa_status launch_fwd_tf32(const float* q, const float* k, const float* v, float* o, float* lse,
                          int B, int H, int N, int d, float scale, bool causal,
                          const LaunchCtx& ctx) {
  const int BH = B * H;
  if (BH > 65535) {
    set_last_error("fa_fwd_f32: B*H = %d exceeds 65535", BH);
    return FA_ERR_UNSUPPORTED;
  }
  if (d == 128)
    return causal ? launch_t<128, true>(q, k, v, o, lse, BH, N, scale, ctx)
                  : launch_t<128, false>(q, k, v, o, lse, BH, N, scale, ctx);
  return causal ? launch_t<64, true>(q, k, v, o, lse, BH, N, scale, ctx)
                : launch_t<64, false>(q, k, v, o, lse, BH, N, scale, ctx);
}

}  // namespace fa
