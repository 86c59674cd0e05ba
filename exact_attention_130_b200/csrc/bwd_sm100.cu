// bwd_sm100.cu -- attention backward by recomputation, B200 (sm_100a).
//
// What it computes ("Bellek Duvarinin Fizigi", section "Geri Yayilim"): the
// forward saved only O and the per-row log-sum-exp L. The backward rebuilds
// every block of P on chip as P = exp(S - L) and forms
//     dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),  dS = P * (dP - D),
//     dQ = scale * dS K,  dK = scale * dS^T Q,
// so neither S nor P is ever stored.
//
// Three kernels on the caller's stream:
//  1. bwd_pre   D_i = sum_c dO_ic O_ic (fp32), the saved LSE converted to
//               base 2, both padded to a multiple of 128 rows (padding rows get
//               LSE = +inf, so their P is exactly 0), and the fp32 dQ
//               accumulator zeroed.
//  2. bwd_main  one CTA per (batch*head, 128-key tile); the K and V tiles stay
//               in shared memory while the Q and dO tiles of every query tile
//               that can see these keys stream past (under the causal mask,
//               query tiles below the diagonal only). Per query tile:
//                 S^T  = K Q^T      (tcgen05, TMEM)
//                 dP^T = V dO^T     (tcgen05, TMEM)
//                 P^T  = 2^(S^T scale log2e - L2), dS^T = scale P^T (dP^T - D)
//                        (one TMEM lane = one key row; P^T goes back to TMEM
//                        as bf16, dS^T to shared memory in the 128-byte
//                        swizzled layout)
//                 dV  += P^T dO     (A from TMEM)
//                 dK  += dS^T Q     (A = dS^T, K-major)
//                 dQ_i = dS K       (A = the same dS^T buffer read MN-major)
//               dV and dK accumulate in TMEM for the whole key tile; dQ_i is
//               added into the fp32 accumulator with vector atomics by four
//               dedicated warps.
//  3. bwd_post  dQ = bf16(accumulator).
// The scale is folded into dS before it is rounded to bf16, so dK and dQ need
// no further scaling.
//
// Warp roles of bwd_main (320 threads):
//   warps 0-3  compute (exp, dS) and the dK/dV epilogue
//   warp  4    TMA producer        warp 5  MMA issuer
//   warps 6-9  dQ readers (TMEM -> atomics into the accumulator)
// TMEM: S^T | dP^T (later dQ_i) | dV | dK = 512 columns at d = 128.
#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kBlk = 128;  // keys per CTA and queries per step
constexpr int kThreads = 320;
constexpr int kLoadWarp = 4;
constexpr int kMmaWarp = 5;
constexpr float kLog2e = 1.4426950408889634f;

enum : int {
  B_KV_FULL = 0,
  B_Q_FULL = 1,    // +stage (2)
  B_Q_EMPTY = 3,   // +stage (2)
  B_S_FULL = 5,
  B_DP_FULL = 6,
  B_P_READY = 7,
  B_DQ_FULL = 8,
  B_DQ_EMPTY = 9,
  B_ACC_DONE = 10,
  B_DRAIN = 11,
  B_COUNT = 12
};

template <int D>
struct BwdLayout {
  static constexpr int kSub = D / 64;
  static constexpr int kSubBytes = 128 * 128;
  static constexpr int kTileBytes = kSub * kSubBytes;  // 128 rows x D bf16
  static constexpr int kStages = 2;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;                       // + s * tile
  static constexpr int kOffDO = kOffQ + kStages * kTileBytes;        // + s * tile
  static constexpr int kOffDS = kOffDO + kStages * kTileBytes;       // 128 x 128 bf16
  static constexpr int kOffBar = kOffDS + 2 * kSubBytes;
  static constexpr int kOffMisc = kOffBar + 8 * B_COUNT;
  static constexpr int kSmemBytes = kOffMisc + 32 + 1024;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
};

struct BwdParams {
  const uint16_t* o;
  const uint16_t* dO;
  const float* lse;
  float* dq_acc;   // [BH, N, D] fp32
  float* lse2;     // [BH, Np] base-2 LSE, +inf in padding rows
  float* dvec;     // [BH, Np] D, 0 in padding rows
  uint16_t* dq;
  uint16_t* dk;
  uint16_t* dv;
  int N, Np, BH, n_tiles;
  float scale, scale_log2;
  unsigned int* status;
  unsigned long long limit_ns;
};

__device__ __forceinline__ float bf16f(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// --------------------------------------------------------------------------
// 1. preprocess: one warp per row
// --------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const BwdParams p) {
  constexpr int kPer = D / 32;
  const int warp = (blockIdx.x * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long total = (long long)p.BH * p.Np;
  if (warp >= total) return;
  const int bh = warp / p.Np;
  const int row = warp % p.Np;
  float dsum = 0.f;
  if (row < p.N) {
    const size_t base = (size_t(bh) * p.N + row) * D + lane * kPer;
    if constexpr (kPer == 4) {
      const uint2 a = *reinterpret_cast<const uint2*>(p.o + base);
      const uint2 b = *reinterpret_cast<const uint2*>(p.dO + base);
      dsum = bf16f(a.x & 0xffffu) * bf16f(b.x & 0xffffu) + bf16f(a.x >> 16) * bf16f(b.x >> 16) +
             bf16f(a.y & 0xffffu) * bf16f(b.y & 0xffffu) + bf16f(a.y >> 16) * bf16f(b.y >> 16);
      *reinterpret_cast<float4*>(p.dq_acc + base) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      const uint32_t a = *reinterpret_cast<const uint32_t*>(p.o + base);
      const uint32_t b = *reinterpret_cast<const uint32_t*>(p.dO + base);
      dsum = bf16f(a & 0xffffu) * bf16f(b & 0xffffu) + bf16f(a >> 16) * bf16f(b >> 16);
      *reinterpret_cast<float2*>(p.dq_acc + base) = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
  }
  if (lane == 0) {
    const size_t o = size_t(bh) * p.Np + row;
    p.dvec[o] = row < p.N ? dsum : 0.f;
    p.lse2[o] = row < p.N ? p.lse[size_t(bh) * p.N + row] * kLog2e : INFINITY;
  }
}

// --------------------------------------------------------------------------
// 2. main kernel
// --------------------------------------------------------------------------
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto BAR = [&](int i) -> uint32_t { return sbase + L::kOffBar + 8u * uint32_t(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // key tiles with the most query tiles first (under the causal mask the
  // lowest key tiles see every query tile), every head of a level together
  const int jt = blockIdx.x / p.BH;  // key tile
  const int bh = blockIdx.x % p.BH;
  const int i0 = CAUSAL ? jt : 0;
  const int n_it = p.n_tiles - i0;

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_KV_FULL), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(BAR(B_Q_FULL + s), 1);
      mbar_init(BAR(B_Q_EMPTY + s), 1);
    }
    mbar_init(BAR(B_S_FULL), 1);
    mbar_init(BAR(B_DP_FULL), 1);
    mbar_init(BAR(B_P_READY), 4);
    mbar_init(BAR(B_DQ_FULL), 1);
    mbar_init(BAR(B_DQ_EMPTY), 4);
    mbar_init(BAR(B_ACC_DONE), 1);
    mbar_init(BAR(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.status, p.limit_ns, KID_BWD};

  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int q_cnt[2] = {0, 0};
      mbar_arrive_expect_tx(BAR(B_KV_FULL), 2 * L::kTileBytes);
      for (int c = 0; c < L::kSub; ++c) {
        tma_load_3d(sbase + L::kOffK + c * L::kSubBytes, &tmK, BAR(B_KV_FULL), c * 64, jt * kBlk, bh);
        tma_load_3d(sbase + L::kOffV + c * L::kSubBytes, &tmV, BAR(B_KV_FULL), c * 64, jt * kBlk, bh);
      }
      for (int it = 0; it < n_it; ++it) {
        const int s = it & 1;
        if (!wait_bounded(BAR(B_Q_EMPTY + s), ((it >> 1) & 1) ^ 1, wc, 1)) break;
        const int i = i0 + it;
        mbar_arrive_expect_tx(BAR(B_Q_FULL + s), 2 * L::kTileBytes);
        for (int c = 0; c < L::kSub; ++c) {
          tma_load_3d(sbase + L::kOffQ + s * L::kTileBytes + c * L::kSubBytes, &tmQ,
                      BAR(B_Q_FULL + s), c * 64, i * kBlk, bh);
          tma_load_3d(sbase + L::kOffDO + s * L::kTileBytes + c * L::kSubBytes, &tmDO,
                      BAR(B_Q_FULL + s), c * 64, i * kBlk, bh);
        }
        ++q_cnt[s];
      }
      if (*abort_flag) {
        wait_bounded(BAR(B_KV_FULL), 0, wc, 2, true);
        for (int s = 0; s < 2; ++s)
          if (q_cnt[s]) wait_bounded(BAR(B_Q_FULL + s), (q_cnt[s] - 1) & 1, wc, 2, true);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_bf16(kBlk, kBlk, false, false);  // S^T, dP^T
      constexpr uint32_t id_kmn = idesc_bf16(kBlk, D, false, true);     // dV, dK
      constexpr uint32_t id_mnmn = idesc_bf16(kBlk, D, true, true);     // dQ
      const uint32_t sK = sbase + L::kOffK, sV = sbase + L::kOffV, sDS = sbase + L::kOffDS;
      bool ok = wait_bounded(BAR(B_KV_FULL), 0, wc, 10);
      for (int it = 0; ok && it < n_it; ++it) {
        const int s = it & 1;
        const uint32_t sQ = sbase + L::kOffQ + s * L::kTileBytes;
        const uint32_t sDO = sbase + L::kOffDO + s * L::kTileBytes;
        ok = wait_bounded(BAR(B_Q_FULL + s), (it >> 1) & 1, wc, 11);
        if (!ok) break;
        tc_fence_after();
        // S^T = K Q^T  (A: K tile, B: Q tile, both K-major)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kSubBytes + (kk & 3) * 32;
          mma_ss(tmem + L::kColS, sdesc_sw128(sK + off, 16, 1024), sdesc_sw128(sQ + off, 16, 1024),
                 id_kk, kk > 0);
        }
        tc_commit(BAR(B_S_FULL));
        // dP^T reuses the columns dQ_{i-1} occupied: wait for its readers
        if (it > 0) {
          ok = wait_bounded(BAR(B_DQ_EMPTY), (it - 1) & 1, wc, 12);
          if (!ok) break;
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kSubBytes + (kk & 3) * 32;
          mma_ss(tmem + L::kColDP, sdesc_sw128(sV + off, 16, 1024), sdesc_sw128(sDO + off, 16, 1024),
                 id_kk, kk > 0);
        }
        tc_commit(BAR(B_DP_FULL));
        ok = wait_bounded(BAR(B_P_READY), it & 1, wc, 13);
        if (!ok) break;
        tc_fence_after();
        // dV += P^T dO   (A: P^T bf16 in TMEM over the S columns; B: dO MN-major)
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk)
          mma_ts(tmem + L::kColDV, tmem + L::kColS + kk * 8,
                 sdesc_sw128(sDO + kk * 2048, L::kSubBytes, 1024), id_kmn, (it > 0 || kk > 0));
        // dK += dS^T Q   (A: dS^T K-major in smem; B: Q MN-major)
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kSubBytes + (kk & 3) * 32;
          mma_ss(tmem + L::kColDK, sdesc_sw128(sDS + off, 16, 1024),
                 sdesc_sw128(sQ + kk * 2048, L::kSubBytes, 1024), id_kmn, (it > 0 || kk > 0));
        }
        // dQ_i = dS K    (A: the dS^T buffer read MN-major; B: K MN-major)
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk)
          mma_ss(tmem + L::kColDP, sdesc_sw128(sDS + kk * 2048, L::kSubBytes, 1024),
                 sdesc_sw128(sK + kk * 2048, L::kSubBytes, 1024), id_mnmn, kk > 0);
        tc_commit(BAR(B_DQ_FULL));
        tc_commit(BAR(B_Q_EMPTY + s));
      }
      tc_commit(BAR(B_ACC_DONE));
      tc_commit(BAR(B_DRAIN));
      wait_bounded(BAR(B_DRAIN), 0, wc, 14, true);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ compute warps
    const int r = warp * 32 + lane;  // key row inside the tile
    const int key = jt * kBlk + r;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t tS = tmem + lane_base + L::kColS;
    const uint32_t tDP = tmem + lane_base + L::kColDP;
    const float c = p.scale_log2;
    uint8_t* ds_row = smem + L::kOffDS + r * 128;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int i = i0 + it;
      const float* l2 = p.lse2 + size_t(bh) * p.Np + size_t(i) * kBlk;
      const float* dv = p.dvec + size_t(bh) * p.Np + size_t(i) * kBlk;
      ok = wait_bounded(BAR(B_S_FULL), it & 1, wc, 20);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld128_wait(tS, sr);
      // P^T row: 2^(s c - L2_q); zero for masked entries
      const bool row_valid = key < p.N;
      const int qlim = (CAUSAL && i == jt) ? r : 0;  // queries q < qlim are masked
      float pr[128];
#pragma unroll
      for (int q4 = 0; q4 < 32; ++q4) {
        const float4 lv = __ldg(reinterpret_cast<const float4*>(l2) + q4);
        const float lq[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int q = 4 * q4 + e;
          const float x = ex2_approx(fmaf(__uint_as_float(sr[q]), c, -lq[e]));
          pr[q] = (row_valid && q >= qlim) ? x : 0.f;
        }
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {  // P^T (bf16) over the first 64 S columns
        uint32_t pk[32];
#pragma unroll
        for (int q = 0; q < 32; ++q)
          pk[q] = pack_bf16x2(pr[64 * half + 2 * q], pr[64 * half + 2 * q + 1]);
        tmem_st32(tS + 32 * half, pk);
      }
      ok = wait_bounded(BAR(B_DP_FULL), it & 1, wc, 21);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // dS^T = scale * P^T (dP^T - D), written to smem in the 128B-swizzled
      // K-major layout: row r, 16-byte chunk ch of group g at
      // g*16KB + r*128 + ((ch ^ (r%8)) * 16)
#pragma unroll
      for (int ch4 = 0; ch4 < 4; ++ch4) {  // 32 queries per TMEM load
        uint32_t dr[32];
        tmem_ld32_wait(tDP + ch4 * 32, dr);
        float dd[32];
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const float4 dvv = __ldg(reinterpret_cast<const float4*>(dv) + ch4 * 8 + q4);
          dd[4 * q4 + 0] = dvv.x;
          dd[4 * q4 + 1] = dvv.y;
          dd[4 * q4 + 2] = dvv.z;
          dd[4 * q4 + 3] = dvv.w;
        }
#pragma unroll
        for (int ck = 0; ck < 4; ++ck) {  // 8 queries = one 16-byte chunk
          const int qb = ch4 * 32 + ck * 8;
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int q0 = qb + 2 * e;
            const float a = pr[q0] * p.scale * (__uint_as_float(dr[ck * 8 + 2 * e]) - dd[ck * 8 + 2 * e]);
            const float b = pr[q0 + 1] * p.scale *
                            (__uint_as_float(dr[ck * 8 + 2 * e + 1]) - dd[ck * 8 + 2 * e + 1]);
            w[e] = pack_bf16x2(a, b);
          }
          const int g = qb >> 6;
          const int chunk = (qb & 63) >> 3;
          *reinterpret_cast<uint4*>(ds_row + g * L::kSubBytes + ((chunk ^ (r & 7)) << 4)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      tmem_st_wait();
      fence_proxy_async_smem();  // make the dS^T stores visible to the tensor core
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_P_READY));
    }
    // epilogue: dV and dK rows of this key tile
    if (ok) {
      ok = wait_bounded(BAR(B_ACC_DONE), 0, wc, 22);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const uint32_t tDV = tmem + lane_base + L::kColDV;
      const uint32_t tDK = tmem + lane_base + L::kColDK;
      const size_t gro = (size_t(bh) * p.N + key) * D;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t src = which ? tDK : tDV;
        uint16_t* dst = (which ? p.dk : p.dv) + gro;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t v[32];
          tmem_ld32_wait(src + ch * 32, v);
          if (key < p.N) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(v[8 * v4 + 0]), __uint_as_float(v[8 * v4 + 1]));
              w.y = pack_bf16x2(__uint_as_float(v[8 * v4 + 2]), __uint_as_float(v[8 * v4 + 3]));
              w.z = pack_bf16x2(__uint_as_float(v[8 * v4 + 4]), __uint_as_float(v[8 * v4 + 5]));
              w.w = pack_bf16x2(__uint_as_float(v[8 * v4 + 6]), __uint_as_float(v[8 * v4 + 7]));
              *reinterpret_cast<uint4*>(dst + ch * 32 + 8 * v4) = w;
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ dQ readers (warps 6-9)
    const int quad = warp & 3;         // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;    // query row inside the tile
    const uint32_t tDQ = tmem + (uint32_t(quad * 32) << 16) + L::kColDP;
    for (int it = 0; it < n_it; ++it) {
      const int q = (i0 + it) * kBlk + r;
      bool ok = wait_bounded(BAR(B_DQ_FULL), it & 1, wc, 30);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float* dst = p.dq_acc + (size_t(bh) * p.N + q) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t v[32];
        tmem_ld32_wait(tDQ + ch * 32, v);
        if (q < p.N) {
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            atomicAdd(reinterpret_cast<float4*>(dst + ch * 32 + 4 * v4),
                      make_float4(__uint_as_float(v[4 * v4]), __uint_as_float(v[4 * v4 + 1]),
                                  __uint_as_float(v[4 * v4 + 2]), __uint_as_float(v[4 * v4 + 3])));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_DQ_EMPTY));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// --------------------------------------------------------------------------
// 3. dQ accumulator -> bf16
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_post_kernel(const float* __restrict__ acc,
                                                       uint16_t* __restrict__ dq, size_t n4) {
  const size_t i = size_t(blockIdx.x) * 256 + threadIdx.x;
  if (i >= n4) return;
  const float4 v = reinterpret_cast<const float4*>(acc)[i];
  uint2 w;
  w.x = pack_bf16x2(v.x, v.y);
  w.y = pack_bf16x2(v.z, v.w);
  reinterpret_cast<uint2*>(dq)[i] = w;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

template <int D, bool CAUSAL>
fa_status launch_main(const CUtensorMap* maps, const BwdParams& p, const LaunchCtx& ctx) {
  auto kern = bwd_main_kernel<D, CAUSAL>;
  const int smem = BwdLayout<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(bwd)");
  const unsigned grid = unsigned(p.n_tiles) * unsigned(p.BH);
  {
    ProfileScope prof(KID_BWD, ctx.stream);
    kern<<<grid, kThreads, smem, ctx.stream>>>(maps[0], maps[1], maps[2], maps[3], p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "bwd main kernel launch");
  return FA_OK;
}

}  // namespace

size_t bwd_workspace_bytes(int B, int H, int N, int d) {
  const size_t bh = size_t(B) * H;
  const size_t np = (size_t(N) + kBlk - 1) / kBlk * kBlk;
  return align256(bh * N * d * 4) + 2 * align256(bh * np * 4);
}

fa_status launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                     float scale, bool causal, void* workspace, const LaunchCtx& ctx) {
  const int BH = B * H;
  if (BH > 65535) {
    set_last_error("fa_bwd: B*H = %d exceeds 65535", BH);
    return FA_ERR_UNSUPPORTED;
  }
  BwdParams p;
  p.o = static_cast<const uint16_t*>(o);
  p.dO = static_cast<const uint16_t*>(dO);
  p.lse = lse;
  p.N = N;
  p.n_tiles = (N + kBlk - 1) / kBlk;
  p.Np = p.n_tiles * kBlk;
  p.BH = BH;
  char* ws = static_cast<char*>(workspace);
  p.dq_acc = reinterpret_cast<float*>(ws);
  p.lse2 = reinterpret_cast<float*>(ws + align256(size_t(BH) * N * d * 4));
  p.dvec = reinterpret_cast<float*>(ws + align256(size_t(BH) * N * d * 4) +
                                    align256(size_t(BH) * p.Np * 4));
  p.dq = static_cast<uint16_t*>(dq);
  p.dk = static_cast<uint16_t*>(dk);
  p.dv = static_cast<uint16_t*>(dv);
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.status = ctx.status_word;
  p.limit_ns = ctx.wait_limit_ns;

  // 1. preprocess
  {
    const long long warps = (long long)BH * p.Np;
    const long long blocks = (warps * 32 + 255) / 256;
    ProfileScope prof(KID_BWD_PRE, ctx.stream);
    if (d == 128)
      bwd_pre_kernel<128><<<unsigned(blocks), 256, 0, ctx.stream>>>(p);
    else
      bwd_pre_kernel<64><<<unsigned(blocks), 256, 0, ctx.stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "bwd preprocess launch");
  }
  // 2. main
  CUtensorMap maps[4];
  const void* srcs[4] = {q, k, v, dO};
  for (int m = 0; m < 4; ++m) {
    fa_status st = make_tmap_3d(&maps[m], srcs[m], true, d, N, BH, 64, 128, true);
    if (st != FA_OK) return st;
  }
  fa_status st;
  if (d == 128)
    st = causal ? launch_main<128, true>(maps, p, ctx) : launch_main<128, false>(maps, p, ctx);
  else
    st = causal ? launch_main<64, true>(maps, p, ctx) : launch_main<64, false>(maps, p, ctx);
  if (st != FA_OK) return st;
  // 3. dQ to bf16
  {
    const size_t n4 = size_t(BH) * N * d / 4;
    ProfileScope prof(KID_BWD_POST, ctx.stream);
    bwd_post_kernel<<<unsigned((n4 + 255) / 256), 256, 0, ctx.stream>>>(p.dq_acc, p.dq, n4);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "bwd dQ conversion launch");
  }
  return FA_OK;
}

}  // namespace fa
