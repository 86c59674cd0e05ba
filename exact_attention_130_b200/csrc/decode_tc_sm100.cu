// decode_tc_sm100.cu -- split-KV decode of a paged KV cache with large groups
// of query heads on the tensor cores ("Bellek Duvarinin Fizigi", sections
// "Duvarin Otesi" -- the KV cache and the grouped-query and paged layouts it
// names -- and "Decode Asamasi: Flash-Decoding").
//
// What it computes is the chunk partials of the split-KV decode: for
// sequence b, KV head hk and chunk c of the cache positions, every query head
// h of the group of hk (h / (Hq / Hkv) = hk) gets o_c = softmax(s) V over the
// chunk's keys and lse_c = log2 sum exp2(s * scale log2 e) (base 2), with
// s_t = q_h . k_t; decode_merge_kernel (decode_sm100.cu) merges the chunks
// by log-sum-exp.
//
// Why tensor cores: the G query heads of a KV head read the same K and V
// rows. On the CUDA cores every row and head costs two dot products per lane
// and a shuffle reduction, which is issue-bound well below HBM bandwidth for
// G >= 4. Here the heads are the M rows of tcgen05.mma (padded with zero
// rows to M = 128; the tensor pipe has far more throughput than a stream from
// HBM needs):
//  * one CTA per (chunk, KV head, sequence); the chunk is walked in tiles of
//    64 keys brought by TMA straight from their pages (a 3-D tensor map over
//    [pages x KV heads, page rows, d], 128-byte swizzle), two stages for K
//    and two for V;
//  * S = Q K^T (M = 128, N = 64, Q written into TMEM by the softmax warps,
//    zero rows past the group), the online softmax of "Online Softmax" on the
//    G valid rows (one warp per 32 heads, one TMEM lane per head), P (bf16)
//    written over the first 32 columns of S, O += P V (N = d) in TMEM;
//    TMEM = S | O | Q, 256 columns, and three 32 KB K/V stages, so two CTAs
//    share an SM and keep ~128 KB of loads in flight per SM;
//  * rows of a page past the sequence length are loaded with the tile: their
//    scores get -inf and, in the sequence's last tile, the softmax warp zeroes
//    their V rows in shared memory before handing over P (a zero probability
//    times a NaN or infinite stale value would still poison O). Runs of rows
//    wholly past the length are not loaded;
//  * every page index is checked against the pool before its rows are read
//    (an index outside it is reported in the device status word);
//  * every mbarrier wait is bounded in time.
#include <cfloat>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kTileKeys = 64;
constexpr int kTcStages = 3;
constexpr int kSoftmaxWarps = 4;  // up to 128 query heads per KV head
constexpr int kLoadWarpTc = 4;
constexpr int kMmaWarpTc = 5;
constexpr int kTcThreads = 32 * 6;
constexpr float kRescaleThresholdTc = 8.0f;

enum : int {
  T_Q_READY = 0,  // the softmax warps have written the Q tile into TMEM (4 warps)
  T_S_FULL = 1,
  T_P_FULL = 2,   // the active softmax warps have stored P
  T_O_FULL = 3,
  T_DRAIN = 4,
  T_K_FULL = 5,
  T_K_EMPTY = T_K_FULL + kTcStages,
  T_V_FULL = T_K_EMPTY + kTcStages,
  T_V_EMPTY = T_V_FULL + kTcStages,
  T_COUNT = T_V_EMPTY + kTcStages
};

template <int D>
struct TcLayout {
  static constexpr int kSub = D / 64;                 // 128-byte column groups of a row
  static constexpr int kKvSubBytes = kTileKeys * 128; // 64 rows x 128 bytes
  static constexpr int kKvTileBytes = kSub * kKvSubBytes;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTcStages * kKvTileBytes;
  static constexpr int kOffBar = kOffV + kTcStages * kKvTileBytes;
  static constexpr int kOffMisc = kOffBar + 8 * T_COUNT;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
  // TMEM: S (64 fp32 columns; P bf16 over its first 32) | O (D) | Q (bf16, D/2)
  static constexpr uint32_t kColS = 0, kColO = kTileKeys, kColQ = kTileKeys + D;
  static constexpr uint32_t kTmemCols = 256;
  static_assert(kColQ + D / 2 <= kTmemCols, "TMEM columns");
};

struct TcParams {
  const uint16_t* q;      // [B, Hq, D]
  const int* seqlens;
  const int* table;       // [B, max_pages]
  float* part_o;          // [B, Hq, C, D]
  float* part_lse;        // [B, Hq, C], base 2
  int Hq, Hkv, group, C;
  int page, max_pages, num_pages, Lmax;
  float scale_log2;
  unsigned int* status;
  unsigned long long limit_ns;
  int debug_skip;
};

template <int D>
__global__ void __launch_bounds__(kTcThreads)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const TcParams p) {
  using L = TcLayout<D>;
  // the merge kernel, launched as a programmatic dependent, may be scheduled
  // now: it waits for this grid's completion before reading anything
  grid_dependents_launch();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * uint32_t(i); };

  const int c = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.group;
  const int nsw = (G + 31) / 32;  // softmax warps with at least one query head

  int Lb = p.seqlens[b];
  Lb = Lb < 0 ? 0 : (Lb > p.Lmax ? p.Lmax : Lb);
  int chunk = (Lb + p.C - 1) / p.C;
  chunk = (chunk + kTileKeys - 1) / kTileKeys * kTileKeys;  // tiles start on 64-key boundaries
  const int t0 = c * chunk, t1 = min(t0 + chunk, Lb);
  if (t0 >= t1) {  // empty chunk: weight 0 in the merge
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
      const size_t part = (size_t(b) * p.Hq + size_t(hk) * G + e / D) * p.C + c;
      p.part_o[part * D + e % D] = 0.f;
      if (e % D == 0) p.part_lse[part] = -INFINITY;
    }
    return;
  }
  const int n_tiles = (t1 - t0 + kTileKeys - 1) / kTileKeys;

  if (threadIdx.x == 0) {
    mbar_init(BAR(T_Q_READY), kSoftmaxWarps);
    mbar_init(BAR(T_S_FULL), 1);
    mbar_init(BAR(T_P_FULL), nsw);
    mbar_init(BAR(T_O_FULL), 1);
    mbar_init(BAR(T_DRAIN), 1);
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(BAR(T_K_FULL + s), 1);
      mbar_init(BAR(T_K_EMPTY + s), 1);
      mbar_init(BAR(T_V_FULL + s), 1);
      mbar_init(BAR(T_V_EMPTY + s), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarpTc) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  if (warp == kLoadWarpTc && lane == 0) {
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.status, p.limit_ns, KID_DECODE};

  if (warp == kLoadWarpTc) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // a 64-key tile in runs of rows that each lie in one page (one run for
      // pages of 64 rows or more); runs wholly past the length are skipped
      const int run = p.page < kTileKeys ? p.page : kTileKeys;
      int k_issued[kTcStages] = {}, v_issued[kTcStages] = {};
      bool skip_pending = p.debug_skip && c == 0 && hk == 0 && b == 0;
      bool ok = true;
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kTcStages;
        const uint32_t ph = ((j / kTcStages) & 1) ^ 1;
        const int tb = t0 + j * kTileKeys;
        const int valid = min(kTileKeys, t1 - tb);
        // bytes of the runs that will be loaded (valid page index, not past the length)
        uint32_t bytes = 0;
        for (int r0 = 0; r0 < valid; r0 += run) {
          const int pg = p.table[size_t(b) * p.max_pages + (tb + r0) / p.page];
          if (pg < 0 || pg >= p.num_pages) {
            atomicCAS(p.status, 0u, (unsigned(KID_DECODE) << 16) | (10u << 8) | 2u);
            continue;  // these rows stay unloaded (results undefined, error reported)
          }
          bytes += uint32_t(run) * 128u * L::kSub;
        }
        for (int which = 0; which < 2 && ok; ++which) {
          const int full = which ? T_V_FULL : T_K_FULL;
          const int empty = which ? T_V_EMPTY : T_K_EMPTY;
          ok = wait_bounded(BAR(empty + s), ph, wc, which ? 2 : 1);
          if (!ok) break;
          if (which && skip_pending) {
            skip_pending = false;  // test hook: this V tile never arrives
            continue;
          }
          mbar_arrive_expect_tx(BAR(full + s), bytes);
          const uint32_t dst0 = sbase + (which ? L::kOffV : L::kOffK) + s * L::kKvTileBytes;
          for (int r0 = 0; r0 < valid; r0 += run) {
            const int tp = tb + r0;
            const int pg = p.table[size_t(b) * p.max_pages + tp / p.page];
            if (pg < 0 || pg >= p.num_pages) continue;
            for (int cs = 0; cs < L::kSub; ++cs)
              tma_load_3d(dst0 + cs * L::kKvSubBytes + r0 * 128, which ? &tmV : &tmK, BAR(full + s),
                          cs * 64, tp % p.page, pg * p.Hkv + hk);
          }
          (which ? v_issued : k_issued)[s] += 1;
        }
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA exits
        for (int s = 0; s < kTcStages; ++s) {
          if (k_issued[s]) wait_bounded(BAR(T_K_FULL + s), (k_issued[s] - 1) & 1, wc, 3, true);
          if (v_issued[s]) wait_bounded(BAR(T_V_FULL + s), (v_issued[s] - 1) & 1, wc, 3, true);
        }
      }
    }
  } else if (warp == kMmaWarpTc) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, kTileKeys, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
      const uint32_t tS = tmem + L::kColS, tO = tmem + L::kColO;
      bool ok = wait_bounded(BAR(T_Q_READY), 0, wc, 10);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kTcStages;
        const uint32_t ph = (j / kTcStages) & 1;
        ok = wait_bounded(BAR(T_K_FULL + s), ph, wc, 11);
        if (!ok) break;
        tc_fence_after();
        // S = Q K^T; issued after P V(j-1), which read P(j-1) from the same columns
        const uint32_t kb = sbase + L::kOffK + s * L::kKvTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * L::kKvSubBytes + (kk & 3) * 32;
          mma_ts(tS, tmem + L::kColQ + kk * 8, sdesc_sw128(kb + koff, 16, 1024), idesc_qk,
                 kk > 0 ? 1u : 0u);
        }
        tc_commit(BAR(T_S_FULL));
        tc_commit(BAR(T_K_EMPTY + s));
        ok = wait_bounded(BAR(T_P_FULL), j & 1, wc, 12);
        if (!ok) break;
        ok = wait_bounded(BAR(T_V_FULL + s), ph, wc, 13);
        if (!ok) break;
        tc_fence_after();
        // O (+)= P V: P (bf16) from the first 32 columns of S, V MN-major
        const uint32_t vb = sbase + L::kOffV + s * L::kKvTileBytes;
#pragma unroll
        for (int kk = 0; kk < kTileKeys / 16; ++kk)
          mma_ts(tO, tS + kk * 8, sdesc_sw128(vb + kk * 16 * 128, L::kKvSubBytes, 1024), idesc_pv,
                 (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(BAR(T_V_EMPTY + s));
        if (j + 1 == n_tiles) tc_commit(BAR(T_O_FULL));
      }
      // every MMA issued above must be finished before TMEM is released
      tc_commit(BAR(T_DRAIN));
      wait_bounded(BAR(T_DRAIN), 0, wc, 16, true);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int r = warp * 32 + lane;  // query head hk * G + r of this CTA, TMEM lane r
    const bool head = r < G;
    // Q tile into TMEM as the A operand of Q K^T (lane r = row r, packed
    // bf16 pairs of d in consecutive columns): head rows from q, the other
    // rows zero
    {
      const uint16_t* qrow = p.q + (size_t(b) * p.Hq + size_t(hk) * G + (head ? r : 0)) * D;
      uint32_t qw[D / 2];
#pragma unroll
      for (int k4 = 0; k4 < D / 8; ++k4) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (head) v = *reinterpret_cast<const uint4*>(qrow + k4 * 8);
        qw[4 * k4 + 0] = v.x;
        qw[4 * k4 + 1] = v.y;
        qw[4 * k4 + 2] = v.z;
        qw[4 * k4 + 3] = v.w;
      }
      const uint32_t tQ = tmem + (uint32_t(warp * 32) << 16) + L::kColQ;
      if constexpr (D == 128) {
        tmem_st64(tQ, qw);
      } else {
        tmem_st32(tQ, qw);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(T_Q_READY));
    }
    if (warp < nsw) {
      const uint32_t lane_base = uint32_t(warp * 32) << 16;
      const uint32_t tS = tmem + lane_base + L::kColS, tO = tmem + lane_base + L::kColO;
      const float cl = p.scale_log2;
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < n_tiles; ++j) {
        const int tb = t0 + j * kTileKeys;
        const int valid = min(kTileKeys, t1 - tb);
        ok = wait_bounded(BAR(T_S_FULL), j & 1, wc, 20);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld64_wait(tS, sr);
        float s[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) s[i] = (i < valid) ? __uint_as_float(sr[i]) : -INFINITY;
        float mx[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) mx[k] = fmaxf(s[k], s[k + 4]);
#pragma unroll
        for (int i = 8; i < 64; i += 8) {
#pragma unroll
          for (int k = 0; k < 4; ++k) mx[k] = max3f(mx[k], s[i + k], s[i + k + 4]);
        }
        const float m_new = fmaxf(m, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * cl);
        if (j == 0) {
          m = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m + kRescaleThresholdTc)) {
          // O~ holds the sum through tile j-1 (that P V finished before S(j),
          // which was issued after it): multiply it by 2^(m_old - m_new)
          const float alpha = ex2_approx(m - m_new);
          m = m_new;
          l *= alpha;
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t orow[32];
            tmem_ld32_wait(tO + ch * 32, orow);
#pragma unroll
            for (int i = 0; i < 32; ++i) orow[i] = __float_as_uint(__uint_as_float(orow[i]) * alpha);
            tmem_st32(tO + ch * 32, orow);
          }
        }
        float sum = 0.f;
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = ex2_approx(fmaf(s[2 * i], cl, -m));
          const float p1 = ex2_approx(fmaf(s[2 * i + 1], cl, -m));
          sum += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        if (valid < kTileKeys && warp == 0) {
          // the sequence's last tile: zero the V rows past its length before
          // the P V MMA reads them (the tile's V copy must have landed)
          const int s_idx = j % kTcStages;
          ok = wait_bounded(BAR(T_V_FULL + s_idx), (j / kTcStages) & 1, wc, 21);
          if (ok) {
            uint8_t* vt = smem + L::kOffV + s_idx * L::kKvTileBytes;
            for (int e = lane; e < (kTileKeys - valid) * 8 * L::kSub; e += 32) {
              const int row = valid + e / (8 * L::kSub), rest = e % (8 * L::kSub);
              *reinterpret_cast<uint4*>(vt + (rest / 8) * L::kKvSubBytes + row * 128 + (rest % 8) * 16) =
                  make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
          }
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tmem_st32(tS, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(T_P_FULL));
        l += sum;
      }
      if (ok) {
        ok = wait_bounded(BAR(T_O_FULL), 0, wc, 22);
        ok = __all_sync(0xffffffffu, ok);
      }
      if (ok) {
        tc_fence_after();
        const float inv_l = 1.0f / l;
        const size_t part = (size_t(b) * p.Hq + size_t(hk) * G + (head ? r : 0)) * p.C + c;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t orow[32];
          tmem_ld32_wait(tO + ch * 32, orow);
          if (head) {
            float4* dst = reinterpret_cast<float4*>(p.part_o + part * D + ch * 32);
#pragma unroll
            for (int v4 = 0; v4 < 8; ++v4)
              dst[v4] = make_float4(__uint_as_float(orow[4 * v4]) * inv_l, __uint_as_float(orow[4 * v4 + 1]) * inv_l,
                                    __uint_as_float(orow[4 * v4 + 2]) * inv_l,
                                    __uint_as_float(orow[4 * v4 + 3]) * inv_l);
          }
        }
        if (head) p.part_lse[part] = m + lg2_approx(l);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarpTc) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

template <int D>
fa_status launch_tc(const CUtensorMap& mk, const CUtensorMap& mv, const TcParams& p, int B,
                    const LaunchCtx& ctx) {
  auto kern = decode_tc_kernel<D>;
  const int smem = TcLayout<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_tc)");
  dim3 grid(p.C, p.Hkv, B);
  {
    ProfileScope prof(KID_DECODE, ctx.stream);
    kern<<<grid, kTcThreads, smem, ctx.stream>>>(mk, mv, p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode tc kernel launch");
  return FA_OK;
}

}  // namespace

// Chunk partials of the paged decode for groups of query heads on the tensor
// cores; the caller merges them (decode_merge_kernel). Requires
// Hq / Hkv <= 128 and a page of 16, 32 or a multiple of 64 rows.
fa_status launch_decode_paged_tc(const void* q, const void* kpages, const void* vpages,
                                 const int* block_table, const int* seqlens, int B, int Hq,
                                 int Hkv, int num_pages, int page_size, int max_pages, int d,
                                 float scale, int chunks, float* part_o, float* part_lse,
                                 const LaunchCtx& ctx) {
  if (Hq / Hkv > 32 * kSoftmaxWarps) {
    set_last_error("fa_decode_paged: more than %d query heads per KV head", 32 * kSoftmaxWarps);
    return FA_ERR_UNSUPPORTED;
  }
  const uint64_t outer = uint64_t(num_pages) * uint64_t(Hkv);
  const uint32_t box_rows = page_size < kTileKeys ? uint32_t(page_size) : uint32_t(kTileKeys);
  CUtensorMap mk, mv;
  fa_status st;
  if ((st = make_tmap_3d(&mk, kpages, 2, d, page_size, outer, 64, box_rows, 128)) != FA_OK)
    return st;
  if ((st = make_tmap_3d(&mv, vpages, 2, d, page_size, outer, 64, box_rows, 128)) != FA_OK)
    return st;
  TcParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.seqlens = seqlens;
  p.table = block_table;
  p.part_o = part_o;
  p.part_lse = part_lse;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.group = Hq / Hkv;
  p.C = chunks;
  p.page = page_size;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  p.Lmax = max_pages * page_size;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = ctx.status_word;
  p.limit_ns = ctx.wait_limit_ns;
  p.debug_skip = ctx.debug_skip_load == KID_DECODE;
  return d == 128 ? launch_tc<128>(mk, mv, p, B, ctx) : launch_tc<64>(mk, mv, p, B, ctx);
}

}  // namespace fa
