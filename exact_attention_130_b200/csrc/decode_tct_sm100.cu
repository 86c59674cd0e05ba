// decode_tct_sm100.cu -- split-KV decode of a paged KV cache for small groups
// of query heads (up to 16 per KV head, d = 128; the library uses it for 4
// to 8) on the tensor cores, with the keys as the MMA's rows ("Bellek Duvarinin Fizigi", sections "Duvarin
// Otesi" -- the KV cache, grouped-query and paged layouts -- and "Decode
// Asamasi: Flash-Decoding").
//
// What it computes is decode_tc_sm100.cu's: for sequence b, KV head hk and
// chunk c of the cache positions, every query head h of the group of hk gets
// o_c = softmax(s) V over the chunk's keys and lse_c = log2 sum exp2(s scale
// log2 e) (base 2), s_t = q_h . k_t; decode_merge_kernel merges the chunks.
//
// Why transposed: with the G query heads as the M rows (decode_tc_sm100.cu)
// a 128-row MMA carries G useful rows, and each softmax lane spends one
// exponential per key whether its row is a head or padding. Here the 128 keys
// of a tile are the M rows and the heads the N columns (N = 16, zero heads
// past G):
//    S^T = K Q^T    (A = the K tile, K-major in shared memory; B = Q, 16 x d)
//    O^T += V^T P^T (A = the V tile read MN-major; B = P^T, 16 x 128 keys,
//                    written to shared memory by the softmax threads)
// so a softmax thread owns one key (one TMEM lane) and computes G useful
// exponentials per tile; the per-head maximum of a tile is a reduction over
// the 128 lanes (warp shuffles, then the four warps' maxima through shared
// memory, handed over by an mbarrier). The running maximum, the lazy rescale
// of O~ and the row sums are those of "Online Softmax", per head.
//
// Layout per CTA (one per (chunk, KV head, sequence); 192 threads: four
// softmax warps, a TMA warp and an MMA warp): tiles of 128 keys, two K stages
// and one V stage of 32 KB each (so two CTAs share an SM), Q and two P^T
// buffers of 4 KB; TMEM = S^T (two buffers of 16 columns) | O^T (16 columns).
// Page handling as in decode_tc_sm100.cu: a tile comes in runs that each lie
// in one page, every page index is checked before use (a bad one is
// reported), runs wholly past the length are not loaded, and in the
// sequence's last tile the V rows past its length are zeroed in shared memory
// before P V reads them (P = 0 there, but 0 times a stale NaN is NaN). Every
// mbarrier wait is bounded in time.
#include <cfloat>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kKeys = 128;        // keys per tile (the M rows)
constexpr int kNH = 16;           // heads per MMA (N), padded with zero rows
constexpr int kD = 128;
constexpr int kKStg = 2;          // K stages
constexpr int kSmWarps = 4;
constexpr int kLoadWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 32 * 6;
constexpr float kRescale = 8.0f;

enum : int {
  X_Q_READY = 0,   // Q written to shared memory (4 warps)
  X_S_FULL = 1,    // +j%2: S^T(j) in TMEM
  X_S_FREE = 3,    // +j%2: the softmax has loaded S^T(j) (4 warps)
  X_MAX = 5,       // +j%2: the four warps' tile maxima are in shared memory (4 warps)
  X_P_FULL = 7,    // +j%2: P^T(j) written (4 warps)
  X_P_EMPTY = 9,   // +j%2: O^T += V^T P^T(j) finished (P^T buffer free, O^T through tile j)
  X_O_FULL = 11,
  X_LSUM = 12,     // the four warps' row sums are in shared memory (4 warps)
  X_DRAIN = 13,
  X_V_FULL = 14,
  X_V_EMPTY = 15,
  X_K_FULL = 16,
  X_K_EMPTY = X_K_FULL + kKStg,
  X_COUNT = X_K_EMPTY + kKStg
};

struct Layout {
  static constexpr int kSubBytes = kKeys * 128;   // 128 keys x 64 dims
  static constexpr int kTileBytes = 2 * kSubBytes;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKStg * kTileBytes;
  static constexpr int kOffQ = kOffV + kTileBytes;      // [2 dim groups][16 heads][128 B]
  static constexpr int kOffP = kOffQ + 2 * kNH * 128;   // [2 buffers][2 key groups][16 heads][128 B]
  static constexpr int kOffRed = kOffP + 2 * 2 * kNH * 128;  // [2][4 warps][16] maxima
  static constexpr int kOffLred = kOffRed + 2 * kSmWarps * kNH * 4;
  static constexpr int kOffBar = kOffLred + kSmWarps * kNH * 4;
  static constexpr int kOffMisc = kOffBar + 8 * X_COUNT;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(2 * kSmemBytes <= 232448, "two CTAs per SM");
  // TMEM: S^T buffers at 0 and 16, O^T at 32 (fp32, 16 columns each)
  static constexpr uint32_t kColO = 2 * kNH;
  static constexpr uint32_t kTmemCols = 64;
};

struct TctParams {
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

__global__ void __launch_bounds__(kThreads)
    decode_tct_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const TctParams p) {
  using L = Layout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kOffBar;
  float* red = reinterpret_cast<float*>(smem + L::kOffRed);
  float* lred = reinterpret_cast<float*>(smem + L::kOffLred);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * uint32_t(i); };

  const int c = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.group;

  int Lb = p.seqlens[b];
  Lb = Lb < 0 ? 0 : (Lb > p.Lmax ? p.Lmax : Lb);
  int chunk = (Lb + p.C - 1) / p.C;
  chunk = (chunk + kKeys - 1) / kKeys * kKeys;  // tiles start on 128-key boundaries
  const int t0 = c * chunk, t1 = min(t0 + chunk, Lb);
  if (t0 >= t1) {  // empty chunk: weight 0 in the merge
    for (int e = threadIdx.x; e < G * kD; e += blockDim.x) {
      const size_t part = (size_t(b) * p.Hq + size_t(hk) * G + e / kD) * p.C + c;
      p.part_o[part * kD + e % kD] = 0.f;
      if (e % kD == 0) p.part_lse[part] = -INFINITY;
    }
    return;
  }
  const int n_tiles = (t1 - t0 + kKeys - 1) / kKeys;

  if (threadIdx.x == 0) {
    mbar_init(BAR(X_Q_READY), kSmWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(X_S_FULL + i), 1);
      mbar_init(BAR(X_S_FREE + i), kSmWarps);
      mbar_init(BAR(X_MAX + i), kSmWarps);
      mbar_init(BAR(X_P_FULL + i), kSmWarps);
      mbar_init(BAR(X_P_EMPTY + i), 1);
    }
    mbar_init(BAR(X_O_FULL), 1);
    mbar_init(BAR(X_LSUM), kSmWarps);
    mbar_init(BAR(X_DRAIN), 1);
    mbar_init(BAR(X_V_FULL), 1);
    mbar_init(BAR(X_V_EMPTY), 1);
    for (int s = 0; s < kKStg; ++s) {
      mbar_init(BAR(X_K_FULL + s), 1);
      mbar_init(BAR(X_K_EMPTY + s), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.status, p.limit_ns, KID_DECODE};

  if (warp == kLoadWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // a 128-key tile in runs of rows that each lie in one page; runs
      // wholly past the length are skipped
      const int run = p.page < kKeys ? p.page : kKeys;
      int k_issued[kKStg] = {}, v_issued = 0;
      bool skip_pending = p.debug_skip && c == 0 && hk == 0 && b == 0;
      bool ok = true;
      auto load_tile = [&](const CUtensorMap* map, uint32_t dst0, uint32_t full, int tb, int valid) {
        uint32_t bytes = 0;
        for (int r0 = 0; r0 < valid; r0 += run) {
          const int pg = p.table[size_t(b) * p.max_pages + (tb + r0) / p.page];
          if (pg < 0 || pg >= p.num_pages) {
            atomicCAS(p.status, 0u, (unsigned(KID_DECODE) << 16) | (11u << 8) | 2u);
            continue;  // these rows stay unloaded (results undefined, error reported)
          }
          bytes += uint32_t(run) * 128u * 2u;
        }
        mbar_arrive_expect_tx(full, bytes);
        for (int r0 = 0; r0 < valid; r0 += run) {
          const int tp = tb + r0;
          const int pg = p.table[size_t(b) * p.max_pages + tp / p.page];
          if (pg < 0 || pg >= p.num_pages) continue;
          for (int cs = 0; cs < 2; ++cs)
            tma_load_3d(dst0 + cs * L::kSubBytes + r0 * 128, map, full, cs * 64, tp % p.page,
                        pg * p.Hkv + hk);
        }
      };
      // K runs up to two tiles ahead of V: tile j's K, then tile j-1's V
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {
          const int s = j % kKStg;
          ok = wait_bounded(BAR(X_K_EMPTY + s), ((j / kKStg) & 1) ^ 1, wc, 1);
          if (!ok) break;
          const int tb = t0 + j * kKeys;
          load_tile(&tmK, sbase + L::kOffK + s * L::kTileBytes, BAR(X_K_FULL + s), tb,
                    min(kKeys, t1 - tb));
          ++k_issued[s];
        }
        if (j >= 1) {
          const int jv = j - 1;
          ok = wait_bounded(BAR(X_V_EMPTY), (jv & 1) ^ 1, wc, 2);
          if (!ok) break;
          if (skip_pending) {
            skip_pending = false;  // test hook: this V tile never arrives
            continue;
          }
          const int tb = t0 + jv * kKeys;
          load_tile(&tmV, sbase + L::kOffV, BAR(X_V_FULL), tb, min(kKeys, t1 - tb));
          ++v_issued;
        }
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA exits
        for (int s = 0; s < kKStg; ++s)
          if (k_issued[s]) wait_bounded(BAR(X_K_FULL + s), (k_issued[s] - 1) & 1, wc, 3, true);
        if (v_issued) wait_bounded(BAR(X_V_FULL), (v_issued - 1) & 1, wc, 3, true);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(kKeys, kNH, false, false);  // K K-major, Q K-major
      constexpr uint32_t idesc_o = idesc_bf16(kD, kNH, true, false);      // V MN-major, P^T K-major
      const uint32_t sQ = sbase + L::kOffQ;
      auto issue_s = [&](int j) -> bool {
        const int s = j % kKStg;
        if (!wait_bounded(BAR(X_K_FULL + s), (j / kKStg) & 1, wc, 10)) return false;
        // S^T buffer j%2 is free once the softmax has loaded S^T(j-2)
        if (j >= 2 && !wait_bounded(BAR(X_S_FREE + (j & 1)), ((j >> 1) - 1) & 1, wc, 11)) return false;
        tc_fence_after();
        const uint32_t kb = sbase + L::kOffK + s * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          mma_ss(tmem + (j & 1) * kNH,
                 sdesc_sw128(kb + (kk >> 2) * L::kSubBytes + (kk & 3) * 32, 16, 1024),
                 sdesc_sw128(sQ + (kk >> 2) * (kNH * 128) + (kk & 3) * 32, 16, 1024), idesc_s,
                 kk > 0 ? 1u : 0u);
        tc_commit(BAR(X_S_FULL + (j & 1)));
        tc_commit(BAR(X_K_EMPTY + s));
        return true;
      };
      bool ok = wait_bounded(BAR(X_Q_READY), 0, wc, 12);
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (j + 1 < n_tiles && !(ok = issue_s(j + 1))) break;
        ok = wait_bounded(BAR(X_P_FULL + (j & 1)), (j >> 1) & 1, wc, 13);
        if (ok) ok = wait_bounded(BAR(X_V_FULL), j & 1, wc, 14);
        if (!ok) break;
        tc_fence_after();
        // O^T (+)= V^T P^T: V read MN-major (d contiguous), P^T K-major
        const uint32_t vb = sbase + L::kOffV;
        const uint32_t pb = sbase + L::kOffP + (j & 1) * (2 * kNH * 128);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          mma_ss(tmem + L::kColO, sdesc_sw128(vb + kk * 16 * 128, L::kSubBytes, 1024),
                 sdesc_sw128(pb + (kk >> 2) * (kNH * 128) + (kk & 3) * 32, 16, 1024), idesc_o,
                 (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(BAR(X_P_EMPTY + (j & 1)));
        tc_commit(BAR(X_V_EMPTY));
        if (j + 1 == n_tiles) tc_commit(BAR(X_O_FULL));
      }
      tc_commit(BAR(X_DRAIN));
      wait_bounded(BAR(X_DRAIN), 0, wc, 16, true);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int t = warp * 32 + lane;  // key of the tile, TMEM lane; dim of O^T at the end
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    // Q as the K-major B operand: 16 head rows of d = 128 (two 64-dim groups
    // of 128-byte rows, 128-byte swizzle), zero rows past the group
    {
      uint8_t* sq = smem + L::kOffQ;
      for (int ch = t; ch < kNH * (kD / 8); ch += kSmWarps * 32) {
        const int h = ch / (kD / 8), cc16 = ch % (kD / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (h < G)
          v = *reinterpret_cast<const uint4*>(p.q + (size_t(b) * p.Hq + size_t(hk) * G + h) * kD +
                                              cc16 * 8);
        const int sub = cc16 >> 3, cc = cc16 & 7;
        *reinterpret_cast<uint4*>(sq + sub * (kNH * 128) + h * 128 + ((cc ^ (h & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(X_Q_READY));
    }
    const float cl = p.scale_log2;
    float m[kNH], lp[kNH];
#pragma unroll
    for (int h = 0; h < kNH; ++h) {
      m[h] = -INFINITY;
      lp[h] = 0.f;
    }
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int tb = t0 + j * kKeys;
      const int valid = min(kKeys, t1 - tb);
      ok = wait_bounded(BAR(X_S_FULL + (j & 1)), (j >> 1) & 1, wc, 20);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[16];
      tmem_ld16_wait(tmem + lane_base + (j & 1) * kNH, sr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(X_S_FREE + (j & 1)));
      // scores in log2 units; keys past the length (and heads past G) -inf
      float x[kNH];
#pragma unroll
      for (int h = 0; h < kNH; ++h)
        x[h] = (t < valid && h < G) ? __uint_as_float(sr[h]) * cl : -INFINITY;
      // the tile's maximum of every head over the 128 keys
      float* rd = red + (j & 1) * kSmWarps * kNH;
#pragma unroll
      for (int h = 0; h < kNH; ++h) {
        if (h < G) {
          float v = x[h];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
          if (lane == 0) rd[warp * kNH + h] = v;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(X_MAX + (j & 1)));
      // X_MAX_j%2: a warp writes this slot again (tile j+2) only after it
      // passed this wait for tile j+1, which all four warps arrive at after
      // reading tile j's maxima
      ok = wait_bounded(BAR(X_MAX + (j & 1)), (j >> 1) & 1, wc, 21);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      bool grow = false;
      float mt[kNH];
#pragma unroll
      for (int h = 0; h < kNH; ++h) {
        mt[h] = -INFINITY;
        if (h < G) {
          mt[h] = fmaxf(fmaxf(rd[h], rd[kNH + h]), fmaxf(rd[2 * kNH + h], rd[3 * kNH + h]));
          grow |= mt[h] > m[h] + kRescale;
        }
      }
      if (j == 0) {
#pragma unroll
        for (int h = 0; h < kNH; ++h) m[h] = mt[h];
      } else if (grow) {
        // (the same decision in every thread: the maxima are the CTA's)
        // O~ must hold the sum through tile j-1: P^T(j-1) V finished
        ok = wait_bounded(BAR(X_P_EMPTY + ((j - 1) & 1)), ((j - 1) >> 1) & 1, wc, 22);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        float alpha[kNH];
#pragma unroll
        for (int h = 0; h < kNH; ++h) {
          const float mn = fmaxf(m[h], mt[h]);
          // a head with no visible key so far has nothing to rescale
          alpha[h] = (h < G && m[h] != -INFINITY) ? ex2_approx(m[h] - mn) : 0.f;
          lp[h] *= alpha[h];
          m[h] = mn;
        }
        uint32_t orow[16];
        tmem_ld16_wait(tmem + lane_base + L::kColO, orow);
#pragma unroll
        for (int h = 0; h < kNH; ++h) orow[h] = __float_as_uint(__uint_as_float(orow[h]) * alpha[h]);
        tmem_st16(tmem + lane_base + L::kColO, orow);
        tmem_st_wait();
      }
      // P^T(j) into buffer j%2 once P^T(j-2) has been read
      if (j >= 2) {
        ok = wait_bounded(BAR(X_P_EMPTY + (j & 1)), ((j >> 1) - 1) & 1, wc, 23);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      uint8_t* pt = smem + L::kOffP + (j & 1) * (2 * kNH * 128) + (t >> 6) * (kNH * 128);
      const int kb = (t & 63) * 2;  // byte of this key in its 128-byte row
#pragma unroll
      for (int h = 0; h < kNH; ++h) {
        if (h < G) {
          // (a head whose keys so far are all masked has m = -inf: its P is 0)
          const float pv = m[h] == -INFINITY ? 0.f : ex2_approx(x[h] - m[h]);
          lp[h] += pv;
          const uint32_t bits = pack_bf16x2(pv, 0.f) & 0xffffu;
          *reinterpret_cast<uint16_t*>(pt + h * 128 + ((((kb >> 4) ^ (h & 7))) << 4) + (kb & 15)) =
              uint16_t(bits);
        }
      }
      if (valid < kKeys && warp == 0) {
        // the sequence's last tile: zero the V rows past its length before
        // O^T += V^T P^T reads them (the tile's V copy must have landed).
        // V has one slot, and S^T(j) can be ready before V(j-1) has landed
        // or after V(j) has: a parity wait on V_FULL alone could be two
        // phases off either way. So first P^T(j-1) V (one phase at most
        // ahead of this thread's last wait on that barrier, tile j-3's, and
        // its next phase needs this tile's P^T): then V(j-1) has landed and
        // V(j) is the only load left, and the parity wait on it is exact.
        ok = j == 0 || wait_bounded(BAR(X_P_EMPTY + ((j - 1) & 1)), ((j - 1) >> 1) & 1, wc, 24);
        if (ok) ok = wait_bounded(BAR(X_V_FULL), j & 1, wc, 24);
        if (ok) {
          uint8_t* vt = smem + L::kOffV;
          for (int e = lane; e < (kKeys - valid) * 16; e += 32) {
            const int row = valid + e / 16, rest = e % 16;
            *reinterpret_cast<uint4*>(vt + (rest / 8) * L::kSubBytes + row * 128 + (rest % 8) * 16) =
                make_uint4(0, 0, 0, 0);
          }
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(X_P_FULL + (j & 1)));
    }
    // row sums over the 128 key lanes, then O = O~ / l and the LSE
    if (ok) {
#pragma unroll
      for (int h = 0; h < kNH; ++h) {
        if (h < G) {
          float v = lp[h];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
          if (lane == 0) lred[warp * kNH + h] = v;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(X_LSUM));
      ok = wait_bounded(BAR(X_LSUM), 0, wc, 25);
      if (ok) ok = wait_bounded(BAR(X_O_FULL), 0, wc, 26);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      uint32_t orow[16];
      tmem_ld16_wait(tmem + lane_base + L::kColO, orow);
#pragma unroll
      for (int h = 0; h < kNH; ++h) {
        if (h < G) {
          const float l = lred[h] + lred[kNH + h] + lred[2 * kNH + h] + lred[3 * kNH + h];
          const size_t part = (size_t(b) * p.Hq + size_t(hk) * G + h) * p.C + c;
          p.part_o[part * kD + t] = __uint_as_float(orow[h]) / l;
          if (t == 0) p.part_lse[part] = m[h] + lg2_approx(l);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace

// Chunk partials of the paged decode for 4 to 16 query heads per KV head and
// d = 128, keys as the MMA rows; the caller merges them (decode_merge_kernel).
fa_status launch_decode_paged_tct(const void* q, const void* kpages, const void* vpages,
                                  const int* block_table, const int* seqlens, int B, int Hq,
                                  int Hkv, int num_pages, int page_size, int max_pages, int d,
                                  float scale, int chunks, float* part_o, float* part_lse,
                                  const LaunchCtx& ctx) {
  if (d != kD || Hq / Hkv > kNH || (page_size > 64 && page_size % kKeys != 0)) {
    set_last_error("fa_decode_paged: the keys-as-rows kernel needs d = 128, <= %d heads per KV "
                   "head and pages of <= 64 rows or a multiple of 128", kNH);
    return FA_ERR_UNSUPPORTED;
  }
  const uint64_t outer = uint64_t(num_pages) * uint64_t(Hkv);
  const uint32_t box_rows = page_size < kKeys ? uint32_t(page_size) : uint32_t(kKeys);
  CUtensorMap mk, mv;
  fa_status st;
  if ((st = make_tmap_3d(&mk, kpages, 2, d, page_size, outer, 64, box_rows, 128)) != FA_OK) return st;
  if ((st = make_tmap_3d(&mv, vpages, 2, d, page_size, outer, 64, box_rows, 128)) != FA_OK) return st;
  TctParams p;
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
  const int smem = Layout::kSmemBytes;
  cudaError_t e =
      cudaFuncSetAttribute(decode_tct_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_tct)");
  dim3 grid(p.C, p.Hkv, B);
  {
    ProfileScope prof(KID_DECODE, ctx.stream);
    decode_tct_kernel<<<grid, kThreads, smem, ctx.stream>>>(mk, mv, p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode tct kernel launch");
  return FA_OK;
}

}  // namespace fa
