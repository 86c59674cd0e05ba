// bwd_sm100.cu -- attention backward by recomputation, B200 (sm_100a).
//
// What it computes ("Bellek Duvarinin Fizigi", section "Geri Yayilim"): the
// forward saved only O and the per-row log-sum-exp L. The backward rebuilds
// every block of P on chip as P = exp(S - L) and forms
//     dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),  dS = P * (dP - D),
//     dQ = scale * dS K,  dK = scale * dS^T Q,
// so neither S nor P (nor dS) is ever stored.
//
// Three kernels on the caller's stream:
//  1. bwd_pre   D_i = sum_c dO_ic O_ic (fp32) and the saved LSE in base 2, both
//               padded to a multiple of 128 rows (padding rows get LSE = +inf,
//               so their P is exactly 0).
//  2. bwd_dkdv  one CTA per (batch*head, 128-key tile). K and V of the tile stay
//               in shared memory; the Q and dO rows of every query that can see
//               these keys stream past in blocks of 64. Per block:
//                 S^T = K Q^T, dP^T = V dO^T          (tcgen05 -> TMEM)
//                 P^T = 2^(S^T scale log2e - L2),
//                 dS^T = scale P^T (dP^T - D)        (CUDA cores, one TMEM lane
//                                                      = one key row)
//                 dV += P^T dO, dK += dS^T Q          (tcgen05, A from TMEM)
//               dV and dK accumulate in TMEM for the whole key tile.
//  3. bwd_dq    one CTA per (batch*head, 128-query tile). Q and dO stay in shared
//               memory; K and V stream past in blocks of 64 keys. Per block:
//                 S = Q K^T, dP = dO V^T; dS = scale P (dP - D); dQ += dS K.
// The scale is folded into dS before it is rounded to bf16.
//
// Splitting dQ from dK/dV recomputes S and dP once more (7 tensor-core GEMMs
// instead of 5) but needs no atomics and keeps the tensor core busy: in both
// kernels two compute warpgroups take alternate 64-wide blocks, each with its
// own S/dP buffer in TMEM, so the exponentials of one block overlap the MMAs of
// the other (TMEM: buffer 0 | buffer 1 | two 128-column accumulators).
//
// Warp roles (320 threads): warps 0-3 compute for buffer 0, warps 4-7 for
// buffer 1, warp 8 TMA producer, warp 9 MMA issuer.
#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kTile = 128;   // rows of the resident tile (keys or queries)
constexpr int kSub = 64;     // rows of a streamed block
constexpr int kThreads = 320;
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kStages = 4;
constexpr float kLog2e = 1.4426950408889634f;

// barrier slots (shared by both kernels)
enum : int {
  B_RES_FULL = 0,      // the resident tiles (K,V or Q,dO)
  B_ST_FULL = 1,       // +stage: a streamed block landed
  B_ST_EMPTY = 5,      // +stage: its MMAs are done
  B_S_FULL = 9,        // +buffer: S and dP of a block are in TMEM
  B_P_READY = 11,      // +buffer: P / dS written back to TMEM
  B_ACC_DONE = 13,
  B_DRAIN = 14,
  B_COUNT = 15
};

struct BwdParams {
  const uint16_t* o;
  const uint16_t* dO;
  const float* lse;
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

// Shared-memory plan. Row-major tiles of bf16 with 128-byte rows, stored as
// D/64 column groups of rows x 128 bytes, 128-byte swizzled (TMA box 64
// columns x rows).
template <int D>
struct Plan {
  static constexpr int kGroups = D / 64;
  static constexpr int kResSub = kTile * 128;            // 16 KB per column group
  static constexpr int kResTile = kGroups * kResSub;      // one resident tile
  static constexpr int kBlkSub = kSub * 128;              // 8 KB per column group
  static constexpr int kBlkTile = kGroups * kBlkSub;      // one streamed tile
  static constexpr int kOffRes0 = 0;
  static constexpr int kOffRes1 = kResTile;
  static constexpr int kOffStage = 2 * kResTile;
  // a stage: two streamed tiles, then (dK/dV kernel) 64 floats of L2 and of D
  static constexpr int kStageBytes = ((2 * kBlkTile + 512) + 1023) / 1024 * 1024;
  static constexpr int kOffBar = kOffStage + kStages * kStageBytes;
  static constexpr int kOffMisc = kOffBar + 8 * B_COUNT;
  static constexpr int kSmemBytes = kOffMisc + 32 + 1024;
  // TMEM columns: buffer b holds S (64 columns) then dP (64 columns)
  static constexpr uint32_t kColAcc0 = 256, kColAcc1 = 256 + D;
  __device__ static constexpr uint32_t col_s(int b) { return b ? 128u : 0u; }
  __device__ static constexpr uint32_t col_dp(int b) { return b ? 192u : 64u; }
};

// --------------------------------------------------------------------------
// 1. preprocess: a row is read by d/8 lanes with 16-byte loads; a warp covers
//    kPreSteps groups of rows and issues all its loads before using them
// --------------------------------------------------------------------------
constexpr int kPreSteps = 4;

template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const BwdParams p) {
  constexpr int kLanesPerRow = D / 8;            // 16 (d = 128) or 8 (d = 64)
  constexpr int kRowsPerStep = 32 / kLanesPerRow;
  const long long gwarp = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane / kLanesPerRow, j = lane % kLanesPerRow;
  const long long total = static_cast<long long>(p.BH) * p.Np;
  const long long row0 = gwarp * kRowsPerStep * kPreSteps;
  uint4 ov[kPreSteps], gv[kPreSteps];
#pragma unroll
  for (int st = 0; st < kPreSteps; ++st) {
    const long long r = row0 + st * kRowsPerStep + sub;
    ov[st] = gv[st] = make_uint4(0, 0, 0, 0);
    if (r < total) {
      const int bh = int(r / p.Np), row = int(r % p.Np);
      if (row < p.N) {
        const size_t off = (size_t(bh) * p.N + row) * D + j * 8;
        ov[st] = *reinterpret_cast<const uint4*>(p.o + off);
        gv[st] = *reinterpret_cast<const uint4*>(p.dO + off);
      }
    }
  }
#pragma unroll
  for (int st = 0; st < kPreSteps; ++st) {
    const uint32_t a[4] = {ov[st].x, ov[st].y, ov[st].z, ov[st].w};
    const uint32_t g[4] = {gv[st].x, gv[st].y, gv[st].z, gv[st].w};
    float dsum = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      dsum += bf16f(a[i] & 0xffffu) * bf16f(g[i] & 0xffffu) + bf16f(a[i] >> 16) * bf16f(g[i] >> 16);
#pragma unroll
    for (int off = kLanesPerRow / 2; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
    const long long r = row0 + st * kRowsPerStep + sub;
    if (j == 0 && r < total) {
      const int bh = int(r / p.Np), row = int(r % p.Np);
      p.dvec[r] = row < p.N ? dsum : 0.f;
      p.lse2[r] = row < p.N ? p.lse[size_t(bh) * p.N + row] * kLog2e : INFINITY;
    }
  }
}

// Common prologue of both main kernels: barriers, TMEM, abort flag.
template <int D>
__device__ __forceinline__ uint32_t setup_cta(uint8_t* smem, int warp, volatile int*& abort_flag) {
  using L = Plan<D>;
  const uint32_t sbase = smem_u32(smem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  if (threadIdx.x == 0) {
    auto bar = [&](int i) { return sbase + L::kOffBar + 8u * i; };
    mbar_init(bar(B_RES_FULL), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B_ST_FULL + s), 1);
      mbar_init(bar(B_ST_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_S_FULL + b), 1);
      mbar_init(bar(B_P_READY + b), 4);
    }
    mbar_init(bar(B_ACC_DONE), 1);
    mbar_init(bar(B_DRAIN), 1);
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
  return *tmem_slot;
}

// MMA of one streamed block against a resident tile, both K-major operands:
// D[128 x 64] = R[128 x D] * B[64 x D]^T
template <int D>
__device__ __forceinline__ void mma_rows_x_block(uint32_t d_tmem, uint32_t res, uint32_t blk) {
  using L = Plan<D>;
  constexpr uint32_t idesc = idesc_bf16(kTile, kSub, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t ra = res + (kk >> 2) * L::kResSub + (kk & 3) * 32;
    const uint32_t rb = blk + (kk >> 2) * L::kBlkSub + (kk & 3) * 32;
    mma_ss(d_tmem, sdesc_sw128(ra, 16, 1024), sdesc_sw128(rb, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}

// Accumulating MMA with A (128 x 64, bf16) in TMEM and B a streamed block of
// 64 rows x D read MN-major: D[128 x D] += A * B
template <int D>
__device__ __forceinline__ void mma_tmem_x_block(uint32_t d_tmem, uint32_t a_tmem, uint32_t blk,
                                                 bool accumulate) {
  using L = Plan<D>;
  constexpr uint32_t idesc = idesc_bf16(kTile, D, false, true);
#pragma unroll
  for (int kk = 0; kk < kSub / 16; ++kk)
    mma_ts(d_tmem, a_tmem + kk * 8, sdesc_sw128(blk + kk * 2048, L::kBlkSub, 1024), idesc,
           (accumulate || kk > 0) ? 1u : 0u);
}

// bf16 row of a TMEM accumulator (this thread's lane) -> global
template <int D>
__device__ __forceinline__ void store_acc_row(uint32_t t_acc, uint16_t* dst, bool valid) {
#pragma unroll
  for (int ch = 0; ch < D / 32; ++ch) {
    uint32_t v[32];
    tmem_ld32_wait(t_acc + ch * 32, v);
    if (valid) {
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

// --------------------------------------------------------------------------
// 2. dK, dV: key-tile-outer
// --------------------------------------------------------------------------
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ64, const __grid_constant__ CUtensorMap tmDO64,
                    const __grid_constant__ CUtensorMap tmK128, const __grid_constant__ CUtensorMap tmV128,
                    const BwdParams p) {
  using L = Plan<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto BAR = [&](int i) -> uint32_t { return sbase + L::kOffBar + 8u * uint32_t(i); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // key tiles that see the most query blocks first, all heads of a level together
  const int jt = blockIdx.x / p.BH;
  const int bh = blockIdx.x % p.BH;
  const int q_start = CAUSAL ? jt * kTile : 0;
  const int n_blk = (p.N - q_start + kSub - 1) / kSub;
  volatile int* abort_flag;
  const uint32_t tmem = setup_cta<D>(smem, warp, abort_flag);
  const WaitCtl wc{abort_flag, p.status, p.limit_ns, KID_BWD};
  const uint32_t sK = sbase + L::kOffRes0, sV = sbase + L::kOffRes1;

  if (warp == kLoadWarp) {
    if (lane == 0) {
      int issued = 0;
      mbar_arrive_expect_tx(BAR(B_RES_FULL), 2 * L::kResTile);
      for (int c = 0; c < L::kGroups; ++c) {
        tma_load_3d(sK + c * L::kResSub, &tmK128, BAR(B_RES_FULL), c * 64, jt * kTile, bh);
        tma_load_3d(sV + c * L::kResSub, &tmV128, BAR(B_RES_FULL), c * 64, jt * kTile, bh);
      }
      for (int it = 0; it < n_blk; ++it) {
        const int s = it % kStages;
        if (!wait_bounded(BAR(B_ST_EMPTY + s), ((it / kStages) & 1) ^ 1, wc, 1)) break;
        const int q0 = q_start + it * kSub;
        const uint32_t st = sbase + L::kOffStage + s * L::kStageBytes;
        mbar_arrive_expect_tx(BAR(B_ST_FULL + s), 2 * L::kBlkTile + 512);
        for (int c = 0; c < L::kGroups; ++c) {
          tma_load_3d(st + c * L::kBlkSub, &tmQ64, BAR(B_ST_FULL + s), c * 64, q0, bh);
          tma_load_3d(st + L::kBlkTile + c * L::kBlkSub, &tmDO64, BAR(B_ST_FULL + s), c * 64, q0, bh);
        }
        const size_t vo = size_t(bh) * p.Np + q0;
        bulk_load(st + 2 * L::kBlkTile, p.lse2 + vo, 256, BAR(B_ST_FULL + s));
        bulk_load(st + 2 * L::kBlkTile + 256, p.dvec + vo, 256, BAR(B_ST_FULL + s));
        ++issued;
      }
      if (*abort_flag) {
        wait_bounded(BAR(B_RES_FULL), 0, wc, 2, true);
        for (int s = 0; s < kStages; ++s) {
          const int cnt = (issued - s + kStages - 1) / kStages;  // loads into stage s
          if (cnt > 0) wait_bounded(BAR(B_ST_FULL + s), (cnt - 1) & 1, wc, 2, true);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      auto stage_addr = [&](int it) { return sbase + L::kOffStage + (it % kStages) * L::kStageBytes; };
      auto issue_sdp = [&](int it) {  // S^T and dP^T of block `it` into buffer it&1
        const int b = it & 1;
        const uint32_t st = stage_addr(it);
        mma_rows_x_block<D>(tmem + L::col_s(b), sK, st);
        mma_rows_x_block<D>(tmem + L::col_dp(b), sV, st + L::kBlkTile);
        tc_commit(BAR(B_S_FULL + b));
      };
      bool ok = wait_bounded(BAR(B_RES_FULL), 0, wc, 10);
      for (int it = 0; ok && it < 2 && it < n_blk; ++it) {
        ok = wait_bounded(BAR(B_ST_FULL + it % kStages), (it / kStages) & 1, wc, 11);
        if (!ok) break;
        tc_fence_after();
        issue_sdp(it);
      }
      for (int it = 0; ok && it < n_blk; ++it) {
        const int b = it & 1;
        ok = wait_bounded(BAR(B_P_READY + b), (it >> 1) & 1, wc, 12);
        if (!ok) break;
        tc_fence_after();
        const uint32_t st = stage_addr(it);
        mma_tmem_x_block<D>(tmem + L::kColAcc0, tmem + L::col_s(b), st + L::kBlkTile, it > 0);  // dV += P^T dO
        mma_tmem_x_block<D>(tmem + L::kColAcc1, tmem + L::col_dp(b), st, it > 0);               // dK += dS^T Q
        tc_commit(BAR(B_ST_EMPTY + it % kStages));
        if (it + 2 < n_blk) {
          ok = wait_bounded(BAR(B_ST_FULL + (it + 2) % kStages), ((it + 2) / kStages) & 1, wc, 13);
          if (!ok) break;
          tc_fence_after();
          issue_sdp(it + 2);
        }
      }
      tc_commit(BAR(B_ACC_DONE));
      tc_commit(BAR(B_DRAIN));
      wait_bounded(BAR(B_DRAIN), 0, wc, 14, true);
    }
  } else {
    // ------------------------------------------------------------ compute warpgroups
    const int b = warp >> 2;          // buffer of this warpgroup
    const int quad = warp & 3;
    const int r = quad * 32 + lane;   // key row in the tile
    const int key = jt * kTile + r;
    const bool row_valid = key < p.N;
    const uint32_t lane_base = uint32_t(quad * 32) << 16;
    const uint32_t tS = tmem + lane_base + L::col_s(b);
    const uint32_t tDP = tmem + lane_base + L::col_dp(b);
    const float c = p.scale_log2;
    bool ok = true;
    for (int it = b; it < n_blk; it += 2) {
      ok = wait_bounded(BAR(B_S_FULL + b), (it >> 1) & 1, wc, 20);
      if (ok) ok = wait_bounded(BAR(B_ST_FULL + it % kStages), (it / kStages) & 1, wc, 21);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int q0 = q_start + it * kSub;
      const float* l2 = reinterpret_cast<const float*>(smem + L::kOffStage + (it % kStages) * L::kStageBytes +
                                                       2 * L::kBlkTile);
      const float* dd = l2 + 64;
      // queries q0 + i with i < qmask are hidden from this key (causal)
      const int qmask = CAUSAL ? min(max(key - q0, 0), kSub) : 0;
      uint32_t sr[64];
      tmem_ld64_wait(tS, sr);
      float pr[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const float x = ex2_approx(fmaf(__uint_as_float(sr[i]), c, -l2[i]));
        pr[i] = (row_valid && i >= qmask) ? x : 0.f;
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(pr[2 * i], pr[2 * i + 1]);
        tmem_st32(tS, pk);  // P^T over the first 32 columns of S^T
      }
      uint32_t dr[64];
      tmem_ld64_wait(tDP, dr);
      {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float a = pr[2 * i] * p.scale * (__uint_as_float(dr[2 * i]) - dd[2 * i]);
          const float e = pr[2 * i + 1] * p.scale * (__uint_as_float(dr[2 * i + 1]) - dd[2 * i + 1]);
          pk[i] = pack_bf16x2(a, e);
        }
        tmem_st32(tDP, pk);  // dS^T over the first 32 columns of dP^T
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_P_READY + b));
    }
    // epilogue: warpgroup 0 writes dV, warpgroup 1 writes dK
    if (ok) {
      ok = wait_bounded(BAR(B_ACC_DONE), 0, wc, 22);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const size_t gro = (size_t(bh) * p.N + key) * D;
      if (b == 0)
        store_acc_row<D>(tmem + lane_base + L::kColAcc0, p.dv + gro, row_valid);
      else
        store_acc_row<D>(tmem + lane_base + L::kColAcc1, p.dk + gro, row_valid);
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
// 3. dQ: query-tile-outer
// --------------------------------------------------------------------------
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ128, const __grid_constant__ CUtensorMap tmDO128,
                  const __grid_constant__ CUtensorMap tmK64, const __grid_constant__ CUtensorMap tmV64,
                  const BwdParams p) {
  using L = Plan<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto BAR = [&](int i) -> uint32_t { return sbase + L::kOffBar + 8u * uint32_t(i); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // query tiles that see the most key blocks first (causal: the last ones)
  const int lvl = blockIdx.x / p.BH;
  const int it_q = CAUSAL ? p.n_tiles - 1 - lvl : lvl;
  const int bh = blockIdx.x % p.BH;
  const int k_end = CAUSAL ? min(p.N, (it_q + 1) * kTile) : p.N;
  const int n_blk = (k_end + kSub - 1) / kSub;
  volatile int* abort_flag;
  const uint32_t tmem = setup_cta<D>(smem, warp, abort_flag);
  const WaitCtl wc{abort_flag, p.status, p.limit_ns, KID_BWD_DQ};
  const uint32_t sQ = sbase + L::kOffRes0, sDO = sbase + L::kOffRes1;

  if (warp == kLoadWarp) {
    if (lane == 0) {
      int issued = 0;
      mbar_arrive_expect_tx(BAR(B_RES_FULL), 2 * L::kResTile);
      for (int c = 0; c < L::kGroups; ++c) {
        tma_load_3d(sQ + c * L::kResSub, &tmQ128, BAR(B_RES_FULL), c * 64, it_q * kTile, bh);
        tma_load_3d(sDO + c * L::kResSub, &tmDO128, BAR(B_RES_FULL), c * 64, it_q * kTile, bh);
      }
      for (int it = 0; it < n_blk; ++it) {
        const int s = it % kStages;
        if (!wait_bounded(BAR(B_ST_EMPTY + s), ((it / kStages) & 1) ^ 1, wc, 1)) break;
        const uint32_t st = sbase + L::kOffStage + s * L::kStageBytes;
        mbar_arrive_expect_tx(BAR(B_ST_FULL + s), 2 * L::kBlkTile);
        for (int c = 0; c < L::kGroups; ++c) {
          tma_load_3d(st + c * L::kBlkSub, &tmK64, BAR(B_ST_FULL + s), c * 64, it * kSub, bh);
          tma_load_3d(st + L::kBlkTile + c * L::kBlkSub, &tmV64, BAR(B_ST_FULL + s), c * 64, it * kSub, bh);
        }
        ++issued;
      }
      if (*abort_flag) {
        wait_bounded(BAR(B_RES_FULL), 0, wc, 2, true);
        for (int s = 0; s < kStages; ++s) {
          const int cnt = (issued - s + kStages - 1) / kStages;  // loads into stage s
          if (cnt > 0) wait_bounded(BAR(B_ST_FULL + s), (cnt - 1) & 1, wc, 2, true);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      auto stage_addr = [&](int it) { return sbase + L::kOffStage + (it % kStages) * L::kStageBytes; };
      auto issue_sdp = [&](int it) {  // S and dP of key block `it` into buffer it&1
        const int b = it & 1;
        const uint32_t st = stage_addr(it);
        mma_rows_x_block<D>(tmem + L::col_s(b), sQ, st);
        mma_rows_x_block<D>(tmem + L::col_dp(b), sDO, st + L::kBlkTile);
        tc_commit(BAR(B_S_FULL + b));
      };
      bool ok = wait_bounded(BAR(B_RES_FULL), 0, wc, 10);
      for (int it = 0; ok && it < 2 && it < n_blk; ++it) {
        ok = wait_bounded(BAR(B_ST_FULL + it % kStages), (it / kStages) & 1, wc, 11);
        if (!ok) break;
        tc_fence_after();
        issue_sdp(it);
      }
      for (int it = 0; ok && it < n_blk; ++it) {
        const int b = it & 1;
        ok = wait_bounded(BAR(B_P_READY + b), (it >> 1) & 1, wc, 12);
        if (!ok) break;
        tc_fence_after();
        mma_tmem_x_block<D>(tmem + L::kColAcc0, tmem + L::col_dp(b), stage_addr(it), it > 0);  // dQ += dS K
        tc_commit(BAR(B_ST_EMPTY + it % kStages));
        if (it + 2 < n_blk) {
          ok = wait_bounded(BAR(B_ST_FULL + (it + 2) % kStages), ((it + 2) / kStages) & 1, wc, 13);
          if (!ok) break;
          tc_fence_after();
          issue_sdp(it + 2);
        }
      }
      tc_commit(BAR(B_ACC_DONE));
      tc_commit(BAR(B_DRAIN));
      wait_bounded(BAR(B_DRAIN), 0, wc, 14, true);
    }
  } else {
    const int b = warp >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;   // query row in the tile
    const int q = it_q * kTile + r;
    const uint32_t lane_base = uint32_t(quad * 32) << 16;
    const uint32_t tS = tmem + lane_base + L::col_s(b);
    const uint32_t tDP = tmem + lane_base + L::col_dp(b);
    const float c = p.scale_log2;
    const float l2q = p.lse2[size_t(bh) * p.Np + it_q * kTile + r];  // +inf past N
    const float dq_ = p.dvec[size_t(bh) * p.Np + it_q * kTile + r];
    bool ok = true;
    for (int it = b; it < n_blk; it += 2) {
      ok = wait_bounded(BAR(B_S_FULL + b), (it >> 1) & 1, wc, 20);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int k0 = it * kSub;
      // keys k0 + i with i >= klim are hidden (causal: key > q; or key >= N)
      int klim = p.N - k0;
      if (CAUSAL) klim = min(klim, q - k0 + 1);
      klim = max(min(klim, kSub), 0);
      uint32_t sr[64];
      tmem_ld64_wait(tS, sr);
      uint32_t dr[64];
      tmem_ld64_wait(tDP, dr);
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(sr[2 * i]), c, -l2q));
        const float p1 = ex2_approx(fmaf(__uint_as_float(sr[2 * i + 1]), c, -l2q));
        const float a = (2 * i < klim) ? p0 * p.scale * (__uint_as_float(dr[2 * i]) - dq_) : 0.f;
        const float e = (2 * i + 1 < klim) ? p1 * p.scale * (__uint_as_float(dr[2 * i + 1]) - dq_) : 0.f;
        pk[i] = pack_bf16x2(a, e);
      }
      tmem_st32(tDP, pk);  // dS over the first 32 columns of dP
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_P_READY + b));
    }
    if (ok) {
      ok = wait_bounded(BAR(B_ACC_DONE), 0, wc, 22);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok && b == 0) {
      tc_fence_after();
      store_acc_row<D>(tmem + lane_base + L::kColAcc0, p.dq + (size_t(bh) * p.N + q) * D, q < p.N);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

template <typename Kern>
fa_status launch_main(Kern kern, unsigned kid, int smem, unsigned grid, const CUtensorMap* m,
                      const BwdParams& p, const LaunchCtx& ctx, const char* what) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, what);
  {
    ProfileScope prof(kid, ctx.stream);
    kern<<<grid, kThreads, smem, ctx.stream>>>(m[0], m[1], m[2], m[3], p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return FA_OK;
}

template <int D, bool CAUSAL>
fa_status launch_all(const void* q, const void* k, const void* v, const void* dO, const BwdParams& p,
                     const LaunchCtx& ctx) {
  const int smem = Plan<D>::kSmemBytes;
  const unsigned grid = unsigned(p.n_tiles) * unsigned(p.BH);
  CUtensorMap m[4];
  fa_status st;
  // dK/dV: queries and dO stream in blocks of 64 rows, K and V tiles of 128
  if ((st = make_tmap_3d(&m[0], q, true, D, p.N, p.BH, 64, kSub, true)) != FA_OK) return st;
  if ((st = make_tmap_3d(&m[1], dO, true, D, p.N, p.BH, 64, kSub, true)) != FA_OK) return st;
  if ((st = make_tmap_3d(&m[2], k, true, D, p.N, p.BH, 64, kTile, true)) != FA_OK) return st;
  if ((st = make_tmap_3d(&m[3], v, true, D, p.N, p.BH, 64, kTile, true)) != FA_OK) return st;
  st = launch_main(bwd_dkdv_kernel<D, CAUSAL>, KID_BWD, smem, grid, m, p, ctx, "bwd dK/dV kernel");
  if (st != FA_OK) return st;
  // dQ: Q and dO tiles of 128 rows, K and V stream in blocks of 64
  if ((st = make_tmap_3d(&m[0], q, true, D, p.N, p.BH, 64, kTile, true)) != FA_OK) return st;
  if ((st = make_tmap_3d(&m[1], dO, true, D, p.N, p.BH, 64, kTile, true)) != FA_OK) return st;
  if ((st = make_tmap_3d(&m[2], k, true, D, p.N, p.BH, 64, kSub, true)) != FA_OK) return st;
  if ((st = make_tmap_3d(&m[3], v, true, D, p.N, p.BH, 64, kSub, true)) != FA_OK) return st;
  return launch_main(bwd_dq_kernel<D, CAUSAL>, KID_BWD_DQ, smem, grid, m, p, ctx, "bwd dQ kernel");
}

}  // namespace

size_t bwd_workspace_bytes(int B, int H, int N, int d) {
  (void)d;
  const size_t bh = size_t(B) * H;
  const size_t np = (size_t(N) + kTile - 1) / kTile * kTile;
  return 2 * align256(bh * np * 4);
}

fa_status launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                     float scale, bool causal, void* workspace, const LaunchCtx& ctx) {
  const int BH = B * H;
  BwdParams p;
  p.o = static_cast<const uint16_t*>(o);
  p.dO = static_cast<const uint16_t*>(dO);
  p.lse = lse;
  p.N = N;
  p.n_tiles = (N + kTile - 1) / kTile;
  p.Np = p.n_tiles * kTile;
  p.BH = BH;
  if ((long long)p.n_tiles * BH > 0x7fffffffLL) {
    set_last_error("fa_bwd: too many tiles");
    return FA_ERR_UNSUPPORTED;
  }
  char* ws = static_cast<char*>(workspace);
  p.lse2 = reinterpret_cast<float*>(ws);
  p.dvec = reinterpret_cast<float*>(ws + align256(size_t(BH) * p.Np * 4));
  p.dq = static_cast<uint16_t*>(dq);
  p.dk = static_cast<uint16_t*>(dk);
  p.dv = static_cast<uint16_t*>(dv);
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.status = ctx.status_word;
  p.limit_ns = ctx.wait_limit_ns;

  {
    const long long rows_per_warp = (32 / (d / 8)) * kPreSteps;
    const long long warps = ((long long)BH * p.Np + rows_per_warp - 1) / rows_per_warp;
    const long long blocks = (warps * 32 + 255) / 256;
    ProfileScope prof(KID_BWD_PRE, ctx.stream);
    if (d == 128)
      bwd_pre_kernel<128><<<unsigned(blocks), 256, 0, ctx.stream>>>(p);
    else
      bwd_pre_kernel<64><<<unsigned(blocks), 256, 0, ctx.stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "bwd preprocess launch");
  }
  if (d == 128)
    return causal ? launch_all<128, true>(q, k, v, dO, p, ctx) : launch_all<128, false>(q, k, v, dO, p, ctx);
  return causal ? launch_all<64, true>(q, k, v, dO, p, ctx) : launch_all<64, false>(q, k, v, dO, p, ctx);
}

}  // namespace fa
