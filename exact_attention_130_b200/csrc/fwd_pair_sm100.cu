// fwd_pair_sm100.cu -- attention forward on CTA pairs (tcgen05 .cta_group::2),
// B200 (sm_100a), bf16, d = 128.
//
// What it computes is fwd_sm100.cu's ("Bellek Duvarinin Fizigi", sections
// "Online Softmax", "Forward gecisin iskeleti", "Maskeleme ve Dropout"):
// O = softmax(scale Q K^T [+ causal mask]) V and the per-row LSE, with the
// running maximum / running sum recurrence and O = O~ / l at the end.
//
// How it differs ("FlashAttention-2, -3 ve -4: Utilizasyon Savasi", the
// Blackwell paragraph: the 2-CTA MMA mode of tcgen05). A cluster of two CTAs
// on two SMs takes 256 query rows of one head: each CTA keeps its own 128
// rows (its Q tile, S, P and O in its own TMEM, its own softmax groups and
// epilogue), and the even CTA issues both products for the pair as
// M = 256 MMAs. The B operand of an M = 256 MMA is split by N between the
// two CTAs, so
//   S = Q K^T : each CTA holds 64 of the tile's 128 keys (all 128 dims),
//   O += P V  : each CTA holds 64 of the 128 dims of V (all 128 keys),
// and each SM loads and feeds the tensor core half as many K/V bytes per
// step as the one-CTA kernel (16 + 16 KB instead of 32 + 32 KB). The
// halved stages leave room for four of each.
//
// Hand-offs between the two CTAs:
//  * the even CTA's commits arrive on the barriers of both CTAs
//    (tcgen05.commit .multicast::cluster): scores ready, P free, O~
//    complete, K/V slots free;
//  * the softmax warps of both CTAs arrive on the even CTA's barriers
//    (scores read, P stored, O read): eight arrivals each. These arrivals
//    and the waits on them use the default (CTA-scope) semantics: the
//    tcgen05 operations they order are fenced by tcgen05.fence, and a
//    release or acquire at cluster scope costs a memory barrier per warp
//    (measured: the pair kernel then ran at 0.6 of its speed without it);
//  * each CTA's TMA loads complete on its own barriers; in the odd CTA the
//    two threads that issue MMAs in the even one instead forward each
//    completed load to the even CTA's barriers, so each CTA can let its own
//    copies land before it exits;
//  * a cluster barrier after set-up (before any remote arrival) and before
//    exit (after the last one).
// No TMA load uses .multicast::cluster.
//
// Work units: (head, 256-row Q pair tile); head-major without the mask;
// under the mask heaviest level first over all heads, dealt to the pairs in
// snake order. Under the mask the pair's steps cover the keys of its last
// row; for the even CTA the pair's last tile is entirely above its rows
// (masked, P = 0).
//
// Every mbarrier wait is bounded in time; a wait that runs out records the
// failure in the device status word and the CTA returns (both CTAs of a pair
// still meet at the final cluster barrier).
#include <cfloat>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kBM = 128;   // query rows per CTA (256 per pair)
constexpr int kBN = 128;   // keys per K/V step
constexpr int kD = 128;
constexpr int kThreads = 384;
constexpr int kRegsAtLaunch = 168;
constexpr int kRegsSoftmax = 208;
constexpr int kRegsControl = 88;
static_assert(128 * (2 * kRegsSoftmax + kRegsControl) <= kThreads * kRegsAtLaunch,
              "register split exceeds the launch allocation");
constexpr int kQkLoadWarp = 8;   // Q and K producer (both CTAs)
constexpr int kQkMmaWarp = 9;    // Q K^T issuer (even CTA); K/Q forwarder (odd CTA); TMEM
constexpr int kVLoadWarp = 10;   // V producer (both CTAs)
constexpr int kPvMmaWarp = 11;   // P V issuer (even CTA); V forwarder (odd CTA)
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kStages = 4;

enum : int {
  B_Q_FULL = 0,       // this CTA's Q tile landed
  B_Q_PEER = 1,       // (even CTA) the odd CTA's Q tile landed
  B_Q_EMPTY = 2,      // both Q tiles have been copied to TMEM (multicast commit)
  B_S_FULL = 3,       // +g%2: Q K^T(g) finished (multicast commit)
  B_S_FREE = 5,       // +g%2 (even CTA): both CTAs' softmax loaded S(g) (8 warps)
  B_P_FULL = 7,       // +g%4 (even CTA): P(g) is in both TMEMs (8 warps)
  B_P_EMPTY = 11,     // +g%2: P V(g) finished (multicast commit)
  B_DEC = 13,         // +g%2: step g's reference maximum (4 warps, this CTA)
  B_LDONE = 15,       // +k%2: the non-final group's row sums (4 warps, this CTA)
  B_O_FULL = 17,      // +f: O~ of a unit complete (multicast commit)
  B_O_EMPTY = 19,     // (even CTA) both CTAs' final groups have read O~ (8 warps)
  B_STG_READY = 20,   // this CTA's final group has written its staging tile
  B_STG_FREE = 21,    // this CTA's previous O store has read the staging tile
  B_DRAIN = 22,       // +issuer: every MMA issued (multicast commit)
  B_K_FULL = 24,
  B_K_PEER = B_K_FULL + kStages,
  B_K_EMPTY = B_K_PEER + kStages,
  B_V_FULL = B_K_EMPTY + kStages,
  B_V_PEER = B_V_FULL + kStages,
  B_V_EMPTY = B_V_PEER + kStages,
  B_COUNT = B_V_EMPTY + kStages
};

struct Layout {
  static constexpr int kSubBytes = 128 * 128;   // 128 rows x 128 bytes
  static constexpr int kQBytes = 2 * kSubBytes;  // Q tile: 128 rows x 128 dims
  static constexpr int kKHalf = 2 * 64 * 128;    // 64 keys x 128 dims (two 64-row column groups)
  static constexpr int kKSub = 64 * 128;         // one 64-row column group
  static constexpr int kVHalf = kSubBytes;       // 128 keys x 64 dims
  static constexpr int kOffQ = 0;
  static constexpr int kOffStg = kQBytes;        // O staging tile (bf16, 128 x 128)
  static constexpr int kOffK = kOffStg + kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKHalf;
  static constexpr int kOffBar = kOffV + kStages * kVHalf;
  static constexpr int kOffMref = kOffBar + 8 * B_COUNT;
  static constexpr int kOffLsum = kOffMref + kBM * 4;
  static constexpr int kOffMisc = kOffLsum + 4 * kBM * 4;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory");
  static constexpr uint32_t kColS1 = 128, kColO = 256, kColQ = 384, kColP = 448;
};

struct PairParams {
  float* lse;
  int N;
  int BH;
  int n_kv;       // K/V tiles per head
  int n_qp;       // 256-row Q pair tiles per head
  int num_items;  // BH * n_qp
  float scale_log2;
  unsigned int* status;
  unsigned long long limit_ns;
};

// The work list every role of both CTAs of a pair walks (G = number of
// pairs, c = this pair). No mask: item i = (head i / n_qp, pair tile
// i % n_qp), pair c takes c, c + G, ... Causal: item i = (level
// n_qp-1 - i / BH, head i % BH), round r gives pair c item r G + c (even r)
// or r G + G-1-c (odd r).
template <bool CAUSAL>
struct Walk {
  int k;
  __device__ __forceinline__ explicit Walk(int start) : k(start) {}
  __device__ __forceinline__ bool next(const PairParams& p, int& bh, int& qp) {
    const int G = int(gridDim.x) / 2, c = int(blockIdx.x) / 2;
    if (CAUSAL) {
      const int idx = k * G + ((k & 1) ? G - 1 - c : c);
      if (idx >= p.num_items) return false;
      qp = p.n_qp - 1 - idx / p.BH;
      bh = idx % p.BH;
      ++k;
      return true;
    }
    if (k >= p.num_items) return false;
    bh = k / p.n_qp;
    qp = k % p.n_qp;
    k += G;
    return true;
  }
};
template <bool CAUSAL>
__device__ __forceinline__ Walk<CAUSAL> walk_start() {
  return Walk<CAUSAL>(CAUSAL ? 0 : int(blockIdx.x) / 2);
}
// K/V steps of a pair tile: every tile without the mask; under it, the
// tiles up to the one holding the pair's last row
template <bool CAUSAL>
__device__ __forceinline__ int steps_of(int qp, int n_kv) {
  return CAUSAL ? min(2 * qp + 2, n_kv) : n_kv;
}

template <bool CAUSAL>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK64,
                    const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmO, const PairParams p) {
  using L = Layout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kOffBar;
  float* m_sh = reinterpret_cast<float*>(smem + L::kOffMref);
  float* lsum = reinterpret_cast<float*>(smem + L::kOffLsum);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * uint32_t(i); };
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues the MMAs
  // a barrier of the even CTA, as a cluster address
  auto LEAD = [&](int i) -> uint32_t { return mapa_shared(BAR(i), 0); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_Q_FULL), 1);
    mbar_init(BAR(B_Q_PEER), 1);
    mbar_init(BAR(B_Q_EMPTY), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(B_S_FULL + i), 1);
      mbar_init(BAR(B_S_FREE + i), 8);
      mbar_init(BAR(B_P_EMPTY + i), 1);
      mbar_init(BAR(B_DEC + i), 4);
      mbar_init(BAR(B_LDONE + i), 4);
      mbar_init(BAR(B_O_FULL + i), 1);
      mbar_init(BAR(B_DRAIN + i), 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(BAR(B_P_FULL + i), 8);
    mbar_init(BAR(B_O_EMPTY), 8);
    mbar_init(BAR(B_STG_READY), 4);
    mbar_init(BAR(B_STG_FREE), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(BAR(B_K_FULL + s), 1);
      mbar_init(BAR(B_K_PEER + s), 1);
      mbar_init(BAR(B_K_EMPTY + s), 1);
      mbar_init(BAR(B_V_FULL + s), 1);
      mbar_init(BAR(B_V_PEER + s), 1);
      mbar_init(BAR(B_V_EMPTY + s), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kQkMmaWarp) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  if (warp == kQkLoadWarp && lane == 0) {
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK64);
    tma_prefetch_map(&tmV);
    tma_prefetch_map(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  // both CTAs' barriers are initialised before either arrives on the other's
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.status, p.limit_ns, KID_FWD};

  if (warp >= 8) {
    regs_decrease<kRegsControl>();
    if (warp == kQkLoadWarp && lane == 0) {
      // ------------------------------------------------------------------ Q and K producer
      int k_issued[kStages] = {};
      int q_issued = 0, kv = 0;
      bool ok = true;
      Walk<CAUSAL> w = walk_start<CAUSAL>();
      int bh, qp;
      for (int u = 0; ok && w.next(p, bh, qp); ++u) {
        const int n = steps_of<CAUSAL>(qp, p.n_kv);
        // the slot is free once both Q tiles of the previous unit are in TMEM
        if (u > 0 && !(ok = wait_bounded(BAR(B_Q_EMPTY), (u - 1) & 1, wc, 1))) break;
        mbar_arrive_expect_tx(BAR(B_Q_FULL), L::kQBytes);
        for (int c = 0; c < 2; ++c)
          tma_load_3d(sbase + L::kOffQ + c * L::kSubBytes, &tmQ, BAR(B_Q_FULL), c * 64,
                      qp * 2 * kBM + int(rank) * kBM, bh);
        ++q_issued;
        for (int j = 0; ok && j < n; ++j, ++kv) {
          const int s = kv % kStages;
          ok = wait_bounded(BAR(B_K_EMPTY + s), ((kv / kStages) & 1) ^ 1, wc, 2);
          if (!ok) break;
          // this CTA's 64 of the tile's 128 keys, in two 64-dim column groups
          mbar_arrive_expect_tx(BAR(B_K_FULL + s), L::kKHalf);
          for (int c = 0; c < 2; ++c)
            tma_load_3d(sbase + L::kOffK + s * L::kKHalf + c * L::kKSub, &tmK64,
                        BAR(B_K_FULL + s), c * 64, j * kBN + int(rank) * 64, bh);
          ++k_issued[s];
        }
      }
      if (*abort_flag) {
        if (q_issued) wait_bounded(BAR(B_Q_FULL), (q_issued - 1) & 1, wc, 3, true);
        for (int s = 0; s < kStages; ++s)
          if (k_issued[s]) wait_bounded(BAR(B_K_FULL + s), (k_issued[s] - 1) & 1, wc, 3, true);
      }
    } else if (warp == kVLoadWarp && lane == 0) {
      // ------------------------------------------------------------------ V producer
      int v_issued[kStages] = {};
      int kv = 0;
      bool ok = true;
      Walk<CAUSAL> w = walk_start<CAUSAL>();
      int bh, qp;
      while (ok && w.next(p, bh, qp)) {
        const int n = steps_of<CAUSAL>(qp, p.n_kv);
        for (int j = 0; ok && j < n; ++j, ++kv) {
          const int s = kv % kStages;
          ok = wait_bounded(BAR(B_V_EMPTY + s), ((kv / kStages) & 1) ^ 1, wc, 4);
          if (!ok) break;
          // all 128 keys of the tile, this CTA's 64 of the 128 dims
          mbar_arrive_expect_tx(BAR(B_V_FULL + s), L::kVHalf);
          tma_load_3d(sbase + L::kOffV + s * L::kVHalf, &tmV, BAR(B_V_FULL + s), int(rank) * 64,
                      j * kBN, bh);
          ++v_issued[s];
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < kStages; ++s)
          if (v_issued[s]) wait_bounded(BAR(B_V_FULL + s), (v_issued[s] - 1) & 1, wc, 5, true);
      }
    } else if (warp == kQkMmaWarp && lane == 0 && rank != 0) {
      // ------------------------------------------------------------------ odd CTA: forward Q, K
      bool ok = true;
      Walk<CAUSAL> w = walk_start<CAUSAL>();
      int bh, qp, kv = 0;
      for (int u = 0; ok && w.next(p, bh, qp); ++u) {
        const int n = steps_of<CAUSAL>(qp, p.n_kv);
        if (!(ok = wait_bounded(BAR(B_Q_FULL), u & 1, wc, 6))) break;
        mbar_arrive_cluster(LEAD(B_Q_PEER));
        for (int j = 0; ok && j < n; ++j, ++kv) {
          const int s = kv % kStages;
          if (!(ok = wait_bounded(BAR(B_K_FULL + s), (kv / kStages) & 1, wc, 7))) break;
          mbar_arrive_cluster(LEAD(B_K_PEER + s));
        }
      }
      // the even CTA's last MMAs read this CTA's shared memory and write its
      // TMEM: they must be finished before this CTA frees TMEM or exits
      wait_bounded(BAR(B_DRAIN + 0), 0, wc, 8, true);
    } else if (warp == kPvMmaWarp && lane == 0 && rank != 0) {
      // ------------------------------------------------------------------ odd CTA: forward V
      bool ok = true;
      Walk<CAUSAL> w = walk_start<CAUSAL>();
      int bh, qp, kv = 0;
      while (ok && w.next(p, bh, qp)) {
        const int n = steps_of<CAUSAL>(qp, p.n_kv);
        for (int j = 0; ok && j < n; ++j, ++kv) {
          const int s = kv % kStages;
          if (!(ok = wait_bounded(BAR(B_V_FULL + s), (kv / kStages) & 1, wc, 9))) break;
          mbar_arrive_cluster(LEAD(B_V_PEER + s));
        }
      }
      wait_bounded(BAR(B_DRAIN + 1), 0, wc, 10, true);
    } else if (warp == kQkMmaWarp && lane == 0) {
      // ------------------------------------------------------------------ even CTA: Q K^T issuer
      constexpr uint32_t idesc_qk = idesc_bf16(2 * kBM, kBN, false, false);
      const uint32_t tQ = tmem + L::kColQ;
      bool ok = true;
      Walk<CAUSAL> w = walk_start<CAUSAL>();
      int bh, qp, g = 0;
      for (int u = 0; ok && w.next(p, bh, qp); ++u) {
        const int n = steps_of<CAUSAL>(qp, p.n_kv);
        // both Q tiles into their CTAs' TMEM (after this thread's last Q K^T
        // of the previous unit, in issue order)
        ok = wait_bounded(BAR(B_Q_FULL), u & 1, wc, 11);
        if (ok) ok = wait_bounded(BAR(B_Q_PEER), u & 1, wc, 12);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kSubBytes + (kk & 3) * 32;
          tmem_cp_pair_128x256b(tQ + kk * 8, sdesc_sw128(sbase + L::kOffQ + off, 16, 1024));
        }
        tc_commit_pair(BAR(B_Q_EMPTY));
        for (int j = 0; ok && j < n; ++j, ++g) {
          const int b = g & 1;
          // S_b is free once both CTAs' softmax loaded S(g-2)
          if (g >= 2 && !(ok = wait_bounded(BAR(B_S_FREE + b), ((g >> 1) - 1) & 1, wc, 13)))
            break;
          const int s = g % kStages;
          ok = wait_bounded(BAR(B_K_FULL + s), (g / kStages) & 1, wc, 14);
          if (ok) ok = wait_bounded(BAR(B_K_PEER + s), (g / kStages) & 1, wc, 15);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kb = sbase + L::kOffK + s * L::kKHalf;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kKSub + (kk & 3) * 32;
            mma_ts_pair(tmem + (b ? L::kColS1 : 0u), tQ + kk * 8, sdesc_sw128(kb + off, 16, 1024),
                        idesc_qk, kk > 0 ? 1u : 0u);
          }
          tc_commit_pair(BAR(B_S_FULL + b));
          tc_commit_pair(BAR(B_K_EMPTY + s));
        }
      }
      tc_commit_pair(BAR(B_DRAIN + 0));
      wait_bounded(BAR(B_DRAIN + 0), 0, wc, 16, true);
    } else if (warp == kPvMmaWarp && lane == 0) {
      // ------------------------------------------------------------------ even CTA: P V issuer
      // V [keys, 64 dims] half tiles, MN-major B; N = 128 dims over the pair
      constexpr uint32_t idesc_pv = idesc_bf16(2 * kBM, kD, false, true);
      const uint32_t tO = tmem + L::kColO, tP = tmem + L::kColP;
      bool ok = true;
      Walk<CAUSAL> w = walk_start<CAUSAL>();
      int bh, qp, g = 0;
      for (int u = 0; ok && w.next(p, bh, qp); ++u) {
        const int n = steps_of<CAUSAL>(qp, p.n_kv);
        for (int j = 0; ok && j < n; ++j, ++g) {
          ok = wait_bounded(BAR(B_P_FULL + (g & 3)), (g >> 2) & 1, wc, 17);
          if (!ok) break;
          const int s = g % kStages;
          ok = wait_bounded(BAR(B_V_FULL + s), (g / kStages) & 1, wc, 18);
          if (ok) ok = wait_bounded(BAR(B_V_PEER + s), (g / kStages) & 1, wc, 19);
          // the epilogues of the previous unit have read O~ in both CTAs
          if (ok && j == 0) ok = wait_bounded(BAR(B_O_EMPTY), (u & 1) ^ 1, wc, 20);
          if (!ok) break;
          tc_fence_after();
          const uint32_t vb = sbase + L::kOffV + s * L::kVHalf;
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            mma_ts_pair(tO, tP + kk * 8, sdesc_sw128(vb + kk * 16 * 128, L::kSubBytes, 1024),
                        idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit_pair(BAR(B_P_EMPTY + (g & 1)));
          tc_commit_pair(BAR(B_V_EMPTY + s));
          if (j + 1 == n) tc_commit_pair(BAR(B_O_FULL + (g & 1)));  // group g % 2 finishes
        }
      }
      tc_commit_pair(BAR(B_DRAIN + 1));
      wait_bounded(BAR(B_DRAIN + 1), 0, wc, 21, true);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kQkMmaWarp) {
      tc_fence_after();
      tmem_dealloc_pair(tmem, 512);
    }
  } else {
    // ------------------------------------------------------------------ softmax groups
    regs_increase<kRegsSoftmax>();
    const int grp = warp >> 2;             // this group takes the steps g with g % 2 == grp
    const int r = (warp & 3) * 32 + lane;  // row inside this CTA's Q tile
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + lane_base + L::kColO;
    const uint32_t tP = tmem + lane_base + L::kColP;
    const bool store_thread = (warp & 3) == 0 && lane == 0;
    const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
    bool ok = true;
    bool store_pending = false;
    Walk<CAUSAL> w = walk_start<CAUSAL>();
    int bh, qp, g = 0, nld = 0, nfin = 0;
    for (int u = 0; ok && w.next(p, bh, qp); ++u) {
      const int n = steps_of<CAUSAL>(qp, p.n_kv);
      const int row0 = qp * 2 * kBM + int(rank) * kBM;
      const int row = row0 + r;
      const bool final_group = ((g + n - 1) & 1) == grp;
      float m_ref = -INFINITY, l_part = 0.f;
      for (int j = 0; j < n; ++j, ++g) {
        if ((g & 1) != grp) continue;
        if (store_pending) {
          if (store_thread) {
            bulk_wait_group_read0();
            mbar_arrive(BAR(B_STG_FREE));
          }
          store_pending = false;
        }
        ok = wait_bounded(BAR(B_S_FULL + (g & 1)), (g >> 1) & 1, wc, 22);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld128_wait(tmem + lane_base + ((g & 1) ? L::kColS1 : 0u), sr);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(LEAD(B_S_FREE + (g & 1)));
        float s[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(sr[i]);
        // keys >= N, and under the mask keys above this row (all of them in
        // the even CTA's last step of a pair tile)
        int limit = p.N - j * kBN;
        if (CAUSAL) limit = min(limit, row - j * kBN + 1);
        if (limit < kBN) {
#pragma unroll
          for (int i = 0; i < 128; ++i) s[i] = (i < limit) ? s[i] : -INFINITY;
        }
        float mx0 = fmaxf(s[0], s[1]), mx1 = fmaxf(s[2], s[3]);
        float mx2 = fmaxf(s[4], s[5]), mx3 = fmaxf(s[6], s[7]);
#pragma unroll
        for (int i = 8; i < 128; i += 8) {
          mx0 = max3f(mx0, s[i], s[i + 1]);
          mx1 = max3f(mx1, s[i + 2], s[i + 3]);
          mx2 = max3f(mx2, s[i + 4], s[i + 5]);
          mx3 = max3f(mx3, s[i + 6], s[i + 7]);
        }
        const float mxc = fmaxf(max3f(mx0, mx1, mx2), mx3) * p.scale_log2;
        if (g > 0) {
          ok = wait_bounded(BAR(B_DEC + ((g - 1) & 1)), ((g - 1) >> 1) & 1, wc, 23);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
        }
        bool pv_prev_done = g == 0;
        auto wait_pv_prev = [&]() -> bool {
          if (pv_prev_done) return true;
          bool w_ok = wait_bounded(BAR(B_P_EMPTY + ((g - 1) & 1)), ((g - 1) >> 1) & 1, wc, 24);
          w_ok = __all_sync(0xffffffffu, w_ok);
          pv_prev_done = w_ok;
          return w_ok;
        };
        if (j == 0) {
          m_ref = mxc;  // the first tile of a pair tile has a visible key for every row
        } else {
          const float m_prev = m_sh[r];
          if (m_prev != m_ref) {
            if (m_ref != -INFINITY) l_part *= ex2_approx(m_ref - m_prev);
            m_ref = m_prev;
          }
          const float m_new = fmaxf(m_ref, mxc);
          if (__any_sync(0xffffffffu, m_new > m_ref + kRescaleThreshold)) {
            ok = wait_pv_prev();
            if (!ok) break;
            tc_fence_after();
            const float alpha = ex2_approx(m_ref - m_new);
            l_part *= alpha;
            m_ref = m_new;
#pragma unroll
            for (int ch = 0; ch < kD / 32; ++ch) {
              uint32_t orow[32];
              tmem_ld32_wait(tO + ch * 32, orow);
#pragma unroll
              for (int i = 0; i < 32; ++i)
                orow[i] = __float_as_uint(__uint_as_float(orow[i]) * alpha);
              tmem_st32(tO + ch * 32, orow);
            }
          }
        }
        m_sh[r] = m_ref;
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_DEC + (g & 1)));
        const uint64_t nm2 = f2_pack(-m_ref, -m_ref);
        uint64_t sum_a = f2_pack(0.f, 0.f), sum_b = sum_a;
        uint32_t pk[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s[2 * i], s[2 * i + 1]), c2, nm2), x0, x1);
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          if (i & 1)
            sum_b = f2_add(sum_b, f2_pack(p0, p1));
          else
            sum_a = f2_add(sum_a, f2_pack(p0, p1));
          pk[i] = pack_bf16x2(p0, p1);
        }
        ok = wait_pv_prev();
        if (!ok) break;
        tc_fence_after();
        tmem_st64(tP, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(LEAD(B_P_FULL + (g & 3)));
        {
          float a0, a1;
          f2_unpack(f2_add(sum_a, sum_b), a0, a1);
          l_part += a0 + a1;
        }
        if (j == n - 2) {
          float* ls = lsum + (nld & 1) * 2 * kBM;
          ls[r] = l_part;
          ls[kBM + r] = m_ref;
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(B_LDONE + (nld & 1)));
        }
      }
      if (!ok) break;
      const int k_ld = nld;
      if (n >= 2) ++nld;
      if (!final_group) continue;
      // ---------------------------------------------------------------- epilogue of unit u
      float l = l_part;
      if (n >= 2) {
        ok = wait_bounded(BAR(B_LDONE + (k_ld & 1)), (k_ld >> 1) & 1, wc, 25);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const float* ls = lsum + (k_ld & 1) * 2 * kBM;
        l += ls[r] * ex2_approx(ls[kBM + r] - m_ref);
      }
      ok = wait_bounded(BAR(B_O_FULL + grp), nfin & 1, wc, 26);
      ++nfin;
      if (ok && u > 0) ok = wait_bounded(BAR(B_STG_FREE), (u - 1) & 1, wc, 27);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t orow[kD];
      tmem_ld128_wait(tO, orow);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(LEAD(B_O_EMPTY));
      if (row < p.N) p.lse[size_t(bh) * p.N + row] = (m_ref + lg2_approx(l)) * kLn2;
      const float inv_l = 1.0f / l;
      uint8_t* stg = smem + L::kOffStg + r * 128;
#pragma unroll
      for (int k16 = 0; k16 < kD / 8; ++k16) {
        uint4 v;
        v.x = pack_bf16x2(__uint_as_float(orow[8 * k16 + 0]) * inv_l,
                          __uint_as_float(orow[8 * k16 + 1]) * inv_l);
        v.y = pack_bf16x2(__uint_as_float(orow[8 * k16 + 2]) * inv_l,
                          __uint_as_float(orow[8 * k16 + 3]) * inv_l);
        v.z = pack_bf16x2(__uint_as_float(orow[8 * k16 + 4]) * inv_l,
                          __uint_as_float(orow[8 * k16 + 5]) * inv_l);
        v.w = pack_bf16x2(__uint_as_float(orow[8 * k16 + 6]) * inv_l,
                          __uint_as_float(orow[8 * k16 + 7]) * inv_l);
        const int gsub = k16 >> 3, cc = k16 & 7;
        *reinterpret_cast<uint4*>(stg + gsub * L::kSubBytes + ((cc ^ (r & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_STG_READY));
      if (store_thread) {
        // (a CTA whose rows all lie past N, the odd one of a last pair tile
        // of at most 128 rows, stores nothing)
        if (wait_bounded(BAR(B_STG_READY), u & 1, wc, 28) && row0 < p.N) {
          for (int gs = 0; gs < 2; ++gs)
            tma_store_3d(&tmO, sbase + L::kOffStg + gs * L::kSubBytes, gs * 64, row0, bh);
          bulk_commit_group();
        }
      }
      store_pending = true;
    }
    if (store_thread) {
      bulk_wait_group0();
      if (store_pending) mbar_arrive(BAR(B_STG_FREE));
    }
    tc_fence_before();
    __syncthreads();
  }
  // the other CTA's last arrivals on this CTA's barriers, and its last reads
  // of its own shared memory by this CTA's MMAs, are done
  cluster_sync_all();
}

template <bool CAUSAL>
fa_status launch(const CUtensorMap& mq, const CUtensorMap& mk64, const CUtensorMap& mv,
                 const CUtensorMap& mo, const PairParams& p, const LaunchCtx& ctx) {
  auto kern = fwd_pair_kernel<CAUSAL>;
  const int smem = Layout::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(fwd pair)");
  cudaFuncAttributes attr;
  e = cudaFuncGetAttributes(&attr, kern);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes(fwd pair)");
  if (attr.numRegs != kRegsAtLaunch) {
    set_last_error("fwd pair kernel built with %d registers per thread, expected %d", attr.numRegs,
                   kRegsAtLaunch);
    return FA_ERR_UNSUPPORTED;
  }
  const int pairs = min(p.num_items, ctx.num_sms / 2);
  {
    ProfileScope prof(KID_FWD, ctx.stream);
    kern<<<2 * pairs, kThreads, smem, ctx.stream>>>(mq, mk64, mv, mo, p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fwd pair kernel launch");
  return FA_OK;
}

}  // namespace

fa_status launch_fwd_pair(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int N, int d, float scale, bool causal,
                          const LaunchCtx& ctx) {
  if (d != 128) {
    set_last_error("the CTA-pair forward is built for d = 128 (got %d)", d);
    return FA_ERR_UNSUPPORTED;
  }
  const uint64_t BH = uint64_t(B) * uint64_t(H);
  CUtensorMap mq, mk64, mv, mo;
  fa_status st;
  if ((st = make_tmap_3d(&mq, q, 2, d, N, BH, 64, 128, 128)) != FA_OK) return st;
  if ((st = make_tmap_3d(&mk64, k, 2, d, N, BH, 64, 64, 128)) != FA_OK) return st;
  if ((st = make_tmap_3d(&mv, v, 2, d, N, BH, 64, 128, 128)) != FA_OK) return st;
  if ((st = make_tmap_3d(&mo, o, 2, d, N, BH, 64, 128, 128)) != FA_OK) return st;
  PairParams p;
  p.lse = lse;
  p.N = N;
  p.BH = int(BH);
  p.n_kv = (N + kBN - 1) / kBN;
  p.n_qp = (N + 2 * kBM - 1) / (2 * kBM);
  p.num_items = p.BH * p.n_qp;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = ctx.status_word;
  p.limit_ns = ctx.wait_limit_ns;
  return causal ? launch<true>(mq, mk64, mv, mo, p, ctx) : launch<false>(mq, mk64, mv, mo, p, ctx);
}

}  // namespace fa
