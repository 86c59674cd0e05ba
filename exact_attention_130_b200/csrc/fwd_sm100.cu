// fwd_sm100.cu -- attention forward for B200 (sm_100a), bf16 in, fp32 accumulate.
//
// What it computes ("Bellek Duvarinin Fizigi", sections "Online Softmax" and
// "Forward gecisin iskeleti"; notation of "FlashAttention'i Anlamak Bolum 1",
// 0.2): for every query row i, O_i = sum_j softmax_j(S_i) V_j with
// S_ij = scale * q_i . k_j, and LSE_i = ln sum_j exp(S_ij). S and P never
// leave the chip: Q, K, V tiles are brought into shared memory by TMA, S and
// the output accumulator O~ sit in tensor memory (TMEM), and the row softmax
// is carried by the running maximum m and running sum l, rescaled by
// exp(m_old - m_new) whenever m grows; O = O~ / l once, at the end.
//
// Exponentials use base 2: scores are multiplied by scale * log2(e) and every
// exp(x) becomes 2^(x log2 e) ("Online Softmax", last paragraph); the saved
// LSE is converted back to the natural logarithm.
//
// Causal mask ("Maskeleme ve Dropout"): K/V tiles wholly above the diagonal
// are never loaded or multiplied; the diagonal tile gets -inf in the masked
// entries before the row maximum is taken.
//
// B200 design (not the pages' A100/H100 kernels):
//  * persistent grid, one CTA per SM, 12 warps:
//      warps 0-3  softmax for Q tile 0 (one TMEM lane = one query row)
//      warps 4-7  softmax for Q tile 1
//      warp  8    TMA producer (Q tiles once per work unit, K/V ring)
//      warp  9    tcgen05 MMA issuer (one thread)
//      warps 10-11 complete the third warpgroup (no work)
//    the control warpgroup hands registers to the softmax warpgroups
//    (setmaxnreg), so the 128 scores of a row stay in registers;
//  * a work unit is 2 Q tiles of 128 rows of one (batch, head); both share
//    every K/V tile, which halves K/V shared-memory traffic per FLOP;
//  * TMEM (512 columns): S_0 | S_1 | O_0 | O_1. The softmax writes P as bf16
//    over the first half of its S columns and the PV MMA reads it from TMEM,
//    so P never touches shared memory;
//  * while one softmax warpgroup works on its S, the tensor core runs the
//    other tile's QK^T and PV (ping-pong between the two Q tiles);
//  * O~ is rescaled only when a row maximum grows by more than 2^8 (the
//    final division by l is exact whatever reference maximum was used), so
//    the O read-modify-write almost never runs;
//  * work units are handed out head-major (K/V reuse in L2); under the
//    causal mask each CTA takes complementary pairs of Q-tile levels, so
//    the persistent CTAs carry equal work;
//  * every mbarrier wait is bounded in time; a wait that runs out records
//    the failure in the device status word and the CTA returns.
#include <cfloat>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kBM = 128;  // query rows per Q tile
constexpr int kBN = 128;  // keys per K/V tile
constexpr int kThreads = 384;  // 3 warpgroups
// Registers per thread: the kernel launches with 168 (65536 / 384, rounded
// down to a multiple of 8); the softmax warpgroups then take 208 and the
// load/MMA warpgroup keeps 88: 2*128*208 + 128*88 = 384*168.
constexpr int kRegsAtLaunch = 168;
constexpr int kRegsSoftmax = 208;
constexpr int kRegsControl = 88;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsControl <= kThreads * kRegsAtLaunch,
              "register split exceeds the launch allocation");
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale when m grows by > 2^8
constexpr float kLn2 = 0.69314718055994530942f;

// barrier slots
enum : int {
  B_Q_FULL = 0,    // +t
  B_Q_EMPTY = 2,   // +t
  B_S_FULL = 4,    // +t
  B_P_FULL = 12,   // +t: P of tile t is in TMEM
  B_O_FULL = 8,    // +t
  B_O_EMPTY = 10,  // +t
  B_DRAIN = 6,
  B_K_FULL = 16,   // +stage
  B_V_FULL = 20,   // +stage
  B_V_EMPTY = 24,  // +stage: both tiles' P V of the stage's step are done
  B_STG_FREE = 28, // the O staging buffer may be rewritten (one arrival per epilogue)
  B_STG_READY = 29, // +t: the 4 warps of softmax group t have written the staging buffer
  B_K_EMPTY = 31,  // +stage: the last Q K^T reading the stage's K tile is done
  B_COUNT = 35
};

template <int D>
struct Layout {
  static constexpr int kSub = D / 64;             // 128-byte column groups per row
  static constexpr int kSubBytes = 128 * 128;     // 128 rows x 128 bytes
  static constexpr int kTileBytes = kSub * kSubBytes;
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffStg = kOffV + kStages * kTileBytes;  // O tile staging for the TMA store
  static constexpr int kOffBar = kOffStg + kTileBytes;
  static constexpr int kOffMisc = kOffBar + 8 * B_COUNT;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
};

struct FwdParams {
  void* o;
  float* lse;
  int N;
  int BH;
  int n_kv;       // K/V tiles per head
  int n_pairs;    // Q-tile pairs per head
  int cpp;        // causal: couples of pairs per head, ceil(n_pairs / 2)
  int num_items;  // work items handed out to the CTAs
  int full_items; // split mode: items before this index are whole units
  int split_s;    // split mode: parts per split unit (along the keys)
  float* part_o;  // split mode: [slot][2 tiles][128 rows][d] fp32, O of each part normalised by its l
  float* part_lse;  // split mode: [slot][2 tiles][128 rows] base-2 LSE of each part
  float scale_log2;
  unsigned int* status;
  unsigned long long limit_ns;
  int debug_skip;
};

// Work list. A unit is one (head, Q-tile pair); every role of a CTA walks the
// same sequence (G = grid size).
//  * no mask: CTA c takes items c, c + G, c + 2G, ...; item = unit,
//    head-major, so the ~G units in flight share few heads and their K/V
//    tiles stay in L2;
//  * causal, couples: item = a couple of pairs (n_pairs-1-k, k) of one head,
//    the heavier first, taken as above; a couple always costs 2 n_pairs + 1 or
//    + 2 K/V tile steps, so equal item counts mean equal work, and the couples
//    of one head run side by side (L2 reuse again). With n_pairs odd the
//    middle pair is a couple on its own.
//  * no mask, split (a separate instantiation, chosen by the host when the
//    units leave the last round of CTAs short): items below full_items are
//    whole units as above; the remaining units are split along the keys into
//    split_s parts each (item full_items + k is part k % split_s of unit
//    full_items + k / split_s), whose partial O and LSE go to slot k and are
//    merged afterwards;
//  * causal, snake (a separate instantiation, chosen by the host when the couples leave the last round
//    of CTAs much emptier than the others, as with few heads and short
//    sequences): item = one pair, sorted by level from the heaviest down
//    (item i: level n_pairs-1-i/BH, head i%BH); round r gives CTA c item
//    r G + c for even r and r G + G-1-c for odd r, which evens out the sums.
// Advances the state and returns the unit, or false at the end.
// Work modes (a template parameter of the kernel).
constexpr int kModePlain = 0, kModeSnake = 1, kModeSplit = 2;

// kv0: first K/V tile of the item; cnt: its K/V tile count, or -1 for "as
// the mask allows"; slot: partial-result slot, or -1 for a whole unit.
template <bool CAUSAL, int MODE>
__device__ __forceinline__ bool next_unit(const FwdParams& p, int& item, int& half, int& bh,
                                          int& pair, int& kv0, int& cnt, int& slot) {
  kv0 = 0;
  cnt = -1;
  slot = -1;
  if (MODE == kModeSnake) {
    // `item` counts the rounds here (it starts at 0)
    const int G = int(gridDim.x), c = int(blockIdx.x);
    const int idx = item * G + ((item & 1) ? G - 1 - c : c);
    if (idx >= p.num_items) return false;
    pair = p.n_pairs - 1 - idx / p.BH;
    bh = idx % p.BH;
    ++item;
    return true;
  }
  // `item` is the item index (it starts at blockIdx.x)
  if (item >= p.num_items) return false;
  if (!CAUSAL) {
    int u = item;
    if (MODE == kModeSplit && item >= p.full_items) {
      const int k = item - p.full_items;
      const int part = k % p.split_s;
      u = p.full_items + k / p.split_s;
      kv0 = part * p.n_kv / p.split_s;
      cnt = (part + 1) * p.n_kv / p.split_s - kv0;
      slot = k;
    }
    bh = u / p.n_pairs;
    pair = u % p.n_pairs;
    item += gridDim.x;
    return true;
  }
  bh = item / p.cpp;
  const int k = item % p.cpp;
  const int hi = p.n_pairs - 1 - k;
  if (half == 0) {
    pair = hi;
    if (hi == k) {
      item += gridDim.x;
    } else {
      half = 1;
    }
  } else {
    pair = k;
    half = 0;
    item += gridDim.x;
  }
  return true;
}

template <bool CAUSAL>
__device__ __forceinline__ int kv_tiles_for(int qtile, int n_kv) {
  if (CAUSAL) return min(qtile + 1, n_kv);
  return n_kv;
}

template <int D, bool CAUSAL, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
               const FwdParams p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * uint32_t(i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(BAR(B_Q_FULL + t), 1);
      mbar_init(BAR(B_Q_EMPTY + t), 1);
      mbar_init(BAR(B_S_FULL + t), 1);
      mbar_init(BAR(B_P_FULL + t), 4);
      mbar_init(BAR(B_O_FULL + t), 1);
      mbar_init(BAR(B_O_EMPTY + t), 4);
    }
    mbar_init(BAR(B_DRAIN), 1);
    mbar_init(BAR(B_STG_FREE), 1);
    mbar_init(BAR(B_STG_READY + 0), 4);
    mbar_init(BAR(B_STG_READY + 1), 4);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(BAR(B_K_FULL + s), 1);
      mbar_init(BAR(B_V_FULL + s), 1);
      mbar_init(BAR(B_K_EMPTY + s), 1);
      mbar_init(BAR(B_V_EMPTY + s), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.status, p.limit_ns, KID_FWD};

  if (warp >= 8) {
    regs_decrease<kRegsControl>();
    if (warp == kLoadWarp) {
      // ------------------------------------------------------------------ TMA producer
      if (lane == 0) {
        // K and V tiles go through separate rings of kStages slots: a K slot
        // is released by the last Q K^T that reads it, a step before the P V
        // that releases the V slot of the same index, so K tiles load that
        // much earlier. Loads started per slot, for the abort path:
        int k_issued[L::kStages] = {}, v_issued[L::kStages] = {};
        int kv_issued = 0, unit_iter = 0;
        int q_issued0 = 0, q_issued1 = 0;
        bool skip_pending = p.debug_skip && blockIdx.x == 0;
        bool ok = true;
        int item = MODE == kModeSnake ? 0 : int(blockIdx.x), half = 0, bh, pair, kv0, cnt, slot;
        for (; ok && next_unit<CAUSAL, MODE>(p, item, half, bh, pair, kv0, cnt, slot); ++unit_iter) {
          const int n1 = cnt >= 0 ? cnt : kv_tiles_for<CAUSAL>(2 * pair + 1, p.n_kv);
          for (int t = 0; t < 2 && ok; ++t) {
            ok = wait_bounded(BAR(B_Q_EMPTY + t), (unit_iter & 1) ^ 1, wc, 1);
            if (!ok) break;
            mbar_arrive_expect_tx(BAR(B_Q_FULL + t), L::kTileBytes);
            for (int c = 0; c < L::kSub; ++c)
              tma_load_3d(sbase + L::kOffQ + t * L::kTileBytes + c * L::kSubBytes, &tmQ,
                          BAR(B_Q_FULL + t), c * 64, (2 * pair + t) * kBM, bh);
            (t ? q_issued1 : q_issued0) += 1;
          }
          for (int j = 0; ok && j < n1; ++j, ++kv_issued) {
            const int s = kv_issued % L::kStages;
            const uint32_t ph = (kv_issued / L::kStages) & 1;
            ok = wait_bounded(BAR(B_K_EMPTY + s), ph ^ 1, wc, 2);
            if (!ok) break;
            mbar_arrive_expect_tx(BAR(B_K_FULL + s), L::kTileBytes);
            for (int c = 0; c < L::kSub; ++c)
              tma_load_3d(sbase + L::kOffK + s * L::kTileBytes + c * L::kSubBytes, &tmK,
                          BAR(B_K_FULL + s), c * 64, (kv0 + j) * kBN, bh);
            ++k_issued[s];
            ok = wait_bounded(BAR(B_V_EMPTY + s), ph ^ 1, wc, 4);
            if (!ok) break;
            if (skip_pending) {
              skip_pending = false;  // test hook: this V tile never arrives
            } else {
              mbar_arrive_expect_tx(BAR(B_V_FULL + s), L::kTileBytes);
              for (int c = 0; c < L::kSub; ++c)
                tma_load_3d(sbase + L::kOffV + s * L::kTileBytes + c * L::kSubBytes, &tmV,
                            BAR(B_V_FULL + s), c * 64, (kv0 + j) * kBN, bh);
              ++v_issued[s];
            }
          }
        }
        if (*abort_flag) {
          // let every copy this thread started land before the CTA exits: the
          // last load into a barrier completes its phase (loads - 1)
          if (q_issued0) wait_bounded(BAR(B_Q_FULL + 0), (q_issued0 - 1) & 1, wc, 3, true);
          if (q_issued1) wait_bounded(BAR(B_Q_FULL + 1), (q_issued1 - 1) & 1, wc, 3, true);
          for (int s = 0; s < L::kStages; ++s) {
            if (k_issued[s]) wait_bounded(BAR(B_K_FULL + s), (k_issued[s] - 1) & 1, wc, 3, true);
            if (v_issued[s]) wait_bounded(BAR(B_V_FULL + s), (v_issued[s] - 1) & 1, wc, 3, true);
          }
        }
      }
    } else if (warp == kMmaWarp) {
      // ------------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        constexpr uint32_t idesc_qk = idesc_bf16(kBM, kBN, false, false);
        constexpr uint32_t idesc_pv = idesc_bf16(kBM, D, false, true);
        auto colS = [](int t) { return t ? L::kColS1 : L::kColS0; };
        auto colO = [](int t) { return t ? L::kColO1 : L::kColO0; };
        auto issue_qk = [&](int t, int stage) {
          const uint32_t qa = sbase + L::kOffQ + t * L::kTileBytes;
          const uint32_t kb = sbase + L::kOffK + stage * L::kTileBytes;
  #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kSubBytes + (kk & 3) * 32;
            mma_ss(tmem + colS(t), sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024),
                   idesc_qk, kk > 0 ? 1u : 0u);
          }
        };
        // O_t (+)= P_t V: P (bf16) from the first 64 TMEM columns of S_t
        auto issue_pv = [&](int t, int stage, bool acc) {
          const uint32_t vb = sbase + L::kOffV + stage * L::kTileBytes;
  #pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            mma_ts(tmem + colO(t), tmem + colS(t) + kk * 8,
                   sdesc_sw128(vb + kk * 16 * 128, L::kSubBytes, 1024), idesc_pv,
                   (acc || kk > 0) ? 1u : 0u);
        };
        int kv_used = 0, unit_iter = 0;
        int p_cnt[2] = {0, 0};
        bool ok = true;
        int item = MODE == kModeSnake ? 0 : int(blockIdx.x), half = 0, bh, pair, kv0, cnt, slot;
        for (; ok && next_unit<CAUSAL, MODE>(p, item, half, bh, pair, kv0, cnt, slot); ++unit_iter) {
          const int n0 = cnt >= 0 ? cnt : kv_tiles_for<CAUSAL>(2 * pair, p.n_kv);
          const int n1 = cnt >= 0 ? cnt : kv_tiles_for<CAUSAL>(2 * pair + 1, p.n_kv);
          for (int t = 0; t < 2 && ok; ++t)
            ok = wait_bounded(BAR(B_Q_FULL + t), unit_iter & 1, wc, 10);
          if (!ok) break;
          {
            const int s0 = kv_used % L::kStages;
            ok = wait_bounded(BAR(B_K_FULL + s0), (kv_used / L::kStages) & 1, wc, 11);
            if (!ok) break;
            tc_fence_after();
            // a Q tile is released after its last QK^T (not its last PV), so
            // the next unit's Q loads while this unit's last steps run
            issue_qk(0, s0);
            tc_commit(BAR(B_S_FULL + 0));
            if (n0 == 1) tc_commit(BAR(B_Q_EMPTY + 0));
            issue_qk(1, s0);
            tc_commit(BAR(B_S_FULL + 1));
            tc_commit(BAR(B_K_EMPTY + s0));  // tile 1 reads every K tile of the unit, last
            if (n1 == 1) tc_commit(BAR(B_Q_EMPTY + 1));
          }
          int k_ready = 0;
          for (int j = 0; ok && j < n1; ++j) {
            const int s = (kv_used + j) % L::kStages;
            ok = wait_bounded(BAR(B_V_FULL + s), ((kv_used + j) / L::kStages) & 1, wc, 12);
            if (!ok) break;
  #pragma unroll
            for (int t = 0; t < 2; ++t) {
              const int nt = t ? n1 : n0;
              if (j >= nt) continue;
              if (j == 0) {
                ok = wait_bounded(BAR(B_O_EMPTY + t), (unit_iter & 1) ^ 1, wc, 13);
                if (!ok) break;
              }
              ok = wait_bounded(BAR(B_P_FULL + t), p_cnt[t] & 1, wc, 14);
              if (!ok) break;
              ++p_cnt[t];
              tc_fence_after();
              issue_pv(t, s, j > 0);
              if (j + 1 < nt) {
                const int s2 = (kv_used + j + 1) % L::kStages;
                if (k_ready < j + 1) {
                  ok = wait_bounded(BAR(B_K_FULL + s2), ((kv_used + j + 1) / L::kStages) & 1, wc,
                                    15);
                  if (!ok) break;
                  k_ready = j + 1;
                  tc_fence_after();
                }
                issue_qk(t, s2);
                tc_commit(BAR(B_S_FULL + t));
                if (t == 1) tc_commit(BAR(B_K_EMPTY + s2));
                if (j + 2 == nt) tc_commit(BAR(B_Q_EMPTY + t));
              } else {
                tc_commit(BAR(B_O_FULL + t));
              }
            }
            if (!ok) break;
            tc_commit(BAR(B_V_EMPTY + s));
          }
          kv_used += n1;
        }
        // every MMA issued above must be finished before TMEM is released
        tc_commit(BAR(B_DRAIN));
        wait_bounded(BAR(B_DRAIN), 0, wc, 16, true);
      }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  } else {
    // ------------------------------------------------------------------ softmax warpgroups
    regs_increase<kRegsSoftmax>();
    const int t = warp >> 2;          // Q tile of this warpgroup
    const int wq = warp & 3;          // TMEM lane quadrant of this warp
    const int r = wq * 32 + lane;     // row inside the Q tile
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    const uint32_t tS = tmem + lane_base + (t ? L::kColS1 : L::kColS0);
    const uint32_t tO = tmem + lane_base + (t ? L::kColO1 : L::kColO0);
    const float c = p.scale_log2;
    int s_cnt = 0, unit_iter = 0;
    bool ok = true;
    int item = MODE == kModeSnake ? 0 : int(blockIdx.x), half = 0, bh, pair, kv0, cnt, slot;
    for (; ok && next_unit<CAUSAL, MODE>(p, item, half, bh, pair, kv0, cnt, slot); ++unit_iter) {
      const int qt = 2 * pair + t;
      const int nt = cnt >= 0 ? cnt : kv_tiles_for<CAUSAL>(qt, p.n_kv);
      const int row = qt * kBM + r;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < nt; ++j) {
        ok = wait_bounded(BAR(B_S_FULL + t), s_cnt & 1, wc, 20);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++s_cnt;
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld128_wait(tS, sr);
        float s[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(sr[i]);
        // mask: the diagonal tile under the causal mask, and keys >= N
        int limit = p.N - (kv0 + j) * kBN;
        if (CAUSAL && j == qt) limit = min(limit, r + 1);
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
        const float m_new = fmaxf(m, fmaxf(max3f(mx0, mx1, mx2), mx3) * c);
        if (j == 0) {
          m = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m + kRescaleThreshold)) {
          // O~ holds the sum up to tile j-1 (its MMA finished before S_j was
          // committed): multiply it by 2^(m_old - m_new)
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
        // P = 2^(s c - m): x = s c - m by one paired FMA per two columns, 2^x
        // on MUFU, row sum by paired adds; P goes to TMEM as bf16 over the
        // first 64 columns of S.
        const float neg_m = (m == -INFINITY) ? 0.f : -m;
        const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(neg_m, neg_m);
        uint64_t sum_a = f2_pack(0.f, 0.f), sum_b = sum_a;
        // P goes to TMEM in 32-column chunks as they are formed, so the stores
        // overlap the remaining exponentials (S is already in registers)
        uint32_t pk[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          if (i > 0 && (i & 15) == 0) tmem_st16(tS + (i - 16), *reinterpret_cast<uint32_t(*)[16]>(pk + i - 16));
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s[2 * i], s[2 * i + 1]), c2, nm2), x0, x1);
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          if (i & 1)
            sum_b = f2_add(sum_b, f2_pack(p0, p1));
          else
            sum_a = f2_add(sum_a, f2_pack(p0, p1));
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + 48, *reinterpret_cast<uint32_t(*)[16]>(pk + 48));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_P_FULL + t));
        {
          float a0, a1;
          f2_unpack(f2_add(sum_a, sum_b), a0, a1);
          l += a0 + a1;
        }
      }
      if (!ok) break;
      // epilogue: O = O~ / l as bf16, staged in shared memory (128-byte
      // swizzle, the layout of the tensor map) and written by TMA stores of
      // 64-column groups, so the rows need no strided global stores; LSE =
      // ln2 * (m + log2 l). One staging buffer serves both groups: the
      // epilogues of a CTA happen in the order their O_FULL commits (tile 0,
      // tile 1, next unit ...), and epilogue e waits until the store of
      // epilogue e-1 has read the buffer.
      const int e = 2 * unit_iter + t;
      ok = wait_bounded(BAR(B_O_FULL + t), unit_iter & 1, wc, 21);
      if (ok && e > 0) ok = wait_bounded(BAR(B_STG_FREE), (e - 1) & 1, wc, 22);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float inv_l = 1.0f / l;
      if (MODE == kModeSplit && slot >= 0) {
        // a part of a split unit: O of this part (normalised by its own l)
        // and its base-2 LSE go to the slot, for the merge kernel. It keeps
        // the staging barriers' sequence (one phase of each per epilogue)
        // without using the buffer.
        float* po = p.part_o + ((size_t(slot) * 2 + t) * kBM + r) * D;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t orow[32];
          tmem_ld32_wait(tO + ch * 32, orow);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            reinterpret_cast<float4*>(po + ch * 32)[v4] =
                make_float4(__uint_as_float(orow[4 * v4 + 0]) * inv_l, __uint_as_float(orow[4 * v4 + 1]) * inv_l,
                            __uint_as_float(orow[4 * v4 + 2]) * inv_l, __uint_as_float(orow[4 * v4 + 3]) * inv_l);
        }
        p.part_lse[(size_t(slot) * 2 + t) * kBM + r] = m + lg2_approx(l);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(BAR(B_O_EMPTY + t));
          mbar_arrive(BAR(B_STG_READY + t));
        }
        if (r == 0 && wait_bounded(BAR(B_STG_READY + t), unit_iter & 1, wc, 24))
          mbar_arrive(BAR(B_STG_FREE));
        continue;
      }
      uint8_t* stg = smem + L::kOffStg + r * 128;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t orow[32];
        tmem_ld32_wait(tO + ch * 32, orow);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(orow[8 * v4 + 0]) * inv_l,
                            __uint_as_float(orow[8 * v4 + 1]) * inv_l);
          w.y = pack_bf16x2(__uint_as_float(orow[8 * v4 + 2]) * inv_l,
                            __uint_as_float(orow[8 * v4 + 3]) * inv_l);
          w.z = pack_bf16x2(__uint_as_float(orow[8 * v4 + 4]) * inv_l,
                            __uint_as_float(orow[8 * v4 + 5]) * inv_l);
          w.w = pack_bf16x2(__uint_as_float(orow[8 * v4 + 6]) * inv_l,
                            __uint_as_float(orow[8 * v4 + 7]) * inv_l);
          const int k16 = ch * 4 + v4;           // 16-byte chunk of the row (8 columns)
          const int g = k16 >> 3, cc = k16 & 7;  // 64-column group, chunk in its 128-byte row
          *reinterpret_cast<uint4*>(stg + g * L::kSubBytes + ((cc ^ (r & 7)) << 4)) = w;
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();  // the staging writes, for the TMA store
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(BAR(B_O_EMPTY + t));
        mbar_arrive(BAR(B_STG_READY + t));
      }
      if (row < p.N) p.lse[size_t(bh) * p.N + row] = (m + lg2_approx(l)) * kLn2;
      if (r == 0) {
        // rows past N fall outside the tensor and are not written
        if (wait_bounded(BAR(B_STG_READY + t), unit_iter & 1, wc, 23)) {
          for (int g = 0; g < L::kSub; ++g)
            tma_store_3d(&tmO, sbase + L::kOffStg + g * L::kSubBytes, g * 64, qt * kBM, bh);
          bulk_commit_group();
          bulk_wait_group_read0();
          mbar_arrive(BAR(B_STG_FREE));
        }
      }
    }
    // the last stores must be complete before the CTA exits
    if (r == 0) bulk_wait_group0();
    tc_fence_before();
    __syncthreads();
  }
}

// O and LSE of the split units from their parts ("Online Softmax": two
// softmax partials over disjoint key sets combine exactly): with the parts'
// base-2 LSEs L_i and normalised O_i, M = max L_i, w_i = 2^(L_i - M),
// O = sum w_i O_i / sum w_i and LSE = ln2 (M + log2 sum w_i). One warp per
// row, lanes striding the d columns.
template <int D>
__global__ void __launch_bounds__(256) fwd_merge_kernel(const FwdParams p, int n_units) {
  const long long gw = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= static_cast<long long>(n_units) * 2 * kBM) return;
  const int k = int(gw / (2 * kBM)), tr = int(gw % (2 * kBM));
  const int t = tr / kBM, r = tr % kBM;
  const int u = p.full_items + k;
  const int bh = u / p.n_pairs, pair = u % p.n_pairs;
  const int row = (2 * pair + t) * kBM + r;
  if (row >= p.N) return;
  const int S = p.split_s;  // 2..4
  auto at = [&](int i) { return (size_t(k) * S + i) * 2 * kBM + size_t(t) * kBM + r; };
  // every load of every part first (S <= 4), then the arithmetic
  constexpr int kMaxParts = 4;
  float L[kMaxParts], v[kMaxParts][D / 32];
#pragma unroll
  for (int i = 0; i < kMaxParts; ++i) {
    L[i] = -INFINITY;
    if (i < S) {
      L[i] = p.part_lse[at(i)];
      const float* po = p.part_o + at(i) * D;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) v[i][q] = po[q * 32 + lane];
    } else {
#pragma unroll
      for (int q = 0; q < D / 32; ++q) v[i][q] = 0.f;
    }
  }
  const float M = fmaxf(fmaxf(L[0], L[1]), fmaxf(L[2], L[3]));
  float acc[D / 32];
#pragma unroll
  for (int q = 0; q < D / 32; ++q) acc[q] = 0.f;
  float wsum = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxParts; ++i) {
    const float w = i < S ? ex2_approx(L[i] - M) : 0.f;
    wsum += w;
#pragma unroll
    for (int q = 0; q < D / 32; ++q) acc[q] = fmaf(w, v[i][q], acc[q]);
  }
  const float inv = 1.0f / wsum;
  uint16_t* orow = reinterpret_cast<uint16_t*>(p.o) + (size_t(bh) * p.N + row) * D;
#pragma unroll
  for (int q = 0; q < D / 32; ++q) orow[q * 32 + lane] = uint16_t(pack_bf16x2(acc[q] * inv, 0.f) & 0xffffu);
  if (lane == 0) p.lse[size_t(bh) * p.N + row] = (M + lg2_approx(wsum)) * kLn2;
}

template <int D, bool CAUSAL, int MODE = kModePlain>
fa_status launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                 const CUtensorMap& mo, const FwdParams& p, const LaunchCtx& ctx) {
  auto kern = fwd_kernel<D, CAUSAL, MODE>;
  const int smem = Layout<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(fwd)");
  // the setmaxnreg split is sized for exactly kRegsAtLaunch registers per
  // thread; with fewer the increase could wait forever, so refuse to launch
  cudaFuncAttributes attr;
  e = cudaFuncGetAttributes(&attr, kern);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes(fwd)");
  if (attr.numRegs != kRegsAtLaunch) {
    set_last_error("fwd kernel built with %d registers per thread, expected %d", attr.numRegs,
                   kRegsAtLaunch);
    return FA_ERR_UNSUPPORTED;
  }
  const int grid = p.num_items < ctx.num_sms ? p.num_items : ctx.num_sms;
  {
    ProfileScope prof(KID_FWD, ctx.stream);
    kern<<<grid, kThreads, smem, ctx.stream>>>(mq, mk, mv, mo, p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fwd kernel launch");
  return FA_OK;
}

}  // namespace

fa_status launch_fwd_bf16(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int N, int d, float scale, bool causal,
                          const LaunchCtx& ctx) {
  const uint64_t BH = uint64_t(B) * uint64_t(H);
  CUtensorMap mq, mk, mv, mo;
  fa_status st;
  if ((st = make_tmap_3d(&mq, q, true, d, N, BH, 64, 128, 128)) != FA_OK) return st;
  if ((st = make_tmap_3d(&mk, k, true, d, N, BH, 64, 128, 128)) != FA_OK) return st;
  if ((st = make_tmap_3d(&mv, v, true, d, N, BH, 64, 128, 128)) != FA_OK) return st;
  if ((st = make_tmap_3d(&mo, o, true, d, N, BH, 64, 128, 128)) != FA_OK) return st;
  FwdParams p;
  p.o = o;
  p.lse = lse;
  p.N = N;
  p.BH = int(BH);
  p.n_kv = (N + kBN - 1) / kBN;
  p.n_pairs = (p.n_kv + 1) / 2;
  p.cpp = (p.n_pairs + 1) / 2;
  bool snake = false;
  p.full_items = 0;
  p.split_s = 1;
  p.part_o = nullptr;
  p.part_lse = nullptr;
  p.num_items = causal ? p.BH * p.cpp : p.BH * p.n_pairs;
  if (causal) {
    // couples carry equal work; if the last round of them leaves many CTAs
    // idle (fraction of a full round below 95%), deal single pairs instead,
    // heaviest first in snake order
    const int G = p.num_items < ctx.num_sms ? p.num_items : ctx.num_sms;
    const long long rounds = (p.num_items + G - 1) / G;
    if (double(p.num_items) / double(G) < 0.95 * double(rounds)) {
      snake = true;
      p.num_items = p.BH * p.n_pairs;
    }
  }
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = ctx.status_word;
  p.limit_ns = ctx.wait_limit_ns;
  p.debug_skip = ctx.debug_skip_load == KID_FWD;
  if (causal) {
    if (d == 128)
      return snake ? launch<128, true, kModeSnake>(mq, mk, mv, mo, p, ctx) : launch<128, true>(mq, mk, mv, mo, p, ctx);
    return snake ? launch<64, true, kModeSnake>(mq, mk, mv, mo, p, ctx) : launch<64, true>(mq, mk, mv, mo, p, ctx);
  }
  // no mask: if the last round of units fills at most half the CTAs, split
  // its units along the keys (2-4 parts, each at least one K/V tile) and
  // merge the parts afterwards
  {
    const int U = p.num_items;
    const int G = U < ctx.num_sms ? U : ctx.num_sms;
    const int full = U / G, rem = U - full * G;
    int S = rem > 0 ? G / rem : 1;
    S = S < 4 ? S : 4;
    S = S < p.n_kv ? S : p.n_kv;
    if (S >= 2) {
      p.full_items = full * G;
      p.split_s = S;
      p.num_items = p.full_items + rem * S;
      const size_t slots = size_t(rem) * S;
      const size_t o_bytes = slots * 2 * kBM * size_t(d) * 4, l_bytes = slots * 2 * kBM * 4;
      void* scratch = nullptr;
      if ((st = scratch_alloc(o_bytes + l_bytes, ctx, &scratch)) != FA_OK) return st;
      p.part_o = static_cast<float*>(scratch);
      p.part_lse = reinterpret_cast<float*>(static_cast<char*>(scratch) + o_bytes);
      st = d == 128 ? launch<128, false, kModeSplit>(mq, mk, mv, mo, p, ctx)
                    : launch<64, false, kModeSplit>(mq, mk, mv, mo, p, ctx);
      if (st == FA_OK) {
        const long long threads = static_cast<long long>(rem) * 2 * kBM * 32;
        const unsigned blocks = unsigned((threads + 255) / 256);
        ProfileScope prof(KID_FWD_MERGE, ctx.stream);
        if (d == 128)
          fwd_merge_kernel<128><<<blocks, 256, 0, ctx.stream>>>(p, rem);
        else
          fwd_merge_kernel<64><<<blocks, 256, 0, ctx.stream>>>(p, rem);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) st = cuda_fail(e, "fwd merge kernel launch");
      }
      scratch_free(scratch, ctx);
      return st;
    }
  }
  return d == 128 ? launch<128, false>(mq, mk, mv, mo, p, ctx) : launch<64, false>(mq, mk, mv, mo, p, ctx);
}

}  // namespace fa
