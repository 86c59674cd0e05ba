// fwd_sm100.cu -- attention forward for B200 (sm_100a): one Q tile per CTA
// at a time, two softmax warpgroups taking turns, two MMA issuing threads.
//
// What it computes ("Bellek Duvarinin Fizigi", sections "Online Softmax",
// "Forward gecisin iskeleti" and "Maskeleme ve Dropout"; notation of
// "FlashAttention'i Anlamak Bolum 1", 0.2): O_i = sum_j softmax_j(S_i) V_j, S_ij = scale * q_i . k_j, and
// LSE_i = ln sum_j exp(S_ij), with the row softmax carried by a running
// maximum and running sum and O = O~ / l once at the end; the causal mask
// skips K/V tiles above the diagonal and puts -inf in the masked entries of
// the diagonal tile before the row maximum.
//
// Design (measured on this hardware: a tcgen05.mma of 128 x 128 x 16 runs
// ~64 cycles and costs its issuing thread ~50, a commit ~50, an mbarrier
// hand-off ~130, and the 128 exponentials of a row take one softmax warp
// ~1500 cycles; with one issuing thread and one softmax warp per row, the
// issuer's serial waits, commits and issues, not the tensor pipe, set the
// pace):
//  * TMEM (512 columns): S_0 | S_1 | O | Q | P. Q (bf16, the A operand of
//    Q K^T) is copied from shared memory by tcgen05.cp once per unit, so
//    Q K^T reads only K from shared memory; P (bf16, the A operand of P V)
//    has its own 64 columns, so a score buffer is free as soon as the
//    softmax has loaded it.
//  * Two issuing threads: one issues Q K^T(g) into S_{g%2} once the softmax
//    has loaded S(g-2); the other issues P V(g) once P(g) is in TMEM. The
//    two streams share no TMEM columns (each thread's tcgen05.commit tracks
//    only its own MMAs), so neither waits for the other's hand-offs.
//  * Two softmax warpgroups take the K/V steps of a tile in turn (group
//    g % 2 does step g), so one group's exponentials overlap the other's
//    load, maximum and hand-offs. They share the reference maximum of each
//    row through shared memory: step g reads the reference left by step
//    g-1, raises it if its own row maximum exceeds it by more than 2^8 (then
//    O~ is rescaled in TMEM after P V(g-1)), and passes it on. Each group
//    keeps its own partial row sum, rescaled whenever the reference moves;
//    the group of a unit's last step adds the other group's sum and writes
//    O (through a swizzled staging tile and TMA stores) and the LSE. P(g)
//    is formed in registers and stored once P V(g-1) has read P(g-1).
//  * 12 warps: 0-3 and 4-7 the softmax groups (one TMEM lane = one query
//    row), 8 the Q/K producer, 9 the Q K^T issuer, 10 the V producer, 11 the
//    P V issuer; the last warpgroup gives registers to the softmax groups
//    via setmaxnreg.
//  * work units (head, Q tile): head-major without the mask; under the mask,
//    heaviest level first over all heads, dealt to the persistent CTAs in
//    snake order (round r gives CTA c item rG + c, or rG + G-1-c for odd r).
//  * every mbarrier wait is bounded in time; a wait that runs out records the
//    failure in the device status word and the CTA returns.
//  * every barrier that more than one warp or thread waits on is either
//    waited for each of its phases in turn by its one waiter, or indexed so
//    that a waiter is never more than one phase away from the phase it
//    waits for (the arguments are given at each barrier).
//
// The FP8 instantiation (F8, d = 128; "FlashAttention-3 (TR)", section
// "FlashAttention-3'un Teknik Yenilikleri", item 3) runs the same pipeline
// on e4m3 codes prepared by fp8_prep.cu: Q and K codes with one scale per
// 128-row block, V transposed ([d, keys] per head, so it is the K-major B
// operand of P V) with one scale per head. Both products are
// tcgen05.mma .kind::f8f6f4 (K = 32 per instruction); the scores of step j
// are scaled by scale * log2(e) * q_scale(Q tile) * k_scale(K tile); P~ is
// rounded to e4m3 (it is at most 2^8, the lazy-rescale bound, inside
// e4m3's 448) while the row sum keeps the fp32 values; the epilogue
// multiplies O~ by v_scale / l.
//
// The EX instantiation (bf16) adds the two options of "FlashAttention'i
// Anlamak Bolum 1", 0.2 (S = Q K^T / sqrt(d) + B) and "Bellek Duvarinin
// Fizigi", "Maskeleme ve Dropout" (dropout on P from a counter-based
// generator driven by a seed and an offset, regenerated in the backward):
//  * bias: each softmax thread adds bias[b, h, row, keys of the tile] / scale
//    to its raw scores before the mask and the row maximum (16-byte loads
//    when rows and strides allow, else 2-byte loads; prefetching them
//    before the wait for S needs 64 more registers than the softmax has);
//  * dropout: Philox4x32-10 with counter (key / 16, row, b H + h, offset)
//    and key = the seed gives one byte per (row, key); the key is kept iff
//    its byte < t, t = round(256 (1 - p)); the calls are made inside the
//    exponential loop, one per 16 keys (forming the bits before the wait
//    for S was slower: more live registers); the row sum uses the undropped
//    P~, the P V operand P~ * 256 / t or 0.
#include <cfloat>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kBM = 128;  // query rows per Q tile
constexpr int kBN = 128;  // keys per K/V tile
constexpr int kThreads = 384;
// 65536 / 384 rounded down to a multiple of 8; softmax groups 208 each and
// control 88: 128 * (2 * 208 + 88) = 384 * 168.
constexpr int kRegsAtLaunch = 168;
constexpr int kRegsSoftmax = 208;
constexpr int kRegsControl = 88;
static_assert(128 * (2 * kRegsSoftmax + kRegsControl) <= kThreads * kRegsAtLaunch,
              "register split exceeds the launch allocation");
constexpr int kQkLoadWarp = 8;  // Q and K producer
constexpr int kQkMmaWarp = 9;   // Q K^T issuer (also allocates TMEM)
constexpr int kVLoadWarp = 10;  // V producer
constexpr int kPvMmaWarp = 11;  // P V issuer
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kMaxStages = 4;

enum : int {
  B_Q_FULL = 0,
  B_Q_EMPTY = 1,      // the Q tile has been copied to TMEM
  B_S_FULL = 2,       // +g%2: Q K^T(g) finished
  B_S_FREE = 4,       // +g%2: the softmax has loaded S(g) (4 warps)
  // +g%4: P(g) is in TMEM (the 4 warps of group g%2). A warp reaches step
  // g+4 only after every warp of its group has passed step g+2 (through the
  // DEC chain), so arrivals of two steps never mix.
  B_P_FULL = 6,
  B_P_EMPTY = 10,     // +g%2: P V(g) finished (P free, O~ through step g)
  // +g%2: step g's reference maximum is in shared memory (the 4 warps of
  // group g%2). Step g waits for phase (g-1)/2 of DEC_(g-1)%2: its previous
  // phase (step g-3) was waited for by this group at step g-2, and its next
  // (step g+1) needs this step's arrival, so the parity wait is exact.
  B_DEC = 12,
  B_LDONE = 14,       // +k%2: the non-final group's row sums of a unit (4 warps)
  // +f: the last P V of a unit whose final step group f does has finished;
  // each group waits for every phase of its own barrier in turn.
  B_O_FULL = 16,
  B_O_EMPTY = 18,     // the final group has read O (4 warps)
  B_STG_READY = 19,   // the final group's 4 warps have written the staging tile
  B_STG_FREE = 20,    // the O store of the previous unit has read the staging tile
  B_DRAIN = 21,       // +issuer
  B_K_FULL = 23,
  B_K_EMPTY = B_K_FULL + kMaxStages,
  B_V_FULL = B_K_EMPTY + kMaxStages,
  B_V_EMPTY = B_V_FULL + kMaxStages,
  B_COUNT = B_V_EMPTY + kMaxStages
};

template <int D, bool F8>
struct Layout {
  static constexpr int kElem = F8 ? 1 : 2;             // bytes per Q/K/V element
  static constexpr int kSub = D * kElem / 128;         // 128-byte column groups per row
  static constexpr int kSubBytes = 128 * 128;          // 128 rows x 128 bytes
  static constexpr int kTileBytes = kSub * kSubBytes;  // a Q, K or V (V^T for F8) tile
  static constexpr int kStgBytes = (D * 2 / 128) * kSubBytes;  // bf16 O staging tile
  static constexpr int kKSteps = D * kElem / 32;       // 32-byte K steps of Q K^T
  static constexpr int kPvSteps = kBN * kElem / 32;    // 32-byte K steps of P V
  static constexpr int kSubElems = 128 / kElem;        // elements per 128-byte group
  static constexpr int kKStages = (F8 || D == 64) ? 4 : 2;
  static constexpr int kVStages = kKStages;
  static_assert(kKStages <= kMaxStages && kVStages <= kMaxStages, "barrier slots");
  static constexpr int kOffQ = 0;
  static constexpr int kOffStg = kTileBytes;  // O staging tile
  static constexpr int kOffK = kOffStg + kStgBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
  static constexpr int kOffMref = kOffBar + 8 * B_COUNT;  // [128] reference maxima
  static constexpr int kOffLsum = kOffMref + kBM * 4;      // [2][2][128] (l, m) of the other group
  static constexpr int kOffMisc = kOffLsum + 4 * kBM * 4;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory");
  // TMEM columns: S_0 | S_1 | O | Q | P (Q and P packed, 4 bytes per column)
  static constexpr uint32_t kColS1 = 128, kColO = 256, kColQ = 256 + D;
  static constexpr uint32_t kColP = kColQ + kKSteps * 8;
  static_assert(kColP + kPvSteps * 8 <= 512, "TMEM columns");
};
struct FwdParams {
  float* lse;
  int N;
  int BH;
  int n_q;        // Q tiles (and K/V tiles) per head
  int num_items;  // BH * n_q
  float scale_log2;
  unsigned int* status;
  unsigned long long limit_ns;
  int debug_skip;
  // F8 only: block scales of the Q and K codes [BH, n_q], V amax [BH]
  const float* q_scale;
  const float* k_scale;
  const float* v_amax;
};
// The bias / dropout options (EX instantiations), a kernel parameter of
// their own: growing FwdParams changed the register allocation of the
// other instantiations.
struct FwdExParams {
  const uint16_t* bias;  // bf16, element strides over b and h, rows of N
  long long bias_sb, bias_sh;
  int H;
  int bias_vec;  // rows and strides are multiples of 8 elements: 16-byte loads
  float inv_scale;
  uint32_t seed_lo, seed_hi, rng_offset;
  int keep_t;    // keep iff byte < keep_t; 256 = no dropout
  float keep_scale;
};

// bias[b, h, row, key0 .. key0 + 127] / scale added to the raw scores s
// (keys >= N are left alone: the mask removes them)
__device__ __forceinline__ void add_bias_row(float (&s)[128], const FwdExParams& p, int N, int bh,
                                             int row, int key0) {
  const int b = bh / p.H, h = bh - b * p.H;
  const uint16_t* src = p.bias + b * p.bias_sb + h * p.bias_sh + size_t(row) * N + key0;
  const int n = min(128, N - key0);
  if (p.bias_vec) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      if (8 * c < n) {
        const uint4 u = *reinterpret_cast<const uint4*>(src + 8 * c);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          s[8 * c + 2 * e] = fmaf(__uint_as_float(w[e] << 16), p.inv_scale, s[8 * c + 2 * e]);
          s[8 * c + 2 * e + 1] =
              fmaf(__uint_as_float(w[e] & 0xffff0000u), p.inv_scale, s[8 * c + 2 * e + 1]);
        }
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 128; ++i)
      if (i < n) s[i] = fmaf(__uint_as_float(uint32_t(src[i]) << 16), p.inv_scale, s[i]);
  }
}

// The work list every role of a CTA walks (G = grid size). No mask: item i
// = (head i / n_q, Q tile i % n_q), CTA c takes c, c + G, ... (the ~G units
// in flight share few heads, whose K/V stay in L2). Causal: item i = (level
// n_q-1 - i / BH, head i % BH), heaviest first, round r gives CTA c item
// r G + c for even r and r G + G-1-c for odd r.
template <bool CAUSAL>
struct Walk {
  int k;
  __device__ __forceinline__ explicit Walk(int start) : k(start) {}
  __device__ __forceinline__ bool next(const FwdParams& p, int& bh, int& qt) {
    if (CAUSAL) {
      const int G = int(gridDim.x), c = int(blockIdx.x);
      const int idx = k * G + ((k & 1) ? G - 1 - c : c);
      if (idx >= p.num_items) return false;
      qt = p.n_q - 1 - idx / p.BH;
      bh = idx % p.BH;
      ++k;
      return true;
    }
    if (k >= p.num_items) return false;
    bh = k / p.n_q;
    qt = k % p.n_q;
    k += int(gridDim.x);
    return true;
  }
};
template <bool CAUSAL>
__device__ __forceinline__ Walk<CAUSAL> walk_start() {
  return Walk<CAUSAL>(CAUSAL ? 0 : int(blockIdx.x));
}
template <bool CAUSAL>
__device__ __forceinline__ int steps_of(int qt, int n_q) {
  return CAUSAL ? qt + 1 : n_q;
}

template <int D, bool CAUSAL, bool F8, bool EX>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                const FwdParams p, const FwdExParams px) {
  static_assert(!F8 || D == 128, "the FP8 forward is built for d = 128");
  static_assert(!(F8 && EX), "bias and dropout are built for the bf16 forward");
  using L = Layout<D, F8>;
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

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_Q_FULL), 1);
    mbar_init(BAR(B_Q_EMPTY), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(B_S_FULL + i), 1);
      mbar_init(BAR(B_S_FREE + i), 4);
      mbar_init(BAR(B_P_EMPTY + i), 1);
      mbar_init(BAR(B_LDONE + i), 4);
      mbar_init(BAR(B_O_FULL + i), 1);
      mbar_init(BAR(B_DRAIN + i), 1);
      mbar_init(BAR(B_DEC + i), 4);
    }
    for (int i = 0; i < 4; ++i) mbar_init(BAR(B_P_FULL + i), 4);
    mbar_init(BAR(B_O_EMPTY), 4);
    mbar_init(BAR(B_STG_READY), 4);
    mbar_init(BAR(B_STG_FREE), 1);
    for (int s = 0; s < L::kKStages; ++s) {
      mbar_init(BAR(B_K_FULL + s), 1);
      mbar_init(BAR(B_K_EMPTY + s), 1);
    }
    for (int s = 0; s < L::kVStages; ++s) {
      mbar_init(BAR(B_V_FULL + s), 1);
      mbar_init(BAR(B_V_EMPTY + s), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kQkMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == kQkLoadWarp && lane == 0) {
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    tma_prefetch_map(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.status, p.limit_ns, KID_FWD};

  if (warp >= 8) {
    regs_decrease<kRegsControl>();
    if (warp == kQkLoadWarp && lane == 0) {
      // ------------------------------------------------------------------ Q and K producer
      int k_issued[L::kKStages] = {};
      int q_issued = 0, kv = 0;
      bool ok = true;
      Walk<CAUSAL> w = walk_start<CAUSAL>();
      int bh, qt;
      for (int u = 0; ok && w.next(p, bh, qt); ++u) {
        const int n = steps_of<CAUSAL>(qt, p.n_q);
        // the slot is free once Q of the previous unit has been copied to TMEM
        if (u > 0) {
          ok = wait_bounded(BAR(B_Q_EMPTY), (u - 1) & 1, wc, 1);
          if (!ok) break;
        }
        mbar_arrive_expect_tx(BAR(B_Q_FULL), L::kTileBytes);
        for (int c = 0; c < L::kSub; ++c)
          tma_load_3d(sbase + L::kOffQ + c * L::kSubBytes, &tmQ, BAR(B_Q_FULL), c * L::kSubElems,
                      qt * kBM, bh);
        ++q_issued;
        for (int j = 0; ok && j < n; ++j, ++kv) {
          const int s = kv % L::kKStages;
          ok = wait_bounded(BAR(B_K_EMPTY + s), ((kv / L::kKStages) & 1) ^ 1, wc, 2);
          if (!ok) break;
          mbar_arrive_expect_tx(BAR(B_K_FULL + s), L::kTileBytes);
          for (int c = 0; c < L::kSub; ++c)
            tma_load_3d(sbase + L::kOffK + s * L::kTileBytes + c * L::kSubBytes, &tmK,
                        BAR(B_K_FULL + s), c * L::kSubElems, j * kBN, bh);
          ++k_issued[s];
        }
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA exits
        if (q_issued) wait_bounded(BAR(B_Q_FULL), (q_issued - 1) & 1, wc, 3, true);
        for (int s = 0; s < L::kKStages; ++s)
          if (k_issued[s]) wait_bounded(BAR(B_K_FULL + s), (k_issued[s] - 1) & 1, wc, 3, true);
      }
    } else if (warp == kVLoadWarp && lane == 0) {
      // ------------------------------------------------------------------ V producer
      int v_issued[L::kVStages] = {};
      int kv = 0;
      bool skip_pending = p.debug_skip && blockIdx.x == 0;
      bool ok = true;
      Walk<CAUSAL> w = walk_start<CAUSAL>();
      int bh, qt;
      while (ok && w.next(p, bh, qt)) {
        const int n = steps_of<CAUSAL>(qt, p.n_q);
        for (int j = 0; ok && j < n; ++j, ++kv) {
          const int s = kv % L::kVStages;
          ok = wait_bounded(BAR(B_V_EMPTY + s), ((kv / L::kVStages) & 1) ^ 1, wc, 4);
          if (!ok) break;
          if (skip_pending) {
            skip_pending = false;  // test hook: this V tile never arrives
            continue;
          }
          mbar_arrive_expect_tx(BAR(B_V_FULL + s), L::kTileBytes);
          if constexpr (F8) {
            // V^T tile: d rows x 128 keys
            tma_load_3d(sbase + L::kOffV + s * L::kTileBytes, &tmV, BAR(B_V_FULL + s), j * kBN, 0,
                        bh);
          } else {
            for (int c = 0; c < L::kSub; ++c)
              tma_load_3d(sbase + L::kOffV + s * L::kTileBytes + c * L::kSubBytes, &tmV,
                          BAR(B_V_FULL + s), c * 64, j * kBN, bh);
          }
          ++v_issued[s];
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < L::kVStages; ++s)
          if (v_issued[s]) wait_bounded(BAR(B_V_FULL + s), (v_issued[s] - 1) & 1, wc, 5, true);
      }
    } else if (warp == kQkMmaWarp && lane == 0) {
      // ------------------------------------------------------------------ Q K^T issuer
      constexpr uint32_t idesc_qk =
          F8 ? idesc_e4m3(kBM, kBN, false, false) : idesc_bf16(kBM, kBN, false, false);
      const uint32_t tQ = tmem + L::kColQ;
      bool ok = true;
      Walk<CAUSAL> w = walk_start<CAUSAL>();
      int bh, qt, g = 0;
      for (int u = 0; ok && w.next(p, bh, qt); ++u) {
        const int n = steps_of<CAUSAL>(qt, p.n_q);
        // Q of the unit into TMEM (after this thread's last Q K^T of the
        // previous unit, in issue order)
        ok = wait_bounded(BAR(B_Q_FULL), u & 1, wc, 10);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < L::kKSteps; ++kk) {
          const uint32_t off = (kk >> 2) * L::kSubBytes + (kk & 3) * 32;
          tmem_cp_128x256b(tQ + kk * 8, sdesc_sw128(sbase + L::kOffQ + off, 16, 1024));
        }
        tc_commit(BAR(B_Q_EMPTY));
        for (int j = 0; ok && j < n; ++j, ++g) {
          const int b = g & 1;
          // S_b is free once the softmax has loaded S(g-2) (this thread
          // waits for every phase of S_FREE_b in turn)
          if (g >= 2) {
            ok = wait_bounded(BAR(B_S_FREE + b), ((g >> 1) - 1) & 1, wc, 11);
            if (!ok) break;
          }
          const int s = g % L::kKStages;
          ok = wait_bounded(BAR(B_K_FULL + s), (g / L::kKStages) & 1, wc, 12);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kb = sbase + L::kOffK + s * L::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < L::kKSteps; ++kk) {
            const uint32_t off = (kk >> 2) * L::kSubBytes + (kk & 3) * 32;
            if constexpr (F8)
              mma_ts_f8(tmem + (b ? L::kColS1 : 0u), tQ + kk * 8, sdesc_sw128(kb + off, 16, 1024),
                        idesc_qk, kk > 0 ? 1u : 0u);
            else
              mma_ts(tmem + (b ? L::kColS1 : 0u), tQ + kk * 8, sdesc_sw128(kb + off, 16, 1024),
                     idesc_qk, kk > 0 ? 1u : 0u);
          }
          tc_commit(BAR(B_S_FULL + b));
          tc_commit(BAR(B_K_EMPTY + s));
        }
      }
      // every MMA issued above must be finished before TMEM is released
      tc_commit(BAR(B_DRAIN + 0));
      wait_bounded(BAR(B_DRAIN + 0), 0, wc, 16, true);
    } else if (warp == kPvMmaWarp && lane == 0) {
      // ------------------------------------------------------------------ P V issuer
      // bf16: V [keys, d] tile, MN-major B; F8: V^T [d, keys] tile, K-major B
      constexpr uint32_t idesc_pv =
          F8 ? idesc_e4m3(kBM, D, false, false) : idesc_bf16(kBM, D, false, true);
      const uint32_t tO = tmem + L::kColO, tP = tmem + L::kColP;
      bool ok = true;
      Walk<CAUSAL> w = walk_start<CAUSAL>();
      int bh, qt, g = 0;
      for (int u = 0; ok && w.next(p, bh, qt); ++u) {
        const int n = steps_of<CAUSAL>(qt, p.n_q);
        for (int j = 0; ok && j < n; ++j, ++g) {
          ok = wait_bounded(BAR(B_P_FULL + (g & 3)), (g >> 2) & 1, wc, 13);
          if (!ok) break;
          const int s = g % L::kVStages;
          ok = wait_bounded(BAR(B_V_FULL + s), (g / L::kVStages) & 1, wc, 14);
          if (!ok) break;
          if (j == 0) {
            // the epilogue of the previous unit has read O
            ok = wait_bounded(BAR(B_O_EMPTY), (u & 1) ^ 1, wc, 15);
            if (!ok) break;
          }
          tc_fence_after();
          const uint32_t vb = sbase + L::kOffV + s * L::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < L::kPvSteps; ++kk) {
            if constexpr (F8)
              mma_ts_f8(tO, tP + kk * 8, sdesc_sw128(vb + kk * 32, 16, 1024), idesc_pv,
                        (j > 0 || kk > 0) ? 1u : 0u);
            else
              mma_ts(tO, tP + kk * 8, sdesc_sw128(vb + kk * 16 * 128, L::kSubBytes, 1024), idesc_pv,
                     (j > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(BAR(B_P_EMPTY + (g & 1)));
          tc_commit(BAR(B_V_EMPTY + s));
          if (j + 1 == n) tc_commit(BAR(B_O_FULL + (g & 1)));  // group g % 2 finishes the unit
        }
      }
      tc_commit(BAR(B_DRAIN + 1));
      wait_bounded(BAR(B_DRAIN + 1), 0, wc, 17, true);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kQkMmaWarp) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  } else {
    // ------------------------------------------------------------------ softmax groups
    regs_increase<kRegsSoftmax>();
    const int grp = warp >> 2;             // this group takes the steps g with g % 2 == grp
    const int r = (warp & 3) * 32 + lane;  // row inside the Q tile
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + lane_base + L::kColO;
    const uint32_t tP = tmem + lane_base + L::kColP;
    const bool store_thread = (warp & 3) == 0 && lane == 0;
    bool ok = true;
    bool store_pending = false;  // this group's last O store is not yet confirmed read
    Walk<CAUSAL> w = walk_start<CAUSAL>();
    int bh, qt, g = 0, nld = 0, nfin = 0;
    for (int u = 0; ok && w.next(p, bh, qt); ++u) {
      const int n = steps_of<CAUSAL>(qt, p.n_q);
      const int row = qt * kBM + r;
      const bool final_group = ((g + n - 1) & 1) == grp;
      // scores -> log2 units: scale * log2(e), times the Q and K block scales for F8
      const float cq = F8 ? p.scale_log2 * p.q_scale[size_t(bh) * p.n_q + qt] : p.scale_log2;
      float m_ref = -INFINITY, l_part = 0.f;
      for (int j = 0; j < n; ++j, ++g) {
        if ((g & 1) != grp) continue;
        // confirm this group's previous O store has read the staging tile
        // (before any wait: the other group's next epilogue waits for it)
        if (store_pending) {
          if (store_thread) {
            bulk_wait_group_read0();
            mbar_arrive(BAR(B_STG_FREE));
          }
          store_pending = false;
        }
        // S(g): this group loaded S(g-2) itself, and Q K^T(g+2) needs this
        // step's S_FREE, so the wait is exact
        const float c = F8 ? cq * p.k_scale[size_t(bh) * p.n_q + j] : cq;
        const uint64_t c2 = f2_pack(c, c);
        ok = wait_bounded(BAR(B_S_FULL + (g & 1)), (g >> 1) & 1, wc, 20);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld128_wait(tmem + lane_base + ((g & 1) ? L::kColS1 : 0u), sr);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_S_FREE + (g & 1)));
        float s[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(sr[i]);
        if constexpr (EX) {
          if (px.bias != nullptr && row < p.N) add_bias_row(s, px, p.N, bh, row, j * kBN);
        }
        // mask: the diagonal tile under the causal mask, and keys >= N
        int limit = p.N - j * kBN;
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
        const float mxc = fmaxf(max3f(mx0, mx1, mx2), mx3) * c;
        // step g-1 (the other group) has published its reference and is done
        // reading m_sh once its DEC arrival is complete (a warp arrives for
        // step g+2 only after DEC(g+1), which waited for all of step g)
        if (g > 0) {
          ok = wait_bounded(BAR(B_DEC + ((g - 1) & 1)), ((g - 1) >> 1) & 1, wc, 21);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
        }
        // P V(g-1) done: this group waited for P V(g-3) at step g-2, and
        // P V(g+1) needs this step's P, so the parity identifies the phase
        bool pv_prev_done = g == 0;
        auto wait_pv_prev = [&]() -> bool {
          if (pv_prev_done) return true;
          bool w_ok = wait_bounded(BAR(B_P_EMPTY + ((g - 1) & 1)), ((g - 1) >> 1) & 1, wc, 22);
          w_ok = __all_sync(0xffffffffu, w_ok);
          pv_prev_done = w_ok;
          return w_ok;
        };
        if (j == 0) {
          m_ref = mxc;  // the first tile of a row always has a visible key
        } else {
          const float m_prev = m_sh[r];
          if (m_prev != m_ref) {
            if (m_ref != -INFINITY) l_part *= ex2_approx(m_ref - m_prev);
            m_ref = m_prev;
          }
          const float m_new = fmaxf(m_ref, mxc);
          if (__any_sync(0xffffffffu, m_new > m_ref + kRescaleThreshold)) {
            // O~ must hold the sum through step g-1
            ok = wait_pv_prev();
            if (!ok) break;
            tc_fence_after();
            // (EX: a row whose keys a -inf bias has hidden so far holds nothing
            // yet, and 2^(-inf - m_new) would be NaN when m_new is -inf too)
            const float alpha = (EX && m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - m_new);
            l_part *= alpha;
            m_ref = m_new;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
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
        // P = 2^(s c - m_ref) by one paired FMA per two columns and MUFU ex2,
        // row sum by paired adds, packed to bf16 (e4m3 for F8) in registers
        // a bias of -inf can hide every key a row has seen so far (m_ref =
        // -inf): its P is then 0, formed against the reference 0
        const float m_use = (EX && m_ref == -INFINITY) ? 0.f : m_ref;
        const uint64_t nm2 = f2_pack(-m_use, -m_use);
        uint64_t sum_a = f2_pack(0.f, 0.f), sum_b = sum_a;
        uint32_t pk[L::kPvSteps * 8];
        uint32_t keep16b = 0;  // EX: keep bits of the current 16-key block
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s[2 * i], s[2 * i + 1]), c2, nm2), x0, x1);
          float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          if (i & 1)
            sum_b = f2_add(sum_b, f2_pack(p0, p1));
          else
            sum_a = f2_add(sum_a, f2_pack(p0, p1));
          if constexpr (EX) {
            if (px.keep_t < 256) {
              // keys j*128 + 2i and + 1: bits 2i % 16 and + 1 of the call for
              // key block (j*128 + 2i) / 16, made every eight pairs
              if ((i & 7) == 0)
                keep16b = keep_bits16(make_uint4(uint32_t(j * (kBN / 16) + i / 8), uint32_t(row),
                                                 uint32_t(bh), px.rng_offset),
                                      px.seed_lo, px.seed_hi, uint32_t(px.keep_t));
              const uint32_t kw = keep16b >> (2 * (i & 7));
              p0 = (kw & 1u) ? p0 * px.keep_scale : 0.f;
              p1 = (kw & 2u) ? p1 * px.keep_scale : 0.f;
            }
          }
          if constexpr (F8) {
            const uint32_t h = pack_e4m3x2(p0, p1);
            pk[i >> 1] = (i & 1) ? (pk[i >> 1] | (h << 16)) : h;
          } else {
            pk[i] = pack_bf16x2(p0, p1);
          }
        }
        // P(g) over P(g-1) once P V(g-1) has read it
        ok = wait_pv_prev();
        if (!ok) break;
        tc_fence_after();
        if constexpr (F8) {
          tmem_st32(tP, pk);
        } else {
          tmem_st64(tP, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_P_FULL + (g & 3)));
        {
          float a0, a1;
          f2_unpack(f2_add(sum_a, sum_b), a0, a1);
          l_part += a0 + a1;
        }
        if (j == n - 2) {
          // the final group (step n-1) adds this group's sum
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
        // LDONE_k%2: its previous phase (index k-2) completed steps ago and
        // the next (k+2) needs this group's later steps
        ok = wait_bounded(BAR(B_LDONE + (k_ld & 1)), (k_ld >> 1) & 1, wc, 23);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const float* ls = lsum + (k_ld & 1) * 2 * kBM;
        l += ls[r] * ex2_approx(ls[kBM + r] - m_ref);
      }
      ok = wait_bounded(BAR(B_O_FULL + grp), nfin & 1, wc, 24);
      ++nfin;
      // the staging tile is free once the store of unit u-1 has read it.
      // Unit u-1's epilogue waited for the store of u-2 before its O_EMPTY,
      // which preceded P V(0) of unit u and so our O_FULL: the wait is exact.
      if (ok && u > 0) ok = wait_bounded(BAR(B_STG_FREE), (u - 1) & 1, wc, 25);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t orow[D];
      if constexpr (D == 128) {
        tmem_ld128_wait(tO, orow);
      } else {
        tmem_ld64_wait(tO, orow);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_O_EMPTY));
      if (row < p.N) p.lse[size_t(bh) * p.N + row] = (m_ref + lg2_approx(l)) * kLn2;
      // O = O~ / l as bf16 into the staging tile (128-byte swizzle, the layout
      // of the tensor map), then TMA stores; rows past N fall outside the tensor
      float inv_l = 1.0f / l;
      if constexpr (F8) {
        const float va = p.v_amax[bh];
        inv_l *= va > 0.f ? __fdiv_rn(va, 448.0f) : 1.0f;  // the V codes' scale
      }
      uint8_t* stg = smem + L::kOffStg + r * 128;
#pragma unroll
      for (int k16 = 0; k16 < D / 8; ++k16) {
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
        // STG_READY: the previous unit's phase completed before its store,
        // which we waited for above; the next needs our store
        if (wait_bounded(BAR(B_STG_READY), u & 1, wc, 26)) {
          for (int gs = 0; gs < L::kStgBytes / L::kSubBytes; ++gs)
            tma_store_3d(&tmO, sbase + L::kOffStg + gs * L::kSubBytes, gs * 64, qt * kBM, bh);
          bulk_commit_group();
        }
      }
      store_pending = true;  // confirmed at this group's next step (or below)
    }
    if (store_thread) {
      // the last stores must be complete before the CTA exits
      bulk_wait_group0();
      if (store_pending) mbar_arrive(BAR(B_STG_FREE));
    }
    tc_fence_before();
    __syncthreads();
  }
}

template <int D, bool CAUSAL, bool F8 = false, bool EX = false>
fa_status launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                  const CUtensorMap& mo, const FwdParams& p, const LaunchCtx& ctx,
                  const FwdExParams& px) {
  auto kern = fwd_kernel<D, CAUSAL, F8, EX>;
  const int smem = Layout<D, F8>::kSmemBytes;
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
    kern<<<grid, kThreads, smem, ctx.stream>>>(mq, mk, mv, mo, p, px);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fwd kernel launch");
  return FA_OK;
}

}  // namespace

fa_status launch_fwd_bf16(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int H, int N, int d, float scale, bool causal,
                           const LaunchCtx& ctx, const FwdExtras* ex) {
  const uint64_t BH = uint64_t(B) * uint64_t(H);
  CUtensorMap mq, mk, mv, mo;
  fa_status st;
  if ((st = make_tmap_3d(&mq, q, 2, d, N, BH, 64, 128, 128)) != FA_OK) return st;
  if ((st = make_tmap_3d(&mk, k, 2, d, N, BH, 64, 128, 128)) != FA_OK) return st;
  if ((st = make_tmap_3d(&mv, v, 2, d, N, BH, 64, 128, 128)) != FA_OK) return st;
  if ((st = make_tmap_3d(&mo, o, 2, d, N, BH, 64, 128, 128)) != FA_OK) return st;
  FwdParams p;
  p.lse = lse;
  p.N = N;
  p.BH = int(BH);
  p.n_q = (N + kBM - 1) / kBM;
  p.num_items = p.BH * p.n_q;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = ctx.status_word;
  p.limit_ns = ctx.wait_limit_ns;
  p.debug_skip = ctx.debug_skip_load == KID_FWD;
  p.q_scale = p.k_scale = p.v_amax = nullptr;
  FwdExParams px;
  px.bias = nullptr;
  px.bias_sb = px.bias_sh = 0;
  px.H = H;
  px.bias_vec = 0;
  px.inv_scale = 1.0f / scale;
  px.seed_lo = px.seed_hi = px.rng_offset = 0;
  px.keep_t = 256;
  px.keep_scale = 1.0f;
  if (ex != nullptr && (ex->bias != nullptr || ex->keep_t < 256)) {
    px.bias = static_cast<const uint16_t*>(ex->bias);
    px.bias_sb = ex->bias_stride_b;
    px.bias_sh = ex->bias_stride_h;
    px.bias_vec = (N % 8 == 0 && ex->bias_stride_b % 8 == 0 && ex->bias_stride_h % 8 == 0) ? 1 : 0;
    px.seed_lo = uint32_t(ex->seed);
    px.seed_hi = uint32_t(ex->seed >> 32);
    px.rng_offset = ex->offset;
    px.keep_t = ex->keep_t;
    px.keep_scale = 256.0f / float(ex->keep_t);
    if (causal)
      return d == 128 ? launch<128, true, false, true>(mq, mk, mv, mo, p, ctx, px)
                      : launch<64, true, false, true>(mq, mk, mv, mo, p, ctx, px);
    return d == 128 ? launch<128, false, false, true>(mq, mk, mv, mo, p, ctx, px)
                    : launch<64, false, false, true>(mq, mk, mv, mo, p, ctx, px);
  }
  if (causal)
    return d == 128 ? launch<128, true>(mq, mk, mv, mo, p, ctx, px)
                    : launch<64, true>(mq, mk, mv, mo, p, ctx, px);
  return d == 128 ? launch<128, false>(mq, mk, mv, mo, p, ctx, px)
                  : launch<64, false>(mq, mk, mv, mo, p, ctx, px);
}

fa_status launch_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* q_scale,
                         const float* k_scale, const float* v_amax, void* o, float* lse, int B,
                         int H, int N, int d, float scale, bool causal, const LaunchCtx& ctx) {
  const uint64_t BH = uint64_t(B) * uint64_t(H);
  const uint64_t n_vt = uint64_t(fp8_vt_keys(N));
  CUtensorMap mq, mk, mv, mo;
  fa_status st;
  if ((st = make_tmap_3d(&mq, q8, 1, d, N, BH, 128, 128, 128)) != FA_OK) return st;
  if ((st = make_tmap_3d(&mk, k8, 1, d, N, BH, 128, 128, 128)) != FA_OK) return st;
  if ((st = make_tmap_3d(&mv, vt8, 1, n_vt, d, BH, 128, 128, 128)) != FA_OK) return st;
  if ((st = make_tmap_3d(&mo, o, 2, d, N, BH, 64, 128, 128)) != FA_OK) return st;
  FwdParams p;
  p.lse = lse;
  p.N = N;
  p.BH = int(BH);
  p.n_q = (N + kBM - 1) / kBM;
  p.num_items = p.BH * p.n_q;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = ctx.status_word;
  p.limit_ns = ctx.wait_limit_ns;
  p.debug_skip = ctx.debug_skip_load == KID_FWD;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.v_amax = v_amax;
  FwdExParams px{};
  px.H = H;
  px.keep_t = 256;
  if (d != 128) {
    set_last_error("the FP8 forward needs d = 128 (got %d)", d);
    return FA_ERR_UNSUPPORTED;
  }
  return causal ? launch<128, true, true>(mq, mk, mv, mo, p, ctx, px)
                : launch<128, false, true>(mq, mk, mv, mo, p, ctx, px);
}

}  // namespace fa
