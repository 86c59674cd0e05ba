// decode_tct_sm100.cu -- split-KV decode of a paged KV cache for small groups
// of query heads (up to 16 per KV head, d = 128; the library uses it for 4
// to 8) on the tensor cores, with the keys as the MMA's rows ("Bellek
// Duvarinin Fizigi", sections "Duvarin Otesi" -- the KV cache, grouped-query
// and paged layouts -- and "Decode Asamasi: Flash-Decoding").
//
// What it computes is decode_tc_sm100.cu's: for sequence b, KV head hk and a
// range of the cache positions, every query head h of the group of hk gets
// o = softmax(s) V over the range's keys and lse = log2 sum exp2(s scale
// log2 e) (base 2), s_t = q_h . k_t; a merge kernel combines the ranges of
// each head by log-sum-exp.
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
// Two schedules of the same kernel:
//  * chunks (a split count given by the caller): one CTA per (chunk, KV
//    head, sequence), chunk c of sequence b covering positions
//    [c ceil(L_b / C), ...) rounded to whole tiles; partials in
//    [B, Hq, C, d], merged by decode_merge_kernel (decode_sm100.cu);
//  * balanced (the automatic split): the tiles of all (sequence, KV head)
//    segments, in sequence-major order, are cut into P equal ranges, one per
//    persistent CTA (two per SM). A CTA walks its range segment by segment
//    and keeps its pipeline running across segment boundaries (the next
//    segment's Q and first tiles load while the current one finishes; two O
//    accumulators in TMEM), so the cost of a CTA start is paid once per CTA
//    slot rather than once per chunk, and every CTA ends within a tile of
//    the others whatever the mix of lengths. The piece of segment s in CTA i
//    writes its partial to slot s + i: for a fixed segment its CTAs are
//    consecutive, and the first CTA of segment s + 1 is no earlier than the
//    last of s, so slots never collide and number at most segments + P - 1.
//    The CTA that starts a segment records the segment's first slot and
//    piece count for decode_merge_slots_kernel.
//
// Layout per CTA (192 threads: four softmax warps, a TMA warp and an MMA
// warp): tiles of 128 keys in a ring of three 32 KB slots shared by K and V
// (so two CTAs share an SM), Q and two P^T buffers of 4 KB; TMEM = S^T (two
// buffers of 16 columns) | O^T (two buffers of 16 columns).
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
// K and V tiles share one ring of three slots, loaded and consumed in the
// order the MMAs use them: K0, K1, V0, K2, V1, K3, V2, ... (S^T of the next
// tile is issued before O^T += V^T P^T of the current one), so V(j) starts to
// load as soon as S^T(j) has read K(j), and lands while the softmax of tile j
// runs
constexpr int kSlots = 3;
constexpr int kSmWarps = 4;
constexpr int kLoadWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 32 * 6;
constexpr float kRescale = 8.0f;
// balanced schedule: at most this many persistent CTAs (two per SM of a
// 148-SM part), and at most this many heads per KV head (the workspace bound)
constexpr int kMaxPersist = 2 * 148;
constexpr int kBalMaxGroup = 8;

enum : int {
  X_Q_FULL = 0,    // Q of the next piece written to shared memory (TMA warp)
  X_Q_EMPTY = 1,   // the last S^T of a piece has read Q
  X_S_FULL = 2,    // +g%2: S^T(g) in TMEM
  X_S_FREE = 4,    // +g%2: the softmax has loaded S^T(g) (4 warps)
  X_MAX = 6,       // +g%2: the four warps' tile maxima are in shared memory (4 warps)
  X_P_FULL = 8,    // +g%2: P^T(g) written (4 warps)
  X_P_EMPTY = 10,  // +g%2: O^T += V^T P^T(g) finished (P^T buffer free, O^T through tile g)
  X_O_FULL = 12,   // +k%2: O^T of piece k complete
  X_O_EMPTY = 14,  // +k%2: the softmax has loaded O^T of piece k (4 warps)
  X_LSUM = 16,     // the four warps' row sums are in shared memory (4 warps)
  X_DRAIN = 17,
  X_FULL = 18,     // +slot: a tile landed
  X_EMPTY = X_FULL + kSlots,  // +slot: its MMA has read it
  X_COUNT = X_EMPTY + kSlots
};

struct Layout {
  static constexpr int kSubBytes = kKeys * 128;   // 128 keys x 64 dims
  static constexpr int kTileBytes = 2 * kSubBytes;
  static constexpr int kOffRing = 0;
  static constexpr int kOffQ = kOffRing + kSlots * kTileBytes;  // [2 dim groups][16 heads][128 B]
  static constexpr int kOffP = kOffQ + 2 * kNH * 128;   // [2 buffers][2 key groups][16 heads][128 B]
  static constexpr int kOffRed = kOffP + 2 * 2 * kNH * 128;  // [2][4 warps][16] maxima
  static constexpr int kOffLred = kOffRed + 2 * kSmWarps * kNH * 4;
  static constexpr int kOffBar = kOffLred + kSmWarps * kNH * 4;
  static constexpr int kOffMisc = kOffBar + 8 * X_COUNT;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  // two CTAs per SM: 228 KB per SM, 1 KB of it reserved per CTA
  static_assert(2 * (kSmemBytes + 1024) <= 233472, "two CTAs per SM");
  // TMEM: S^T buffers at 0 and 16, O^T buffers at 32 and 48 (fp32, 16 columns each)
  static constexpr uint32_t kColO = 2 * kNH;
  static constexpr uint32_t kTmemCols = 64;
};

struct TctParams {
  const uint16_t* q;      // [B, Hq, D]
  const int* seqlens;
  const int* table;       // [B, max_pages]
  float* part_o;          // chunks: [B, Hq, C, D]; balanced: [slots, G, D]
  float* part_lse;        // chunks: [B, Hq, C]; balanced: [slots, G]; base 2
  int2* seg_meta;         // balanced: [B, Hkv] (first slot, piece count)
  int B, Hq, Hkv, group, C;
  int page, max_pages, num_pages, Lmax;
  float scale_log2;
  unsigned int* status;
  unsigned long long limit_ns;
  int debug_skip;
};

__device__ __forceinline__ int seq_len(const TctParams& p, int b) {
  const int L = p.seqlens[b];
  return L < 0 ? 0 : (L > p.Lmax ? p.Lmax : L);
}
__device__ __forceinline__ int tiles_of(int L) { return (L + kKeys - 1) / kKeys; }

// The slow path of a bounded wait as a call: this kernel has some twenty
// wait sites, and inlining the polling loop at each of them made the code
// large enough for instruction fetch to stall the softmax warps.
__device__ __noinline__ bool wait_slow_call(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                            unsigned int* status, unsigned long long limit,
                                            unsigned int code, bool drain) {
  return wait_bounded_slow(bar, parity, abort_flag, status, limit, code, drain);
}
__device__ __forceinline__ bool wait_nb(uint32_t bar, uint32_t parity, const WaitCtl& w,
                                        uint32_t site, bool drain = false) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow_call(bar, parity, w.abort_flag, w.status_word, w.limit_ns,
                        (w.kernel_id << 16) | ((site & 0xffu) << 8) | 1u, drain);
}

// The maximum of v over the warp (one instruction on sm_100a).
__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// TMEM loads and stores of N 32-bit columns per lane (N = 4, 8 or 16), then
// the wait for the loads / stores.
template <int N>
__device__ __forceinline__ void tmem_ldn_wait(uint32_t taddr, uint32_t (&r)[N]) {
  if constexpr (N == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];\n"
                 "tcgen05.wait::ld.sync.aligned;\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr) : "memory");
  } else if constexpr (N == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n"
                 "tcgen05.wait::ld.sync.aligned;\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr) : "memory");
  } else {
    static_assert(N == 16, "4, 8 or 16 columns");
    tmem_ld16_wait(taddr, r);
  }
}
template <int N>
__device__ __forceinline__ void tmem_stn_wait(uint32_t taddr, const uint32_t (&r)[N]) {
  if constexpr (N == 4) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};\n"
                 :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]) : "memory");
  } else if constexpr (N == 8) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n"
                 :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
                    "r"(r[6]), "r"(r[7]) : "memory");
  } else {
    static_assert(N == 16, "4, 8 or 16 columns");
    tmem_st16(taddr, r);
  }
  tmem_st_wait();
}

// A piece: the keys [k0, k1) of segment (b, hk) that one CTA processes in one
// go (k0 a multiple of 128), with where its partial goes.
struct Piece {
  int b, hk, k0, k1;
  long long part;  // partial of head g at part + g * stride (in rows of D floats)
  int meta;     // balanced, piece that starts its segment: pieces of the segment; else 0
};

// The pieces of one CTA, in order. Every role of the CTA walks its own copy.
template <bool BAL>
struct Walker {
  // balanced: global tiles [pos, hi) left of T, cut over P CTAs; the
  // segment and tile at pos
  long long pos, hi, T, P;
  int b, hk, t;
  bool done;  // chunks: the one piece was handed out

  __device__ __forceinline__ bool next(const TctParams& p, Piece& pc) {
    if constexpr (!BAL) {
      if (done) return false;
      done = true;
      const int c = blockIdx.x;
      pc.b = blockIdx.z;
      pc.hk = blockIdx.y;
      const int Lb = seq_len(p, pc.b);
      int chunk = (Lb + p.C - 1) / p.C;
      chunk = (chunk + kKeys - 1) / kKeys * kKeys;  // tiles start on 128-key boundaries
      pc.k0 = c * chunk;
      pc.k1 = min(pc.k0 + chunk, Lb);
      pc.part = ((long long)pc.b * p.Hq + (long long)pc.hk * p.group) * p.C + c;
      pc.meta = 0;
      return pc.k0 < pc.k1;
    } else {
      if (pos >= hi) return false;
      const int Lb = seq_len(p, b), nb = tiles_of(Lb);
      const long long left = hi - pos;
      const int len = left < (long long)(nb - t) ? int(left) : nb - t;
      pc.b = b;
      pc.hk = hk;
      pc.k0 = t * kKeys;
      pc.k1 = min((t + len) * kKeys, Lb);
      const int s = b * p.Hkv + hk;
      pc.part = ((long long)s + blockIdx.x) * p.group;
      pc.meta = 0;
      if (t == 0) {
        // the CTA holding the segment's last tile x: the largest i with
        // floor(i T / P) <= x is floor(((x + 1) P - 1) / T)
        const long long x = pos + nb - 1;
        const long long i1 = ((x + 1) * P - 1) / T;
        pc.meta = int(i1 - (long long)blockIdx.x) + 1;
      }
      pos += len;
      t += len;
      if (t == nb) {
        t = 0;
        if (++hk == p.Hkv) {
          hk = 0;
          // skip empty sequences (tiles remain, so a later sequence has some)
          do {
            ++b;
          } while (pos < hi && tiles_of(seq_len(p, b)) == 0);
        }
      }
      return true;
    }
  }
};

// The tiles of one CTA, in order: piece index, keys, first and last of a piece.
template <bool BAL>
struct TileIter {
  Walker<BAL> w;
  Piece pc;
  int k = -1;   // piece index
  int kb = 0;   // first key of the current tile
  __device__ __forceinline__ bool next(const TctParams& p) {
    if (k >= 0 && kb + kKeys < pc.k1) {
      kb += kKeys;
      return true;
    }
    if (!w.next(p, pc)) return false;
    ++k;
    kb = pc.k0;
    return true;
  }
  __device__ __forceinline__ bool first() const { return kb == pc.k0; }
  __device__ __forceinline__ bool last() const { return kb + kKeys >= pc.k1; }
  __device__ __forceinline__ int valid() const { return min(kKeys, pc.k1 - kb); }
};

// Balanced schedule, computed by a whole warp: T = all tiles, P = min(grid,
// T) CTAs (so that none of them has an empty range, and the CTAs of a
// segment's slots all exist), this CTA's range [lo, hi) = [floor(i T / P),
// floor((i + 1) T / P)), and the segment and tile at lo. Returns false for a
// CTA past P.
__device__ __forceinline__ bool balanced_start(const TctParams& p, int lane, Walker<true>& w) {
  long long acc = 0;
  for (int base = 0; base < p.B; base += 32) {
    const int b = base + lane;
    if (b < p.B) acc += tiles_of(seq_len(p, b));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  const long long T = acc * p.Hkv;
  const long long P = T < (long long)gridDim.x ? T : (long long)gridDim.x, i = blockIdx.x;
  if (i >= P) return false;
  const long long lo = i * T / P, hi = (i + 1) * T / P;
  // the sequence holding global tile lo: a warp-wide scan of Hkv * tiles
  long long run = 0;
  for (int base = 0;; base += 32) {
    const int b = base + lane;
    const long long v = b < p.B ? (long long)tiles_of(seq_len(p, b)) * p.Hkv : 0;
    long long incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long u = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += u;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, run + incl > lo);
    if (hit) {
      const int l = __ffs(hit) - 1;
      const long long before = run + __shfl_sync(0xffffffffu, incl - v, l);
      const int nb = int(__shfl_sync(0xffffffffu, v, l) / p.Hkv);
      w.b = base + l;
      w.hk = int((lo - before) / nb);
      w.t = int((lo - before) % nb);
      break;
    }
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  w.pos = lo;
  w.hi = hi;
  w.T = T;
  w.P = P;
  w.done = false;
  return true;
}

// GH: the heads of a group the softmax handles (4, 8 or 16; a group of G <
// GH heads masks the rest).
template <bool BAL, int GH>
__global__ void __launch_bounds__(kThreads)
    decode_tct_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const TctParams p) {
  using L = Layout;
  // the merge kernel, launched as a programmatic dependent, may be scheduled
  // now: it waits for this grid's completion before reading anything
  grid_dependents_launch();
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

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.group;

  // the CTA's schedule (every warp computes the same)
  Walker<BAL> w0;
  long long n_total;  // tiles of this CTA
  if constexpr (BAL) {
    if (!balanced_start(p, lane, w0)) return;
    n_total = w0.hi - w0.pos;
  } else {
    w0.done = false;
    Walker<BAL> probe = w0;
    Piece pc;
    if (!probe.next(p, pc)) {  // empty chunk: weight 0 in the merge
      for (int e = threadIdx.x; e < G * kD; e += blockDim.x) {
        const size_t part = size_t(pc.part) + size_t(e / kD) * size_t(p.C);
        p.part_o[part * kD + e % kD] = 0.f;
        if (e % kD == 0) p.part_lse[part] = -INFINITY;
      }
      return;
    }
    n_total = (pc.k1 - pc.k0 + kKeys - 1) / kKeys;
  }
  const int part_stride = BAL ? 1 : p.C;

  if (threadIdx.x == 0) {
    mbar_init(BAR(X_Q_FULL), 1);
    mbar_init(BAR(X_Q_EMPTY), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(X_S_FULL + i), 1);
      mbar_init(BAR(X_S_FREE + i), kSmWarps);
      mbar_init(BAR(X_MAX + i), kSmWarps);
      mbar_init(BAR(X_P_FULL + i), kSmWarps);
      mbar_init(BAR(X_P_EMPTY + i), 1);
      mbar_init(BAR(X_O_FULL + i), 1);
      mbar_init(BAR(X_O_EMPTY + i), kSmWarps);
    }
    mbar_init(BAR(X_LSUM), kSmWarps);
    mbar_init(BAR(X_DRAIN), 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(BAR(X_FULL + s), 1);
      mbar_init(BAR(X_EMPTY + s), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  // Q's rows past the group stay zero (the B operand's padding heads)
  for (int ch = threadIdx.x; ch < 2 * kNH * 8; ch += kThreads)
    reinterpret_cast<uint4*>(smem + L::kOffQ)[ch] = make_uint4(0, 0, 0, 0);
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
  // ring position of V(g): the order is K0, K1, V0, K2, V1, ..., so V(g) is
  // at 2g + 2, except the CTA's last tile's V, which follows it at 2g + 1
  auto v_pos = [&](int g) -> int { return 2 * g + (g + 1 < n_total ? 2 : 1); };

  if (warp == kLoadWarp) {
    // ------------------------------------------------------------------ TMA producer + Q
    // (all lanes walk the schedule; lane 0 issues the copies and waits)
    const int run = p.page < kKeys ? p.page : kKeys;
    int issued[kSlots] = {};
    int pos = 0;  // ring position of the next load
    bool skip_pending = p.debug_skip && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0;
    auto load_tile = [&](const CUtensorMap* map, uint32_t dst0, uint32_t full, const Piece& pc,
                         int tb, int valid) {
      uint32_t bytes = 0;
      for (int r0 = 0; r0 < valid; r0 += run) {
        const int pg = p.table[size_t(pc.b) * p.max_pages + (tb + r0) / p.page];
        if (pg < 0 || pg >= p.num_pages) {
          atomicCAS(p.status, 0u, (unsigned(KID_DECODE) << 16) | (11u << 8) | 2u);
          continue;  // these rows stay unloaded (results undefined, error reported)
        }
        bytes += uint32_t(run) * 128u * 2u;
      }
      mbar_arrive_expect_tx(full, bytes);
      for (int r0 = 0; r0 < valid; r0 += run) {
        const int tp = tb + r0;
        const int pg = p.table[size_t(pc.b) * p.max_pages + tp / p.page];
        if (pg < 0 || pg >= p.num_pages) continue;
        for (int cs = 0; cs < 2; ++cs)
          tma_load_3d(dst0 + cs * L::kSubBytes + r0 * 128, map, full, cs * 64, tp % p.page,
                      pg * p.Hkv + pc.hk);
      }
    };
    // one ring position: K (which = 0) or V (1) of the iterator's tile
    auto next = [&](int which, const TileIter<BAL>& it) -> bool {
      bool r = true;
      if (lane == 0) {
        const int sl = pos % kSlots;
        r = wait_nb(BAR(X_EMPTY + sl), ((pos / kSlots) & 1) ^ 1, wc, which ? 2 : 1);
        if (r) {
          if (which && skip_pending) {
            skip_pending = false;  // test hook: this V tile never arrives
          } else {
            load_tile(which ? &tmV : &tmK, sbase + L::kOffRing + sl * L::kTileBytes,
                      BAR(X_FULL + sl), it.pc, it.kb, it.valid());
            ++issued[sl];
          }
        }
      }
      ++pos;
      return __shfl_sync(0xffffffffu, r, 0);
    };
    // Q of a piece (its G heads as 16 B-operand rows, 128-byte swizzle) once
    // the last S^T of the previous piece has read the buffer
    auto write_q = [&](const TileIter<BAL>& it) -> bool {
      const uint16_t* src = p.q + (size_t(it.pc.b) * p.Hq + size_t(it.pc.hk) * G) * kD;
      constexpr int kPer = kNH * (kD / 8) / 32;  // 16-byte chunks per lane
      uint4 v[kPer];
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        const int ch = lane + 32 * e, h = ch / (kD / 8);
        v[e] = h < G ? *reinterpret_cast<const uint4*>(src + ch * 8) : make_uint4(0, 0, 0, 0);
      }
      bool r = true;
      if (lane == 0 && it.k > 0) r = wait_nb(BAR(X_Q_EMPTY), (it.k - 1) & 1, wc, 4);
      r = __shfl_sync(0xffffffffu, r, 0);
      if (!r) return false;
      uint8_t* sq = smem + L::kOffQ;
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        const int ch = lane + 32 * e, h = ch / (kD / 8), cc16 = ch % (kD / 8);
        const int sub = cc16 >> 3, cc = cc16 & 7;
        if (h < G)
          *reinterpret_cast<uint4*>(sq + sub * (kNH * 128) + h * 128 + ((cc ^ (h & 7)) << 4)) = v[e];
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(X_Q_FULL));
      return true;
    };
    // Q of a new piece is written after the loads of its first K and of the
    // previous tile's V have been issued: its wait (the previous piece's
    // last S^T) would otherwise hold those loads back
    TileIter<BAL> kit, vit;
    kit.w = w0;
    vit.w = w0;
    kit.next(p);
    vit.next(p);
    bool ok = next(0, kit);
    if (ok) ok = write_q(kit);
    while (ok) {
      const bool has_k = kit.next(p);
      if (has_k && !(ok = next(0, kit))) break;
      if (!(ok = next(1, vit)) || !has_k) break;
      if (kit.first() && !(ok = write_q(kit))) break;
      vit.next(p);
    }
    if (lane == 0 && *abort_flag) {
      // let every copy this thread started land before the CTA exits
      for (int sl = 0; sl < kSlots; ++sl)
        if (issued[sl]) wait_nb(BAR(X_FULL + sl), (issued[sl] - 1) & 1, wc, 3, true);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(kKeys, kNH, false, false);  // K K-major, Q K-major
      constexpr uint32_t idesc_o = idesc_bf16(kD, kNH, true, false);      // V MN-major, P^T K-major
      const uint32_t sQ = sbase + L::kOffQ;
      int pos = 0;  // ring position of the next tile to consume (the producer's order)
      auto issue_s = [&](const TileIter<BAL>& it, int g) -> bool {
        if (it.first() && !wait_nb(BAR(X_Q_FULL), it.k & 1, wc, 12)) return false;
        const int s = pos % kSlots;
        if (!wait_nb(BAR(X_FULL + s), (pos / kSlots) & 1, wc, 10)) return false;
        ++pos;
        // S^T buffer g%2 is free once the softmax has loaded S^T(g-2)
        if (g >= 2 && !wait_nb(BAR(X_S_FREE + (g & 1)), ((g >> 1) - 1) & 1, wc, 11)) return false;
        tc_fence_after();
        const uint32_t kb = sbase + L::kOffRing + s * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          mma_ss(tmem + (g & 1) * kNH,
                 sdesc_sw128(kb + (kk >> 2) * L::kSubBytes + (kk & 3) * 32, 16, 1024),
                 sdesc_sw128(sQ + (kk >> 2) * (kNH * 128) + (kk & 3) * 32, 16, 1024), idesc_s,
                 kk > 0 ? 1u : 0u);
        tc_commit(BAR(X_S_FULL + (g & 1)));
        tc_commit(BAR(X_EMPTY + s));
        if (it.last()) tc_commit(BAR(X_Q_EMPTY));
        return true;
      };
      TileIter<BAL> sit, oit;
      sit.w = w0;
      oit.w = w0;
      sit.next(p);
      oit.next(p);
      bool ok = issue_s(sit, 0);
      for (int g = 0; ok; ++g) {
        const bool has_next = sit.next(p);
        if (has_next && !(ok = issue_s(sit, g + 1))) break;
        const int ob = oit.k & 1;
        // O^T buffer of piece k is free once the softmax has loaded piece k-2's
        if (oit.first() && oit.k >= 2 &&
            !(ok = wait_nb(BAR(X_O_EMPTY + ob), ((oit.k >> 1) - 1) & 1, wc, 15)))
          break;
        const int vs = pos % kSlots;
        ok = wait_nb(BAR(X_P_FULL + (g & 1)), (g >> 1) & 1, wc, 13);
        if (ok) ok = wait_nb(BAR(X_FULL + vs), (pos / kSlots) & 1, wc, 14);
        if (!ok) break;
        ++pos;
        tc_fence_after();
        // O^T (+)= V^T P^T: V read MN-major (d contiguous), P^T K-major
        const uint32_t vb = sbase + L::kOffRing + vs * L::kTileBytes;
        const uint32_t pb = sbase + L::kOffP + (g & 1) * (2 * kNH * 128);
        const bool fresh = oit.first();
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          mma_ss(tmem + L::kColO + ob * kNH, sdesc_sw128(vb + kk * 16 * 128, L::kSubBytes, 1024),
                 sdesc_sw128(pb + (kk >> 2) * (kNH * 128) + (kk & 3) * 32, 16, 1024), idesc_o,
                 (!fresh || kk > 0) ? 1u : 0u);
        tc_commit(BAR(X_P_EMPTY + (g & 1)));
        tc_commit(BAR(X_EMPTY + vs));
        if (oit.last()) tc_commit(BAR(X_O_FULL + ob));
        if (!has_next) break;
        oit.next(p);
      }
      tc_commit(BAR(X_DRAIN));
      wait_nb(BAR(X_DRAIN), 0, wc, 16, true);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int t = warp * 32 + lane;  // key of the tile, TMEM lane; dim of O^T at the end
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const float cl = p.scale_log2;
    auto on = [&](int h) { return GH == 4 || h < G; };  // (a compile-time true for GH = 4)
    float m[GH], lp[GH];
#pragma unroll
    for (int h = 0; h < GH; ++h) {
      m[h] = -INFINITY;
      lp[h] = 0.f;
    }
    bool ok = true;
    TileIter<BAL> it;
    it.w = w0;
    for (int g = 0; ok && it.next(p); ++g) {
      const int valid = it.valid();
      const int ob = it.k & 1;
      if (it.first()) {
#pragma unroll
        for (int h = 0; h < GH; ++h) {
          m[h] = -INFINITY;
          lp[h] = 0.f;
        }
      }
      ok = wait_nb(BAR(X_S_FULL + (g & 1)), (g >> 1) & 1, wc, 20);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[GH];
      tmem_ldn_wait<GH>(tmem + lane_base + (g & 1) * kNH, sr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(X_S_FREE + (g & 1)));
      // scores in log2 units; keys past the length (and heads past G) -inf
      float x[GH];
#pragma unroll
      for (int h = 0; h < GH; ++h)
        x[h] = (t < valid && on(h)) ? __uint_as_float(sr[h]) * cl : -INFINITY;
      // the tile's maximum of every head over the 128 keys (heads past G
      // carry -inf throughout: no branch per head, so the GH reductions
      // overlap)
      float* rd = red + (g & 1) * kSmWarps * kNH;
#pragma unroll
      for (int h = 0; h < GH; ++h) {
        const float v = warp_max(x[h]);
        if (lane == 0) rd[warp * kNH + h] = v;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(X_MAX + (g & 1)));
      // X_MAX_g%2: a warp writes this slot again (tile g+2) only after it
      // passed this wait for tile g+1, which all four warps arrive at after
      // reading tile g's maxima
      ok = wait_nb(BAR(X_MAX + (g & 1)), (g >> 1) & 1, wc, 21);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      bool grow = false;
      float mt[GH];
#pragma unroll
      for (int h = 0; h < GH; ++h) {
        mt[h] = fmaxf(fmaxf(rd[h], rd[kNH + h]), fmaxf(rd[2 * kNH + h], rd[3 * kNH + h]));
        grow |= mt[h] > m[h] + kRescale;  // (false for a masked head: -inf > -inf)
      }
      if (it.first()) {
#pragma unroll
        for (int h = 0; h < GH; ++h) m[h] = mt[h];
      } else if (grow) {
        // (the same decision in every thread: the maxima are the CTA's)
        // O~ must hold the sum through tile g-1 (of this piece): P^T(g-1) V finished
        ok = wait_nb(BAR(X_P_EMPTY + ((g - 1) & 1)), ((g - 1) >> 1) & 1, wc, 22);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        float alpha[GH];
#pragma unroll
        for (int h = 0; h < GH; ++h) {
          const float mn = fmaxf(m[h], mt[h]);
          // a head with no visible key so far has nothing to rescale
          alpha[h] = (on(h) && m[h] != -INFINITY) ? ex2_approx(m[h] - mn) : 0.f;
          lp[h] *= alpha[h];
          m[h] = mn;
        }
        uint32_t orow[GH];
        tmem_ldn_wait<GH>(tmem + lane_base + L::kColO + ob * kNH, orow);
#pragma unroll
        for (int h = 0; h < GH; ++h) orow[h] = __float_as_uint(__uint_as_float(orow[h]) * alpha[h]);
        tmem_stn_wait<GH>(tmem + lane_base + L::kColO + ob * kNH, orow);
      }
      // P^T(g) into buffer g%2 once P^T(g-2) has been read
      if (g >= 2) {
        ok = wait_nb(BAR(X_P_EMPTY + (g & 1)), ((g >> 1) - 1) & 1, wc, 23);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      uint8_t* pt = smem + L::kOffP + (g & 1) * (2 * kNH * 128) + (t >> 6) * (kNH * 128);
      const int kb = (t & 63) * 2;  // byte of this key in its 128-byte row
#pragma unroll
      for (int h = 0; h < GH; ++h) {
        // (a head whose keys so far are all masked, a head past G among
        // them, has m = -inf: its P is 0)
        const float pv = m[h] == -INFINITY ? 0.f : ex2_approx(x[h] - m[h]);
        lp[h] += pv;
        const uint32_t bits = pack_bf16x2(pv, 0.f) & 0xffffu;
        *reinterpret_cast<uint16_t*>(pt + h * 128 + ((((kb >> 4) ^ (h & 7))) << 4) + (kb & 15)) =
            uint16_t(bits);
      }
      if (valid < kKeys && warp == 0) {
        // the sequence's last tile: zero the V rows past its length before
        // O^T += V^T P^T reads them (the tile's V copy must have landed). The
        // slot's previous position, 3 before V(g), is K(g) (or an earlier
        // one), consumed before S^T(g) was seen, so the parity wait is exact
        const int vp = v_pos(g), vs = vp % kSlots;
        ok = wait_nb(BAR(X_FULL + vs), (vp / kSlots) & 1, wc, 24);
        if (ok) {
          uint8_t* vt = smem + L::kOffRing + vs * L::kTileBytes;
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
      if (lane == 0) mbar_arrive(BAR(X_P_FULL + (g & 1)));
      if (!it.last()) continue;

      // ---- end of a piece: row sums over the 128 key lanes, then O = O~ / l
      // and the LSE of each head
#pragma unroll
      for (int h = 0; h < GH; ++h) {
        if (on(h)) {
          float v = lp[h];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
          if (lane == 0) lred[warp * kNH + h] = v;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(X_LSUM));
      // (a warp writes lred again only at the next piece's end, after the
      // X_MAX waits of that piece's tiles, which need every warp past here)
      ok = wait_nb(BAR(X_LSUM), it.k & 1, wc, 25);
      if (ok) ok = wait_nb(BAR(X_O_FULL + ob), (it.k >> 1) & 1, wc, 26);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t orow[GH];
      tmem_ldn_wait<GH>(tmem + lane_base + L::kColO + ob * kNH, orow);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(X_O_EMPTY + ob));
#pragma unroll
      for (int h = 0; h < GH; ++h) {
        if (on(h)) {
          const float l = lred[h] + lred[kNH + h] + lred[2 * kNH + h] + lred[3 * kNH + h];
          const size_t part = size_t(it.pc.part) + size_t(h) * part_stride;
          p.part_o[part * kD + t] = __uint_as_float(orow[h]) / l;
          if (t == 0) p.part_lse[part] = m[h] + lg2_approx(l);
        }
      }
      if (BAL && t == 0 && it.pc.meta > 0)
        p.seg_meta[size_t(it.pc.b) * p.Hkv + it.pc.hk] = make_int2(int(it.pc.part / G), it.pc.meta);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// Merge of the balanced schedule's partials: for each (sequence, query
// head), the pieces of its segment (slots first .. first + count - 1) by the
// same log-sum-exp rescale decode_merge_kernel applies to chunks, in slot
// order. A slot range outside the workspace (a record the split kernel did
// not write, after a failed launch) is reported, never read.
__global__ void __launch_bounds__(kD) decode_merge_slots_kernel(const TctParams p, int slots,
                                                                uint16_t* o, float* lse) {
  grid_dependency_wait();  // the split kernel's partials and records
  const int h = blockIdx.x, b = blockIdx.y, i = threadIdx.x;
  const size_t bh = size_t(b) * p.Hq + h;
  const int hk = h / p.group, g = h % p.group;
  constexpr float kLn2 = 0.69314718055994530942f;
  if (seq_len(p, b) == 0) {  // no key at all
    o[bh * kD + i] = 0;
    if (i == 0) lse[bh] = -INFINITY;
    return;
  }
  const int2 meta = p.seg_meta[b * p.Hkv + hk];
  if (meta.y < 1 || meta.x < 0 || meta.x > slots - meta.y) {
    if (i == 0) atomicCAS(p.status, 0u, (unsigned(KID_DECODE_MERGE) << 16) | (1u << 8) | 2u);
    return;
  }
  const float* pl = p.part_lse + size_t(meta.x) * p.group + g;
  const float* po = p.part_o + (size_t(meta.x) * p.group + g) * kD;
  float mx = -INFINITY;
  for (int c = 0; c < meta.y; ++c) mx = fmaxf(mx, pl[size_t(c) * p.group]);
  if (mx == -INFINITY) {
    o[bh * kD + i] = 0;
    if (i == 0) lse[bh] = -INFINITY;
    return;
  }
  float wsum = 0.f, acc = 0.f;
  for (int c = 0; c < meta.y; ++c) {
    const float lc = pl[size_t(c) * p.group];
    if (lc == -INFINITY) continue;
    const float wgt = ex2_approx(lc - mx);
    wsum += wgt;
    acc = fmaf(wgt, po[size_t(c) * p.group * kD + i], acc);
  }
  const float out = acc / wsum;
  // round to nearest even bf16
  const uint32_t u = __float_as_uint(out);
  o[bh * kD + i] = uint16_t((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
  if (i == 0) lse[bh] = (mx + lg2_approx(wsum)) * kLn2;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

// Workspace of the balanced schedule: partials of at most B Hkv + P - 1
// slots of G heads (<= B Hq + P G rows), their LSEs and the per-segment
// records.
size_t decode_balanced_workspace_bytes(int B, int H, int d) {
  const size_t rows = size_t(B) * H + size_t(kMaxPersist) * kBalMaxGroup;
  return align256(rows * d * 4) + align256(rows * 4) + align256(size_t(B) * H * 8);
}

// Chunk partials (chunks > 0, merged by the caller) or the balanced schedule
// and its merge (chunks == 0, a workspace of decode_balanced_workspace_bytes)
// of the paged decode for 4 to 16 query heads per KV head and d = 128.
fa_status launch_decode_paged_tct(const void* q, const void* kpages, const void* vpages,
                                  const int* block_table, const int* seqlens, int B, int Hq,
                                  int Hkv, int num_pages, int page_size, int max_pages, int d,
                                  float scale, int chunks, float* part_o, float* part_lse,
                                  void* workspace, void* o, float* lse, const LaunchCtx& ctx) {
  if (d != kD || Hq / Hkv > kNH || (page_size > 64 && page_size % kKeys != 0) ||
      (chunks == 0 && Hq / Hkv > kBalMaxGroup)) {
    set_last_error("fa_decode_paged: the keys-as-rows kernel needs d = 128, <= %d heads per KV "
                   "head (%d for the automatic split) and pages of <= 64 rows or a multiple of 128",
                   kNH, kBalMaxGroup);
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
  p.B = B;
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
  if (chunks > 0) {
    p.part_o = part_o;
    p.part_lse = part_lse;
    p.seg_meta = nullptr;
    auto kern = p.group == 4   ? decode_tct_kernel<false, 4>
                : p.group <= 8 ? decode_tct_kernel<false, 8>
                               : decode_tct_kernel<false, 16>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_tct)");
    dim3 grid(p.C, p.Hkv, B);
    {
      ProfileScope prof(KID_DECODE, ctx.stream);
      kern<<<grid, kThreads, smem, ctx.stream>>>(mk, mv, p);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "decode tct kernel launch");
    return FA_OK;
  }
  // balanced: P persistent CTAs, no more than there can be tiles
  const long long max_tiles = (long long)B * Hkv * ((p.Lmax + kKeys - 1) / kKeys);
  long long P = 2LL * (ctx.num_sms > 0 ? ctx.num_sms : 148);
  if (P > kMaxPersist) P = kMaxPersist;
  if (P > max_tiles) P = max_tiles;
  if (P < 1) P = 1;
  const int slots = int((long long)B * Hkv + P - 1);
  const size_t rows = size_t(B) * Hq + size_t(kMaxPersist) * kBalMaxGroup;
  char* ws = static_cast<char*>(workspace);
  p.part_o = reinterpret_cast<float*>(ws);
  p.part_lse = reinterpret_cast<float*>(ws + align256(rows * kD * 4));
  p.seg_meta = reinterpret_cast<int2*>(ws + align256(rows * kD * 4) + align256(rows * 4));
  auto kern = p.group == 4 ? decode_tct_kernel<true, 4> : decode_tct_kernel<true, 8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_tct)");
  {
    ProfileScope prof(KID_DECODE, ctx.stream);
    kern<<<dim3(unsigned(P)), kThreads, smem, ctx.stream>>>(mk, mv, p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode tct kernel launch");
  {
    ProfileScope prof(KID_DECODE_MERGE, ctx.stream);
    e = launch_dependent(decode_merge_slots_kernel, dim3(Hq, B), dim3(kD), 0, ctx.stream, p, slots,
                         static_cast<uint16_t*>(o), lse);
    if (e != cudaSuccess) return cuda_fail(e, "decode merge kernel launch");
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode merge kernel launch");
  return FA_OK;
}

}  // namespace fa
