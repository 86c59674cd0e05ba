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
//  1. bwd_pre   D_i = sum_c dO_ic O_ic (fp32) and the saved LSE in base 2,
//               stored negated and D pre-multiplied by -scale (the forms the
//               paired FMAs of the main kernels add), both padded to a
//               multiple of 128 rows (padding rows get -L2 = -inf, so their P
//               is exactly 0, and -scale D = 0).
//  2. bwd_dkdv  one CTA per (batch*head, 128-key tile). K and V of the tile stay
//               in shared memory; the Q and dO rows of every query that can see
//               these keys stream past in blocks of 128. Per block:
//                 S^T = K Q^T, dP^T = V dO^T          (tcgen05 -> TMEM)
//                 P^T = 2^(S^T scale log2e - L2)     (phase 1, CUDA cores)
//                 dV += P^T dO                        (tcgen05, A = P^T in TMEM)
//                 dS^T = P^T (scale dP^T - scale D)  (phase 2)
//                 dK += dS^T Q                        (tcgen05, A = dS^T in TMEM)
//               dV and dK accumulate in TMEM for the whole key tile.
//  3. bwd_dq    one CTA per (batch*head, 128-query tile). Q and dO stay in
//               shared memory; K and V stream past in blocks of 128 keys:
//                 S = Q K^T, dP = dO V^T; dS = scale P (dP - D); dQ += dS K.
// The scale is folded into dS before it is rounded to bf16.
//
// The EX instantiations add the bias and dropout options of the forward
// ("FlashAttention'i Anlamak Bolum 1", 0.2; "Bellek Duvarinin Fizigi",
// "Maskeleme ve Dropout": the backward regenerates the forward's dropout
// mask from the same seed and offset instead of storing it). With the keep
// factor z = keep * 256/t (0 for a dropped pair):
//     P = exp(S + bias - L), dV = (P z)^T dO, dS = P (z dP - D),
// and dQ, dK as before. The bias (an input, no gradient) is added to the raw
// scores before the exponential: in the dQ kernel a thread reads its query
// row (16-byte loads when possible), in the dK/dV kernel a warp reads 32
// consecutive keys of one query row per load. The keep bits come from the
// same Philox4x32-10 calls as the forward (counter (key / 16, query, b H + h,
// offset)): a dQ thread makes four calls for its 64 keys; in the dK/dV
// kernel, whose threads own keys, each lane makes four calls for
// (query, 16 keys) pairs of its warp, reduces them to 16 keep bits, and a
// warp shuffle per query hands every lane its bit. The dK/dV kernel's TMEM
// holds dP^T - D (D enters through the extension step), so there
// scale (z dP - D) = z u + (1 - z)(-scale D) with u = scale (dP - D), and
// -scale D is read per query column.
//
// Splitting dQ from dK/dV recomputes S and dP once more (7 tensor-core GEMMs
// instead of 5) but needs no atomics and gives deterministic results. Both
// kernels use 128-wide blocks, so every MMA is M = 128, N = 128 (the full-rate
// shape), with one buffer per operand in TMEM; the overlap comes from splitting
// the per-block CUDA-core work in two phases and issuing each dependent MMA as
// soon as its phase ends, interleaved with the next block's S and dP MMAs:
//   dK/dV kernel:  ... dV_i | S^T_i+1 | dK_i | dP^T_i+1 | dV_i+1 ...
//                  phase 1 of block i+1 (the exponentials) runs during
//                  dK_i and dP^T_i+1;
//   dQ kernel:     S_j+1 is issued as soon as S_j has been read into
//                  registers, so phase 1 of block j+1 starts right after
//                  phase 2 of block j, during dQ_j and dP_j+1.
//
// Warp roles (384 threads, three warpgroups): warps 0-7 compute, warp 8 TMA
// producer, warp 9 MMA issuer, warps 10-11 idle (they only complete the third
// warpgroup, which setmaxnreg needs whole). A row (one TMEM lane) is shared by two compute warps of the same lane
// quadrant, warp w taking columns 0-63 and warp w+4 columns 64-127, so each
// thread keeps 64 probabilities in registers between the phases and two warps
// per SMSP hide each other's latencies. Each half writes its bf16 P or dS
// inside its own 64 columns, so the A operand of the K-step kk of the next MMA
// starts at column (kk/4)*64 + (kk%4)*8.
#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kTile = 128;   // rows of the resident tile and of a streamed block
constexpr int kThreads = 384;
// Registers per thread: the kernels launch with 168 (65536 / 384, rounded down
// to a multiple of 8); the compute warpgroups then take 208 and the control
// warpgroup keeps 88: 2*128*208 + 128*88 = 384*168.
constexpr int kRegsAtLaunch = 168;
constexpr int kRegsCompute = 208;
constexpr int kRegsControl = 88;
static_assert(2 * 128 * kRegsCompute + 128 * kRegsControl <= kThreads * kRegsAtLaunch,
              "register split exceeds the launch allocation");
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kComputeWarps = 8;
constexpr int kHalfCols = kTile / 2;  // columns of a row each compute warp owns
constexpr int kStages = 2;
constexpr int kKSlots = 3;   // dQ kernel: K ring depth (its V ring has kStages slots)
constexpr float kLog2e = 1.4426950408889634f;

// barrier slots (shared by both kernels)
enum : int {
  B_RES_FULL = 0,      // the resident tiles (K,V or Q,dO)
  B_ST_FULL = 1,       // +stage: a streamed block landed
  B_ST_EMPTY = 3,      // +stage: its MMAs are done
  B_S_FULL = 5,        // S of the current block is in TMEM
  B_DP_FULL = 6,       // dP of the current block is in TMEM
  B_PHASE1 = 7,        // S of the current block read into registers
  B_PHASE2 = 8,        // dS (and in the dK/dV kernel P) written back to TMEM
  B_ACC_DONE = 9,
  B_DRAIN = 10,
  B_DO_FULL = 11,      // +stage, dK/dV kernel: the dO block landed (B_ST_FULL: the Q block)
  B_DO_EMPTY = 13,     // +stage, dK/dV kernel: dV has read the dO block (B_ST_EMPTY: dK the Q block)
  B_OUT_READY = 15,    // +stage: the compute warps have staged an item's output tiles in that slot
                       // (one arrival per warp)
  B_RES_EMPTY = 17,    // the item's last S and dP MMAs have read the resident tiles
  B_ACC_EMPTY = 18,    // the compute warps have read the accumulators (one arrival per warp)
  B_K_FULL = 19,       // +slot (3), dQ kernel: a K block landed (B_DO_FULL: a V block)
  B_K_EMPTY = 22,      // +slot (3), dQ kernel: dQ has read the K block (B_DO_EMPTY: dP the V block)
  B_KOUT_READY = 25,   // +slot (3), dQ kernel: dQ staged in that K slot (one arrival per warp)
  B_COUNT = 28
};

struct BwdParams {
  const uint16_t* o;
  const uint16_t* dO;
  const float* lse;
  float* lse2;     // [BH, Np] minus the base-2 LSE, -inf in padding rows
  float* dvec;     // [BH, Np] -scale D, 0 in padding rows
  uint16_t* qext;  // [BH, Np, 16] bf16: -L/scale split in three (hi, mid, lo), then zeros
  uint16_t* dext;  // [BH, Np, 16] bf16: -D split in three, then zeros
  uint16_t* dq;
  uint16_t* dk;
  uint16_t* dv;
  int N, Np, BH, n_tiles;
  float scale, scale_log2;
  unsigned int* status;
  unsigned long long limit_ns;
  int debug_skip;  // test hook: kernel id whose CTA 0 leaves out one load (0: none)
  // EX only: bias (bf16, element strides over b and h, rows of N) and dropout
  const uint16_t* bias;
  long long bias_sb, bias_sh;
  int H;
  int bias_vec;  // rows and strides are multiples of 8 elements: 16-byte loads
  float inv_scale;
  uint32_t seed_lo, seed_hi, rng_offset;
  int keep_t;    // keep iff byte < keep_t; 256 = no dropout
  float keep_scale;
};

__device__ __forceinline__ const uint16_t* bias_head(const BwdParams& p, int bh) {
  const int b = bh / p.H, h = bh - b * p.H;
  return p.bias + b * p.bias_sb + h * p.bias_sh;
}

// keep bits of query q for keys 16 kb .. 16 kb + 15 (bit e: key 16 kb + e)
__device__ __forceinline__ uint32_t keep16(const BwdParams& p, int bh, int q, int kb) {
  return keep_bits16(make_uint4(uint32_t(kb), uint32_t(q), uint32_t(bh), p.rng_offset), p.seed_lo,
                     p.seed_hi, uint32_t(p.keep_t));
}

__device__ __forceinline__ float bf16f(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// v as hi + mid + lo, each rounded to bf16 (round to nearest even): the sum
// recovers v to about 2^-24 relative, the precision of fp32. Packed as the
// first three bf16 of 8 (the rest zero).
__device__ __forceinline__ uint4 split3_bf16(float v) {
  const uint32_t hi = pack_bf16x2(v, 0.f) & 0xffffu;
  const float r1 = v - bf16f(hi);
  const uint32_t mid = pack_bf16x2(r1, 0.f) & 0xffffu;
  const float r2 = r1 - bf16f(mid);
  const uint32_t lo = pack_bf16x2(r2, 0.f) & 0xffffu;
  return make_uint4(hi | (mid << 16), lo, 0u, 0u);
}

// Shared-memory plan. Row-major bf16 tiles of 128 rows, stored as D/64 column
// groups of 128 rows x 128 bytes, 128-byte swizzled (TMA box 64 x 128).
// Extension tiles are 128 rows x 16 bf16 (32 bytes), 32-byte swizzled.
template <int D>
struct Plan {
  static constexpr int kGroups = D / 64;
  static constexpr int kSubBytes = kTile * 128;        // 16 KB per column group
  static constexpr int kTileBytes = kGroups * kSubBytes;
  static constexpr int kExtBytes = kTile * 32;         // 4 KB
  static constexpr int kOffRes0 = 0;
  static constexpr int kOffRes1 = kTileBytes;
  static constexpr int kOffOnes = 2 * kTileBytes;      // dK/dV kernel: 128 x 16 ones
  static constexpr int kOffStage = kOffOnes + kExtBytes;
  // a stage: two streamed tiles, then (dK/dV kernel) the extension tiles of
  // the Q block and of the dO block
  static constexpr int kStageBytes = 2 * kTileBytes + 2 * kExtBytes;
  // dQ kernel: resident Q, dO at kOffRes0/1, then a ring of kKSlots K tiles
  // and a ring of kStages V tiles (no extension tiles, no ones tile)
  static constexpr int kOffKRing = 2 * kTileBytes;
  static constexpr int kOffVRing = kOffKRing + kKSlots * kTileBytes;
  static constexpr int kDqEnd = kOffVRing + kStages * kTileBytes;
  static constexpr int kStageEnd = kOffStage + kStages * kStageBytes;
  static constexpr int kOffBar = kStageEnd > kDqEnd ? kStageEnd : kDqEnd;
  static constexpr int kOffMisc = kOffBar + 8 * B_COUNT;
  static constexpr int kSmemBytes = kOffMisc + 32 + 1024;
  // TMEM columns; the dQ kernel keeps its resident Q and dO tiles (bf16, A
  // operands) in the columns the second accumulator would use
  static constexpr uint32_t kColS = 0, kColDP = 128, kColAcc0 = 256, kColAcc1 = 256 + D;
  static constexpr uint32_t kColQT = 256 + D, kColDOT = 256 + D + D / 2;
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
  // a warp's rows never cross a (batch, head): Np is a multiple of 128 and a
  // warp covers kRowsPerStep * kPreSteps rows (8 or 16), a divisor of 128, so
  // one division per thread
  static_assert(kTile % (kRowsPerStep * kPreSteps) == 0, "a warp's rows must stay in one head");
  const int bh0 = int(row0 / p.Np), rowb = int(row0 - static_cast<long long>(bh0) * p.Np);
  uint4 ov[kPreSteps], gv[kPreSteps];
#pragma unroll
  for (int st = 0; st < kPreSteps; ++st) {
    const long long r = row0 + st * kRowsPerStep + sub;
    ov[st] = gv[st] = make_uint4(0, 0, 0, 0);
    if (r < total) {
      const int bh = bh0, row = rowb + st * kRowsPerStep + sub;
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
      const int bh = bh0, row = rowb + st * kRowsPerStep + sub;
      const bool valid = row < p.N;
      const float lse = valid ? p.lse[size_t(bh) * p.N + row] : 0.f;
      p.dvec[r] = valid ? -p.scale * dsum : 0.f;
      p.lse2[r] = valid ? -lse * kLog2e : -INFINITY;
      // extension rows: -L/scale (added to S by the MMA, so that scale log2e
      // times the sum is the exponent of P) and -D (added to dP); a padding
      // query gets a hugely negative S, so its P is exactly 0
      const uint4 qx = valid ? split3_bf16(-lse / p.scale) : make_uint4(0xF149u, 0, 0, 0);  // bf16, about -1e30
      const uint4 dx = valid ? split3_bf16(-dsum) : make_uint4(0, 0, 0, 0);
      uint4* qo = reinterpret_cast<uint4*>(p.qext + size_t(r) * 16);
      uint4* dout = reinterpret_cast<uint4*>(p.dext + size_t(r) * 16);
      qo[0] = qx;
      qo[1] = make_uint4(0, 0, 0, 0);
      dout[0] = dx;
      dout[1] = make_uint4(0, 0, 0, 0);
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
      mbar_init(bar(B_DO_FULL + s), 1);
      mbar_init(bar(B_DO_EMPTY + s), 1);
    }
    mbar_init(bar(B_S_FULL), 1);
    mbar_init(bar(B_DP_FULL), 1);
    mbar_init(bar(B_PHASE1), kComputeWarps);  // one arrival per compute warp
    mbar_init(bar(B_PHASE2), kComputeWarps);
    mbar_init(bar(B_ACC_DONE), 1);
    mbar_init(bar(B_DRAIN), 1);
    mbar_init(bar(B_OUT_READY), kComputeWarps);
    mbar_init(bar(B_OUT_READY + 1), kComputeWarps);
    mbar_init(bar(B_RES_EMPTY), 1);
    mbar_init(bar(B_ACC_EMPTY), kComputeWarps);
    for (int s = 0; s < kKSlots; ++s) {
      mbar_init(bar(B_K_FULL + s), 1);
      mbar_init(bar(B_K_EMPTY + s), 1);
      mbar_init(bar(B_KOUT_READY + s), kComputeWarps);
    }
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

// D[128 x 128] = R[128 x D] * B[128 x D]^T, both K-major in shared memory
template <int D>
__device__ __forceinline__ void mma_rows_x_rows(uint32_t d_tmem, uint32_t r, uint32_t b) {
  using L = Plan<D>;
  constexpr uint32_t idesc = idesc_bf16(kTile, kTile, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * L::kSubBytes + (kk & 3) * 32;
    mma_ss(d_tmem, sdesc_sw128(r + off, 16, 1024), sdesc_sw128(b + off, 16, 1024), idesc,
           kk > 0 ? 1u : 0u);
  }
}

// D[128 x 128] = A[128 x D] * B[128 x D]^T with A in TMEM (K-major: element
// k of row m in lane m, column k/2) and B K-major in shared memory
template <int D>
__device__ __forceinline__ void mma_tmem_rows_x_rows(uint32_t d_tmem, uint32_t a_tmem, uint32_t b) {
  using L = Plan<D>;
  constexpr uint32_t idesc = idesc_bf16(kTile, kTile, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * L::kSubBytes + (kk & 3) * 32;
    mma_ts(d_tmem, a_tmem + kk * 8, sdesc_sw128(b + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}

// a resident 128 x D tile (K-major, 128-byte swizzle) into TMEM as an A
// operand: D/16 copies of one K step each
template <int D>
__device__ __forceinline__ void copy_tile_to_tmem(uint32_t t_dst, uint32_t src) {
  using L = Plan<D>;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * L::kSubBytes + (kk & 3) * 32;
    tmem_cp_128x256b(t_dst + kk * 8, sdesc_sw128(src + off, 16, 1024));
  }
}

// D[128 x 128] += ONES[128 x 16] * X[128 x 16]^T: adds sum_j X[n][j] to every
// row of column n (one more K step, both operands 32-byte-swizzled K-major)
__device__ __forceinline__ void mma_ext(uint32_t d_tmem, uint32_t ones, uint32_t x) {
  constexpr uint32_t idesc = idesc_bf16(kTile, kTile, false, false);
  mma_ss(d_tmem, sdesc_sw32_kmajor(ones), sdesc_sw32_kmajor(x), idesc, 1u);
}

// D[128 x D] (+)= A[128 x 128] * B[128 x D]: A bf16 in TMEM, K-major, its two
// halves at columns 0-31 and 64-95 of a 128-column region (see the warp roles
// above); B a tile in shared memory read MN-major
template <int D>
__device__ __forceinline__ void mma_tmem_x_rows(uint32_t d_tmem, uint32_t a_tmem, uint32_t b,
                                                bool accumulate) {
  using L = Plan<D>;
  constexpr uint32_t idesc = idesc_bf16(kTile, D, false, true);
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)
    mma_ts(d_tmem, a_tmem + (kk >> 2) * 64 + (kk & 3) * 8, sdesc_sw128(b + kk * 2048, L::kSubBytes, 1024), idesc,
           (accumulate || kk > 0) ? 1u : 0u);
}

// This thread's half of an accumulator row (TMEM lane r, columns half*D/2 ..)
// as bf16 into a staged output tile: D/64 column groups of 128 rows x 128
// bytes with the 128-byte swizzle of the tensor maps (16-byte chunk c of row
// r at chunk c ^ (r % 8)), ready for TMA stores.
template <int D>
__device__ __forceinline__ void stage_acc_half(uint32_t t_acc, uint8_t* stg, int r, int half) {
  constexpr int kSubBytes = kTile * 128;
#pragma unroll
  for (int ch = 0; ch < D / 64; ++ch) {
    const int c0 = half * (D / 2) + ch * 32;
    uint32_t v[32];
    tmem_ld32_wait(t_acc + c0, v);
#pragma unroll
    for (int v4 = 0; v4 < 4; ++v4) {
      uint4 w;
      w.x = pack_bf16x2(__uint_as_float(v[8 * v4 + 0]), __uint_as_float(v[8 * v4 + 1]));
      w.y = pack_bf16x2(__uint_as_float(v[8 * v4 + 2]), __uint_as_float(v[8 * v4 + 3]));
      w.z = pack_bf16x2(__uint_as_float(v[8 * v4 + 4]), __uint_as_float(v[8 * v4 + 5]));
      w.w = pack_bf16x2(__uint_as_float(v[8 * v4 + 6]), __uint_as_float(v[8 * v4 + 7]));
      const int k16 = c0 / 8 + v4;          // 16-byte chunk of the row
      const int g = k16 >> 3, cc = k16 & 7;  // column group, chunk in its 128-byte row
      *reinterpret_cast<uint4*>(stg + g * kSubBytes + r * 128 + ((cc ^ (r & 7)) << 4)) = w;
    }
  }
}

// dS = P (scale dP - scale D) for this warp's 64 columns of a row, in paired
// fp32 arithmetic: dP read from TMEM 32 columns at a time, dS written back as
// bf16 over the first 32 of the 64 (chunk 1 overwrites columns chunk 0 has
// already read). nsd4(j) gives -scale D for local columns 4j..4j+3 (a
// per-column vector in the dK/dV kernel, one value per row in the dQ kernel).
template <typename NsdFn>
__device__ __forceinline__ void write_ds_half(uint32_t t_dp, const uint64_t (&pr2)[kHalfCols / 2], uint64_t scale2,
                                              NsdFn nsd4) {
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    uint32_t dr[32];
    tmem_ld32_wait(t_dp + ch * 32, dr);
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 n = nsd4(ch * 8 + j);
      const uint64_t t0 = f2_fma(f2_pack(__uint_as_float(dr[4 * j]), __uint_as_float(dr[4 * j + 1])), scale2,
                                 f2_pack(n.x, n.y));
      const uint64_t t1 = f2_fma(f2_pack(__uint_as_float(dr[4 * j + 2]), __uint_as_float(dr[4 * j + 3])), scale2,
                                 f2_pack(n.z, n.w));
      pk[2 * j] = f2_to_bf16x2(f2_mul(pr2[ch * 16 + 2 * j], t0));
      pk[2 * j + 1] = f2_to_bf16x2(f2_mul(pr2[ch * 16 + 2 * j + 1], t1));
    }
    tmem_st16(t_dp + ch * 16, pk);
  }
}

// write_ds_half with the dropout factor: column i of dP is scaled by szk
// when bit i of keep64 is set, else by 0
template <typename NsdFn>
__device__ __forceinline__ void write_ds_half_z(uint32_t t_dp, const uint64_t (&pr2)[kHalfCols / 2],
                                                uint64_t keep64, float szk, NsdFn nsd4) {
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    uint32_t dr[32];
    tmem_ld32_wait(t_dp + ch * 32, dr);
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = ch * 32 + 4 * j;
      const float4 n = nsd4(ch * 8 + j);
      const float z0 = (keep64 >> c) & 1 ? szk : 0.f, z1 = (keep64 >> (c + 1)) & 1 ? szk : 0.f;
      const float z2 = (keep64 >> (c + 2)) & 1 ? szk : 0.f, z3 = (keep64 >> (c + 3)) & 1 ? szk : 0.f;
      const uint64_t t0 = f2_fma(f2_pack(__uint_as_float(dr[4 * j]), __uint_as_float(dr[4 * j + 1])),
                                 f2_pack(z0, z1), f2_pack(n.x, n.y));
      const uint64_t t1 = f2_fma(f2_pack(__uint_as_float(dr[4 * j + 2]), __uint_as_float(dr[4 * j + 3])),
                                 f2_pack(z2, z3), f2_pack(n.z, n.w));
      pk[2 * j] = f2_to_bf16x2(f2_mul(pr2[ch * 16 + 2 * j], t0));
      pk[2 * j + 1] = f2_to_bf16x2(f2_mul(pr2[ch * 16 + 2 * j + 1], t1));
    }
    tmem_st16(t_dp + ch * 16, pk);
  }
}

// P for this warp's 64 columns of a row: 2^(s c + nl2) in pairs, where nl2 is
// minus the base-2 LSE of the query (the row's one value, or a per-column
// vector); nl4(j) gives it for local columns 4j..4j+3. Columns with
// hidden(i) true get P = 0.
template <bool MASK, typename Nl2Fn, typename HideFn>
__device__ __forceinline__ void form_p_half(const uint32_t (&sr)[kHalfCols], uint64_t c2, Nl2Fn nl4,
                                            HideFn hidden, uint64_t (&pr2)[kHalfCols / 2]) {
#pragma unroll
  for (int j = 0; j < kHalfCols / 4; ++j) {
    const float4 n = nl4(j);
    const uint64_t x0 = f2_fma(f2_pack(__uint_as_float(sr[4 * j]), __uint_as_float(sr[4 * j + 1])), c2,
                               f2_pack(n.x, n.y));
    const uint64_t x1 = f2_fma(f2_pack(__uint_as_float(sr[4 * j + 2]), __uint_as_float(sr[4 * j + 3])), c2,
                               f2_pack(n.z, n.w));
    float a, b, e, f;
    f2_unpack(x0, a, b);
    f2_unpack(x1, e, f);
    a = ex2_approx(a);
    b = ex2_approx(b);
    e = ex2_approx(e);
    f = ex2_approx(f);
    if (MASK) {
      a = hidden(4 * j) ? 0.f : a;
      b = hidden(4 * j + 1) ? 0.f : b;
      e = hidden(4 * j + 2) ? 0.f : e;
      f = hidden(4 * j + 3) ? 0.f : f;
    }
    pr2[2 * j] = f2_pack(a, b);
    pr2[2 * j + 1] = f2_pack(e, f);
  }
}

// --------------------------------------------------------------------------
// 2. dK, dV: key-tile-outer
// --------------------------------------------------------------------------
// Persistent work list of both main kernels: item = (b*h, tile), heaviest
// level first (under the causal mask the key tiles that see the most query
// blocks, and the query tiles that see the most key blocks); round r gives
// CTA c item r G + c for even r and r G + G-1-c for odd r (G = grid size),
// which evens out the sums.
__device__ __forceinline__ bool bwd_item(const BwdParams& p, int round, int& bh, int& level) {
  const int G = int(gridDim.x), c = int(blockIdx.x);
  const int idx = round * G + ((round & 1) ? G - 1 - c : c);
  if (idx >= p.n_tiles * p.BH) return false;
  level = idx / p.BH;
  bh = idx % p.BH;
  return true;
}

template <int D, bool CAUSAL, bool EX>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmQX, const __grid_constant__ CUtensorMap tmDX,
                    const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                    const BwdParams p) {
  using L = Plan<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto BAR = [&](int i) -> uint32_t { return sbase + L::kOffBar + 8u * uint32_t(i); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // items: (b*h, key tile jt); an item streams the query blocks i0 + it,
  // it = 0 .. n_blk-1, that can see its keys
  auto blocks_of = [&](int jt) { return CAUSAL ? p.n_tiles - jt : p.n_tiles; };
  // the all-ones tile that multiplies the extension columns (uniform, so its
  // swizzle does not matter); visible to the tensor core after the fence and
  // the barrier in setup_cta
  for (int i = threadIdx.x; i < L::kExtBytes / 16; i += kThreads)
    reinterpret_cast<uint4*>(smem + L::kOffOnes)[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  fence_proxy_async_smem();
  volatile int* abort_flag;
  const uint32_t tmem = setup_cta<D>(smem, warp, abort_flag);
  const WaitCtl wc{abort_flag, p.status, p.limit_ns, KID_BWD};
  const uint32_t sK = sbase + L::kOffRes0, sV = sbase + L::kOffRes1;
  // stage slot s (global block g of this CTA uses slot g % 2): the Q block
  // (+ its extension rows) and the dO block (+ its own), each with full /
  // empty barriers (Q is released by dK, dO by dV). After an item's last
  // block the slot of that block stages the item's dV and dK tiles for the
  // TMA stores, which the producer issues before its next load into it.
  auto q_addr = [&](int g) { return sbase + L::kOffStage + (g % kStages) * L::kStageBytes; };
  auto do_addr = [&](int g) { return q_addr(g) + L::kTileBytes; };
  auto qx_addr = [&](int g) { return q_addr(g) + 2 * L::kTileBytes; };
  auto dx_addr = [&](int g) { return qx_addr(g) + L::kExtBytes; };
  const uint32_t sOnes = sbase + L::kOffOnes;
  const uint32_t tP = tmem + L::kColDP;        // P^T as bf16: columns 0-31 and 64-95 of the dP region
  const uint32_t tDS = tmem + L::kColDP + 32;  // dS^T as bf16: columns 32-63 and 96-127

  if (warp >= 8) {
    regs_decrease<kRegsControl>();
    if (warp == kLoadWarp) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        // loads started into each stage slot (the abort path waits for them)
        int q_issued[kStages] = {0, 0}, do_issued[kStages] = {0, 0}, res_issued = 0;
        bool skip_pending = p.debug_skip == KID_BWD && blockIdx.x == 0;
        // the item whose output is staged in slot s and not yet stored (-1:
        // none), with its coordinates, and how many stagings slot s has seen
        int pend_jt[kStages] = {-1, -1}, pend_bh[kStages] = {0, 0}, staged[kStages] = {0, 0};
        auto flush = [&](int s) -> bool {
          if (pend_jt[s] < 0) return true;
          if (!wait_bounded(BAR(B_OUT_READY + s), staged[s] & 1, wc, 4)) return false;
          ++staged[s];
          const uint32_t stg = sbase + L::kOffStage + s * L::kStageBytes;
          for (int c = 0; c < L::kGroups; ++c) {
            tma_store_3d(&tmDV, stg + c * L::kSubBytes, c * 64, pend_jt[s] * kTile, pend_bh[s]);
            tma_store_3d(&tmDK, stg + L::kTileBytes + c * L::kSubBytes, c * 64, pend_jt[s] * kTile,
                         pend_bh[s]);
          }
          bulk_commit_group();
          bulk_wait_group_read0();
          pend_jt[s] = -1;
          return true;
        };
        bool ok = true;
        int g = 0, bh, jt;
        for (int round = 0; ok && bwd_item(p, round, bh, jt); ++round) {
          const int i0 = CAUSAL ? jt : 0, n_blk = blocks_of(jt);
          // resident K, V: the previous item's last S^T and dP^T have read them
          if (!wait_bounded(BAR(B_RES_EMPTY), (round & 1) ^ 1, wc, 5)) break;
          mbar_arrive_expect_tx(BAR(B_RES_FULL), 2 * L::kTileBytes);
          for (int c = 0; c < L::kGroups; ++c) {
            tma_load_3d(sK + c * L::kSubBytes, &tmK, BAR(B_RES_FULL), c * 64, jt * kTile, bh);
            tma_load_3d(sV + c * L::kSubBytes, &tmV, BAR(B_RES_FULL), c * 64, jt * kTile, bh);
          }
          ++res_issued;
          for (int it = 0; it < n_blk; ++it, ++g) {
            const int s = g % kStages, ph = ((g / kStages) & 1) ^ 1;
            const int q0 = (i0 + it) * kTile;
            if (!(ok = wait_bounded(BAR(B_ST_EMPTY + s), ph, wc, 1))) break;
            if (!(ok = flush(s))) break;
            const uint32_t sq = q_addr(g);
            mbar_arrive_expect_tx(BAR(B_ST_FULL + s), L::kTileBytes + L::kExtBytes);
            for (int c = 0; c < L::kGroups; ++c)
              tma_load_3d(sq + c * L::kSubBytes, &tmQ, BAR(B_ST_FULL + s), c * 64, q0, bh);
            tma_load_3d(qx_addr(g), &tmQX, BAR(B_ST_FULL + s), 0, q0, bh);
            ++q_issued[s];
            if (!(ok = wait_bounded(BAR(B_DO_EMPTY + s), ph, wc, 3))) break;
            if (skip_pending) {
              skip_pending = false;  // test hook: this dO block never arrives
            } else {
              mbar_arrive_expect_tx(BAR(B_DO_FULL + s), L::kTileBytes + L::kExtBytes);
              for (int c = 0; c < L::kGroups; ++c)
                tma_load_3d(do_addr(g) + c * L::kSubBytes, &tmDO, BAR(B_DO_FULL + s), c * 64, q0, bh);
              tma_load_3d(dx_addr(g), &tmDX, BAR(B_DO_FULL + s), 0, q0, bh);
              ++do_issued[s];
            }
            if (it == n_blk - 1) {  // this slot will stage the item's output
              pend_jt[s] = jt;
              pend_bh[s] = bh;
            }
          }
        }
        // the outputs still staged, oldest first
        if (ok) ok = flush(g % kStages);
        if (ok) ok = flush((g + 1) % kStages);
        bulk_wait_group0();
        if (*abort_flag) {
          if (res_issued) wait_bounded(BAR(B_RES_FULL), (res_issued - 1) & 1, wc, 2, true);
          // the last load into a barrier completes its phase (loads - 1)
          for (int s = 0; s < kStages; ++s) {
            if (q_issued[s]) wait_bounded(BAR(B_ST_FULL + s), (q_issued[s] - 1) & 1, wc, 2, true);
            if (do_issued[s]) wait_bounded(BAR(B_DO_FULL + s), (do_issued[s] - 1) & 1, wc, 2, true);
          }
        }
      }
    } else if (warp == kMmaWarp) {
      // ------------------------------------------------------------ MMA issuer
      // per block g: S^T of the next block (which may open the next item) as
      // soon as S^T_g is in registers; then, once P^T and dS^T are in TMEM,
      // dK_g, dV_g and dP^T of the next block (the in-order tensor pipe makes
      // it overwrite the dP region only after dK_g and dV_g have read it).
      // An item's resident K, V are released after its last S^T and dP^T; a
      // new item's first dK, dV (which overwrite the accumulators) wait until
      // the compute warps have read the previous item's.
      if (lane == 0) {
        int round = 0, bh, jt;
        bool ok = bwd_item(p, 0, bh, jt);
        int n_blk = ok ? blocks_of(jt) : 0;
        // the block after (round, it): (nround, nit), valid if has_next
        int nround = 0, nit = 0, nbh = bh, njt = jt, nn_blk = n_blk;
        auto issue_s = [&](int g, int r, int it_, int nb) -> bool {
          if (it_ == 0 && !wait_bounded(BAR(B_RES_FULL), r & 1, wc, 10)) return false;
          if (!wait_bounded(BAR(B_ST_FULL + g % kStages), (g / kStages) & 1, wc, 11)) return false;
          tc_fence_after();
          mma_rows_x_rows<D>(tmem + L::kColS, sK, q_addr(g));  // S^T - L/scale
          mma_ext(tmem + L::kColS, sOnes, qx_addr(g));
          tc_commit(BAR(B_S_FULL));
          (void)nb;
          return true;
        };
        auto issue_dp = [&](int g, int it_, int nb) -> bool {
          if (!wait_bounded(BAR(B_DO_FULL + g % kStages), (g / kStages) & 1, wc, 16)) return false;
          tc_fence_after();
          mma_rows_x_rows<D>(tmem + L::kColDP, sV, do_addr(g));  // dP^T - D
          mma_ext(tmem + L::kColDP, sOnes, dx_addr(g));
          tc_commit(BAR(B_DP_FULL));
          if (it_ == nb - 1) tc_commit(BAR(B_RES_EMPTY));  // the item's last reads of K, V
          return true;
        };
        if (ok) ok = issue_s(0, 0, 0, n_blk) && issue_dp(0, 0, n_blk);
        for (int g = 0, it = 0; ok; ++g) {
          // the next block
          bool has_next = true;
          if (it + 1 < n_blk) {
            nround = round, nit = it + 1, nbh = bh, njt = jt, nn_blk = n_blk;
          } else {
            nround = round + 1, nit = 0;
            has_next = bwd_item(p, nround, nbh, njt);
            nn_blk = has_next ? blocks_of(njt) : 0;
          }
          const int s = g % kStages;
          // within an item the next S^T goes first; across items it goes after
          // this block's dK, dV, since it waits for the next item's K and V
          // (loaded only once this item's last S^T and dP^T have read the
          // resident tiles) and must not hold back the item's ACC_DONE
          const bool next_same_item = has_next && nit != 0;
          if (next_same_item) {
            ok = wait_bounded(BAR(B_PHASE1), g & 1, wc, 12);
            if (ok) ok = issue_s(g + 1, nround, nit, nn_blk);
            if (!ok) break;
          }
          ok = wait_bounded(BAR(B_PHASE2), g & 1, wc, 14);
          if (ok && it == 0 && round > 0) ok = wait_bounded(BAR(B_ACC_EMPTY), (round - 1) & 1, wc, 17);
          if (!ok) break;
          tc_fence_after();
          mma_tmem_x_rows<D>(tmem + L::kColAcc1, tDS, q_addr(g), it > 0);   // dK += dS^T Q
          tc_commit(BAR(B_ST_EMPTY + s));
          mma_tmem_x_rows<D>(tmem + L::kColAcc0, tP, do_addr(g), it > 0);   // dV += P^T dO
          tc_commit(BAR(B_DO_EMPTY + s));
          if (it == n_blk - 1) tc_commit(BAR(B_ACC_DONE));
          if (!has_next) break;
          if (!next_same_item) {
            ok = wait_bounded(BAR(B_PHASE1), g & 1, wc, 12);
            if (ok) ok = issue_s(g + 1, nround, nit, nn_blk);
            if (!ok) break;
          }
          if (!(ok = issue_dp(g + 1, nit, nn_blk))) break;
          round = nround, it = nit, bh = nbh, jt = njt, n_blk = nn_blk;
        }
        tc_commit(BAR(B_DRAIN));
        wait_bounded(BAR(B_DRAIN), 0, wc, 15, true);
      }
    }
  } else {
    regs_increase<kRegsCompute>();
    // ------------------------------------------------------------ compute warps
    // warp w: TMEM lanes (key rows) 32 (w % 4) .., columns (queries) 64 (w / 4) ..
    const int quad = warp & 3, half = warp >> 2;
    const int r = quad * 32 + lane;   // key row in the tile
    const uint32_t lane_base = uint32_t(quad * 32) << 16;
    const uint32_t tS = tmem + lane_base + L::kColS + half * kHalfCols;
    const uint32_t tDP = tmem + lane_base + L::kColDP + half * kHalfCols;
    const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
    const uint64_t scale2 = f2_pack(p.scale, p.scale);
    // the per-query terms -L/scale and -D arrive inside S^T and dP^T (the
    // extension K step of their MMAs), so these warps read no shared memory:
    // while the tensor core streams its operands, shared-memory reads queue for
    // hundreds of cycles and would stall the exponentials and the barrier
    // arrivals behind them
    const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
    bool ok = true;
    int g = 0, bh, jt;
    for (int round = 0; ok && bwd_item(p, round, bh, jt); ++round) {
      const int i0 = CAUSAL ? jt : 0, n_blk = blocks_of(jt);
      const int key = jt * kTile + r;
      for (int it = 0; it < n_blk; ++it, ++g) {
        const int q0 = (i0 + it) * kTile;
        // EX dropout: keep bit c of this key for query q0 + 64 half + c. Lane L
        // computes the calls for queries qb + 16 rnd + L/2, key block of
        // keys key - lane + 16 (L % 2); lane src = 2 qq + lane/16 holds the bits
        // of query qq of the round for this lane's 16-key block.
        uint64_t keep64 = ~0ull;
        if constexpr (EX) {
          if (p.keep_t < 256) {
            keep64 = 0;
            const int qb = q0 + half * kHalfCols;
            const int kb0 = (key - lane) / 16;
#pragma unroll
            for (int rnd = 0; rnd < 4; ++rnd) {
              const uint32_t m16 = keep16(p, bh, qb + 16 * rnd + (lane >> 1), kb0 + (lane & 1));
#pragma unroll
              for (int qq = 0; qq < 16; ++qq) {
                const uint32_t bits = __shfl_sync(0xffffffffu, m16, 2 * qq + (lane >> 4));
                keep64 |= uint64_t((bits >> (lane & 15)) & 1u) << (16 * rnd + qq);
              }
            }
          }
        }
        // EX bias: bias[q][key] of the 64 query columns, loaded before the
        // wait for S^T so that the loads overlap it (lanes read 32
        // consecutive keys of one row per load)
        uint32_t bpre[kHalfCols];
        const bool bias_on = EX && p.bias != nullptr && key < p.N;
        if constexpr (EX) {
          if (bias_on) {
            const uint16_t* bcol = bias_head(p, bh) + key;
            const int qb = q0 + half * kHalfCols;
#pragma unroll
            for (int c = 0; c < kHalfCols; ++c)
              bpre[c] = qb + c < p.N ? uint32_t(bcol[size_t(qb + c) * p.N]) : 0u;
          }
        }
        ok = wait_bounded(BAR(B_S_FULL), g & 1, wc, 20);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        // phase 1: read S^T - L/scale (after which the next S^T may overwrite
        // it) and form P^T = 2^(scale log2e (s - L_q/scale)) in registers. Only
        // the first block under the causal mask hides queries (q < key). Rows
        // past N are not masked: each row of dV and dK depends on its own row
        // of P^T and dS^T only, and those rows are never stored.
        uint64_t pr2[kHalfCols / 2];
        {
          uint32_t sr[kHalfCols];
          tmem_ld64_wait(tS, sr);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(B_PHASE1));
          if constexpr (EX) {
            if (bias_on) {
#pragma unroll
              for (int c = 0; c < kHalfCols; ++c)
                sr[c] = __float_as_uint(fmaf(bf16f(bpre[c]), p.inv_scale, __uint_as_float(sr[c])));
            }
          }
          auto nl4 = [&](int) { return zero4; };
          if (CAUSAL && it == 0) {
            const int qlim = key - q0 - half * kHalfCols;  // local columns below qlim are hidden
            form_p_half<true>(sr, c2, nl4, [&](int i) { return i < qlim; }, pr2);
          } else {
            form_p_half<false>(sr, c2, nl4, [](int) { return false; }, pr2);
          }
        }
        // phase 2: dS^T = P^T scale (dP^T - D_q); P^T and dS^T (bf16) then
        // replace this warp's 64 dP^T columns: P^T in the first 32, dS^T in the
        // last 32. Both chunks of dP^T are read before either store.
        ok = wait_bounded(BAR(B_DP_FULL), g & 1, wc, 22);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        {
          uint32_t pk_ds[kHalfCols / 2];
          const bool drop = EX && p.keep_t < 256;
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t dr[32];
            tmem_ld32_wait(tDP + ch * 32, dr);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              uint64_t t0 = f2_mul(f2_pack(__uint_as_float(dr[4 * j]), __uint_as_float(dr[4 * j + 1])), scale2);
              uint64_t t1 = f2_mul(f2_pack(__uint_as_float(dr[4 * j + 2]), __uint_as_float(dr[4 * j + 3])), scale2);
              if constexpr (EX) {
                if (drop) {
                  // z u + (1 - z)(-scale D_q), u = scale (dP - D)
                  const int c0 = ch * 32 + 4 * j;
                  const float* nsd = p.dvec + size_t(bh) * p.Np + q0 + half * kHalfCols + c0;
                  float u[4];
                  f2_unpack(t0, u[0], u[1]);
                  f2_unpack(t1, u[2], u[3]);
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const float z = (keep64 >> (c0 + e)) & 1 ? p.keep_scale : 0.f;
                    u[e] = fmaf(z, u[e], (1.f - z) * nsd[e]);
                  }
                  t0 = f2_pack(u[0], u[1]);
                  t1 = f2_pack(u[2], u[3]);
                }
              }
              pk_ds[ch * 16 + 2 * j] = f2_to_bf16x2(f2_mul(pr2[ch * 16 + 2 * j], t0));
              pk_ds[ch * 16 + 2 * j + 1] = f2_to_bf16x2(f2_mul(pr2[ch * 16 + 2 * j + 1], t1));
            }
          }
          uint32_t pk_p[kHalfCols / 2];
#pragma unroll
          for (int i = 0; i < kHalfCols / 2; ++i) {
            if constexpr (EX) {
              if (drop) {
                float a, b;
                f2_unpack(pr2[i], a, b);
                a = (keep64 >> (2 * i)) & 1 ? a * p.keep_scale : 0.f;
                b = (keep64 >> (2 * i + 1)) & 1 ? b * p.keep_scale : 0.f;
                pk_p[i] = pack_bf16x2(a, b);
                continue;
              }
            }
            pk_p[i] = f2_to_bf16x2(pr2[i]);
          }
          tmem_st32(tDP, pk_p);
          tmem_st32(tDP + 32, pk_ds);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_PHASE2));
      }
      if (!ok) break;
      // epilogue of the item: dV and dK as bf16 into the slot of its last
      // block (idle once every MMA of the item is done); the producer stores
      // them with TMA before it loads into that slot again. Key rows past N
      // fall outside the tensor.
      ok = wait_bounded(BAR(B_ACC_DONE), round & 1, wc, 23);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int s = (g - 1) % kStages;
      uint8_t* stg = smem + L::kOffStage + s * L::kStageBytes;
      stage_acc_half<D>(tmem + lane_base + L::kColAcc0, stg, r, half);
      stage_acc_half<D>(tmem + lane_base + L::kColAcc1, stg + L::kTileBytes, r, half);
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(BAR(B_ACC_EMPTY));
        mbar_arrive(BAR(B_OUT_READY + s));
      }
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
template <int D, bool CAUSAL, bool EX>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap,
                  const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap,
                  const BwdParams p) {
  using L = Plan<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto BAR = [&](int i) -> uint32_t { return sbase + L::kOffBar + 8u * uint32_t(i); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // items: (b*h, query tile it_q), the tiles that see the most key blocks
  // first (causal: the last ones); an item streams key blocks 0 .. n_blk-1
  auto tile_of = [&](int level) { return CAUSAL ? p.n_tiles - 1 - level : level; };
  auto blocks_of = [&](int it_q) { return CAUSAL ? it_q + 1 : p.n_tiles; };
  volatile int* abort_flag;
  const uint32_t tmem = setup_cta<D>(smem, warp, abort_flag);
  const WaitCtl wc{abort_flag, p.status, p.limit_ns, KID_BWD_DQ};
  const uint32_t sQ = sbase + L::kOffRes0, sDO = sbase + L::kOffRes1;
  // global block g of this CTA takes K slot g % 3 and V slot g % 2: K (read
  // by S and, last, by dQ) gets one more block of prefetch than V (last read
  // by dP). After an item's last block its K slot stages the item's dQ tile,
  // which the producer stores with TMA before its next load into that slot.
  auto k_addr = [&](int g) { return sbase + L::kOffKRing + (g % kKSlots) * L::kTileBytes; };
  auto v_addr = [&](int g) { return sbase + L::kOffVRing + (g % kStages) * L::kTileBytes; };

  if (warp >= 8) {
    regs_decrease<kRegsControl>();
    if (warp == kLoadWarp) {
      if (lane == 0) {
        // loads started into each ring slot (the abort path waits for them)
        int k_issued[kKSlots] = {0, 0, 0}, v_issued[kStages] = {0, 0}, res_issued = 0;
        bool skip_pending = p.debug_skip == KID_BWD_DQ && blockIdx.x == 0;
        int pend_q[kKSlots] = {-1, -1, -1}, pend_bh[kKSlots] = {0, 0, 0}, staged[kKSlots] = {0, 0, 0};
        auto flush = [&](int s) -> bool {
          if (pend_q[s] < 0) return true;
          if (!wait_bounded(BAR(B_KOUT_READY + s), staged[s] & 1, wc, 4)) return false;
          ++staged[s];
          for (int c = 0; c < L::kGroups; ++c)
            tma_store_3d(&tmDQ, sbase + L::kOffKRing + s * L::kTileBytes + c * L::kSubBytes, c * 64,
                         pend_q[s] * kTile, pend_bh[s]);
          bulk_commit_group();
          bulk_wait_group_read0();
          pend_q[s] = -1;
          return true;
        };
        bool ok = true;
        int g = 0, bh, lvl;
        for (int round = 0; ok && bwd_item(p, round, bh, lvl); ++round) {
          const int it_q = tile_of(lvl), n_blk = blocks_of(it_q);
          if (!wait_bounded(BAR(B_RES_EMPTY), (round & 1) ^ 1, wc, 5)) break;
          mbar_arrive_expect_tx(BAR(B_RES_FULL), 2 * L::kTileBytes);
          for (int c = 0; c < L::kGroups; ++c) {
            tma_load_3d(sQ + c * L::kSubBytes, &tmQ, BAR(B_RES_FULL), c * 64, it_q * kTile, bh);
            tma_load_3d(sDO + c * L::kSubBytes, &tmDO, BAR(B_RES_FULL), c * 64, it_q * kTile, bh);
          }
          ++res_issued;
          for (int it = 0; it < n_blk; ++it, ++g) {
            const int ks = g % kKSlots, vs = g % kStages;
            if (!(ok = wait_bounded(BAR(B_K_EMPTY + ks), ((g / kKSlots) & 1) ^ 1, wc, 1))) break;
            if (!(ok = flush(ks))) break;
            mbar_arrive_expect_tx(BAR(B_K_FULL + ks), L::kTileBytes);
            for (int c = 0; c < L::kGroups; ++c)
              tma_load_3d(k_addr(g) + c * L::kSubBytes, &tmK, BAR(B_K_FULL + ks), c * 64, it * kTile, bh);
            ++k_issued[ks];
            if (!(ok = wait_bounded(BAR(B_DO_EMPTY + vs), ((g / kStages) & 1) ^ 1, wc, 3))) break;
            if (skip_pending) {
              skip_pending = false;  // test hook: this V block never arrives
            } else {
              mbar_arrive_expect_tx(BAR(B_DO_FULL + vs), L::kTileBytes);
              for (int c = 0; c < L::kGroups; ++c)
                tma_load_3d(v_addr(g) + c * L::kSubBytes, &tmV, BAR(B_DO_FULL + vs), c * 64, it * kTile, bh);
              ++v_issued[vs];
            }
            if (it == n_blk - 1) {
              pend_q[ks] = it_q;
              pend_bh[ks] = bh;
            }
          }
        }
        // the outputs still staged, oldest first
        for (int j = 0; ok && j < kKSlots; ++j) ok = flush((g + j) % kKSlots);
        bulk_wait_group0();
        if (*abort_flag) {
          if (res_issued) wait_bounded(BAR(B_RES_FULL), (res_issued - 1) & 1, wc, 2, true);
          // the last load into a barrier completes its phase (loads - 1)
          for (int s = 0; s < kKSlots; ++s)
            if (k_issued[s]) wait_bounded(BAR(B_K_FULL + s), (k_issued[s] - 1) & 1, wc, 2, true);
          for (int s = 0; s < kStages; ++s)
            if (v_issued[s]) wait_bounded(BAR(B_DO_FULL + s), (v_issued[s] - 1) & 1, wc, 2, true);
        }
      }
    } else if (warp == kMmaWarp) {
      // per block g: S of the next block of the same item once S_g is in
      // registers; dQ_g after phase 2; then (for a new item, after dQ_g, since
      // it waits for the item's resident Q and dO) S of the next block, and
      // dP of the next block. A new item's first dQ (which overwrites the
      // accumulator) waits until the compute warps have read the previous one.
      if (lane == 0) {
        int round = 0, bh, lvl;
        bool ok = bwd_item(p, 0, bh, lvl);
        int n_blk = ok ? blocks_of(tile_of(lvl)) : 0;
        int nround = 0, nit = 0, nbh = bh, nlvl = lvl, nn_blk = n_blk;
        // an item's Q and dO go from shared memory into TMEM once (the A
        // operands of its S and dP MMAs, which then read only K or V from
        // shared memory); the shared copies are released right after, so the
        // next item's Q and dO can load during this one
        auto issue_s = [&](int g, int r, int it_) -> bool {
          if (it_ == 0) {
            if (!wait_bounded(BAR(B_RES_FULL), r & 1, wc, 10)) return false;
            tc_fence_after();
            copy_tile_to_tmem<D>(tmem + L::kColQT, sQ);
            copy_tile_to_tmem<D>(tmem + L::kColDOT, sDO);
            tc_commit(BAR(B_RES_EMPTY));
          }
          if (!wait_bounded(BAR(B_K_FULL + g % kKSlots), (g / kKSlots) & 1, wc, 11)) return false;
          tc_fence_after();
          mma_tmem_rows_x_rows<D>(tmem + L::kColS, tmem + L::kColQT, k_addr(g));  // S = Q K^T
          tc_commit(BAR(B_S_FULL));
          return true;
        };
        auto issue_dp = [&](int g, int it_, int nb) -> bool {
          (void)it_;
          (void)nb;
          if (!wait_bounded(BAR(B_DO_FULL + g % kStages), (g / kStages) & 1, wc, 16)) return false;
          tc_fence_after();
          mma_tmem_rows_x_rows<D>(tmem + L::kColDP, tmem + L::kColDOT, v_addr(g));  // dP = dO V^T
          tc_commit(BAR(B_DP_FULL));
          tc_commit(BAR(B_DO_EMPTY + g % kStages));  // V read
          return true;
        };
        if (ok && (ok = issue_s(0, 0, 0))) ok = issue_dp(0, 0, n_blk);
        for (int g = 0, it = 0; ok; ++g) {
          bool has_next = true;
          if (it + 1 < n_blk) {
            nround = round, nit = it + 1, nbh = bh, nlvl = lvl, nn_blk = n_blk;
          } else {
            nround = round + 1, nit = 0;
            has_next = bwd_item(p, nround, nbh, nlvl);
            nn_blk = has_next ? blocks_of(tile_of(nlvl)) : 0;
          }
          const bool next_same_item = has_next && nit != 0;
          if (next_same_item) {
            ok = wait_bounded(BAR(B_PHASE1), g & 1, wc, 12);
            if (ok) ok = issue_s(g + 1, nround, nit);
            if (!ok) break;
          }
          ok = wait_bounded(BAR(B_PHASE2), g & 1, wc, 14);
          if (ok && it == 0 && round > 0) ok = wait_bounded(BAR(B_ACC_EMPTY), (round - 1) & 1, wc, 17);
          if (!ok) break;
          tc_fence_after();
          mma_tmem_x_rows<D>(tmem + L::kColAcc0, tmem + L::kColDP, k_addr(g), it > 0);  // dQ += dS K
          tc_commit(BAR(B_K_EMPTY + g % kKSlots));
          if (it == n_blk - 1) tc_commit(BAR(B_ACC_DONE));
          if (!has_next) break;
          if (!next_same_item) {
            ok = wait_bounded(BAR(B_PHASE1), g & 1, wc, 12);
            if (ok) ok = issue_s(g + 1, nround, nit);
            if (!ok) break;
          }
          if (!(ok = issue_dp(g + 1, nit, nn_blk))) break;
          round = nround, it = nit, bh = nbh, lvl = nlvl, n_blk = nn_blk;
        }
        tc_commit(BAR(B_DRAIN));
        wait_bounded(BAR(B_DRAIN), 0, wc, 15, true);
      }
    }
  } else {
    regs_increase<kRegsCompute>();
    // warp w: TMEM lanes (query rows) 32 (w % 4) .., columns (keys) 64 (w / 4) ..
    const int quad = warp & 3, half = warp >> 2;
    const int r = quad * 32 + lane;   // query row in the tile
    const uint32_t lane_base = uint32_t(quad * 32) << 16;
    const uint32_t tS = tmem + lane_base + L::kColS + half * kHalfCols;
    const uint32_t tDP = tmem + lane_base + L::kColDP + half * kHalfCols;
    const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
    const uint64_t scale2 = f2_pack(p.scale, p.scale);
    bool ok = true;
    int g = 0, bh, lvl;
    // this row's -L2 and -scale D (-inf and 0 past N; q < Np always), read one
    // item ahead so the load hides behind the previous item's epilogue
    bool have = bwd_item(p, 0, bh, lvl);
    float nl2q = 0.f, nsdq = 0.f;
    if (have) {
      const size_t at = size_t(bh) * p.Np + tile_of(lvl) * kTile + r;
      nl2q = p.lse2[at];
      nsdq = p.dvec[at];
    }
    for (int round = 0; ok && have; ++round) {
      const int it_q = tile_of(lvl), n_blk = blocks_of(it_q);
      const int q = it_q * kTile + r;
      const float4 nl2q4 = make_float4(nl2q, nl2q, nl2q, nl2q);
      const float4 nsdq4 = make_float4(nsdq, nsdq, nsdq, nsdq);
      for (int it = 0; it < n_blk; ++it, ++g) {
        const int k0 = it * kTile;
        // EX dropout: keep bit c of this query for key k0 + 64 half + c
        uint64_t keep64 = ~0ull;
        if constexpr (EX) {
          if (p.keep_t < 256) {
            const int kb = (k0 + half * kHalfCols) / 16;
            keep64 = uint64_t(keep16(p, bh, q, kb)) | (uint64_t(keep16(p, bh, q, kb + 1)) << 16) |
                     (uint64_t(keep16(p, bh, q, kb + 2)) << 32) |
                     (uint64_t(keep16(p, bh, q, kb + 3)) << 48);
          }
        }
        // EX bias (16-byte rows): this half's 64 keys of row q, loaded before
        // the wait for S so that the loads overlap it
        uint4 bq[kHalfCols / 8];
        const bool bias_pf = EX && p.bias != nullptr && p.bias_vec && q < p.N;
        if constexpr (EX) {
          if (bias_pf) {
            const int kb0 = k0 + half * kHalfCols;
            const uint16_t* brow = bias_head(p, bh) + size_t(q) * p.N + kb0;
            const int n = min(kHalfCols, p.N - kb0);
#pragma unroll
            for (int c8 = 0; c8 < kHalfCols / 8; ++c8)
              bq[c8] = 8 * c8 < n ? *reinterpret_cast<const uint4*>(brow + 8 * c8) : make_uint4(0, 0, 0, 0);
          }
        }
        ok = wait_bounded(BAR(B_S_FULL), g & 1, wc, 20);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        // phase 1: read S (then the MMA may overwrite it) and form P
        uint32_t sr[kHalfCols];
        tmem_ld64_wait(tS, sr);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_PHASE1));
        if constexpr (EX) {
          // bias[q][keys] / scale for this half's 64 keys
          if (p.bias != nullptr && q < p.N) {
            const int kb0 = k0 + half * kHalfCols;
            const uint16_t* brow = bias_head(p, bh) + size_t(q) * p.N + kb0;
            const int n = min(kHalfCols, p.N - kb0);
            if (bias_pf) {
#pragma unroll
              for (int c8 = 0; c8 < kHalfCols / 8; ++c8) {
                if (8 * c8 < n) {
                  const uint4 u = bq[c8];
                  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    sr[8 * c8 + 2 * e] = __float_as_uint(
                        fmaf(bf16f(w[e] & 0xffffu), p.inv_scale, __uint_as_float(sr[8 * c8 + 2 * e])));
                    sr[8 * c8 + 2 * e + 1] = __float_as_uint(
                        fmaf(bf16f(w[e] >> 16), p.inv_scale, __uint_as_float(sr[8 * c8 + 2 * e + 1])));
                  }
                }
              }
            } else {
#pragma unroll
              for (int c = 0; c < kHalfCols; ++c)
                if (c < n)
                  sr[c] = __float_as_uint(fmaf(bf16f(brow[c]), p.inv_scale, __uint_as_float(sr[c])));
            }
          }
        }
        uint64_t pr2[kHalfCols / 2];
        auto nl4 = [&](int) { return nl2q4; };
        // keys past N, or (causal) past q, are hidden: only the last block has any
        if ((CAUSAL && it == n_blk - 1) || k0 + kTile > p.N) {
          int klim = p.N - k0;
          if (CAUSAL) klim = min(klim, q - k0 + 1);
          klim -= half * kHalfCols;  // local columns at or above klim are hidden
          form_p_half<true>(sr, c2, nl4, [&](int i) { return i >= klim; }, pr2);
        } else {
          form_p_half<false>(sr, c2, nl4, [](int) { return false; }, pr2);
        }
        // phase 2: dS = P (scale dP - scale D_q), written back over dP as bf16
        ok = wait_bounded(BAR(B_DP_FULL), g & 1, wc, 21);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        if constexpr (EX) {
          if (p.keep_t < 256) {
            // dS = P (scale z dP - scale D): the scale of each dP entry is scale z
            const float szk = p.scale * p.keep_scale;
            write_ds_half_z(tDP, pr2, keep64, szk, [&](int) { return nsdq4; });
          } else {
            write_ds_half(tDP, pr2, scale2, [&](int) { return nsdq4; });
          }
        } else {
          write_ds_half(tDP, pr2, scale2, [&](int) { return nsdq4; });
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_PHASE2));
      }
      if (!ok) break;
      // the next item's row terms, then the epilogue of this one: dQ as bf16
      // into the K part of the last block's slot (idle once every MMA of the
      // item is done); the producer stores it with TMA (rows past N clipped)
      have = bwd_item(p, round + 1, bh, lvl);
      if (have) {
        const size_t at = size_t(bh) * p.Np + tile_of(lvl) * kTile + r;
        nl2q = p.lse2[at];
        nsdq = p.dvec[at];
      }
      ok = wait_bounded(BAR(B_ACC_DONE), round & 1, wc, 22);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int s = (g - 1) % kKSlots;
      stage_acc_half<D>(tmem + lane_base + L::kColAcc0, smem + L::kOffKRing + s * L::kTileBytes, r, half);
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(BAR(B_ACC_EMPTY));
        mbar_arrive(BAR(B_KOUT_READY + s));
      }
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
  // the setmaxnreg split is sized for exactly kRegsAtLaunch registers per
  // thread; with fewer the increase could wait forever, so refuse to launch
  cudaFuncAttributes attr;
  e = cudaFuncGetAttributes(&attr, kern);
  if (e != cudaSuccess) return cuda_fail(e, what);
  if (attr.numRegs != kRegsAtLaunch) {
    set_last_error("%s built with %d registers per thread, expected %d", what, attr.numRegs, kRegsAtLaunch);
    return FA_ERR_UNSUPPORTED;
  }
  {
    ProfileScope prof(kid, ctx.stream);
    kern<<<grid, kThreads, smem, ctx.stream>>>(m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return FA_OK;
}

template <int D, bool CAUSAL, bool EX>
fa_status launch_all(const void* q, const void* k, const void* v, const void* dO, const BwdParams& p,
                     const LaunchCtx& ctx) {
  // maps 0-3: Q, dO, K, V; 4-5: extension rows; 6-7: outputs (dK, dV for the
  // key-tile kernel, dQ for the query-tile kernel)
  const int smem = Plan<D>::kSmemBytes;
  const unsigned grid = unsigned(p.n_tiles) * unsigned(p.BH);
  CUtensorMap m[8], mq[8];
  const void* src[4] = {q, dO, k, v};
  for (int i = 0; i < 4; ++i) {
    fa_status st = make_tmap_3d(&m[i], src[i], 2, D, p.N, p.BH, 64, kTile, 128);
    if (st != FA_OK) return st;
  }
  fa_status st = make_tmap_3d(&m[4], p.qext, 2, 16, p.Np, p.BH, 16, kTile, 32);
  if (st == FA_OK) st = make_tmap_3d(&m[5], p.dext, 2, 16, p.Np, p.BH, 16, kTile, 32);
  if (st == FA_OK) st = make_tmap_3d(&m[6], p.dk, 2, D, p.N, p.BH, 64, kTile, 128);
  if (st == FA_OK) st = make_tmap_3d(&m[7], p.dv, 2, D, p.N, p.BH, 64, kTile, 128);
  if (st != FA_OK) return st;
  for (int i = 0; i < 6; ++i) mq[i] = m[i];
  st = make_tmap_3d(&mq[6], p.dq, 2, D, p.N, p.BH, 64, kTile, 128);
  if (st != FA_OK) return st;
  mq[7] = mq[6];
  // both kernels are persistent: one CTA per SM walks its items
  const unsigned grid_kv = grid < unsigned(ctx.num_sms) ? grid : unsigned(ctx.num_sms);
  st = launch_main(bwd_dkdv_kernel<D, CAUSAL, EX>, KID_BWD, smem, grid_kv, m, p, ctx, "bwd dK/dV kernel");
  if (st != FA_OK) return st;
  return launch_main(bwd_dq_kernel<D, CAUSAL, EX>, KID_BWD_DQ, smem, grid_kv, mq, p, ctx, "bwd dQ kernel");
}

}  // namespace

size_t bwd_workspace_bytes(int B, int H, int N, int d) {
  (void)d;
  const size_t bh = size_t(B) * H;
  const size_t np = (size_t(N) + kTile - 1) / kTile * kTile;
  return 2 * align256(bh * np * 4) + 2 * align256(bh * np * 32);
}

fa_status launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                     float scale, bool causal, void* workspace, const LaunchCtx& ctx,
                     const FwdExtras* ex) {
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
  const size_t vec_bytes = align256(size_t(BH) * p.Np * 4), ext_bytes = align256(size_t(BH) * p.Np * 32);
  p.lse2 = reinterpret_cast<float*>(ws);
  p.dvec = reinterpret_cast<float*>(ws + vec_bytes);
  p.qext = reinterpret_cast<uint16_t*>(ws + 2 * vec_bytes);
  p.dext = reinterpret_cast<uint16_t*>(ws + 2 * vec_bytes + ext_bytes);
  p.dq = static_cast<uint16_t*>(dq);
  p.dk = static_cast<uint16_t*>(dk);
  p.dv = static_cast<uint16_t*>(dv);
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.status = ctx.status_word;
  p.limit_ns = ctx.wait_limit_ns;
  p.debug_skip = ctx.debug_skip_load;
  const bool use_ex = ex != nullptr && (ex->bias != nullptr || ex->keep_t < 256);
  p.bias = use_ex ? static_cast<const uint16_t*>(ex->bias) : nullptr;
  p.bias_sb = use_ex ? ex->bias_stride_b : 0;
  p.bias_sh = use_ex ? ex->bias_stride_h : 0;
  p.H = H;
  p.bias_vec = (use_ex && N % 8 == 0 && p.bias_sb % 8 == 0 && p.bias_sh % 8 == 0) ? 1 : 0;
  p.inv_scale = 1.0f / scale;
  p.seed_lo = use_ex ? uint32_t(ex->seed) : 0u;
  p.seed_hi = use_ex ? uint32_t(ex->seed >> 32) : 0u;
  p.rng_offset = use_ex ? ex->offset : 0u;
  p.keep_t = use_ex ? ex->keep_t : 256;
  p.keep_scale = 256.0f / float(p.keep_t);

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
  if (use_ex) {
    if (d == 128)
      return causal ? launch_all<128, true, true>(q, k, v, dO, p, ctx)
                    : launch_all<128, false, true>(q, k, v, dO, p, ctx);
    return causal ? launch_all<64, true, true>(q, k, v, dO, p, ctx)
                  : launch_all<64, false, true>(q, k, v, dO, p, ctx);
  }
  if (d == 128)
    return causal ? launch_all<128, true, false>(q, k, v, dO, p, ctx)
                  : launch_all<128, false, false>(q, k, v, dO, p, ctx);
  return causal ? launch_all<64, true, false>(q, k, v, dO, p, ctx)
                : launch_all<64, false, false>(q, k, v, dO, p, ctx);
}

}  // namespace fa
