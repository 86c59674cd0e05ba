// decode_sm100.cu -- split-KV decode: one query token per (sequence, head)
// against a KV cache ("Bellek Duvarinin Fizigi", "Decode Asamasi:
// Flash-Decoding").
//
// The cache axis of each sequence is cut into C chunks. Chunk c of sequence b
// covers cache positions [c*ceil(L_b/C), min((c+1)*ceil(L_b/C), L_b)). Each
// chunk yields its own triple (m_c, l_c, O~_c), stored as the normalised
// partial o_c = O~_c / l_c and lse_c = m_c + log2 l_c (base 2). A second
// kernel merges the chunks of each (b, h) by the rescale identity the page
// states for the online softmax, applied across chunks:
//     LSE = log sum_c exp(lse_c),   O = sum_c exp(lse_c - LSE) o_c,
// in a fixed chunk order, so the result is the same on every run.
//
// The work is a stream over the cache: about 4 bytes read per FLOP, so the
// bound is HBM bandwidth, not the tensor cores (a single query row is not a
// dense contraction). B200 design:
//  * one CTA per (chunk, head, sequence); a producer warp streams the
//    chunk's K and V rows into a 3-stage shared-memory ring with plain bulk
//    copies (cp.async.bulk: the rows of one chunk are contiguous), up to
//    96 KB per CTA and two CTAs per SM;
//  * eight consumer warps; each half-warp owns 4 rows of every 64-row stage
//    and a lane d/16 elements of q and of the output accumulator, so one
//    16-byte shared-memory load per lane reads a row;
//  * the four partial dot products of a half-warp are summed across its 16
//    lanes together (5 shuffles for 4 rows instead of 4 per row), and the
//    running maximum moves once per 4 rows;
//  * positions at or past seqlens[b] are never read;
//  * grouped query heads ("Duvarin Otesi": GQA / MQA): query head h reads
//    KV head h / (Hq / Hkv); a CTA serves up to 4 query heads of one KV head
//    from a single shared-memory copy of each K/V row (each lane keeps q, the
//    running statistics and the output slice of every head), and the CTAs
//    of the remaining heads of the group run side by side, so a chunk is
//    read from HBM once and through L2 Hq / Hkv / 4 times at most;
//  * paged caches (the same section: PagedAttention): a separate
//    instantiation whose producer finds each 64-row stage's page in the
//    sequence's block table (chunks then start on 64-row boundaries); a
//    page index outside the pool is never dereferenced but reported in the
//    device status word;
//  * all waits are bounded in time (see sm100_ptx.cuh).
#include <mutex>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kStageTok = 64;     // cache rows per pipeline stage
constexpr int kStages = 3;
constexpr int kConsumerWarps = 8;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kRowsPerHalf = kStageTok / (2 * kConsumerWarps);  // 4
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kSmHint = 148;      // B200 SM count, for the automatic split
constexpr int kTcMinGroup = 4;    // query heads per KV head from which the tensor-core path runs
constexpr int kTcMaxGroup = 128;  // its M rows; larger groups run on the CUDA cores
// up to this many heads per KV head, keys as the M rows (measured: as fast
// as heads-as-rows at 4 and 8 heads, 6% slower at 16)
constexpr int kTctMaxGroup = 8;

template <int D>
struct DecLayout {
  static constexpr int kTileBytes = kStageTok * D * 2;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kStages * kTileBytes;
  static constexpr int kOffBar = 2 * kStages * kTileBytes;       // full[s], empty[s]
  static constexpr int kOffMisc = kOffBar + 8 * 2 * kStages;     // abort flag
  static constexpr int kSmemBytes = kOffMisc + 16 + 128;
  // after the stream: per half-warp and query head m, l, acc[D], over the
  // stage buffers (no copy is in flight by then)
  static constexpr int kOffMerge = 0;
  static_assert(2 * kConsumerWarps * 4 * (D + 2) * 4 <= 2 * kStages * kTileBytes, "merge area");
};

struct DecParams {
  const uint16_t* q;
  const uint16_t* kc;   // contiguous [B, Hkv, Lmax, D], or pages [num_pages, Hkv, page, D]
  const uint16_t* vc;
  const int* seqlens;
  const int* table;     // paged: [B, max_pages] page of each page-sized run of positions
  int group;            // query heads per KV head (Hq / Hkv)
  int Hkv;
  int page, max_pages, num_pages;  // paged layout
  float* part_o;    // [B, H, C, D]
  float* part_lse;  // [B, H, C], base 2
  uint16_t* o;
  float* lse;
  int H, Lmax, C;
  float scale_log2;
  unsigned int* status;
  unsigned long long limit_ns;
  int debug_skip;   // test hook: CTA (0,0,0) leaves out its first tile's loads
};

// kPer bf16 of one cached row (this lane's part) -> fp32
template <int kPer>
__device__ __forceinline__ void load_row_part(const uint8_t* row, int j, float (&x)[kPer]) {
  if constexpr (kPer == 8) {
    const uint4 w = *reinterpret_cast<const uint4*>(row + j * 16);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(ws[i] << 16);
      x[2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u);
    }
  } else {
    const uint2 w = *reinterpret_cast<const uint2*>(row + j * 8);
    const uint32_t ws[2] = {w.x, w.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      x[2 * i] = __uint_as_float(ws[i] << 16);
      x[2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u);
    }
  }
}

// One CTA per (chunk, head, sequence): a producer warp streams the chunk's
// K and V rows into a 3-stage ring; each half-warp of the 8 consumer warps
// owns 4 rows of every 64-row stage. A lane holds d/16 elements of q and of
// its output accumulator, so one 16-byte shared load per lane reads a whole
// row per half-warp.
template <int D, bool PAGED, int GH>
__global__ void __launch_bounds__(kThreads, 2)
    decode_split_kernel(const DecParams p) {
  using L = DecLayout<D>;
  // the merge kernel, launched as a programmatic dependent, may be scheduled
  // now: it waits for this grid's completion before reading anything
  grid_dependents_launch();
  constexpr int kPer = D / 16;  // elements per lane (16 lanes per row)
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc);
  float* merge = reinterpret_cast<float*>(smem + L::kOffMerge);
  auto FULL = [&](int s) -> uint32_t { return sbase + L::kOffBar + 8u * s; };
  auto EMPTY = [&](int s) -> uint32_t { return sbase + L::kOffBar + 8u * (kStages + s); };

  // GH query heads h0 .. h0+GH-1 that share KV head hkv (GH divides the group)
  const int c = blockIdx.x, h0 = blockIdx.y * GH, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t bh0 = size_t(b) * p.H + h0;
  const int hkv = h0 / p.group;

  int Lb = p.seqlens[b];
  Lb = Lb < 0 ? 0 : (Lb > p.Lmax ? p.Lmax : Lb);
  int chunk = (Lb + p.C - 1) / p.C;
  if (PAGED) chunk = (chunk + kStageTok - 1) / kStageTok * kStageTok;  // stages start on 64-row boundaries
  const int t0 = c * chunk;
  const int t1 = min(t0 + chunk, Lb);
  if (t0 >= t1) {  // empty chunk: weight 0 in the merge
    for (int g = 0; g < GH; ++g) {
      const size_t part = (bh0 + g) * p.C + c;
      for (int i = threadIdx.x; i < D; i += blockDim.x) p.part_o[part * D + i] = 0.f;
      if (threadIdx.x == 0) p.part_lse[part] = -INFINITY;
    }
    return;
  }
  const int n_tok = t1 - t0;
  const int n_tiles = (n_tok + kStageTok - 1) / kStageTok;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(FULL(s), 1);
      mbar_init(EMPTY(s), kConsumerWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const WaitCtl wc{abort_flag, p.status, p.limit_ns, KID_DECODE};

  if (warp == kConsumerWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const size_t bkv = size_t(b) * p.Hkv + hkv;
      const uint16_t* kb = PAGED ? p.kc : p.kc + (bkv * p.Lmax + t0) * D;  // contiguous cache only
      const uint16_t* vb = PAGED ? p.vc : p.vc + (bkv * p.Lmax + t0) * D;
      int issued = 0, skip_stage = -1;
      const bool skip = p.debug_skip && c == 0 && h0 == 0 && b == 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % kStages;
        if (!wait_bounded(EMPTY(s), ((i / kStages) & 1) ^ 1, wc, 1)) break;
        if (skip && i == 0) {  // test hook: this tile never arrives
          skip_stage = s;
          ++issued;
          continue;
        }
        const int rows = min(kStageTok, n_tok - i * kStageTok);
        if (!PAGED) {
          const uint32_t bytes = uint32_t(rows) * D * 2;
          mbar_arrive_expect_tx(FULL(s), 2 * bytes);
          bulk_load(sbase + L::kOffK + s * L::kTileBytes, kb + size_t(i) * kStageTok * D, bytes, FULL(s));
          bulk_load(sbase + L::kOffV + s * L::kTileBytes, vb + size_t(i) * kStageTok * D, bytes, FULL(s));
        } else {
          // the stage's rows [t, t + rows) in runs that each lie in one page
          // (one run when the page holds a multiple of 64 rows, 64 / page
          // runs for pages of 16 or 32 rows); every page index is checked
          // against the pool before its rows are read
          const int t = t0 + i * kStageTok;
          const int run = p.page < kStageTok ? p.page : kStageTok;
          uint32_t total = 0;
          for (int r0 = 0; r0 < rows; r0 += run) {
            const int tp = t + r0;
            const int pg = p.table[size_t(b) * p.max_pages + tp / p.page];
            if (pg < 0 || pg >= p.num_pages) {
              atomicCAS(p.status, 0u, (unsigned(KID_DECODE) << 16) | (9u << 8) | 2u);
              continue;  // these rows stay unread (results undefined, error reported)
            }
            total += uint32_t(min(run, rows - r0)) * D * 2;
          }
          mbar_arrive_expect_tx(FULL(s), 2 * total);
          for (int r0 = 0; r0 < rows; r0 += run) {
            const int tp = t + r0;
            const int pg = p.table[size_t(b) * p.max_pages + tp / p.page];
            if (pg < 0 || pg >= p.num_pages) continue;
            const uint32_t bytes = uint32_t(min(run, rows - r0)) * D * 2;
            const size_t src = ((size_t(pg) * p.Hkv + hkv) * p.page + tp % p.page) * D;
            const uint32_t dst = uint32_t(r0) * D * 2;
            bulk_load(sbase + L::kOffK + s * L::kTileBytes + dst, p.kc + src, bytes, FULL(s));
            bulk_load(sbase + L::kOffV + s * L::kTileBytes + dst, p.vc + src, bytes, FULL(s));
          }
        }
        ++issued;
      }
      if (*abort_flag)
        for (int s = 0; s < kStages; ++s) {
          const int cnt = (issued - s + kStages - 1) / kStages - (s == skip_stage ? 1 : 0);
          if (cnt > 0) wait_bounded(FULL(s), (cnt - 1) & 1, wc, 2, true);  // the last load into s
        }
    }
  } else {
    // ---------------------------------------------------------------- consumers
    const int half = lane >> 4;   // which of the two rows a step covers
    const int j = lane & 15;      // this lane's slice of a row
    // the row whose full score this lane holds after the reduction below
    const int u_own = 2 * ((j >> 3) & 1) + ((j >> 2) & 1);
    float qv[GH][kPer];
#pragma unroll
    for (int g = 0; g < GH; ++g) {
      const uint16_t* qp = p.q + (bh0 + g) * D + j * kPer;
#pragma unroll
      for (int i = 0; i < kPer; ++i) qv[g][i] = __uint_as_float(uint32_t(qp[i]) << 16) * p.scale_log2;
    }
    float m[GH], l[GH], acc[GH][kPer];
#pragma unroll
    for (int g = 0; g < GH; ++g) {
      m[g] = -INFINITY;
      l[g] = 0.f;
#pragma unroll
      for (int i = 0; i < kPer; ++i) acc[g][i] = 0.f;
    }

    for (int it = 0; it < n_tiles; ++it) {
      const int s = it % kStages;
      bool ok = wait_bounded(FULL(s), (it / kStages) & 1, wc, 3);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const int rows = min(kStageTok, n_tok - it * kStageTok);
      const uint8_t* ktile = smem + L::kOffK + s * L::kTileBytes;
      const uint8_t* vtile = smem + L::kOffV + s * L::kTileBytes;
      // partial q.k of this lane's slice for the half-warp's 4 rows, every
      // query head from the one shared-memory read of the row
      float sc[GH][kRowsPerHalf];
#pragma unroll
      for (int u = 0; u < kRowsPerHalf; ++u) {
        const int r = warp * 2 * kRowsPerHalf + 2 * u + half;
        float kx[kPer];
        if (r < rows) {
          load_row_part<kPer>(ktile + r * D * 2, j, kx);
        } else {
#pragma unroll
          for (int i = 0; i < kPer; ++i) kx[i] = 0.f;
        }
#pragma unroll
        for (int g = 0; g < GH; ++g) {
          float dot = 0.f;
#pragma unroll
          for (int i = 0; i < kPer; ++i) dot = fmaf(qv[g][i], kx[i], dot);
          sc[g][u] = dot;
        }
      }
      // sum over the 16 lanes of the half for all 4 rows at once: each
      // exchange halves the number of rows a lane carries
      const bool b3 = (j >> 3) & 1, b2 = (j >> 2) & 1;
      const int r_own = warp * 2 * kRowsPerHalf + 2 * u_own + half;
      const bool valid = r_own < rows;
      float sv[GH], mt[GH];
#pragma unroll
      for (int g = 0; g < GH; ++g) {
        float t0v = b3 ? sc[g][2] : sc[g][0], t1v = b3 ? sc[g][3] : sc[g][1];
        t0v += __shfl_xor_sync(0xffffffffu, b3 ? sc[g][0] : sc[g][2], 8);
        t1v += __shfl_xor_sync(0xffffffffu, b3 ? sc[g][1] : sc[g][3], 8);
        float v = b2 ? t1v : t0v;
        v += __shfl_xor_sync(0xffffffffu, b2 ? t0v : t1v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        sv[g] = valid ? v : -INFINITY;
        float x = fmaxf(sv[g], __shfl_xor_sync(0xffffffffu, sv[g], 4));
        mt[g] = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
      }
      // warp-uniform (the shuffles below span both halves); a half with no
      // valid row in this stage keeps its state: alpha = 1 (or 0 before its
      // first row), p = 0
      if (__any_sync(0xffffffffu, valid)) {
        float pr[GH];
#pragma unroll
        for (int g = 0; g < GH; ++g) {
          const float m_new = fmaxf(m[g], mt[g]);
          const float alpha = (m[g] == -INFINITY) ? 0.f : ex2_approx(m[g] - m_new);
          m[g] = m_new;
          pr[g] = valid ? ex2_approx(sv[g] - m[g]) : 0.f;
          float ps = pr[g] + __shfl_xor_sync(0xffffffffu, pr[g], 4);
          ps += __shfl_xor_sync(0xffffffffu, ps, 8);
          l[g] = l[g] * alpha + ps;
#pragma unroll
          for (int i = 0; i < kPer; ++i) acc[g][i] *= alpha;
        }
#pragma unroll
        for (int u = 0; u < kRowsPerHalf; ++u) {
          // row u's probability sits in lanes with (j>>3, j>>2) = (u>>1, u&1)
          const int src = half * 16 + 8 * (u >> 1) + 4 * (u & 1);
          float pu[GH];
#pragma unroll
          for (int g = 0; g < GH; ++g) pu[g] = __shfl_sync(0xffffffffu, pr[g], src);
          const int r = warp * 2 * kRowsPerHalf + 2 * u + half;
          if (r < rows) {
            float vx[kPer];
            load_row_part<kPer>(vtile + r * D * 2, j, vx);
#pragma unroll
            for (int g = 0; g < GH; ++g)
#pragma unroll
              for (int i = 0; i < kPer; ++i) acc[g][i] = fmaf(pu[g], vx[i], acc[g][i]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(EMPTY(s));
    }
    // every copy has landed and been read (or the CTA is aborting, and the
    // producer lets its copies land before the barrier below)
    __syncthreads();
    if (*abort_flag) return;
    // per half-warp and head state to shared memory (over the stage buffers)
#pragma unroll
    for (int g = 0; g < GH; ++g) {
      float* mw = merge + ((warp * 2 + half) * GH + g) * (D + 2);
      if (j == 0) {
        mw[0] = m[g];
        mw[1] = l[g];
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i) mw[2 + j * kPer + i] = acc[g][i];
    }
  }
  // the producer warp joins the consumers' first barrier here
  if (warp == kConsumerWarps) {
    __syncthreads();
    if (*abort_flag) return;
  }
  __syncthreads();
  // merge the 16 half-warp states (base-2 statistics) of each head into this
  // chunk's partial
  constexpr int kStates = 2 * kConsumerWarps;
  for (int e = threadIdx.x; e < GH * D; e += blockDim.x) {
    const int g = e / D, i = e % D;
    float mm = -INFINITY;
    for (int w = 0; w < kStates; ++w) mm = fmaxf(mm, merge[(w * GH + g) * (D + 2)]);
    float ll = 0.f, oo = 0.f;
    for (int w = 0; w < kStates; ++w) {
      const float* st = merge + (w * GH + g) * (D + 2);
      if (st[0] == -INFINITY) continue;
      const float f = ex2_approx(st[0] - mm);
      ll = fmaf(st[1], f, ll);
      oo = fmaf(st[2 + i], f, oo);
    }
    const size_t part = (bh0 + g) * p.C + c;
    p.part_o[part * D + i] = oo / ll;
    if (i == 0) p.part_lse[part] = mm + lg2_approx(ll);
  }
}

// One CTA per (head, sequence); thread i owns output element i. Chunks are
// combined in index order.
template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(const DecParams p) {
  grid_dependency_wait();  // the split kernel's partials
  const int h = blockIdx.x, b = blockIdx.y;
  const size_t bh = size_t(b) * p.H + h;
  const float* pl = p.part_lse + bh * p.C;
  const float* po = p.part_o + bh * p.C * D;
  float mx = -INFINITY;
  for (int c = 0; c < p.C; ++c) mx = fmaxf(mx, pl[c]);
  const int i = threadIdx.x;
  if (mx == -INFINITY) {  // no visible key at all
    p.o[bh * D + i] = 0;
    if (i == 0) p.lse[bh] = -INFINITY;
    return;
  }
  float wsum = 0.f, acc = 0.f;
  for (int c = 0; c < p.C; ++c) {
    const float lc = pl[c];
    if (lc == -INFINITY) continue;
    const float w = ex2_approx(lc - mx);
    wsum += w;
    acc = fmaf(w, po[size_t(c) * D + i], acc);
  }
  const float out = acc / wsum;
  // round to nearest even bf16
  const uint32_t u = __float_as_uint(out);
  p.o[bh * D + i] = uint16_t((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
  if (i == 0) p.lse[bh] = (mx + lg2_approx(wsum)) * kLn2;
}

template <int D>
fa_status launch_merge(const DecParams& p, int B, const LaunchCtx& ctx) {
  dim3 g2(p.H, B);
  {
    ProfileScope prof(KID_DECODE_MERGE, ctx.stream);
    cudaError_t e = launch_dependent(decode_merge_kernel<D>, g2, dim3(D), 0, ctx.stream, p);
    if (e != cudaSuccess) return cuda_fail(e, "decode merge kernel launch");
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode merge kernel launch");
  return FA_OK;
}

template <int D, bool PAGED, int GH>
fa_status launch(const DecParams& p, int B, const LaunchCtx& ctx) {
  const int smem = DecLayout<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, PAGED, GH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode)");
  dim3 g1(p.C, p.H / GH, B);
  {
    ProfileScope prof(KID_DECODE, ctx.stream);
    decode_split_kernel<D, PAGED, GH><<<g1, kThreads, smem, ctx.stream>>>(p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode split kernel launch");
  dim3 g2(p.H, B);
  {
    ProfileScope prof(KID_DECODE_MERGE, ctx.stream);
    e = launch_dependent(decode_merge_kernel<D>, g2, dim3(D), 0, ctx.stream, p);
    if (e != cudaSuccess) return cuda_fail(e, "decode merge kernel launch");
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode merge kernel launch");
  return FA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

int decode_num_chunks(int B, int H, int Lmax, int num_splits, int /*num_sms*/) {
  if (num_splits > 0) return num_splits;
  // enough CTAs for ~4 per SM, chunks of at most 2048 positions, but never
  // chunks shorter than 256 positions
  const long long bh = (long long)B * H;
  long long c = (4LL * kSmHint + bh - 1) / bh;
  const long long by_len = (Lmax + 2047) / 2048;
  if (c < by_len) c = by_len;
  const long long max_c = (Lmax + 255) / 256;
  if (c > max_c) c = max_c;
  if (c < 1) c = 1;
  if (c > 1024) c = 1024;
  return int(c);
}

size_t decode_workspace_bytes(int B, int H, int d, int chunks) {
  const size_t parts = size_t(B) * H * chunks;
  return align256(parts * d * 4) + align256(parts * 4);
}

fa_status launch_decode(const void* q, const void* kcache, const void* vcache, const int* seqlens,
                        void* o, float* lse, int B, int H, int Lmax, int d, float scale,
                        int chunks, void* workspace, const LaunchCtx& ctx, const char* caller) {
  if ((long long)B * H > 65535LL * 65535LL || H > 65535 || B > 65535) {
    set_last_error("%s: B and H must each be <= 65535", caller);
    return FA_ERR_UNSUPPORTED;
  }
  DecParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.kc = static_cast<const uint16_t*>(kcache);
  p.vc = static_cast<const uint16_t*>(vcache);
  p.seqlens = seqlens;
  p.table = nullptr;
  p.group = 1;
  p.Hkv = H;
  p.page = p.max_pages = p.num_pages = 0;
  const size_t parts = size_t(B) * H * chunks;
  p.part_o = static_cast<float*>(workspace);
  p.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(parts * d * 4));
  p.o = static_cast<uint16_t*>(o);
  p.lse = lse;
  p.H = H;
  p.Lmax = Lmax;
  p.C = chunks;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = ctx.status_word;
  p.limit_ns = ctx.wait_limit_ns;
  p.debug_skip = ctx.debug_skip_load == KID_DECODE;
  return d == 128 ? launch<128, false, 1>(p, B, ctx) : launch<64, false, 1>(p, B, ctx);
}

fa_status launch_decode_paged(const void* q, const void* kpages, const void* vpages,
                              const int* block_table, const int* seqlens, void* o, float* lse,
                              int B, int Hq, int Hkv, int num_pages, int page_size, int max_pages,
                              int d, float scale, int chunks, bool auto_split, void* workspace,
                              const LaunchCtx& ctx) {
  if (Hq > 65535 || B > 65535) {
    set_last_error("fa_decode_paged: B and Hq must each be <= 65535");
    return FA_ERR_UNSUPPORTED;
  }
  DecParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.kc = static_cast<const uint16_t*>(kpages);
  p.vc = static_cast<const uint16_t*>(vpages);
  p.seqlens = seqlens;
  p.table = block_table;
  p.group = Hq / Hkv;
  p.Hkv = Hkv;
  p.page = page_size;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  const size_t parts = size_t(B) * Hq * chunks;
  p.part_o = static_cast<float*>(workspace);
  p.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(parts * d * 4));
  p.o = static_cast<uint16_t*>(o);
  p.lse = lse;
  p.H = Hq;
  p.Lmax = max_pages * page_size;
  p.C = chunks;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = ctx.status_word;
  p.limit_ns = ctx.wait_limit_ns;
  p.debug_skip = ctx.debug_skip_load == KID_DECODE;
  if (p.group >= kTcMinGroup && p.group <= kTcMaxGroup) {
    // groups of 4 to 8 heads at d = 128: the keys as the M rows of the
    // tensor cores (decode_tct_sm100.cu); larger groups or d = 64: the query
    // heads as the M rows (decode_tc_sm100.cu); then the same merge
    // (its 128-key tiles must split into runs inside one page: pages of at
    // most 64 rows, or of a multiple of 128). With the automatic split the
    // keys-as-rows kernel balances whole tiles over persistent CTAs and
    // merges its own partials.
    const bool keys_as_rows = d == 128 && p.group <= kTctMaxGroup &&
                              (page_size <= 64 || page_size % 128 == 0);
    if (keys_as_rows && auto_split)
      return launch_decode_paged_tct(q, kpages, vpages, block_table, seqlens, B, Hq, Hkv,
                                     num_pages, page_size, max_pages, d, scale, 0, nullptr,
                                     nullptr, workspace, o, lse, ctx);
    fa_status st =
        keys_as_rows
            ? launch_decode_paged_tct(q, kpages, vpages, block_table, seqlens, B, Hq, Hkv,
                                      num_pages, page_size, max_pages, d, scale, chunks, p.part_o,
                                      p.part_lse, nullptr, nullptr, nullptr, ctx)
            : launch_decode_paged_tc(q, kpages, vpages, block_table, seqlens, B, Hq, Hkv,
                                     num_pages, page_size, max_pages, d, scale, chunks, p.part_o,
                                     p.part_lse, ctx);
    if (st != FA_OK) return st;
    return d == 128 ? launch_merge<128>(p, B, ctx) : launch_merge<64>(p, B, ctx);
  }
  // query heads per CTA: up to 4 of the heads that share a KV head
  const int gh = (p.group % 4 == 0) ? 4 : (p.group % 2 == 0) ? 2 : 1;
  if (d == 128)
    return gh == 4 ? launch<128, true, 4>(p, B, ctx)
                   : gh == 2 ? launch<128, true, 2>(p, B, ctx) : launch<128, true, 1>(p, B, ctx);
  return gh == 4 ? launch<64, true, 4>(p, B, ctx)
                 : gh == 2 ? launch<64, true, 2>(p, B, ctx) : launch<64, true, 1>(p, B, ctx);
}

}  // namespace fa

// ---------------------------------------------------------------------------
// Decode without any device allocation.
//
// fa_decode_splitkv needs a caller-provided workspace for the per-chunk
// partial results. Some callers cannot allocate device memory at the moment
// they decode: a serving loop whose allocator forbids cudaMalloc on its hot
// path (cudaMalloc can synchronise the device and stall every other
// stream), or a host framework that passes the library only its inputs and
// outputs and keeps no memory pool for it. For them the partials live in
// the fixed buffer below, which is part of the library image: every GPU
// that loads the library reserves kStaticScratchBytes of device memory for
// it until the process exits. Nothing here calls cudaMalloc, cudaFree or
// any allocating routine. The fa_debug_skip_load test hook does not apply
// to this entry point (a skip armed by it stays armed for the next call
// that honours it).
// ---------------------------------------------------------------------------
namespace fa {
namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB per device
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

constexpr int kMaxScratchDevices = 64;
void* g_scratch_ptr[kMaxScratchDevices] = {};  // device address per device
std::mutex g_scratch_mu;

}  // namespace
}  // namespace fa

extern "C" fa_status fa_decode_splitkv_static(const void* q, const void* kcache,
                                              const void* vcache, const int* seqlens, void* o,
                                              float* lse, int B, int H, int Lmax, int d,
                                              float scale, int num_splits, cudaStream_t stream) {
  using namespace fa;
  auto bad = [](fa_status st, const char* msg) {
    set_last_error("fa_decode_splitkv_static: %s", msg);
    return st;
  };
  const void* ptrs[5] = {q, kcache, vcache, o, lse};
  for (const void* ptr : ptrs) {
    if (ptr == nullptr) return bad(FA_ERR_INVALID_ARG, "null tensor pointer");
    if (reinterpret_cast<uintptr_t>(ptr) & 15u)
      return bad(FA_ERR_ALIGNMENT, "a tensor pointer is not 16-byte aligned");
  }
  if (seqlens == nullptr || (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return bad(FA_ERR_INVALID_ARG, "seqlens must be a non-null, 4-byte aligned int32 array");
  if (B < 1 || H < 1 || Lmax < 1 || (long long)B * H * Lmax > 0x7fffffffLL)
    return bad(FA_ERR_INVALID_ARG, "B, H, Lmax must be >= 1 with B*H*Lmax < 2^31");
  if (d != 64 && d != 128) return bad(FA_ERR_UNSUPPORTED, "head dim must be 64 or 128");
  if (!(scale > 0.f) || scale == INFINITY) return bad(FA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (num_splits < 0 || num_splits > 1024)
    return bad(FA_ERR_INVALID_ARG, "num_splits must be in [0, 1024]");
  const int chunks = decode_num_chunks(B, H, Lmax, num_splits, 0);
  const size_t need = decode_workspace_bytes(B, H, d, chunks);
  if (need > kStaticScratchBytes) {
    set_last_error(
        "fa_decode_splitkv_static: this shape needs %zu bytes of scratch, more than the %zu "
        "bytes built into the library; call fa_decode_splitkv with a workspace instead",
        need, kStaticScratchBytes);
    return FA_ERR_WORKSPACE;
  }
  LaunchCtx ctx;
  fa_status st = current_launch_ctx(stream, &ctx);
  if (st != FA_OK) return st;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxScratchDevices) return bad(FA_ERR_UNSUPPORTED, "device index too large");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
      // once per device, with that device current: the host-side name of the
      // array is only a stand-in, the kernel needs its device address
      void* addr = nullptr;
      e = cudaGetSymbolAddress(&addr, g_decode_scratch);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static decode scratch)");
      g_scratch_ptr[dev] = addr;
    }
    scratch = g_scratch_ptr[dev];
  }
  // every chunk writes its own partial (empty chunks write weight 0), so no
  // part of the scratch has to start at zero
  return launch_decode(q, kcache, vcache, seqlens, o, lse, B, H, Lmax, d, scale, chunks, scratch,
                       ctx, "fa_decode_splitkv_static");
}
