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
//    chunk's K and V rows into a 4-stage shared-memory ring with plain bulk
//    copies (cp.async.bulk: the rows of one chunk are contiguous), keeping up
//    to 64 KB per CTA and ~190 KB per SM in flight;
//  * four consumer warps take every fourth token of a stage; a lane owns
//    d/32 consecutive elements of q and of its output accumulator, so a
//    warp reads one cached row as one contiguous 256-byte line;
//  * scores of a warp's 8 tokens are formed together and the running
//    maximum is updated once per 8 tokens, so the exponentials cost about one
//    per token;
//  * positions at or past seqlens[b] are never read;
//  * all waits are bounded in time (see sm100_ptx.cuh).
#include <mutex>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kTileT = 32;        // cache rows per pipeline stage
constexpr int kStages = 4;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kTokPerWarp = kTileT / kConsumerWarps;  // 8
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kSmHint = 148;      // B200 SM count, for the automatic split

template <int D>
struct DecLayout {
  static constexpr int kTileBytes = kTileT * D * 2;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kStages * kTileBytes;
  static constexpr int kOffBar = 2 * kStages * kTileBytes;       // full[s], empty[s]
  static constexpr int kOffMisc = kOffBar + 8 * 2 * kStages;     // abort flag
  static constexpr int kOffMerge = kOffMisc + 16;                // per-warp m, l, acc[D]
  static constexpr int kSmemBytes = kOffMerge + kConsumerWarps * (D + 2) * 4 + 128;
};

struct DecParams {
  const uint16_t* q;
  const uint16_t* kc;
  const uint16_t* vc;
  const int* seqlens;
  float* part_o;    // [B, H, C, D]
  float* part_lse;  // [B, H, C], base 2
  uint16_t* o;
  float* lse;
  int H, Lmax, C;
  float scale_log2;
  unsigned int* status;
  unsigned long long limit_ns;
};

__device__ __forceinline__ float bf16_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

template <int D>
__global__ void __launch_bounds__(kThreads)
    decode_split_kernel(const DecParams p) {
  using L = DecLayout<D>;
  constexpr int kPer = D / 32;  // elements per lane
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc);
  float* merge = reinterpret_cast<float*>(smem + L::kOffMerge);
  auto FULL = [&](int s) -> uint32_t { return sbase + L::kOffBar + 8u * s; };
  auto EMPTY = [&](int s) -> uint32_t { return sbase + L::kOffBar + 8u * (kStages + s); };

  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t bh = size_t(b) * p.H + h;
  const size_t part = bh * p.C + c;

  int Lb = p.seqlens[b];
  Lb = Lb < 0 ? 0 : (Lb > p.Lmax ? p.Lmax : Lb);
  const int chunk = (Lb + p.C - 1) / p.C;
  const int t0 = c * chunk;
  const int t1 = min(t0 + chunk, Lb);
  if (t0 >= t1) {  // empty chunk: weight 0 in the merge
    for (int i = threadIdx.x; i < D; i += blockDim.x) p.part_o[part * D + i] = 0.f;
    if (threadIdx.x == 0) p.part_lse[part] = -INFINITY;
    return;
  }
  const int n_tok = t1 - t0;
  const int n_tiles = (n_tok + kTileT - 1) / kTileT;

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
      const uint16_t* kb = p.kc + (bh * p.Lmax + t0) * D;
      const uint16_t* vb = p.vc + (bh * p.Lmax + t0) * D;
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % kStages;
        if (!wait_bounded(EMPTY(s), ((i / kStages) & 1) ^ 1, wc, 1)) break;
        const int rows = min(kTileT, n_tok - i * kTileT);
        const uint32_t bytes = uint32_t(rows) * D * 2;
        mbar_arrive_expect_tx(FULL(s), 2 * bytes);
        bulk_load(sbase + L::kOffK + s * L::kTileBytes, kb + size_t(i) * kTileT * D, bytes, FULL(s));
        bulk_load(sbase + L::kOffV + s * L::kTileBytes, vb + size_t(i) * kTileT * D, bytes, FULL(s));
        ++issued;
      }
      if (*abort_flag)
        for (int s = 0; s < kStages; ++s) {
          const int cnt = (issued - s + kStages - 1) / kStages;  // loads into stage s
          if (cnt > 0) wait_bounded(FULL(s), (cnt - 1) & 1, wc, 2, true);
        }
    }
  } else {
    // ---------------------------------------------------------------- consumers
    float qv[kPer];
    {
      const uint16_t* qp = p.q + bh * D + lane * kPer;
#pragma unroll
      for (int i = 0; i < kPer; ++i) qv[i] = bf16_to_f32(qp[i]) * p.scale_log2;
    }
    float m = -INFINITY, l = 0.f, acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.f;

    for (int it = 0; it < n_tiles; ++it) {
      const int s = it % kStages;
      bool ok = wait_bounded(FULL(s), (it / kStages) & 1, wc, 3);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const int rows = min(kTileT, n_tok - it * kTileT);
      const uint8_t* ktile = smem + L::kOffK + s * L::kTileBytes;
      const uint8_t* vtile = smem + L::kOffV + s * L::kTileBytes;
      float sc[kTokPerWarp];
      float mx = -INFINITY;
#pragma unroll
      for (int u = 0; u < kTokPerWarp; ++u) {
        const int tt = warp + u * kConsumerWarps;
        float dot = 0.f;
        if (tt < rows) {
          const uint16_t* kr = reinterpret_cast<const uint16_t*>(ktile + tt * D * 2) + lane * kPer;
          if constexpr (kPer == 4) {
            const uint2 w = *reinterpret_cast<const uint2*>(kr);
            dot = fmaf(qv[0], bf16_to_f32(w.x & 0xffffu), dot);
            dot = fmaf(qv[1], bf16_to_f32(w.x >> 16), dot);
            dot = fmaf(qv[2], bf16_to_f32(w.y & 0xffffu), dot);
            dot = fmaf(qv[3], bf16_to_f32(w.y >> 16), dot);
          } else {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(kr);
            dot = fmaf(qv[0], bf16_to_f32(w & 0xffffu), dot);
            dot = fmaf(qv[1], bf16_to_f32(w >> 16), dot);
          }
        }
        sc[u] = dot;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
        for (int u = 0; u < kTokPerWarp; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], off);
      }
#pragma unroll
      for (int u = 0; u < kTokPerWarp; ++u) {
        const int tt = warp + u * kConsumerWarps;
        if (tt >= rows) sc[u] = -INFINITY;
        mx = fmaxf(mx, sc[u]);
      }
      if (mx != -INFINITY) {
        const float m_new = fmaxf(m, mx);
        const float alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - m_new);
        m = m_new;
        float rs = 0.f;
#pragma unroll
        for (int i = 0; i < kPer; ++i) acc[i] *= alpha;
#pragma unroll
        for (int u = 0; u < kTokPerWarp; ++u) {
          const int tt = warp + u * kConsumerWarps;
          if (tt < rows) {
            const float pr = ex2_approx(sc[u] - m);
            rs += pr;
            const uint16_t* vr =
                reinterpret_cast<const uint16_t*>(vtile + tt * D * 2) + lane * kPer;
            if constexpr (kPer == 4) {
              const uint2 w = *reinterpret_cast<const uint2*>(vr);
              acc[0] = fmaf(pr, bf16_to_f32(w.x & 0xffffu), acc[0]);
              acc[1] = fmaf(pr, bf16_to_f32(w.x >> 16), acc[1]);
              acc[2] = fmaf(pr, bf16_to_f32(w.y & 0xffffu), acc[2]);
              acc[3] = fmaf(pr, bf16_to_f32(w.y >> 16), acc[3]);
            } else {
              const uint32_t w = *reinterpret_cast<const uint32_t*>(vr);
              acc[0] = fmaf(pr, bf16_to_f32(w & 0xffffu), acc[0]);
              acc[1] = fmaf(pr, bf16_to_f32(w >> 16), acc[1]);
            }
          }
        }
        l = l * alpha + rs;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(EMPTY(s));
    }
    // per-warp state to shared memory for the merge
    float* mw = merge + warp * (D + 2);
    if (lane == 0) {
      mw[0] = m;
      mw[1] = l;
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) mw[2 + lane * kPer + i] = acc[i];
  }
  __syncthreads();
  if (*abort_flag) return;
  // merge the consumer warps (base-2 statistics) into this chunk's partial
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    float mm = -INFINITY;
    for (int w = 0; w < kConsumerWarps; ++w) mm = fmaxf(mm, merge[w * (D + 2)]);
    float ll = 0.f, oo = 0.f;
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float mw = merge[w * (D + 2)];
      if (mw == -INFINITY) continue;
      const float f = ex2_approx(mw - mm);
      ll = fmaf(merge[w * (D + 2) + 1], f, ll);
      oo = fmaf(merge[w * (D + 2) + 2 + i], f, oo);
    }
    p.part_o[part * D + i] = oo / ll;
    if (i == 0) p.part_lse[part] = mm + lg2_approx(ll);
  }
}

// One CTA per (head, sequence); thread i owns output element i. Chunks are
// combined in index order.
template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(const DecParams p) {
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
fa_status launch(const DecParams& p, int B, const LaunchCtx& ctx) {
  const int smem = DecLayout<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode)");
  dim3 g1(p.C, p.H, B);
  {
    ProfileScope prof(KID_DECODE, ctx.stream);
    decode_split_kernel<D><<<g1, kThreads, smem, ctx.stream>>>(p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode split kernel launch");
  dim3 g2(p.H, B);
  {
    ProfileScope prof(KID_DECODE_MERGE, ctx.stream);
    decode_merge_kernel<D><<<g2, D, 0, ctx.stream>>>(p);
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
                        int chunks, void* workspace, const LaunchCtx& ctx) {
  if ((long long)B * H > 65535LL * 65535LL || H > 65535 || B > 65535) {
    set_last_error("fa_decode_splitkv: B and H must each be <= 65535");
    return FA_ERR_UNSUPPORTED;
  }
  DecParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.kc = static_cast<const uint16_t*>(kcache);
  p.vc = static_cast<const uint16_t*>(vcache);
  p.seqlens = seqlens;
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
  return d == 128 ? launch<128>(p, B, ctx) : launch<64>(p, B, ctx);
}

}  // namespace fa

// ---------------------------------------------------------------------------
// Decode without any device allocation.
//
// fa_decode_splitkv needs a caller-provided workspace for the per-chunk
// partial results. Some callers cannot allocate device memory at the moment
// they decode: code running inside a stream capture, code driven by an
// allocator that forbids cudaMalloc on the hot path, or a host that owns no
// memory pool of its own. For them the partials live in the fixed buffer
// below, which is part of the library image: every GPU that loads the
// library reserves kStaticScratchBytes of device memory for it until the
// process exits. Nothing here calls cudaMalloc, cudaFree or any allocating
// routine.
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
                       ctx);
}
