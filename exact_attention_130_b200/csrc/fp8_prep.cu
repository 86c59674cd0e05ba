// fp8_prep.cu -- incoherent processing and FP8 quantisation of Q, K and V
// for the FP8 forward (fwd_sm100.cu, F8 instantiation).
//
// What it computes ("FlashAttention-3 (TR)", section "FlashAttention-3'un
// Teknik Yenilikleri", item 3, and "Bellek Duvarinin Fizigi", section
// "FlashAttention-2, -3 ve -4: Utilizasyon Savasi"): Q and K are multiplied
// by the orthogonal matrix diag(sigma) H_d / sqrt(d) (random signs sigma,
// Sylvester Hadamard H_d), which spreads outlier coordinates over all
// coordinates and cancels in Q K^T, then quantised to e4m3 with one scale per
// 128-row block of each head; V is quantised as it is, with one scale per
// head. Here the unnormalised H_d is applied and Q's block scales carry the
// 1/d (a power of two, so the product is exact): dequantised Q^ K^T is
// Q K^T up to the FP8 rounding.
//
// Exact conventions (the codes are bit-for-bit reproducible):
//  * rotation in fp32: x * sign(sigma), then butterflies of stride 1, 2, 4,
//    ..., d/2 in that order, each pair (i, i + h) (bit h of i clear)
//    becoming (x_i + x_{i+h}, x_i - x_{i+h});
//  * block scale s = fp32(max |x|) / 448 (IEEE division; 1 for an all-zero
//    block), code = e4m3(x / s) rounded to nearest even, saturating at 448;
//  * V: v_amax[bh] = max |v| over the head (bits of a non-negative float, so
//    an integer atomicMax orders them); its scale v_amax / 448 is
//    recomputed by the forward the same way.
//
// Layout: one CTA per (128-row block, head, tensor); warp w holds rows
// 16 w .. 16 w + 15 of the block, lane l columns 4 l .. 4 l + 3 (d = 128),
// so a row's butterflies of stride >= 4 are warp shuffles. The transposed V
// ([B, H, d, n_vt] codes, n_vt = N rounded up to 16, zero codes past N) goes
// through a shared-memory tile so that both the loads and the stores are
// coalesced (see fp8_prep_vt_kernel for the lane mapping).
#include <cstdint>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kPrepD = 128;
constexpr int kPrepRows = 128;  // rows per quantisation block
constexpr int kPrepThreads = 256;
constexpr int kRowsPerWarp = kPrepRows / (kPrepThreads / 32);
constexpr float kE4m3Max = 448.0f;

// (x * sign(sigma)) H_128 of one row held by a warp (4 columns per lane).
// Every lane of the warp must call it (shuffles).
__device__ __forceinline__ void rotate_row(float (&x)[4], const bool (&neg)[4], int lane) {
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] = neg[e] ? -x[e] : x[e];
  float a, b;
  // stride 1: pairs (0, 1) and (2, 3) of the lane
  a = x[0], b = x[1], x[0] = a + b, x[1] = a - b;
  a = x[2], b = x[3], x[2] = a + b, x[3] = a - b;
  // stride 2: pairs (0, 2) and (1, 3)
  a = x[0], b = x[2], x[0] = a + b, x[2] = a - b;
  a = x[1], b = x[3], x[1] = a + b, x[3] = a - b;
  // strides 4 .. 64: the partner lane is lane ^ (stride / 4)
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool lower = (lane & m) == 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float o = __shfl_xor_sync(0xffffffffu, x[e], m);
      x[e] = lower ? x[e] + o : o - x[e];
    }
  }
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < kPrepThreads / 32; ++w) r = fmaxf(r, red[w]);
  return r;
}

__device__ __forceinline__ uint32_t codes4(const float (&x)[4], float s) {
  return pack_e4m3x2(__fdiv_rn(x[0], s), __fdiv_rn(x[1], s)) |
         (pack_e4m3x2(__fdiv_rn(x[2], s), __fdiv_rn(x[3], s)) << 16);
}

// blockIdx = (128-row block, head, tensor: 0 Q, 1 K, 2 V). Q and K: rotate
// (when signs is given), block scale, codes. V: only the head's amax.
__global__ void __launch_bounds__(kPrepThreads)
    fp8_prep_qkv_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                        const uint16_t* __restrict__ v, const float* __restrict__ signs, int N,
                        int n_blk, uint8_t* __restrict__ q8, uint8_t* __restrict__ k8,
                        float* __restrict__ q_scale, float* __restrict__ k_scale,
                        unsigned int* __restrict__ v_amax_bits) {
  __shared__ float red[kPrepThreads / 32];
  const int blk = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint16_t* src = which == 0 ? q : which == 1 ? k : v;
  const size_t head_row0 = size_t(bh) * N;
  const bool rot = which < 2 && signs != nullptr;
  bool neg[4] = {false, false, false, false};
  if (rot) {
#pragma unroll
    for (int e = 0; e < 4; ++e) neg[e] = signbit(signs[lane * 4 + e]);
  }
  // all of the warp's row loads first (16 in flight per thread), then the
  // rotations: loading and rotating row by row left the kernel waiting on
  // one load at a time
  uint2 raw[kRowsPerWarp];
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int row = blk * kPrepRows + warp * kRowsPerWarp + i;  // the same for the whole warp
    raw[i] = make_uint2(0u, 0u);
    if (row < N)
      raw[i] = *reinterpret_cast<const uint2*>(src + (head_row0 + row) * kPrepD + lane * 4);
  }
  float x[kRowsPerWarp][4];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    x[i][0] = __uint_as_float(raw[i].x << 16);
    x[i][1] = __uint_as_float(raw[i].x & 0xffff0000u);
    x[i][2] = __uint_as_float(raw[i].y << 16);
    x[i][3] = __uint_as_float(raw[i].y & 0xffff0000u);
    // (rows past N are zero and stay zero under the rotation)
    if (rot) rotate_row(x[i], neg, lane);
#pragma unroll
    for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(x[i][e]));
  }
  amax = block_max(amax, red);
  if (which == 2) {
    if (threadIdx.x == 0) atomicMax(v_amax_bits + bh, __float_as_uint(amax));
    return;
  }
  const float s = amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.0f;
  uint8_t* dst = which == 0 ? q8 : k8;
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int row = blk * kPrepRows + warp * kRowsPerWarp + i;
    if (row < N)
      *reinterpret_cast<uint32_t*>(dst + (head_row0 + row) * kPrepD + lane * 4) = codes4(x[i], s);
  }
  if (threadIdx.x == 0) {
    float* out = which == 0 ? q_scale : k_scale;
    out[size_t(bh) * n_blk + blk] = (which == 0 && rot) ? s * (1.0f / kPrepD) : s;
  }
}

// blockIdx = (128-key block, head): V codes with the head's scale, written
// transposed ([d, n_vt] per head). Lane l of a warp takes the dims l, l + 32,
// l + 64, l + 96 of four consecutive keys (each load of the warp reads 64
// contiguous bytes of one key row), packs the four keys' codes of a dim into
// one word and stores it into a shared-memory tile of dim rows whose pitch is
// an odd number of words, so the 32 lanes' stores hit 32 different banks;
// the tile then leaves in 16-byte global stores along the keys.
__global__ void __launch_bounds__(kPrepThreads)
    fp8_prep_vt_kernel(const uint16_t* __restrict__ v, int N, int n_vt,
                       const float* __restrict__ v_amax, uint8_t* __restrict__ vt8) {
  constexpr int kPitchW = kPrepRows / 4 + 1;  // words per transposed row (odd)
  __shared__ uint32_t t[kPrepD * kPitchW];
  const int blk = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float va = v_amax[bh];
  const float s = va > 0.f ? __fdiv_rn(va, kE4m3Max) : 1.0f;
  constexpr int kWarps = kPrepThreads / 32;
#pragma unroll 1
  for (int k4 = warp; k4 < kPrepRows / 4; k4 += kWarps) {  // a group of four keys
    uint16_t raw[4][4];  // [key][dim group]
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int row = blk * kPrepRows + k4 * 4 + kk;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        raw[kk][e] = row < N ? v[(size_t(bh) * N + row) * kPrepD + e * 32 + lane] : uint16_t(0);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uint32_t w = 0;
#pragma unroll
      for (int kk = 0; kk < 4; kk += 2) {
        const float a = __uint_as_float(uint32_t(raw[kk][e]) << 16);
        const float b = __uint_as_float(uint32_t(raw[kk + 1][e]) << 16);
        w |= pack_e4m3x2(__fdiv_rn(a, s), __fdiv_rn(b, s)) << (8 * kk);
      }
      t[(e * 32 + lane) * kPitchW + k4] = w;
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < kPrepD * (kPrepRows / 16); idx += kPrepThreads) {
    const int dcol = idx / (kPrepRows / 16), chunk = idx % (kPrepRows / 16);
    const int key0 = blk * kPrepRows + chunk * 16;
    if (key0 < n_vt) {
      const uint32_t* src = t + dcol * kPitchW + chunk * 4;
      *reinterpret_cast<uint4*>(vt8 + (size_t(bh) * kPrepD + dcol) * n_vt + key0) =
          make_uint4(src[0], src[1], src[2], src[3]);
    }
  }
}

}  // namespace

fa_status launch_fp8_prepare(const void* q, const void* k, const void* v, const float* signs,
                             int B, int H, int N, int d, void* q8, void* k8, void* vt8,
                             float* q_scale, float* k_scale, float* v_amax,
                             const LaunchCtx& ctx) {
  if (d != kPrepD) {
    set_last_error("the FP8 preparation needs d = 128 (got %d)", d);
    return FA_ERR_UNSUPPORTED;
  }
  const int BH = B * H;  // <= 65535, checked by the caller
  const int n_blk = (N + kPrepRows - 1) / kPrepRows;
  cudaError_t e = cudaMemsetAsync(v_amax, 0, size_t(BH) * sizeof(float), ctx.stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(v_amax)");
  {
    ProfileScope prof(KID_FP8_PREP, ctx.stream);
    fp8_prep_qkv_kernel<<<dim3(n_blk, BH, 3), kPrepThreads, 0, ctx.stream>>>(
        static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
        static_cast<const uint16_t*>(v), signs, N, n_blk, static_cast<uint8_t*>(q8),
        static_cast<uint8_t*>(k8), q_scale, k_scale, reinterpret_cast<unsigned int*>(v_amax));
    fp8_prep_vt_kernel<<<dim3(n_blk, BH), kPrepThreads, 0, ctx.stream>>>(
        static_cast<const uint16_t*>(v), N, fp8_vt_keys(N), v_amax, static_cast<uint8_t*>(vt8));
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fp8 preparation launch");
  return FA_OK;
}

}  // namespace fa
