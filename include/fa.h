/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library libfa_sm100.so
 *
 * The library computes exact scaled dot-product attention
 *
 *     S = scale * Q K^T  (+ causal mask),  P = softmax_row(S),  O = P V
 *
 * without ever writing S or P to device memory: K/V tiles stream through
 * shared memory, S and the output accumulator live in tensor memory, and the
 * row softmax is carried by the running maximum / running sum recurrence.
 * Definitions followed:
 *   - "FlashAttention'i Anlamak Bolum 1" (blog.edumints.com), 0.2 Notasyon:
 *     the function S = QK^T/sqrt(d) + B, P = softmax_row(S), O = PV.
 *   - "Bellek Duvarinin Fizigi" (webturing Principia): "Online Softmax" and
 *     "Forward gecisin iskeleti" (tiling, running max/sum, final division),
 *     "Maskeleme ve Dropout" (causal mask with skipped tiles),
 *     "Geri Yayilim" (backward by recomputing P from the saved log-sum-exp),
 *     "Decode Asamasi: Flash-Decoding" (split-KV decode merged by LSE).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Layout: row-major [B, H, N, d], contiguous (head dim fastest). The
 *    per-row log-sum-exp is fp32 [B, H, N]. bf16 tensors are passed as
 *    void* holding IEEE bfloat16.
 *  - LSE_i = ln sum_j exp(S_ij), natural logarithm, scale already inside S.
 *  - Causal: query i sees key j iff j <= i (N_q = N_k = N).
 *  - Ownership: every pointer is caller-owned DEVICE memory; the library
 *    never frees or retains it past the call. The library allocates no
 *    device memory per call (it keeps one 4-byte device status word per
 *    device, a __device__ variable of the library).
 *  - Alignment: every tensor pointer must be 16-byte aligned (TMA needs
 *    16-byte global addresses), else FA_ERR_ALIGNMENT.
 *  - Execution: all device work is enqueued on `stream` (0 = legacy default
 *    stream) and the call returns without synchronising. Argument errors are
 *    returned before anything is launched and leave outputs untouched.
 *  - Errors: FA_ERR_CUDA carries the CUDA error text (fa_last_error()).
 *    A kernel wait that exceeds its time limit does not hang the GPU: the
 *    kernel records it in the device status word and returns; the host sees
 *    it as FA_ERR_TIMEOUT from fa_device_status().
 *  - The library never aborts or exits the process.
 */
#ifndef FA_SM100_H
#define FA_SM100_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, non-finite scale   */
    FA_ERR_UNSUPPORTED = 2,   /* head dim or device not supported           */
    FA_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned           */
    FA_ERR_WORKSPACE = 4,     /* workspace missing or smaller than needed   */
    FA_ERR_CUDA = 5,          /* a CUDA runtime/driver call failed          */
    FA_ERR_TIMEOUT = 6        /* a device-side wait gave up (see above)     */
} fa_status;

/* Static, human-readable name of a status code. */
const char* fa_status_string(fa_status s);

/* Text of the last FA_ERR_CUDA / validation failure on the calling thread. */
const char* fa_last_error(void);

/* Version of this ABI (major * 100 + minor). */
int fa_abi_version(void);

/*
 * fa_fwd -- attention forward, bf16 in / bf16 out, fp32 accumulation.
 *   q, k, v : bf16 [B, H, N, d]          (input, device)
 *   o       : bf16 [B, H, N, d]          (output, device)
 *   lse     : fp32 [B, H, N]             (output, device; natural log)
 *   B, H, N : >= 1;  B*H*N <= 2^31 - 1
 *   d       : 64 or 128 (else FA_ERR_UNSUPPORTED)
 *   scale   : finite, usually 1/sqrt(d)
 *   causal  : 0 or 1
 * Passages: "Forward gecisin iskeleti" (tiles of Q, K, V; running m, l and
 * O~; O = diag(l)^-1 O~ at the end), "Online Softmax" (exp2 form with the
 * scores pre-scaled by log2 e), "Maskeleme ve Dropout" (tiles above the
 * diagonal skipped, the diagonal tile masked before the row maximum).
 * Allocates nothing: O and LSE are written once each, straight from the
 * kernel (one 128-row query tile per work unit).
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o,
                 float* lse, int B, int H, int N, int d, float scale,
                 int causal, cudaStream_t stream);

/*
 * fa_fwd_pair -- fa_fwd computed on pairs of CTAs that share each tensor-core
 * product ("FlashAttention-2, -3 ve -4: Utilizasyon Savasi", the Blackwell
 * paragraph: the 2-CTA MMA mode of tcgen05). Same arguments, layouts,
 * results (within the same tolerances) and error behaviour as fa_fwd, for
 * d = 128 only (else FA_ERR_UNSUPPORTED). A cluster of two CTAs takes 256
 * query rows of one head; one CTA issues M = 256 MMAs whose K and V
 * operands are split between the two CTAs' shared memory, so each SM loads
 * half of every K/V tile. Allocates nothing; the work units are dealt in a
 * fixed order, so results are bitwise repeatable.
 */
fa_status fa_fwd_pair(const void* q, const void* k, const void* v, void* o,
                      float* lse, int B, int H, int N, int d, float scale,
                      int causal, cudaStream_t stream);

/*
 * fa_fwd_f32 -- the same forward on fp32 tensors, computed in fp32.
 *   q, k, v, o : fp32 [B, H, N, d];  lse : fp32 [B, H, N]
 *   d : 64 or 128; N <= 4096 (a small-problem path: fp32 inputs are not
 *   rounded to a tensor-core type, so this path runs on the CUDA cores).
 * Passages as for fa_fwd.
 */
fa_status fa_fwd_f32(const float* q, const float* k, const float* v, float* o,
                     float* lse, int B, int H, int N, int d, float scale,
                     int causal, cudaStream_t stream);

/*
 * fa_fwd_tf32 -- the forward of fa_fwd_f32 (fp32 tensors in and out, same
 * arguments and errors) with both products on the tensor cores in TF32
 * (tcgen05 .kind::tf32: a 10-bit mantissa, fp32 accumulation). Q, K, V and
 * P are rounded to TF32 to nearest before the products (the tensor cores
 * would otherwise truncate, which biases every product toward zero). The
 * price is precision: errors of ~1e-4 to 1e-3 in O and LSE on N(0,1)
 * inputs, inside the 1e-2 / 1e-3 bars of the bf16 forward but far from
 * fa_fwd_f32's ~1e-6; the gain is speed (one 128-row tile per CTA, 64-key
 * tiles, no pipelining: about 15% on a 128-row head, 2x at N = 1000).
 * Passages as for fa_fwd.
 */
fa_status fa_fwd_tf32(const float* q, const float* k, const float* v, float* o,
                      float* lse, int B, int H, int N, int d, float scale,
                      int causal, cudaStream_t stream);

/*
 * fa_fwd_ex / fa_bwd_ex -- fa_fwd / fa_bwd with the two options of the
 * attention definition and of dropout ("FlashAttention'i Anlamak Bolum 1",
 * 0.2: S = Q K^T / sqrt(d) + B, B an optional mask or bias; "Bellek
 * Duvarinin Fizigi", "Maskeleme ve Dropout": dropout on P from a
 * counter-based generator driven by a seed and an offset, the backward
 * regenerating the same mask).
 *   bias    : bf16, element (b, h, i, j) at bias[b*bias_stride_b +
 *             h*bias_stride_h + i*N + j] (rows of N keys contiguous; a
 *             stride of 0 broadcasts), or NULL. 16-byte aligned. Added to
 *             the scaled scores before the causal mask and the row maximum;
 *             an input only (fa_bwd_ex returns no gradient for it); -inf
 *             entries mask (every row needs one finite score).
 *   p_drop  : dropout probability in [0, 1); 0 = no dropout.
 *   seed, offset : the generator's key and sequence offset. Pair (i, j) of
 *             head (b, h) takes byte (j % 16) % 4 of word (j % 16) / 4 of
 *             Philox4x32-10(counter = (j / 16, i, b*H + h, offset),
 *             key = (seed mod 2^32, seed >> 32)); it is kept iff that byte
 *             < t = round(256 (1 - p_drop)) (ties to even, 1 <= t <= 256),
 *             and a kept P is scaled by 256 / t.
 * O = (P * keep * 256/t) V; the LSE is that of the undropped P. fa_bwd_ex
 * must get the same bias, p_drop, seed and offset as the forward that made
 * o and lse. Other arguments, workspace and errors as for fa_fwd / fa_bwd.
 */
/* The keep threshold t that fa_fwd_ex / fa_bwd_ex use for p_drop
 * (round(256 (1 - p_drop)), ties to even, clamped to [1, 256]), or -1 for a
 * p_drop outside [0, 1). */
int fa_dropout_keep_threshold(float p_drop);

fa_status fa_fwd_ex(const void* q, const void* k, const void* v, void* o,
                    float* lse, int B, int H, int N, int d, float scale,
                    int causal, const void* bias, long long bias_stride_b,
                    long long bias_stride_h, float p_drop,
                    unsigned long long seed, unsigned int offset,
                    cudaStream_t stream);
fa_status fa_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                    const float* lse, const void* dO, void* dq, void* dk,
                    void* dv, int B, int H, int N, int d, float scale,
                    int causal, const void* bias, long long bias_stride_b,
                    long long bias_stride_h, float p_drop,
                    unsigned long long seed, unsigned int offset,
                    void* workspace, size_t workspace_bytes,
                    cudaStream_t stream);

/*
 * FP8 forward with incoherent processing ("FlashAttention-3 (TR)", section
 * "FlashAttention-3'un Teknik Yenilikleri", item 3: Q and K multiplied by a
 * random orthogonal matrix before FP8 quantisation, which spreads outliers
 * and cancels in Q K^T; "Bellek Duvarinin Fizigi", section
 * "FlashAttention-2, -3 ve -4: Utilizasyon Savasi": block-wise scaling and
 * random signs). Two calls: fa_fp8_prepare makes the e4m3 operands once,
 * fa_fwd_fp8 runs attention on them. d = 128 only (else FA_ERR_UNSUPPORTED).
 *
 * fa_fp8_vt_keys -- keys per row of the transposed V codes: N rounded up
 * to a multiple of 16 (0 for N < 1).
 */
int fa_fp8_vt_keys(int N);

/*
 * fa_fp8_prepare -- rotation and e4m3 quantisation.
 *   q, k, v  : bf16 [B, H, N, 128]          (input, device)
 *   signs    : fp32 [128] or NULL            (input, device; only the sign
 *              of each entry is used; NULL = no rotation)
 *   q8, k8   : e4m3 codes [B, H, N, 128]     (output, device, uint8)
 *   vt8      : e4m3 codes [B, H, 128, fa_fp8_vt_keys(N)] (output; V
 *              transposed, zero codes past N)
 *   q_scale, k_scale : fp32 [B, H, ceil(N/128)] (output) one scale per
 *              128-row block; q_scale includes the rotation's 1/128
 *   v_amax   : fp32 [B, H] (output) max |v| of each head; V's scale is
 *              v_amax / 448 (1 when v_amax is 0)
 *   B*H <= 65535. Rotation: x * sign(signs) times the unnormalised
 *   Sylvester Hadamard matrix, as fp32 butterflies of stride 1, 2, ..., 64
 *   (pair (i, i+h) -> (x_i + x_{i+h}, x_i - x_{i+h})). Block scale
 *   s = max|x| / 448 (fp32 division; 1 for a zero block); code =
 *   e4m3(x / s), nearest even, saturating. The codes are reproducible bit
 *   for bit. Pointers 16-byte aligned except signs (4). Allocates nothing.
 */
fa_status fa_fp8_prepare(const void* q, const void* k, const void* v,
                         const float* signs, int B, int H, int N, int d,
                         void* q8, void* k8, void* vt8, float* q_scale,
                         float* k_scale, float* v_amax, cudaStream_t stream);

/*
 * fa_fwd_fp8 -- attention forward on fa_fp8_prepare's operands.
 *   q8, k8, vt8, q_scale, k_scale, v_amax : as written by fa_fp8_prepare
 *   o   : bf16 [B, H, N, 128] (output)   lse : fp32 [B, H, N] (output)
 *   scale, causal : as for fa_fwd (scale applies to the original Q K^T)
 * Both products run on the tensor cores in e4m3 with fp32 accumulation;
 * P~ is rounded to e4m3 before P V, the row sums stay fp32. Result: the
 * attention of the dequantised operands, up to that rounding of P~.
 */
fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* vt8,
                     const float* q_scale, const float* k_scale,
                     const float* v_amax, void* o, float* lse, int B, int H,
                     int N, int d, float scale, int causal,
                     cudaStream_t stream);

/*
 * fa_bwd_workspace_size -- bytes of scratch fa_bwd needs: two fp32 vectors
 * [B, H, Np] (the saved LSE in base 2, and D = rowsum(dO * O), in the forms
 * the kernels add) and two bf16 arrays [B, H, Np, 16] (-L/scale and -D, each
 * split into three bf16 terms, which the tensor cores add to S and dP), Np =
 * N rounded up to a multiple of 128, each part starting on a 256-byte
 * boundary. Returns 0 for invalid sizes.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * fa_bwd -- attention backward by recomputation.
 *   q, k, v, o, dO : bf16 [B, H, N, d]   (input; o is fa_fwd's output)
 *   lse            : fp32 [B, H, N]      (input; fa_fwd's output)
 *   dq, dk, dv     : bf16 [B, H, N, d]   (output)
 *   workspace      : device scratch of >= fa_bwd_workspace_size() bytes,
 *                    16-byte aligned; its contents on entry do not matter
 *                    and are overwritten.
 * Computes D = rowsum(dO * O), then recomputes P = exp(S - LSE) block by
 * block and forms dV = P^T dO, dP = dO V^T, dS = P * (dP - D),
 * dK = scale dS^T Q ("Geri Yayilim") in a key-tile-outer kernel and
 * dQ = scale dS K in a query-tile-outer kernel. d : 64 or 128.
 * Deterministic: bitwise identical results on every run.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o,
                 const float* lse, const void* dO, void* dq, void* dk,
                 void* dv, int B, int H, int N, int d, float scale,
                 int causal, void* workspace, size_t workspace_bytes,
                 cudaStream_t stream);

/*
 * fa_decode_workspace_size -- bytes of scratch fa_decode_splitkv and
 * fa_decode_paged need for per-chunk partial results: fp32 [B, H, C, d]
 * outputs and fp32 [B, H, C] log-sum-exps, C = the chunk count the call will
 * use (num_splits, or the automatic choice when num_splits == 0). With
 * num_splits == 0 the size also covers the paged decode's balanced split
 * (fa_decode_paged below): at most B H + 2368 partials of d + 1 floats and
 * 8 bytes per (sequence, KV head), whichever is larger.
 */
size_t fa_decode_workspace_size(int B, int H, int Lmax, int d, int num_splits);

/*
 * fa_decode_splitkv -- one query token per (sequence, head) against a KV
 * cache, split along the cache into C chunks whose partial (o_c, lse_c) are
 * merged by log-sum-exp ("Decode Asamasi: Flash-Decoding").
 *   q               : bf16 [B, H, d]
 *   kcache, vcache  : bf16 [B, H, Lmax, d]
 *   seqlens         : int32 [B] on the device; keys 0 .. seqlens[b]-1 are
 *                     visible; 1 <= seqlens[b] <= Lmax is the caller's
 *                     contract (values outside it are clamped to [0, Lmax]
 *                     and a sequence with no visible key gets O = 0 and
 *                     LSE = -inf)
 *   o               : bf16 [B, H, d];  lse : fp32 [B, H]
 *   num_splits      : chunks per sequence, 0 = automatic, <= 1024
 *   workspace       : >= fa_decode_workspace_size(B, H, Lmax, d, num_splits)
 * Cache positions at or past seqlens[b] are never read. d : 128 or 64.
 * Deterministic: chunks are merged in a fixed order.
 */
fa_status fa_decode_splitkv(const void* q, const void* kcache,
                            const void* vcache, const int* seqlens, void* o,
                            float* lse, int B, int H, int Lmax, int d,
                            float scale, int num_splits, void* workspace,
                            size_t workspace_bytes, cudaStream_t stream);

/*
 * fa_decode_paged -- the split-KV decode of fa_decode_splitkv over a paged
 * KV cache, with grouped query heads ("Bellek Duvarinin Fizigi", section
 * "Duvarin Otesi": the KV cache, and the paged / grouped-query layouts it
 * names as the inference-side IO methods; "Decode Asamasi: Flash-Decoding"
 * for the split and the log-sum-exp merge).
 *   q              : bf16 [B, Hq, d]                       (input, device)
 *   kpages, vpages : bf16 [num_pages, Hkv, page_size, d]   (input, device);
 *                    page p holds page_size consecutive cache positions of
 *                    every KV head
 *   block_table    : int32 [B, max_pages] (device): cache position t of
 *                    sequence b is row t % page_size of page
 *                    block_table[b * max_pages + t / page_size]; entries past
 *                    a sequence's last page are never read
 *   seqlens        : int32 [B] (device); keys 0 .. seqlens[b]-1 are visible
 *                    (clamped to [0, max_pages * page_size]; a sequence with
 *                    no key gets O = 0, LSE = -inf)
 *   o              : bf16 [B, Hq, d];  lse : fp32 [B, Hq]  (outputs, device)
 *   Hq, Hkv        : Hq a multiple of Hkv; query head h reads KV head
 *                    h / (Hq / Hkv) (Hkv = 1: multi-query; Hkv = Hq: one KV
 *                    head per query head). Groups of 4 to 128 query heads
 *                    per KV head run on the tensor cores (the group's heads
 *                    are the rows of the MMA), the others on the CUDA cores
 *                    (up to four heads of a group per CTA)
 *   page_size      : 16, 32 or a multiple of 64
 *   num_splits     : chunks per sequence, 0 = automatic, <= 1024. With 0,
 *                    groups of 4 to 8 query heads at d = 128 (and pages of
 *                    <= 64 rows or a multiple of 128) split the cache by
 *                    whole 128-key tiles instead: all tiles of all
 *                    (sequence, KV head) pairs are dealt out in equal
 *                    contiguous ranges to persistent CTAs (two per SM),
 *                    whatever the mix of lengths
 *   workspace      : >= fa_decode_workspace_size(B, Hq, max_pages *
 *                    page_size, d, num_splits) bytes (caller-owned, device)
 * Validation errors return before any launch. A block-table entry outside
 * [0, num_pages) is never dereferenced: the kernel leaves those rows unread
 * and records the fault in the device status word, and the next
 * fa_device_status returns FA_ERR_INVALID_ARG (the outputs of that call are
 * undefined). d : 128 or 64. Deterministic, like fa_decode_splitkv.
 */
fa_status fa_decode_paged(const void* q, const void* kpages, const void* vpages,
                          const int* block_table, const int* seqlens, void* o,
                          float* lse, int B, int Hq, int Hkv, int num_pages,
                          int page_size, int max_pages, int d, float scale,
                          int num_splits, void* workspace,
                          size_t workspace_bytes, cudaStream_t stream);

/*
 * fa_decode_splitkv_static -- fa_decode_splitkv for callers that cannot
 * allocate device memory when they decode: a serving loop whose allocator
 * forbids cudaMalloc on its hot path (cudaMalloc can synchronise the device
 * and stall every other stream), or a host framework that passes the
 * library only its inputs and outputs and keeps no memory pool for it.
 * No counterpart on the pages: it is the same computation,
 * with the per-chunk partials kept in an 8 MiB buffer that is part of the
 * library image instead of a caller workspace. Arguments as for
 * fa_decode_splitkv, minus the workspace.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *    Every GPU that loads the library holds the 8 MiB until the process
 *    exits.
 *  - The first call on each device looks up the buffer's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Shapes whose partials exceed 8 MiB (B * H * C * (d + 1) * 4 bytes, C the
 *    chunk count) are rejected with FA_ERR_WORKSPACE and a message saying so.
 *  - All calls share the one buffer, which keeps the last call's contents;
 *    nothing in it needs to start at zero. Calls that can overlap on the GPU
 *    (different streams without ordering between them) race on it and give
 *    wrong results: serialise them.
 *  - The test hook fa_debug_skip_load does not apply here; a skip armed by
 *    it stays armed for the next call that honours it.
 */
fa_status fa_decode_splitkv_static(const void* q, const void* kcache,
                                   const void* vcache, const int* seqlens,
                                   void* o, float* lse, int B, int H, int Lmax,
                                   int d, float scale, int num_splits,
                                   cudaStream_t stream);

/*
 * fa_device_status -- synchronises `stream`, reads and clears the current
 * device's status word. Returns FA_ERR_TIMEOUT if any kernel of this
 * library gave up a wait since the last check, FA_ERR_INVALID_ARG if a
 * kernel found an invalid value in device memory (a block-table entry of
 * fa_decode_paged outside the page pool), FA_ERR_CUDA if the
 * synchronisation itself failed, else FA_OK. *detail (may be NULL) gets the
 * raw word of the first such event: kernel id << 16 | site << 8 | kind,
 * kind 1 = a wait gave up, 2 = an invalid value.
 */
fa_status fa_device_status(cudaStream_t stream, unsigned int* detail);

/*
 * fa_set_wait_limit -- time limit of every device-side wait, in
 * nanoseconds, for launches made after the call (default 2e9, i.e. 2 s;
 * 0 restores the default). Process-wide.
 */
void fa_set_wait_limit(unsigned long long nanoseconds);

/*
 * fa_debug_skip_load -- test hook for the bounded waits. kernel_id names the
 * kernel (ids as in fa_profile_end) whose first CTA leaves out one load in
 * the next call: 1 the forward (a V tile), 4 the backward dK/dV kernel (a dO
 * block), 5 the backward dQ kernel (a V block), 6 the decode split kernel (its
 * first tile). The wait for that load runs out, the kernel records
 * FA_ERR_TIMEOUT in the device status word (fa_device_status) and returns
 * without a fault; its outputs are then undefined. The next call of fa_fwd,
 * fa_bwd or fa_decode_splitkv consumes the setting, whichever kernel it names;
 * 0 or a negative value clears it.
 */
void fa_debug_skip_load(int kernel_id);

/*
 * Per-kernel timing, off by default. Between fa_profile_begin() and
 * fa_profile_end() every kernel this library launches is bracketed by a pair
 * of CUDA events recorded on its launching stream. fa_profile_end()
 * synchronises those events, stops recording and writes, for each kernel id
 * k in [0, capacity), the number of launches (launches[k]) and their summed
 * device time in milliseconds (total_ms[k]). Kernel ids: 1 forward (bf16),
 * 2 forward (fp32), 3 backward preprocess, 4 backward dK/dV, 5 backward
 * dQ, 6 decode split, 7 decode merge, 9 FP8 preparation (8 is not used;
 * the FP8 forward reports as 1).
 * Returns the number of ids (10), or -1 if a CUDA call failed. Not thread-safe against concurrent
 * begin/end pairs; launches from several threads are recorded.
 */
void fa_profile_begin(void);
int fa_profile_end(int* launches, double* total_ms, int capacity);

#ifdef __cplusplus
}
#endif

#endif /* FA_SM100_H */
