/*
 * attn.h -- C ABI of libattn_b200: exact tiled attention forward and paged-KV
 * decode for NVIDIA B200 (sm_100a), one GPU.
 *
 * What the library computes
 *   O = softmax(Q K^T * scale [+ causal mask]) V, exactly (no approximation of
 *   the softmax), in tiles with an online softmax so the T x T score matrix is
 *   never written to device memory; and the gradients of that attention from the
 *   saved log-sum-exp by recomputing the tiles. Definitions:
 *   - Scores = Q K^T / sqrt(d_k), row-wise softmax, times V, computed per head:
 *     "Self-attention, CUDA kernels and FlashAttention" (russian.itimpress.au),
 *     section 1, the Scores and Attention(Q,K,V) formulas.
 *   - Tiles of Q, K, V held on chip, a running max and normaliser that rescale
 *     partial outputs, only O written back, small normalisation statistics
 *     saved: same page, section 3 (tiling, the online-softmax trick,
 *     recomputation in the backward pass).
 *   - causal=True and fewer K/V heads than query heads: "Flash Attention"
 *     skill page (hermes-agent-app.ru), Scenario 2, steps 2 and 3.
 *   - Paged KV cache with a block table, block size 16: "Fast attention
 *     kernels and operator fusion" (the-ai.news), section on FlashAttention-
 *     style and paged attention.
 *
 * Conventions for every call
 *   - Pointers: device memory owned by the caller (e.g. from cudaMalloc or a
 *     framework's allocator). The library keeps no pointer after the call
 *     returns and allocates no device memory per call.
 *   - Streams: `stream` is a cudaStream_t passed as void*; NULL means the legacy
 *     default stream. Calls enqueue work and return; they never synchronise the
 *     device. Results are valid once the stream reaches that point.
 *   - Errors: every call returns an attn_status_t and never aborts. Arguments
 *     are validated before anything is launched; on a non-OK return nothing was
 *     enqueued. A launch failure returns ATTN_ERR_CUDA. Device-side bounded
 *     waits and device-side index checks report through
 *     attn_get_device_status().
 *   - There is no CPU fallback: without an sm_100 device the compute calls
 *     return ATTN_ERR_DEVICE.
 *   - Dtypes: f16 or bf16 in and out (fp32 is not accepted, as on the pages);
 *     scores, softmax and accumulation run in fp32; lse is fp32.
 */
#ifndef TILED_ATTENTION_19_B200_ATTN_H
#define TILED_ATTENTION_19_B200_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_F16 = 0,
    ATTN_BF16 = 1
} attn_dtype_t;

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID = -1,     /* null pointer, negative size, H_q % H_kv != 0,
                                  scale not finite and > 0, bad table sizes */
    ATTN_ERR_UNSUPPORTED = -2, /* D not in {64, 128}, dtype, block_size != 16,
                                  H_q / H_kv > 16 (paged), a size past the limits */
    ATTN_ERR_MISALIGNED = -3,  /* a tensor base pointer not 16-byte aligned
                                  (lse, block_table, seq_lens: 4-byte) */
    ATTN_ERR_DEVICE = -4,      /* no CUDA device, or the current device is not
                                  compute capability 10.0 (B200) */
    ATTN_ERR_CUDA = -5,        /* a CUDA call (tensor-map encode, launch) failed */
    ATTN_ERR_TIMEOUT = -6,     /* from attn_get_device_status: a device-side
                                  bounded wait expired; the kernel gave up */
    ATTN_ERR_WORKSPACE = -7,   /* workspace NULL or smaller than required */
    ATTN_ERR_BAD_INDEX = -8,   /* from attn_get_device_status: a block-table entry
                                  or sequence length out of range was skipped */
    ATTN_ERR_SCRATCH_LIMIT = -9 /* attn_fwd_paged_noalloc: the problem needs more
                                  scratch than the fixed 4 MiB buffer holds */
} attn_status_t;

/*
 * attn_fwd -- dense attention forward (prefill), tcgen05 tensor cores.
 *
 *   q    [B, H_q,  Lq, D]  dtype, contiguous, 16-byte aligned
 *   k    [B, H_kv, Lk, D]  dtype, contiguous, 16-byte aligned
 *   v    [B, H_kv, Lk, D]  dtype, contiguous, 16-byte aligned
 *   out  [B, H_q,  Lq, D]  dtype, written (every element)
 *   lse  [B, H_q,  Lq]     fp32, written if non-NULL: natural-log
 *        log-sum-exp of the row's scaled, masked scores
 *
 *   Query head h reads K/V head h / (H_q / H_kv) (consecutive query heads share
 *   a K/V head; H_q must be a multiple of H_kv). With causal != 0, key j is
 *   visible to query i iff j <= i + (Lk - Lq) (bottom-right aligned; top-left
 *   when Lq == Lk). A row that sees no key gets O = 0 and lse = -inf.
 *   scale multiplies Q K^T; pass 1/sqrt(D) for the textbook scaling. It must be
 *   finite and > 0.
 *
 *   D in {64, 128}. H_q, H_kv >= 1; B, Lq, Lk >= 0. B == 0 or Lq == 0 is a
 *   no-op (every pointer may then be NULL). Lk == 0 writes O = 0, lse = -inf
 *   (k and v may then be NULL). Lq, Lk <= 2^22.
 */
attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                       int B, int H_q, int H_kv, int Lq, int Lk, int D, float scale,
                       int causal, attn_dtype_t dtype, void* stream);

/*
 * attn_fwd_window -- attn_fwd with a sliding window (local attention): the
 * window_size = (left, right) of the "Flash Attention" skill page (hermes-agent-app.ru),
 * Scenario 2, step 3. With i' = i + (Lk - Lq), key j is visible to query i iff
 * i' - window_left <= j <= i' + window_right; -1 leaves that side unbounded, and
 * causal != 0 caps the right side at i' (window_right is then ignored). Key tiles
 * outside every row's window are never loaded. (-1, -1) without causal is attn_fwd's
 * full attention; (-1, -1) with causal is attn_fwd's causal attention. Rows that see no
 * key get O = 0 and lse = -inf. Returns ATTN_ERR_INVALID for a bound below -1; all
 * other arguments as attn_fwd.
 */
attn_status_t attn_fwd_window(const void* q, const void* k, const void* v, void* out, float* lse,
                              int B, int H_q, int H_kv, int Lq, int Lk, int D, float scale,
                              int causal, int window_left, int window_right, attn_dtype_t dtype,
                              void* stream);

/*
 * attn_strides_t -- element strides of a tensor of shape [B, H, L, D] whose D elements
 * are contiguous: element (b, h, l, d) sits at base + b*batch + h*head + l*seq + d.
 * The contiguous layout [B, H, L, D] is {H*L*D, L*D, D}; flash_attn's [B, L, H, D] is
 * {L*H*D, D, H*D}.
 */
typedef struct {
    int64_t batch;
    int64_t head;
    int64_t seq;
} attn_strides_t;

/*
 * attn_fwd_strided -- attn_fwd_window on tensors with arbitrary strides: the layouts
 * of [B, L, H, D] tensors (flash_attn_func's q, k, v and output, "Flash Attention"
 * skill page (hermes-agent-app.ru), Scenario 2), of q, k and v sliced from a packed
 * QKV projection, or of any view whose D elements are contiguous.
 *
 *   q, k, v, out  base pointers, 16-byte aligned, with the strides in q_strides,
 *                 k_strides, v_strides, out_strides (a NULL strides pointer means the
 *                 contiguous [B, H, L, D] layout). Each stride of a dimension longer than
 *                 1 must be positive, a multiple of 8 elements (16 bytes) and below 2^38;
 *                 a stride of a dimension of length 1 is ignored.
 *   lse           [B, H_q, Lq] fp32, contiguous, written if non-NULL.
 *
 *   out must not overlap q, k or v. All other arguments, results and errors as
 *   attn_fwd_window (window_left = window_right = -1 for no window). Returns
 *   ATTN_ERR_INVALID for a non-positive or oversized stride and ATTN_ERR_MISALIGNED
 *   for a stride that is not a multiple of 8.
 */
attn_status_t attn_fwd_strided(const void* q, const attn_strides_t* q_strides, const void* k,
                               const attn_strides_t* k_strides, const void* v,
                               const attn_strides_t* v_strides, void* out,
                               const attn_strides_t* out_strides, float* lse, int B, int H_q,
                               int H_kv, int Lq, int Lk, int D, float scale, int causal,
                               int window_left, int window_right, attn_dtype_t dtype,
                               void* stream);

/*
 * attn_paged_workspace_size -- bytes of device workspace attn_fwd_paged needs
 * for these sizes (0 when no sequence is ever split). The workspace holds the
 * partial results of the split-KV chunks (one per CTA of the balanced
 * schedule) and one completion counter per (sequence, K/V head).
 */
size_t attn_paged_workspace_size(int num_seqs, int H_q, int H_kv, int D,
                                 int max_blocks_per_seq, int block_size);

/*
 * attn_fwd_paged -- decode attention over a paged KV cache (one query token per
 * sequence), memory-bound, split over KV chunks with an in-kernel combine.
 *
 *   q            [num_seqs, H_q, D]                        dtype
 *   k_cache      [num_blocks, H_kv, block_size, D]         dtype
 *   v_cache      [num_blocks, H_kv, block_size, D]         dtype
 *   block_table  [num_seqs, max_blocks_per_seq] int32: token t of sequence s
 *                is row t % block_size of physical block block_table[s][t / block_size]
 *   seq_lens     [num_seqs] int32, 0 <= seq_lens[s] <= max_blocks_per_seq * block_size
 *   out          [num_seqs, H_q, D] dtype, written
 *   lse          [num_seqs, H_q] fp32, written if non-NULL
 *
 *   block_size must be 16; H_q / H_kv <= 16; D in {64, 128}. Entries of
 *   block_table past ceil(seq_lens[s] / 16) are never read. The cache rows of a
 *   sequence's last block past seq_lens[s] may hold anything (even NaN): they are
 *   masked out of both products. An entry outside
 *   [0, num_blocks), or a seq_len past the table, is skipped on the device and
 *   reported as ATTN_ERR_BAD_INDEX by attn_get_device_status(). A sequence of
 *   length 0 gets O = 0 and lse = -inf. num_seqs == 0 is a no-op (every
 *   pointer may then be NULL).
 *
 *   workspace: device memory of at least attn_paged_workspace_size(...) bytes,
 *   256-byte aligned, ZERO-FILLED BEFORE ITS FIRST USE (its first bytes are
 *   the completion counters). Every call that completes returns the counters
 *   to zero, so one workspace serves any number of calls without clearing, as
 *   long as the calls do not overlap on the device. May be NULL only when the
 *   size query returns 0.
 */
attn_status_t attn_fwd_paged(const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_table, const int32_t* seq_lens,
                             int block_size, void* out, float* lse, int num_seqs, int H_q,
                             int H_kv, int D, int max_blocks_per_seq, int num_blocks,
                             float scale, attn_dtype_t dtype, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * attn_fwd_paged_noalloc -- attn_fwd_paged without a caller-supplied workspace.
 * (The pages have no counterpart: this entry point is a property of this
 * library, not of the attention method.)
 *
 * Some callers cannot allocate device memory. A plugin may be handed only its
 * input and output buffers by a host framework that owns the allocator. A
 * latency-critical path may not accept cudaMalloc's implicit device
 * synchronisation. A deployment may have reserved all device memory up front.
 * This entry point serves them: it allocates nothing and calls no allocating
 * routine. Its scratch is one fixed array of 4 MiB (4,194,304 bytes) inside the
 * library's device module, which every GPU that loads the library holds until
 * the process exits.
 *
 * Arguments, layouts, results and errors are those of attn_fwd_paged, without
 * the workspace. A problem whose attn_paged_workspace_size() exceeds 4 MiB is
 * rejected with ATTN_ERR_SCRATCH_LIMIT before anything is enqueued. The
 * decode workload of 16 sequences, 12/2 heads, D = 128, 256 blocks per
 * sequence needs 916,736 bytes.
 *
 * The first call on a device looks up the array's device address with that
 * device current (cudaGetSymbolAddress); make that first call before any
 * stream capture. The address is looked up again when the device's current
 * context changes (after a device reset the library's module, and the array
 * with it, is loaded anew); the first call after such a reset is then again a
 * set-up call. Every argument check and the tensor-map encoding run before
 * anything is enqueued; then each call clears the array's completion counters
 * on `stream` and launches the kernel.
 *
 * Every call on a device shares the one array, which keeps the last call's
 * contents: calls that overlap on the GPU (different streams, or different
 * host threads without ordering) race and may produce wrong results. Order
 * them on one stream, or use attn_fwd_paged with a workspace per stream.
 */
attn_status_t attn_fwd_paged_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_table, const int32_t* seq_lens,
                                     int block_size, void* out, float* lse, int num_seqs,
                                     int H_q, int H_kv, int D, int max_blocks_per_seq,
                                     int num_blocks, float scale, attn_dtype_t dtype,
                                     void* stream);

/*
 * attn_bwd_workspace_size -- bytes of device workspace attn_bwd needs:
 * 8 * B * H_q * ceil(Lq / 128) * 128 (two fp32 values per query row, rows padded
 * to a multiple of 128).
 */
size_t attn_bwd_workspace_size(int B, int H_q, int Lq);

/*
 * attn_bwd -- dense attention backward pass: the gradients dQ, dK, dV of a scalar
 * loss given dO = dLoss/dO, for the attention attn_fwd computed. The attention
 * tiles are recomputed from q, k, v and the forward pass's lse; the score matrix is
 * never written to device memory ("Self-attention, CUDA kernels and
 * FlashAttention" (russian.itimpress.au), section 3: recomputation in the backward
 * pass from the saved normalisation statistics). With P the attention probabilities
 * and delta_i = dO_i . O_i:
 *   dV_j = sum_i P_ij dO_i
 *   dS_ij = P_ij (dO_i . v_j - delta_i)
 *   dQ_i = scale sum_j dS_ij k_j
 *   dK_j = scale sum_i dS_ij q_i
 * Grouped K/V heads get the sum over the query heads that read them.
 *
 *   q, k, v  as attn_fwd (the forward pass's inputs)
 *   out      [B, H_q, Lq, D] dtype: the forward pass's O
 *   dout     [B, H_q, Lq, D] dtype: dLoss/dO
 *   lse      [B, H_q, Lq] fp32: the forward pass's lse (-inf for rows that see no key)
 *   dq       [B, H_q, Lq, D] dtype, written (every element)
 *   dk, dv   [B, H_kv, Lk, D] dtype, written (every element)
 *
 *   causal and all sizes as attn_fwd. Tensor pointers 16-byte aligned (lse:
 *   4-byte). workspace: device memory of at least attn_bwd_workspace_size(B, H_q,
 *   Lq) bytes, 16-byte aligned, no initial contents required; it is overwritten on
 *   `stream` by every call, so calls that overlap on the device need separate
 *   workspaces. B == 0 is a no-op (pointers may be NULL); Lq == 0 writes dK = dV = 0;
 *   Lk == 0 writes dQ = 0. No atomics: results do not depend on scheduling.
 *   Returns ATTN_ERR_WORKSPACE for a missing or short workspace.
 */
attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* out,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv,
                       int B, int H_q, int H_kv, int Lq, int Lk, int D, float scale,
                       int causal, attn_dtype_t dtype, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * attn_bwd_window -- attn_bwd for attn_fwd_window's sliding-window attention
 * (window_left, window_right, causal as there); arguments otherwise as attn_bwd.
 */
attn_status_t attn_bwd_window(const void* q, const void* k, const void* v, const void* out,
                              const void* dout, const float* lse, void* dq, void* dk, void* dv,
                              int B, int H_q, int H_kv, int Lq, int Lk, int D, float scale,
                              int causal, int window_left, int window_right,
                              attn_dtype_t dtype, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * attn_bwd_strided -- attn_bwd_window on tensors of any layout with a contiguous last
 * dimension (for example the [B, L, H, D] layout: batch stride L*H*D, head stride D,
 * row stride H*D). Each of q, k, v, out, dout, dq, dk, dv takes its own
 * attn_strides_t (in elements; each stride times the element size a multiple of 16
 * bytes), or NULL for the contiguous [B, H, L, D] layout; lse stays [B, H_q, Lq]
 * contiguous. Gradients are written through their strides, every element of the
 * described views and nothing else. causal, window_left and window_right as
 * attn_fwd_window (pass -1, -1 with causal = 0 for dense attention); all other
 * arguments and errors as attn_bwd, plus ATTN_ERR_MISALIGNED for a stride that breaks
 * the 16-byte rule. The results are bit-identical to attn_bwd_window on contiguous
 * copies of the same values.
 */
attn_status_t attn_bwd_strided(const void* q, const attn_strides_t* q_strides, const void* k,
                               const attn_strides_t* k_strides, const void* v,
                               const attn_strides_t* v_strides, const void* out,
                               const attn_strides_t* out_strides, const void* dout,
                               const attn_strides_t* dout_strides, const float* lse, void* dq,
                               const attn_strides_t* dq_strides, void* dk,
                               const attn_strides_t* dk_strides, void* dv,
                               const attn_strides_t* dv_strides, int B, int H_q, int H_kv, int Lq,
                               int Lk, int D, float scale, int causal, int window_left,
                               int window_right, attn_dtype_t dtype, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * attn_fwd_fp8 -- dense attention forward on 8-bit inputs: q, k and v in FP8 E4M3, the
 * tensor-core products in 8 bits (tcgen05 kind::f8f6f4), softmax and accumulation in
 * fp32, O in bf16 ("Flash Attention" skill page (hermes-agent-app.ru), Scenario 3: the
 * FP8 forward of FlashAttention-3, for maximum performance, on inputs cast to
 * float8_e4m3fn; forward only).
 *
 *   q, k, v  e4m3 bytes, shapes and strides as attn_fwd_strided (strides in elements =
 *            bytes, multiples of 16); the values they stand for are q * descale_q,
 *            k * descale_k and v * descale_v (pass 1 for plain casts)
 *   out      [B, H_q, Lq, D] bf16, strides as attn_fwd_strided; lse as attn_fwd
 *
 *   The attention weights P are rounded to e4m3 before P.V (relative error up to 2^-4
 *   per weight; the normaliser and lse use the unrounded fp32 weights). D must be 128;
 *   causal as attn_fwd (no window). scale and the three descale factors must be finite
 *   and > 0. Other arguments, results and errors as attn_fwd_strided.
 */
attn_status_t attn_fwd_fp8(const void* q, const attn_strides_t* q_strides, const void* k,
                           const attn_strides_t* k_strides, const void* v,
                           const attn_strides_t* v_strides, void* out,
                           const attn_strides_t* out_strides, float* lse, int B, int H_q, int H_kv,
                           int Lq, int Lk, int D, float scale, float descale_q, float descale_k,
                           float descale_v, int causal, void* stream);

/*
 * attn_fwd_paged_prefill -- prefill attention over a paged KV cache: each sequence's
 * chunk of queries attends to its keys in the cache, resolved block by block through
 * the block table inside the kernel ("Fast attention kernels and operator fusion"
 * (the-ai.news), section on FlashAttention-style and paged attention: long prefill,
 * and a paged cache whose positions the kernel translates through the table). Runs
 * the tcgen05 prefill kernel of attn_fwd with its K/V tiles gathered from 16-token
 * blocks.
 *
 *   q            [num_seqs, H_q, Lq, D] dtype, strides as attn_fwd_strided (q_strides
 *                NULL: contiguous); sequence s's chunk is its first q_lens[s] rows
 *   k_cache      [num_blocks, H_kv, block_size, D] dtype, contiguous
 *   v_cache      [num_blocks, H_kv, block_size, D] dtype, contiguous
 *   block_table  [num_seqs, max_blocks_per_seq] int32, as attn_fwd_paged
 *   seq_lens     [num_seqs] int32: keys of sequence s, 0 <= seq_lens[s] <=
 *                max_blocks_per_seq * block_size (they include the chunk's own keys)
 *   q_lens       [num_seqs] int32, 0 <= q_lens[s] <= Lq, or NULL for all Lq
 *   out          [num_seqs, H_q, Lq, D] dtype, written (every element; out_strides as
 *                q_strides)
 *   lse          [num_seqs, H_q, Lq] fp32, contiguous, written if non-NULL
 *
 *   The chunk's queries are the sequence's last q_lens[s] positions: with causal != 0,
 *   query i sees keys j <= i + seq_lens[s] - q_lens[s] (attn_fwd's bottom-right mask
 *   with Lq = q_lens[s], Lk = seq_lens[s]); without it every query sees all
 *   seq_lens[s] keys. Rows i >= q_lens[s], and rows that see no key, get O = 0 and
 *   lse = -inf. block_size must be 16; H_q a multiple of H_kv; D in {64, 128}.
 *   Table entries past ceil(seq_lens[s] / 16) are never read. A length out of range is
 *   clamped, an entry outside [0, num_blocks) is replaced by block 0, and both are
 *   reported as ATTN_ERR_BAD_INDEX by attn_get_device_status(). The cache rows of a
 *   sequence's last block past seq_lens[s] are read but weigh nothing; they must hold
 *   finite values (a NaN there would reach the output through 0 * NaN).
 *   num_seqs == 0 or Lq == 0 is a no-op (pointers may be NULL).
 */
attn_status_t attn_fwd_paged_prefill(const void* q, const attn_strides_t* q_strides,
                                     const void* k_cache, const void* v_cache,
                                     const int32_t* block_table, const int32_t* seq_lens,
                                     const int32_t* q_lens, int block_size, void* out,
                                     const attn_strides_t* out_strides, float* lse, int num_seqs,
                                     int H_q, int H_kv, int Lq, int D, int max_blocks_per_seq,
                                     int num_blocks, float scale, int causal, attn_dtype_t dtype,
                                     void* stream);

/* Static text for a status code (never NULL). */
const char* attn_error_string(attn_status_t status);

/*
 * attn_get_device_status -- read and clear the device-side status word that
 * kernels set when a bounded wait expires (ATTN_ERR_TIMEOUT) or an index is out
 * of range (ATTN_ERR_BAD_INDEX). Synchronises `stream` to read it. Returns
 * ATTN_OK if no kernel on the current device reported anything since the last
 * call, ATTN_ERR_CUDA if the read itself failed.
 */
attn_status_t attn_get_device_status(void* stream);

/*
 * attn_selftest_bounded_wait -- exercise the kernels' failure detection without a
 * fault. Launches one CTA that waits, through the same bounded wait the attention
 * kernels use, on a barrier that nothing completes. The wait gives up after about a
 * second, sets ATTN_ERR_TIMEOUT in the device status word and the kernel returns; the
 * context stays usable. Returns ATTN_OK once enqueued (ATTN_ERR_DEVICE without an
 * sm_100 device); read the outcome with attn_get_device_status().
 */
attn_status_t attn_selftest_bounded_wait(void* stream);

/*
 * attn_selftest_fill_noalloc_scratch -- test hook for attn_fwd_paged_noalloc:
 * overwrites every byte of its fixed 4 MiB scratch array on the current device with
 * (byte_value & 0xFF), enqueued on `stream`. This stands in for what an interrupted
 * call (one whose bounded wait expired) can leave behind: completion counters that
 * are not zero and stale partial results. Tests use it to check that the next
 * no-allocation call does not depend on what the array held. Like any call that
 * touches the array, it races with no-allocation calls in flight on other streams.
 * Returns ATTN_OK once enqueued, ATTN_ERR_DEVICE without an sm_100 device,
 * ATTN_ERR_CUDA if the array's address cannot be looked up or the fill fails to
 * enqueue.
 */
attn_status_t attn_selftest_fill_noalloc_scratch(int byte_value, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TILED_ATTENTION_19_B200_ATTN_H */
