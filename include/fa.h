/*
 * fa.h - C ABI of the B200 (sm_100a) exact-attention library (libfa.so).
 *
 * The library computes exact softmax attention
 *
 *     O = softmax(scale * Q K^T + mask) V
 *
 * (page "PyTorch-CUDA-v2.9镜像中使用FlashAttention提升训练速度", the Attention(Q,K,V)
 * formula) tile by tile with an online softmax, so that the N x N score matrix never
 * reaches device memory (page "告别OOM和训练慢：用Flash Attention加速你的PyTorch大模型
 * （含A100环境配置）" §2.1 tiling, §2.2 online softmax), and the training backward,
 * which recomputes P from the per-row log-sum-exp saved by the forward (same page
 * §2.2, "only the normalisation factors are stored").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Tensors.  q, k, v, o, dout, dq, dk, dv are bf16 tensors of shape
 *   (B, H, N, d) = (batch, heads, seq_len, head_dim), fully contiguous, row-major
 *   (page "Flash Attention 3.7 核心原理与实战" §3.2 states the problem in this shape).
 *   lse is fp32 (B, H, N): the natural-log log-sum-exp of each row of the scaled,
 *   masked scores.
 *   Query and key sequences have the same length N.
 * Sizes.  d must be 64 or 128 (else FA_ERR_UNSUPPORTED: the pages list 64 and 128
 *   as the common head sizes and report "no available kernel" otherwise, page
 *   "Flash Attention 3.7 …" §5). B, H, N >= 0; if any is 0 the call does nothing and
 *   returns FA_OK. Each tensor must have fewer than 2^31 elements (else
 *   FA_ERR_UNSUPPORTED).
 * Scale.  scale multiplies Q K^T before the mask. It is used exactly as given and
 *   must be finite and > 0 (else FA_ERR_INVALID_ARG); pass 1/sqrt(d) for the usual
 *   default (`softmax_scale=None`, page "告别OOM和训练慢…" §4.2).
 * Mask.  Key j is visible from query i iff
 *     (window.left  < 0 or j >= i - window.left) and
 *     (window.right < 0 or j <= i + window.right),
 *   with -1 meaning unbounded (`window_size=(-1,-1)`, page "告别OOM和训练慢…" §4.2).
 *   causal != 0 masks future positions, i.e. forces window.right = 0 when it is -1
 *   or positive. Values below -1 give FA_ERR_INVALID_ARG. Every query sees at least
 *   itself, so no row is fully masked unless key padding (fa_options_t) removes all of
 *   its keys.
 * Memory.  Every pointer is caller-owned device memory that is only used during the
 *   call's kernels; the library keeps nothing and allocates nothing. Pointers must be
 *   non-null (FA_ERR_INVALID_ARG) and 16-byte aligned (FA_ERR_MISALIGNED: the
 *   tensors are fetched by the Tensor Memory Accelerator, page "告别OOM和训练慢…" §4.3
 *   "misaligned address").
 * Streams.  stream is a cudaStream_t (NULL = the legacy default stream). All checks
 *   run on the host before any launch and return synchronously; kernels are then
 *   enqueued on the stream and the call returns without waiting. Launch failures
 *   return FA_ERR_CUDA. Calls on distinct streams may run concurrently.
 * Faults.  Every wait inside the kernels is bounded (about two seconds). A kernel
 *   whose wait runs out abandons its work, records FA_ERR_TIMEOUT in a device
 *   status word and exits; fa_debug_status() reports and clears it.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad scale or window  */
    FA_ERR_UNSUPPORTED = 2,  /* head_dim not 64/128, or a tensor of >= 2^31 elements */
    FA_ERR_MISALIGNED = 3,   /* a pointer that is not 16-byte aligned               */
    FA_ERR_WORKSPACE = 4,    /* workspace (or the no-alloc array) too small         */
    FA_ERR_CUDA = 5,         /* a CUDA runtime or driver call failed                */
    FA_ERR_TIMEOUT = 6       /* a kernel abandoned a bounded wait (fa_debug_status) */
} fa_status_t;

/* Sliding window (`window_size=(left,right)`): keys j with i-left <= j <= i+right. */
typedef struct {
    int left;
    int right;
} fa_window_t;

/*
 * Optional inputs and outputs of the _ex entry points (and of the backward's phase entry
 * points). A null fa_options_t pointer, or a zero-initialised struct, means none of them.
 *
 *   alibi_slopes  H fp32 slopes, device memory, 4-byte aligned, or NULL: the ALiBi bias
 *                 (see fa_fwd_alibi).
 *   key_padding   (B, N) bytes, device memory, any alignment, or NULL: nonzero marks key
 *                 n of batch entry b as padding. The attention layer of page "PyTorch-
 *                 CUDA-v2.9镜像中使用FlashAttention提升训练速度" takes such a `key_padding_mask`
 *                 (True = padded), and the reference layer of page "Flash Attention 3.7 核心
 *                 原理与实战" §4.2 applies it with masked_fill(-inf) to every head and query:
 *                 a padded key's score is -inf before the softmax. A query left with no visible,
 *                 unpadded key gets O = 0, LSE = -inf and no gradient (the backward must
 *                 get the same flags as the forward).
 *   o_low         bf16 (B, H, N, d), device memory, 16-byte aligned, or NULL. The forward
 *                 writes there what rounding O to bf16 left out, O_fp32 - bf16(O), itself
 *                 rounded to bf16; the backward then forms delta = rowsum(dO o O) from
 *                 o + o_low, about 16 significant bits instead of 8. This matters for rows
 *                 whose softmax is nearly one-hot: there dS = P o (dP - delta) cancels
 *                 almost completely and the bf16 rounding of O alone would move dQ and dK
 *                 by several percent. Costs one more bf16 tensor written by the forward and
 *                 read by the backward.
 *   dropout_p, dropout_seed, dropout_offset
 *                 dropout on the attention weights (`dropout_p` of flash_attn_fn, page
 *                 "告别OOM和训练慢…" §4.2; the reference layer of page "Flash Attention 3.7
 *                 核心原理与实战" §4.2 applies it to the softmax weights before the product with
 *                 V): O = (P o Z / (1 - p')) V, LSE unchanged. The keep flags Z are drawn from
 *                 Philox4x32-10 (Salmon et al., SC 2011) under key dropout_seed (low, high
 *                 32 bits) at counter (key / 16, query, b*H + h, dropout_offset): key j uses
 *                 byte j mod 4 of output word (j mod 16) / 4 and is dropped iff that byte is
 *                 below t = floor(256 p + 1/2); p' = t / 256 (p rounded to a multiple of
 *                 1/256). dropout_p must be in [0, 1) with t <= 255, and dropout_offset below
 *                 2^32 (else FA_ERR_INVALID_ARG); t = 0 is no dropout. The backward must get
 *                 the same three values; it regenerates the flags instead of storing them.
 *                 Use a new offset (or seed) per call to draw new flags.
 *   flags         FA_BWD_FUSED or 0 (see below).
 *   seq_lengths   B int32 real lengths, device memory, 4-byte aligned, or NULL: a
 *                 variable-length batch (the `lengths` of the dynamic batching of page
 *                 "告别OOM和训练慢…" §6, each sample's real length). Batch entry b holds
 *                 L_b real tokens at the start of its rows: query i and key j interact only
 *                 if i < L_b and j < L_b. Rows past L_b get O = 0, LSE = -inf and zero
 *                 gradients, and no tile that lies wholly past L_b is computed, so a batch
 *                 costs what its real lengths cost. Values are clamped to [0, N]. The
 *                 backward must get the same lengths.
 *   cu_seqlens, total_tokens
 *                 a packed batch, or NULL / 0: the B sequences stored back to back with no
 *                 padding (the page's dynamic batching groups sequences to avoid padding
 *                 waste, page "告别OOM和训练慢…" §6). cu_seqlens holds B + 1 int32 cumulative
 *                 lengths in device memory, 4-byte aligned: sequence b is tokens
 *                 cu_seqlens[b] .. cu_seqlens[b+1]-1 of q, k, v, o, dout, dq, dk, dv (and
 *                 o_low), which are then (total_tokens, H, d) bf16 instead of (B, H, N, d);
 *                 lse is (H, total_tokens) fp32. N is the longest length the call handles:
 *                 a sequence is cut at N (its tokens past N are not written) and empty or
 *                 decreasing entries count as length 0. The offsets must lie in
 *                 [0, total_tokens]; the kernels write no token at or past total_tokens.
 *                 Masks, scale, ALiBi, key padding ((B, N) flags by position in the
 *                 sequence) and dropout apply per sequence as in the padded layout; the
 *                 results of each sequence are bit-identical to those of the same sequence
 *                 in a (B, H, N, d) batch with seq_lengths (and finite padding). Exclusive
 *                 with seq_lengths
 *                 (FA_ERR_INVALID_ARG); not with FA_BWD_FUSED (FA_ERR_UNSUPPORTED); the
 *                 backward must get the same two values, and its workspace
 *                 (fa_bwd_workspace_bytes_ex) then holds the schedule tables as with
 *                 seq_lengths. total_tokens < 0 gives FA_ERR_INVALID_ARG; 0 is an empty call.
 * The layout is that of a C struct with natural alignment (72 bytes on LP64).
 */
typedef struct {
    const float *alibi_slopes;
    const unsigned char *key_padding;
    void *o_low;
    float dropout_p;
    unsigned int flags;                 /* FA_BWD_* bits below; 0 = none */
    unsigned long long dropout_seed;
    unsigned long long dropout_offset;
    const int *seq_lengths;
    const int *cu_seqlens;
    int total_tokens;
} fa_options_t;

/*
 * flags: FA_BWD_FUSED selects, at head_dim 64, the backward that computes dK, dV and dQ in
 * one pass over key tiles (fa_bwd_fused): each (query tile, key tile) pair's share of dQ is
 * added into an fp32 accumulator by TMA bulk reduce-adds at L2, in no fixed order, so dQ is
 * reproducible to fp32 rounding only (dK, dV stay bit-identical), and the workspace must
 * also hold the accumulator (fa_bwd_workspace_bytes_ex). It does 2/7 less tensor work than
 * the default, but moves P and dS through shared memory and is not faster on B200 (see the
 * design notes). Without it (and always at head_dim 128) the backward runs the dK/dV pass
 * and a separate dQ pass: bit-identical results from run to run. Other bits give
 * FA_ERR_INVALID_ARG.
 */
#define FA_BWD_FUSED 1u

/*
 * Forward pass.
 *   in : q, k, v  (B,H,N,d) bf16
 *   out: o (B,H,N,d) bf16, rounded to nearest even from fp32;
 *        lse (B,H,N) fp32, natural log.
 * One fused kernel: S = scale Q K^T is formed tile by tile in tensor memory, the
 * running max m and sum l are updated per row (page "告别OOM和训练慢…" §2.2), the output
 * accumulates P V in tensor memory and is divided by l at the end; only O and LSE are
 * written to device memory.
 */
fa_status_t fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                   int B, int H, int N, int d, float scale, int causal,
                   fa_window_t window, void *stream);

/*
 * fa_fwd with the optional inputs and outputs of `options` (may be NULL). Misaligned
 * slopes or o_low give FA_ERR_MISALIGNED; dropout values out of range FA_ERR_INVALID_ARG.
 */
fa_status_t fa_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse,
                      int B, int H, int N, int d, float scale, int causal,
                      fa_window_t window, const fa_options_t *options, void *stream);

/*
 * Forward pass on 8-bit inputs (page "告别OOM和训练慢…" §6 lists FP8 support among the next
 * steps of the method). q, k, v are e4m3 (OCP FP8 E4M3, one byte per value) tensors of shape
 * (B, H, N, d); the values they stand for are q * q_scale, k * k_scale, v * v_scale (per-tensor
 * descales, finite and > 0, else FA_ERR_INVALID_ARG). S = Q K^T and P V run on the tensor core
 * in FP8 (tcgen05 kind::f8f6f4) with fp32 accumulation; P is rounded to e4m3 for the second
 * product, so O carries a relative error of a few percent (the 3-bit mantissa of each weight),
 * while LSE, formed from the fp32 scores, is as exact as in fa_fwd.
 *   out: o (B,H,N,d) bf16 (the attention of the descaled values); lse (B,H,N) fp32.
 * d must be 128 (else FA_ERR_UNSUPPORTED). Masks, scale, errors and memory rules as fa_fwd; no
 * options. There is no FP8 backward.
 */
fa_status_t fa_fwd_fp8(const void *q, const void *k, const void *v, float q_scale,
                       float k_scale, float v_scale, void *o, float *lse, int B, int H, int N,
                       int d, float scale, int causal, fa_window_t window, void *stream);

/*
 * Bytes of device workspace fa_bwd() needs: two fp32 arrays of B*H*Np values, where
 * Np = N rounded up to a multiple of 128 (the row statistics of the backward, see
 * fa_bwd_preprocess), rounded up to 256 bytes. Returns 0 for an empty problem or invalid
 * sizes.
 */
size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * The same for fa_bwd_ex with `options` (may be NULL): with FA_BWD_FUSED at head_dim 64 the
 * row statistics are followed by the fused pass's fp32 dQ accumulator of B*H*Np*64 values;
 * with seq_lengths (and B <= 8192) the last part holds the tables of the variable-length
 * work schedule, 2*(Np/128 + 1) + B ints rounded up to 256 bytes, which fa_bwd_preprocess
 * writes and the passes read (items ordered by their tile's distance from the start or end
 * of its sequence, so that the persistent CTAs get even shares of uneven sequences).
 * Returns 0 for an empty problem, invalid sizes or invalid options.
 */
size_t fa_bwd_workspace_bytes_ex(int B, int H, int N, int d, const fa_options_t *options);

/*
 * Backward pass: the gradient of the scalar <O, dO> with respect to q, k and v.
 *   in : q, k, v, o, dout (B,H,N,d) bf16; lse (B,H,N) fp32 from fa_fwd with the
 *        same q, k, v, scale and mask.
 *   out: dq, dk, dv (B,H,N,d) bf16.
 *   workspace: caller-owned device scratch of at least fa_bwd_workspace_bytes()
 *        bytes (FA_ERR_WORKSPACE if workspace_bytes is smaller), 16-byte aligned.
 * The pages state only that the backward recomputes the attention matrix from the
 * stored normalisation factors (page "告别OOM和训练慢…" §2.2; page "PyTorch-CUDA-v2.9
 * 镜像…", "3. 重计算策略"); the steps are the chain rule of softmax attention:
 *   delta_i = sum_c dO_ic O_ic                 (fa_bwd_preprocess)
 *   P = exp(scale Q K^T - LSE), dP = dO V^T, dS = P o (dP - delta),
 *   dV = P^T dO, dK = scale dS^T Q             (fa_bwd_dkdv, one pass per key tile)
 *   dQ = scale dS K                            (fa_bwd_dq, one pass per query tile)
 * The kernels run in that order on the stream; results are deterministic. (fa_bwd_ex with
 * FA_BWD_FUSED replaces the two passes by one at head_dim 64, see FA_BWD_FUSED.)
 */
fa_status_t fa_bwd(const void *q, const void *k, const void *v, const void *o,
                   const void *dout, const float *lse, void *dq, void *dk, void *dv,
                   int B, int H, int N, int d, float scale, int causal,
                   fa_window_t window, void *workspace, size_t workspace_bytes,
                   void *stream);

/*
 * fa_bwd with the optional inputs of `options` (may be NULL): the same alibi_slopes,
 * key_padding and dropout values as the forward had, and o_low if the forward wrote it.
 */
fa_status_t fa_bwd_ex(const void *q, const void *k, const void *v, const void *o,
                      const void *dout, const float *lse, void *dq, void *dk, void *dv,
                      int B, int H, int N, int d, float scale, int causal,
                      fa_window_t window, const fa_options_t *options, void *workspace,
                      size_t workspace_bytes, void *stream);

/*
 * ALiBi: fa_fwd and fa_bwd with a linear bias. Page "告别OOM和训练慢…(含A100环境配置)" §4.2
 * lists `alibi_slopes` among the parameters of flash_attn_fn and calls it a linear bias;
 * the reading taken is that of ALiBi: head h has a slope m_h, and -m_h * |i - j| is added
 * to the scaled score of query i and key j before masking and softmax (LSE includes it).
 *   alibi_slopes: device pointer to H fp32 slopes, shared by all batch entries; 4-byte
 *        aligned; not null (FA_ERR_INVALID_ARG). The slopes must be finite.
 * All other arguments, layouts, errors and guarantees are those of fa_fwd / fa_bwd;
 * fa_bwd_alibi needs the lse of fa_fwd_alibi with the same slopes.
 */
fa_status_t fa_fwd_alibi(const void *q, const void *k, const void *v, void *o, float *lse,
                         int B, int H, int N, int d, float scale, int causal,
                         fa_window_t window, const float *alibi_slopes, void *stream);

fa_status_t fa_bwd_alibi(const void *q, const void *k, const void *v, const void *o,
                         const void *dout, const float *lse, void *dq, void *dk, void *dv,
                         int B, int H, int N, int d, float scale, int causal,
                         fa_window_t window, const float *alibi_slopes, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * Step 1 of fa_bwd alone: fills `workspace` (at least fa_bwd_workspace_bytes(), or
 * fa_bwd_workspace_bytes_ex() with the same options when they carry FA_BWD_FUSED or
 * seq_lengths: the workspace is not bounds-checked here) with
 * the per-row statistics the two passes read, each as B*H rows of Np = N rounded up to
 * 128 fp32 values (padding rows: +inf and 0):
 *   workspace[0 .. B*H*Np)          LSE * log2(e)      (from `lse`)
 *   workspace[B*H*Np .. 2*B*H*Np)   delta = rowsum(dout * o), summed in fp32
 *                                   (o + options->o_low when o_low is given)
 * The padding lets each 128-row tile of both arrays be fetched with one bulk copy.
 * With FA_BWD_FUSED at head_dim 64 it also zeroes the fused pass's dQ accumulator, and
 * with seq_lengths it writes the tables of the variable-length schedule (both after the
 * statistics, as fa_bwd_workspace_bytes_ex() lays them out).
 * `options` may be NULL; its o_low, flags and seq_lengths are used here.
 */
fa_status_t fa_bwd_preprocess(const void *o, const void *dout, const float *lse,
                              void *workspace, int B, int H, int N, int d,
                              const fa_options_t *options, void *stream);

/* Step 2 of fa_bwd alone: dk, dv from q, k, v, dout and the workspace of step 1
 * (`options`: alibi_slopes, key_padding, dropout, and seq_lengths or cu_seqlens with
 * total_tokens, as given to step 1; or NULL). */
fa_status_t fa_bwd_dkdv(const void *q, const void *k, const void *v, const void *dout,
                        const void *workspace, void *dk, void *dv,
                        int B, int H, int N, int d, float scale, int causal,
                        fa_window_t window, const fa_options_t *options, void *stream);

/* Step 3 of fa_bwd alone: dq from q, k, v, dout and the workspace of step 1
 * (`options`: alibi_slopes, key_padding, dropout, and seq_lengths or cu_seqlens with
 * total_tokens, as given to step 1; or NULL). */
fa_status_t fa_bwd_dq(const void *q, const void *k, const void *v, const void *dout,
                      const void *workspace, void *dq,
                      int B, int H, int N, int d, float scale, int causal,
                      fa_window_t window, const fa_options_t *options, void *stream);

/*
 * Step 2 of the fused backward alone (head_dim 64, else FA_ERR_UNSUPPORTED): dk, dv, and
 * dQ / scale added into the accumulator part of `workspace` (which fa_bwd_preprocess,
 * called with FA_BWD_FUSED, zeroed). `options`: alibi_slopes, key_padding, dropout and
 * seq_lengths, or NULL.
 */
fa_status_t fa_bwd_fused(const void *q, const void *k, const void *v, const void *dout,
                         void *workspace, void *dk, void *dv,
                         int B, int H, int N, int d, float scale, int causal,
                         fa_window_t window, const fa_options_t *options, void *stream);

/* Step 3 of the fused backward alone: dq = bf16(scale * accumulator). */
fa_status_t fa_bwd_dq_convert(void *workspace, void *dq, int B, int H, int N, int d,
                              float scale, void *stream);

/*
 * Backward pass for callers that cannot allocate device memory. (The pages have no
 * counterpart of this entry point; it is an interface addition of this library.)
 *
 * Some callers may not allocate: an engine that reserves all of its device memory up
 * front and may not grow it while serving, or a framework plugin whose enqueue step
 * is not allowed to call cudaMalloc. fa_bwd_noalloc computes exactly what fa_bwd
 * computes, with the same arguments except the workspace: its row
 * statistics go to a fixed 8 MiB array in device memory that the library holds on every
 * GPU that loads it, until the process exits. It calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *   Limit: 2 * B * H * Np * 4 bytes must fit in 8 MiB, i.e. B * H * Np <= 1,048,576
 *   with Np = N rounded up to a multiple of 128; larger problems return
 *   FA_ERR_WORKSPACE before anything is launched.
 *   Set-up: in host code the array's name is only a host-side stand-in, so the first
 *   call in each CUDA context (with that context current) looks up the array's device
 *   address with cudaGetSymbolAddress. The address belongs to that context, so it is
 *   cached by the driver's context id: a second context on the same device, or the new
 *   primary context after a cudaDeviceReset, gets its own lookup. Make the first call in a
 *   context before any stream capture.
 *   Sharing: every call on a device uses the same array. The statistics are fully
 *   rewritten by each call, so nothing carries over, but calls whose kernels overlap
 *   on the GPU (different streams, or several threads) race on the array: serialise
 *   them.
 */
fa_status_t fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                           const void *dout, const float *lse, void *dq, void *dk, void *dv,
                           int B, int H, int N, int d, float scale, int causal,
                           fa_window_t window, void *stream);

/* Static, human-readable name of a status code (never NULL). */
const char *fa_status_string(fa_status_t status);

/*
 * Synchronises `stream`, then reads and clears the device status word the kernels of
 * the current device write when a bounded wait runs out. Returns FA_ERR_TIMEOUT if it
 * was set, FA_ERR_CUDA if the synchronisation failed, FA_OK otherwise.
 */
fa_status_t fa_debug_status(void *stream);

/*
 * Test hook for the timeout path (no GPU fault is involved). fault = 1: fa_fwd calls
 * made afterwards in this process launch with their copy warp skipping every V tile, so
 * the MMA warps' bounded waits for V run out after about two seconds; the kernel then
 * abandons its work, drains the copies and products already in flight, frees its tensor
 * memory and exits, and fa_debug_status() returns FA_ERR_TIMEOUT. fault = 0 restores
 * normal operation. Other values return FA_ERR_INVALID_ARG.
 */
fa_status_t fa_debug_set_fault(int fault);

/* Library version, major * 10000 + minor * 100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
