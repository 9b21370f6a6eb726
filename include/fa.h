/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library (libfa.so).
 *
 * The operation is exact scaled dot-product attention
 *
 *     O = softmax(scale * Q K^T + mask) V
 *
 * as defined on the FlashAttention case-study slides (nmj0.github.io,
 * "Attention is where tokens meet"), computed as on the slide "FlashAttention:
 * the idea": one fused, tiled kernel that never writes the score matrix S or
 * the probability matrix P to device memory, combining key tiles with the
 * running (m, l, o) update of "Online softmax: divide once, at the end" and
 * dividing by l once per row.  The backward pass recomputes the scores from
 * the saved row log-sum-exp instead of storing them (lastdictionary.com,
 * "FlashAttention", definition paragraph).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers    Every tensor pointer is DEVICE memory owned by the caller and
 *             must be 16-byte aligned.  The library keeps no pointer after a
 *             call returns and allocates no device memory per call (the
 *             backward's scratch comes from the caller's `workspace`).
 * Layout      q, o, dO, dq: [B, H, Nq, D]; k, v, dk, dv: [B, H, Nk, D];
 *             contiguous, row-major, D fastest (the "reshape to [h x n x d_k]"
 *             of the slides' "Queries, keys and values").  All share `dtype`.
 *             lse: [B, H, Nq] float32.  key_bias: [B, Nk] float32.
 * dtype       FA_F16 or FA_BF16 (storage and tensor-core input type; all
 *             accumulation is float32).
 * D           64 or 128.
 * Sizes       B, H >= 1; Nq, Nk >= 0.  Nq == 0 is a no-op (no pointer is
 *             read).  Nk == 0 makes every row empty (O = 0, LSE = -inf);
 *             k, v (and dk, dv) may then be NULL.
 * scale       Multiplies Q K^T before the mask; finite and > 0 (pass
 *             1/sqrt(D) for standard attention).
 * causal      0 or 1.  Bottom-right aligned: key j is visible to query i iff
 *             j <= i + (Nk - Nq), which is j <= i when Nq == Nk.
 * key_bias    Optional (NULL = none).  Additive per-key term added to the
 *             scaled scores of batch b, shared by all heads and queries;
 *             entries are finite or -inf (-inf = masked key).
 * Empty rows  A query row that sees no key gets O = 0 and LSE = -inf.
 * stream      A cudaStream_t passed as void*; NULL = the legacy default
 *             stream.  Work is enqueued asynchronously on it.
 * Errors      Argument errors are reported synchronously, before anything is
 *             launched.  Kernel launch failures return FA_ERR_CUDA.  A device
 *             wait that exceeds its time limit makes the kernel give up
 *             cleanly and latch FA_ERR_DEVICE_TIMEOUT in a per-device error
 *             word, read and cleared by fa_device_status().
 * Threads     Calls on different streams may run concurrently, except
 *             fa_bwd_noalloc(), whose calls all share one scratch array
 *             (see its description below).
 */
#ifndef FA_H
#define FA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,     /* null/misaligned pointer, bad size, bad scale */
    FA_ERR_UNSUPPORTED = 2,     /* D not in {64, 128}, unknown dtype, no sm_100 device */
    FA_ERR_CUDA = 3,            /* a CUDA runtime/driver call failed */
    FA_ERR_DEVICE_TIMEOUT = 4,  /* a bounded device-side wait gave up */
    FA_ERR_WORKSPACE = 5,       /* backward workspace missing or too small */
    FA_ERR_INTERNAL = 6         /* a kernel's own layout check failed; it did no work */
} fa_status;

typedef enum { FA_F16 = 0, FA_BF16 = 1 } fa_dtype;

/*
 * Forward pass.  Writes o [B,H,Nq,D] (dtype) and lse [B,H,Nq] (float32,
 * natural log of sum_j exp(scale * q_i . k_j + bias_j) over visible keys).
 * Inputs are read once per query tile from HBM; S and P live only on chip.
 */
int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
           int B, int H, int Nq, int Nk, int D, int causal, float scale,
           int dtype, const float *key_bias, void *stream);

/*
 * Forward pass with 8-bit floating-point inputs, the low-precision tensor-core
 * path the lastdictionary.com "FlashAttention" entry credits to
 * FlashAttention-3 (definition paragraph: "exploited asynchrony and FP8").
 *   q, k, v    [B,H,N,D] OCP FP8 E4M3 values (1 byte each, the finite-only
 *              "e4m3fn" encoding); D must be 128.  The attention inputs are
 *              q_descale * q, k_descale * k and v_descale * v (per-tensor
 *              scale factors, finite and > 0; 1 for unscaled data).
 *   o          [B,H,Nq,D] bf16;  lse [B,H,Nq] float32 as in fa_fwd().
 * S = Q K^T runs on the tensor cores with E4M3 operands and an fp32
 * accumulator; the probabilities P are rounded to E4M3 (round to nearest
 * even) for the P V product, while the row sum l adds the unrounded fp32
 * values.  Everything else (masking, causal alignment, empty rows, errors)
 * is as in fa_fwd().  D != 128 returns FA_ERR_UNSUPPORTED.
 */
int fa_fwd_fp8(const void *q, const void *k, const void *v, void *o, float *lse,
               int B, int H, int Nq, int Nk, int D, int causal, float scale,
               float q_descale, float k_descale, float v_descale,
               const float *key_bias, void *stream);

/*
 * Split-KV forward, for few query rows and many keys (decoding): the keys are
 * cut into num_splits contiguous ranges of whole 128-key tiles, each range is
 * processed by its own CTAs into a partial (O_s, LSE_s) in fp32, and a second
 * kernel merges the partials with the associative log-sum-exp merge
 *   LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s
 * (the "secretly associative" softmax merge of the algebra digest,
 * setupai.cc, "Mastering FlashAttention: The Algebraic Foundation").  Same
 * arguments, layouts and results as fa_fwd() plus:
 *   num_splits   1 .. 256 (1 is allowed and equals fa_fwd());
 *   workspace    device memory of fa_fwd_splitkv_workspace_bytes() bytes,
 *                16-byte aligned, caller-owned; contents on entry irrelevant.
 * A split whose keys are all masked for a row contributes LSE_s = -inf.
 */
size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int Nk, int D, int num_splits);

/*
 * A num_splits for fa_fwd_splitkv() on these sizes (host arithmetic only, no
 * device call unless num_sms is 0).  The forward runs units of 256 query rows
 * per (b, h); with few units the SMs idle, and splitting the keys multiplies
 * the units.  The count minimises waves * (key tiles per split + 1), where
 * waves = ceil(units * splits / num_sms) and the +1 charges each unit's fixed
 * cost (Q load, pipeline fill, partial write) as one key tile; ties go to
 * fewer splits.  Returns 1 when the units already fill the SMs, when there is
 * a single key tile, or for invalid sizes.  num_sms: the device's SM count,
 * or 0 for that of the current device (148 on B200).
 */
int fa_splitkv_num_splits(int B, int H, int Nq, int Nk, int num_sms);
int fa_fwd_splitkv(const void *q, const void *k, const void *v, void *o, float *lse,
                   int B, int H, int Nq, int Nk, int D, int causal, float scale,
                   int dtype, const float *key_bias, int num_splits, void *workspace,
                   size_t workspace_bytes, void *stream);

/*
 * Bytes of device scratch fa_bwd() needs for these sizes: the per-row term
 * D_i = rowsum(dO * O), one float32 per query row (O(n) memory).
 */
size_t fa_bwd_workspace_bytes(int B, int H, int Nq, int Nk, int D);

/*
 * Backward pass of L = sum(O * dO): writes dq, dk, dv (dtype, same layouts as
 * q, k, v).  o and lse must be the outputs of fa_fwd() for the same inputs.
 * Scores and probabilities are recomputed tile by tile from q, k and lse;
 * no atomics are used, so the result is bitwise reproducible.
 * workspace: device memory of at least fa_bwd_workspace_bytes() bytes,
 * 16-byte aligned, owned by the caller; its contents on entry do not matter.
 * The mask and key_bias receive no gradient.
 */
int fa_bwd(const void *q, const void *k, const void *v, const void *o,
           const float *lse, const void *dO, void *dq, void *dk, void *dv,
           int B, int H, int Nq, int Nk, int D, int causal, float scale,
           int dtype, const float *key_bias, void *workspace,
           size_t workspace_bytes, void *stream);

/*
 * Forward and backward with a general additive mask: the "+ mask" of the SDPA
 * formula in full ("Attention is where tokens meet"),
 *     S = scale * Q K^T + M,   O = softmax(S) V,
 * with M a float32 [mask_B, mask_H, Nq, ldm] array in device memory (row i,
 * columns [0, Nk) of plane (b, h) are M_ij for batch b, head h):
 *   mask_B   1 (the same planes for every batch) or B;
 *   mask_H   1 (the same plane for every head) or H;
 *   ldm      row stride in elements: ldm >= Nk, a multiple of 4 (rows start
 *            16-byte aligned); columns [Nk, ldm) are never read.
 * Entries are finite or -inf (-inf = key hidden from that query).  causal may
 * be combined with the mask; there is no separate key bias (fold it into M).
 * A row whose keys are all hidden gets O = 0 and LSE = -inf.  The mask
 * receives no gradient.  Arguments, layouts and results are otherwise those
 * of fa_fwd() and fa_bwd(); the mask adds Nq * Nk * 4 bytes of reads per
 * plane, so these calls are bound by memory bandwidth rather than the tensor
 * cores.  Invalid mask arguments return FA_ERR_INVALID_ARG.
 *
 * tile_flags (optional, NULL = visit every tile) is the mask's tile summary
 * written by fa_mask_tile_flags() for the same mask and sizes: device bytes
 * [mask_B * mask_H, ceil(Nq/128), ceil(Nk/128)], 1 where a 128 x 128 tile
 * has an entry above -inf.  Tiles marked 0 contribute exactly nothing and are
 * skipped (not loaded, not multiplied), so masks that hide whole blocks --
 * packed documents, sliding windows -- cost only their visible tiles.  One
 * summary serves the forward and the backward and every call with that mask.
 */
size_t fa_mask_tile_flags_bytes(int mask_B, int mask_H, int Nq, int Nk);
int fa_mask_tile_flags(const float *mask, int mask_B, int mask_H, int Nq, int Nk,
                       long long ldm, unsigned char *flags, size_t flags_bytes, void *stream);
int fa_fwd_mask(const void *q, const void *k, const void *v, void *o, float *lse,
                int B, int H, int Nq, int Nk, int D, int causal, float scale, int dtype,
                const float *mask, int mask_B, int mask_H, long long ldm,
                const unsigned char *tile_flags, void *stream);
int fa_bwd_mask(const void *q, const void *k, const void *v, const void *o,
                const float *lse, const void *dO, void *dq, void *dk, void *dv,
                int B, int H, int Nq, int Nk, int D, int causal, float scale,
                int dtype, const float *mask, int mask_B, int mask_H, long long ldm,
                const unsigned char *tile_flags, void *workspace, size_t workspace_bytes,
                void *stream);

/*
 * Forward and backward of packed variable-length sequences: num_seqs
 * independent attention problems of different lengths stored one after
 * another along the row axis (the "Nq != Nk / variable lengths" case; each
 * sequence is exact attention as in fa_fwd() / fa_bwd(), with no attention
 * across sequences).
 *   q, o, dO, dq   [H, total_q, D];  k, v, dk, dv  [H, total_k, D];
 *   lse            [H, total_q] float32 (same dtype and D rules as fa_fwd()).
 *   cu_seqlens_q, cu_seqlens_k   DEVICE int32 [num_seqs + 1], non-decreasing,
 *                  starting at 0 and ending at total_q / total_k: sequence b
 *                  owns query rows [cu_q[b], cu_q[b+1]) and key rows
 *                  [cu_k[b], cu_k[b+1]) of every head.
 *   max_seqlen_q, max_seqlen_k   upper bounds of the sequence lengths (they
 *                  size the grid; a longer sequence is cut at the bound).
 * causal is bottom-right aligned within each sequence.  Rows of the packed
 * tensors that belong to no sequence are not written.  The library reads the
 * tables only on the device and clamps every start and length into [0, total]
 * and [0, max_seqlen], so a malformed table gives wrong values, never an
 * access outside the tensors.  The backward's workspace must hold
 * fa_bwd_workspace_bytes(1, H, total_q, total_k, D) bytes.
 */
int fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                  const int *cu_seqlens_q, const int *cu_seqlens_k, int num_seqs, int H,
                  int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int D,
                  int causal, float scale, int dtype, void *stream);
int fa_bwd_varlen(const void *q, const void *k, const void *v, const void *o,
                  const float *lse, const void *dO, void *dq, void *dk, void *dv,
                  const int *cu_seqlens_q, const int *cu_seqlens_k, int num_seqs, int H,
                  int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int D,
                  int causal, float scale, int dtype, void *workspace,
                  size_t workspace_bytes, void *stream);

/*
 * Largest B * H * Nq that fa_bwd_noalloc() accepts.
 */
#define FA_BWD_NOALLOC_MAX_ROWS 1048576

/*
 * fa_bwd() for callers that cannot allocate device memory: services that
 * reserve their whole memory budget at start-up and allow no allocation while
 * serving, plugin hosts that give a library only its input and output
 * buffers, and latency-critical paths that cannot afford an allocation or its
 * failure.  No page describes this entry point; it exists for those callers.
 *
 * Arguments, layouts and results are those of fa_bwd() without the workspace:
 * the per-row scratch lives in a fixed array compiled into the library
 * (4 * FA_BWD_NOALLOC_MAX_ROWS bytes plus 256, held on every GPU that loads the
 * library until the process exits).  Nothing is allocated by this call.
 *   - Argument errors are reported as by fa_bwd(); then
 *     B * H * Nq > FA_BWD_NOALLOC_MAX_ROWS returns FA_ERR_WORKSPACE; both
 *     before any CUDA call.
 *   - The first call on a device asks the CUDA runtime for the array's device
 *     address (cudaGetSymbolAddress); make that first call before any stream
 *     capture begins.
 *   - All calls share the one array and every call writes the parts it reads,
 *     so what an earlier call left there does not matter; but two calls whose
 *     work overlaps on the GPU (different streams without ordering between
 *     them) race on it and may return wrong gradients.
 */
int fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                   const float *lse, const void *dO, void *dq, void *dk, void *dv,
                   int B, int H, int Nq, int Nk, int D, int causal, float scale,
                   int dtype, const float *key_bias, void *stream);

/* Static, human-readable name of a status code (never NULL). */
const char *fa_status_string(int status);

/*
 * Synchronises `stream`, then returns and clears the current device's error
 * word: FA_OK, or FA_ERR_DEVICE_TIMEOUT if a kernel gave up on a wait since
 * the last call.  FA_ERR_CUDA if the synchronisation itself failed.
 */
int fa_device_status(void *stream);

/*
 * Number of kernels this library has launched in this process (all devices,
 * all streams) since it was loaded; for accounting in benchmarks.
 */
unsigned long long fa_launch_count(void);

/*
 * Per-kernel device timing, a measurement aid.  While enabled on the calling
 * host thread, every kernel the library launches from that thread is
 * bracketed by two CUDA events recorded on its stream.  fa_profile_read()
 * waits for those events, writes each kernel's elapsed milliseconds (launch
 * order) into ms[0 .. *count) and, if names is not NULL, a static kernel name
 * into names[i]; then it forgets them.  Records beyond `capacity` are dropped.
 * Profiling stays enabled until fa_profile_enable(0).
 */
int fa_profile_enable(int on);
int fa_profile_read(float *ms, const char **names, int capacity, int *count);

/*
 * Self-test of the bounded-wait mechanism: launches one block that waits on a
 * barrier nothing will ever complete, with a limit of `timeout_us`
 * microseconds; the kernel must give up, latch FA_ERR_DEVICE_TIMEOUT and
 * return.  Returns FA_OK if the launch succeeded (read the outcome with
 * fa_device_status()).
 */
int fa_debug_wait_timeout(unsigned timeout_us, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_H */
