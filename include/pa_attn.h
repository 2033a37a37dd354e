/*
 * pa_attn.h - blockwise (ring-step) attention for NVIDIA B200 (sm_100a).
 *
 * A C ABI whose two core entry points are:
 *
 *   pa_attn_fwd    attention of every query row against ONE key/value chunk,
 *                  returning the normalised partial output O and the natural
 *                  log-sum-exp LSE of the scaled logits over that chunk;
 *   pa_attn_merge  the exact combination of n such partial results, computed
 *                  over disjoint key chunks, into the full-sequence result.
 *
 * Around them: pa_attn_fwd_accum (fold one chunk into a running fp32 O and
 * LSE, the local step of a ring that receives chunks one at a time),
 * pa_attn_fwd_chunks (up to 8 chunks in one launch, no partials),
 * pa_attn_fwd_fp8 / pa_attn_fwd_fp8_dev with pa_quantize_e4m3 (e4m3 inputs),
 * pa_attn_chunks_noalloc (chunks + merge with library-owned static scratch),
 * and the status helpers at the end of this file.
 *
 * Together they are the per-device step of Ring Attention as the diffusers
 * guide "Context parallelism" describes it (section "Ring Attention": each
 * device attends with the K/V block it holds and passes the block on; after a
 * full turn every device has seen the K/V of every token).  Chunks of any
 * length are accepted (section "Ring Anything Attention": blocks are trimmed
 * to their real length before attention, so padding never enters the
 * softmax).  Attention is the non-causal, unmasked scaled-dot-product
 * attention of the guide "Accelerate inference" (section "Scaled dot product
 * attention"; inference only, attn_mask None), computed on bf16 inputs (same
 * guide, section "Model data type") with fp32 accumulation.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Layouts are contiguous, row-major, head dimension innermost:
 *     q, o   [B, H, Nq, d] bf16          k, v   [B, H, Nk, d] bf16
 *     (q, k, v are one-byte e4m3 codes in the fp8 entry points; o stays bf16)
 *     lse    [B, H, Nq]    fp32, natural log
 * - All tensor pointers are DEVICE pointers on the current CUDA device, owned
 *   and allocated by the caller.  The library allocates no memory in any call.
 *   Inputs and outputs must not overlap.
 * - q, k, v, o and o_parts must be 16-byte aligned (TMA / vector access);
 *   lse and lse_parts 4-byte aligned.
 * - d must be 64 or 128 (128 for the e4m3 entry points).
 * - `stream` is a cudaStream_t (0 = legacy default stream).  Calls are fully
 *   asynchronous: they validate arguments on the host, enqueue kernels on
 *   `stream` and return.  They never synchronise the host and never copy
 *   between host and device.
 * - Return values: PA_OK or a negative PA_ERR_* code for errors the host can
 *   see before or at launch.  Errors raised later on the device (a bounded
 *   wait that gave up, a bad value read on the device) are reported by
 *   pa_poll_device_status(); the outputs of the work that raised one are
 *   undefined.  A caller that needs to know polls after synchronising.
 */
#ifndef PA_ATTN_H_
#define PA_ATTN_H_

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define PA_OK 0
#define PA_ERR_INVALID_ARG (-1) /* null pointer, size out of range, non-finite or non-positive scale,
                                   host (non-device) pointer, overlapping input/output */
#define PA_ERR_UNSUPPORTED (-2) /* d not in {64, 128}, device not sm_100, B*H > 65535 */
#define PA_ERR_MISALIGNED (-3)  /* a pointer breaks the alignment rule above */
#define PA_ERR_CUDA (-4)        /* CUDA runtime / driver error; see pa_last_error() */
#define PA_ERR_TIMEOUT (-5)     /* a device-side bounded wait gave up (from pa_poll_device_status) */
#define PA_ERR_BAD_INPUT (-6)   /* a value read on the device (a dequantisation scale, a quantiser's
                                   amax) was not finite or not positive (from pa_poll_device_status) */

/* Flags of pa_attn_fwd_accum. */
#define PA_ACCUM_FIRST 1 /* no incoming state: o_acc / lse_acc are only written */
#define PA_ACCUM_FINAL 2 /* write the result as bf16 into o (and lse_acc), not into o_acc */

/*
 * pa_attn_fwd - attention of Q against one K/V chunk.
 *
 * For each b < B, h < H and query row i < Nq, over the keys j < Nk of the
 * chunk (diffusers "Context parallelism", section "Ring Attention"):
 *     s_ij    = scale * sum_c q[b,h,i,c] k[b,h,j,c]
 *     lse[i]  = ln sum_j exp(s_ij)
 *     o[i,:]  = sum_j exp(s_ij - lse[i]) v[b,h,j,:]        (rounded to bf16)
 *
 * q      [B,H,Nq,d] bf16, device, 16-byte aligned       (input)
 * k, v   [B,H,Nk,d] bf16, device, 16-byte aligned       (input)
 * o      [B,H,Nq,d] bf16, device, 16-byte aligned       (output, fully written)
 * lse    [B,H,Nq]   fp32, device, 4-byte aligned        (output, fully written)
 * B, H   >= 1, B*H <= 65535
 * Nq     >= 0 (0 is a no-op returning PA_OK); Nk >= 1 (an empty chunk has no
 *        attention: pass it to pa_attn_merge with lse = -inf instead)
 * d      64 or 128
 * scale  finite and > 0 (typically 1/sqrt(d))
 * stream cudaStream_t
 *
 * Errors: PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_MISALIGNED before
 * anything is enqueued; PA_ERR_CUDA if the launch fails.
 */
int pa_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                int Nq, int Nk, int d, float scale, void* stream);

/*
 * pa_attn_fwd_accum - fold the attention over one more K/V chunk into a
 * running result.
 *
 * The step a device takes each time a block arrives on the ring (diffusers
 * "Context parallelism", section "Ring Attention": attend with the block held,
 * pass it on; once every block has been seen the result is the full-sequence
 * attention).  The running state is the result over the chunks folded so far,
 * kept in fp32: a normalised output o_acc and its natural-log LSE lse_acc.
 * One call replaces it by the merge (as pa_attn_merge defines it) of that
 * state with the attention of q over this chunk's keys:
 *     o_acc, lse_acc  <-  merge((o_acc, lse_acc), attention(q, k, v))
 * without rounding any partial output to bf16 and without a separate merge.
 *
 * q, k, v   as pa_attn_fwd (bf16, device, 16-byte aligned)           (input)
 * o_acc     [B,H,Nq,d] fp32, device, 16-byte aligned     (state: read unless
 *           PA_ACCUM_FIRST, written unless PA_ACCUM_FINAL)
 * lse_acc   [B,H,Nq]   fp32, device, 4-byte aligned      (state: read unless
 *           PA_ACCUM_FIRST, always written).  A row whose lse_acc is -inf
 *           counts as empty (its o_acc row is not read).  Values must
 *           otherwise be finite.
 * o         [B,H,Nq,d] bf16, device, 16-byte aligned: with PA_ACCUM_FINAL
 *           the final output goes here (and the final LSE to lse_acc);
 *           without it o must be NULL
 * flags     0, PA_ACCUM_FIRST, PA_ACCUM_FINAL or both (both = pa_attn_fwd
 *           with the LSE written to lse_acc)
 * B, H, Nq, Nk, d, scale, stream   as pa_attn_fwd
 *
 * The state is read and written in place, row by row, by the thread that
 * owns the row; no other call may use it concurrently.  Errors: as
 * pa_attn_fwd; PA_ERR_INVALID_ARG for unknown flags, a missing o with
 * PA_ACCUM_FINAL or an o without it, and overlapping buffers.
 */
int pa_attn_fwd_accum(const void* q, const void* k, const void* v, float* o_acc, float* lse_acc, void* o,
                      int B, int H, int Nq, int Nk, int d, float scale, int flags, void* stream);

/*
 * pa_attn_fwd_fp8 - pa_attn_fwd with e4m3 (fp8) Q, K and V.
 *
 * The pages' fp8 path quantises activations dynamically to fp8 (diffusers
 * "ParaAttention" guide, fp8 section); this entry applies the same storage
 * format to the attention inputs.  Each input is one scaled e4m3 tensor:
 *     q_real = q_scale * decode(q),  k_real = k_scale * decode(k),
 *     v_real = v_scale * decode(v)              (decode: OCP E4M3FN)
 * and o, lse are the attention of pa_attn_fwd over q_real, k_real, v_real.
 * Q.K^T and P.V run on the tensor cores in e4m3 with fp32 accumulation; the
 * softmax is fp32 and P is rounded to e4m3 (range 2^-9 .. 448) before P.V,
 * which is the dominant error: about 2^-4 relative per weight.
 *
 * q        [B,H,Nq,d] e4m3 (1 byte), device, 16-byte aligned     (input)
 * k, v     [B,H,Nk,d] e4m3, device, 16-byte aligned              (input)
 * q_scale, k_scale, v_scale   finite and > 0
 * o        [B,H,Nq,d] bf16; lse [B,H,Nq] fp32                      (outputs)
 * d        128 only (PA_ERR_UNSUPPORTED otherwise)
 * B, H, Nq, Nk, scale, stream   as pa_attn_fwd
 *
 * Errors: as pa_attn_fwd; PA_ERR_INVALID_ARG for a bad scale.
 */
int pa_attn_fwd_fp8(const void* q, const void* k, const void* v, float q_scale, float k_scale,
                    float v_scale, void* o, float* lse, int B, int H, int Nq, int Nk, int d,
                    float scale, void* stream);

/*
 * pa_attn_fwd_fp8_dev - pa_attn_fwd_fp8 with the three dequantisation scales
 * read from device memory (each a float, e.g. written by pa_quantize_e4m3),
 * so that quantising and attending need no host synchronisation.
 *
 * q_scale, k_scale, v_scale   device pointers to one float each, 4-byte aligned;
 *                             read on the device, where a value that is not
 *                             finite and > 0 raises PA_ERR_BAD_INPUT in the
 *                             device status word (outputs then undefined)
 * everything else             as pa_attn_fwd_fp8
 *
 * Errors: as pa_attn_fwd_fp8; PA_ERR_INVALID_ARG for a null or host scale
 * pointer, PA_ERR_MISALIGNED for a misaligned one.
 */
int pa_attn_fwd_fp8_dev(const void* q, const void* k, const void* v, const float* q_scale,
                        const float* k_scale, const float* v_scale, void* o, float* lse, int B, int H,
                        int Nq, int Nk, int d, float scale, void* stream);

/*
 * pa_quantize_e4m3 - per-tensor e4m3 quantisation of a bf16 tensor.
 *
 *     amax  = max_i |x[i]|
 *     scale = amax / 448 in fp32 (1 if amax = 0)     (written to *scale)
 *     inv   = 448 / amax in fp32 (1 if amax = 0)
 *     q[i]  = e4m3 nearest to x[i] * inv (fp32 multiply), ties to even,
 *             saturated to +-448                 (OCP E4M3FN codes)
 * so that x ~= scale * decode(q); *scale is written on the device.  This is
 * the dynamic per-tensor fp8 quantisation the pages apply to activations
 * (diffusers "ParaAttention" guide, fp8 section), as input to
 * pa_attn_fwd_fp8_dev.
 *
 * x      n bf16 values, device, 16-byte aligned             (input)
 * q      n bytes, device, 16-byte aligned                    (output)
 * scale  one float, device, 4-byte aligned                   (output; also
 *        used as the reduction word while the call runs)
 * n      >= 1
 *
 * Errors: PA_ERR_INVALID_ARG (null, n < 1, overlapping buffers, host memory),
 * PA_ERR_MISALIGNED, PA_ERR_CUDA.  An Inf or NaN in x leaves no usable scale:
 * it raises PA_ERR_BAD_INPUT in the device status word.  Three kernels and
 * one memset are enqueued on `stream`; nothing is allocated.
 */
int pa_quantize_e4m3(const void* x, long long n, void* q, float* scale, void* stream);

/*
 * pa_attn_fwd_chunks - attention of Q over several K/V chunks in one launch.
 *
 * The local loop of Ring Attention fused (diffusers "Context parallelism",
 * section "Ring Attention": attend to each block held, and after all blocks
 * the result is the full-sequence attention): the keys are the concatenation
 * of the chunks, in order, so o and lse are the exact attention over all of
 * them, the same as pa_attn_fwd per chunk followed by pa_attn_merge, with no
 * partial results written.  Chunks of unequal, ragged length are accepted
 * (section "Ring Anything Attention": each block keeps its real length).
 *
 * q            [B,H,Nq,d] bf16, device, 16-byte aligned               (input)
 * k_chunks[c], v_chunks[c]  [B,H,nk_chunks[c],d] bf16, device, 16-byte
 *              aligned; the three arrays are HOST arrays of n_chunks entries
 * n_chunks     1 .. 8; nk_chunks[c] >= 1
 * o, lse, B, H, Nq, d, scale, stream   as pa_attn_fwd
 *
 * Errors: as pa_attn_fwd, for every chunk.
 */
int pa_attn_fwd_chunks(const void* q, const void* const* k_chunks, const void* const* v_chunks,
                       const int* nk_chunks, int n_chunks, void* o, float* lse, int B, int H, int Nq, int d,
                       float scale, void* stream);

/*
 * pa_attn_merge - combine n partial results over disjoint key chunks.
 *
 * For every row r of the B*H*N rows (same section as above: the per-block
 * results combine into the exact full attention):
 *     M = max_p lse_parts[p,r];  w_p = exp(lse_parts[p,r] - M);  L = sum_p w_p
 *     o[r,:] = sum_p w_p o_parts[p,r,:] / L;     lse[r] = M + ln L
 * A part with lse = -inf carries no weight and its o_parts row is not read;
 * a row whose parts are all -inf gets o = 0 and lse = -inf.  n_parts = 1 is a
 * copy.
 *
 * o_parts   [n_parts,B,H,N,d] bf16, device, 16-byte aligned   (input)
 * lse_parts [n_parts,B,H,N]   fp32, device, 4-byte aligned    (input)
 * o         [B,H,N,d] bf16, device, 16-byte aligned           (output)
 * lse       [B,H,N]   fp32, device, 4-byte aligned            (output)
 * n_parts >= 1; B, H >= 1; N >= 0 (0 is a no-op); d 64 or 128.
 *
 * Errors: as pa_attn_fwd.
 */
int pa_attn_merge(const void* o_parts, const float* lse_parts, int n_parts, void* o, float* lse,
                  int B, int H, int N, int d, void* stream);

/*
 * pa_residual_diff - First Block Cache's residual difference.
 *
 * diffusers "ParaAttention" guide, section "First Block Cache": the change of
 * the first transformer block's residual output between two denoising steps
 * approximates the change of the model's output, and the cached residuals
 * are reused while it stays below a threshold (0.08 by default for FLUX).
 * The guide gives no formula; this computes the relative L1 difference
 *     out[0] = sum_i |cur_i - prev_i| / sum_i |prev_i|
 * over the n elements (0 when both sums are 0, +inf when only the
 * denominator is), accumulated in fp32 in a fixed order: the same inputs give
 * the same bits on the same device.
 *
 * cur, prev  [n] bf16, device, 16-byte aligned                (inputs; may be the same buffer)
 * out        [1] fp32, device, 4-byte aligned                 (output)
 * n >= 1.
 *
 * Two launches on `stream`.  The block partials live in a small array the
 * library reserves statically on each GPU: calls that overlap on the GPU
 * (different streams, no ordering) race on it; calls ordered on one stream
 * do not.
 *
 * Errors: PA_ERR_INVALID_ARG (null pointer, n < 1, out overlapping an input),
 * PA_ERR_MISALIGNED, PA_ERR_CUDA (including pointers that are not device
 * memory).
 */
int pa_residual_diff(const void* cur, const void* prev, long long n, float* out, void* stream);

/*
 * pa_attn_chunks_noalloc - attention of Q over several K/V chunks, allocating
 * nothing.
 *
 * Not part of the method: the pages have no counterpart for this call.  It is
 * for callers that cannot allocate device memory on the call path: code that
 * runs under a framework's caching allocator with a fixed memory budget,
 * loops where cudaMalloc's implicit device-wide synchronisation is not
 * acceptable, or plug-ins that are handed only their input and output
 * buffers.  It gives the same result as pa_attn_fwd on each chunk into
 * caller-allocated partial buffers followed by pa_attn_merge, but keeps the
 * partials in a fixed 32 MiB array that the library reserves statically on
 * every GPU that loads it (for as long as the process lives).
 *
 * q            [B,H,Nq,d] bf16, device, 16-byte aligned               (input)
 * k_chunks[c], v_chunks[c]  [B,H,nk_chunks[c],d] bf16, device,
 *              16-byte aligned, c < n_chunks; the three arrays are HOST arrays
 * o, lse       as pa_attn_fwd                                         (output)
 * n_chunks     1 .. 64; with n_chunks >= 2 the partials need
 *              round_up(n*B*H*Nq*d*2, 256) + n*B*H*Nq*4 bytes, at most 32 MiB
 *              (PA_ERR_INVALID_ARG beyond it, before anything is enqueued)
 * B, H, Nq, d, scale, stream   as pa_attn_fwd; nk_chunks[c] >= 1
 *
 * Calls no allocating routine of any kind.  The first call on a device looks
 * up the array's device address (once per device, with that device current);
 * make that first call before any stream capture.  All calls on a device share
 * the one array: calls whose work overlaps on the GPU (different streams, or
 * other host threads) race on it and must be serialised by the caller.  The
 * array keeps the last call's contents; each call writes every partial it
 * reads, so nothing needs clearing.  Errors as pa_attn_fwd.
 */
int pa_attn_chunks_noalloc(const void* q, const void* const* k_chunks, const void* const* v_chunks,
                           const int* nk_chunks, int n_chunks, void* o, float* lse, int B, int H, int Nq,
                           int d, float scale, void* stream);

/* Static, human-readable name of a status code. */
const char* pa_status_string(int code);

/*
 * Detail of the last PA_ERR_* returned on the calling host thread (the CUDA
 * error string for PA_ERR_CUDA, the failed check otherwise).  The pointer
 * stays valid until the next library call on this thread.
 */
const char* pa_last_error(void);

/*
 * Read and clear the device status word of the current device.  Kernels set
 * it (first error wins) when a bounded wait inside them gives up (the kernel
 * then releases its resources and exits instead of hanging; the outputs it
 * did not write keep their old contents) or when they read a bad value.
 * Returns PA_OK, PA_ERR_TIMEOUT, PA_ERR_BAD_INPUT, or PA_ERR_CUDA if the word
 * could not be read.  This call synchronises with the device (it copies 4
 * bytes device -> host): call it after the work of interest has completed,
 * never on a hot path.
 */
int pa_poll_device_status(void);

/*
 * Exercise the bounded-wait path on the device: launch one CTA that waits on
 * a shared-memory barrier nothing will ever complete, with a limit of
 * `limit_us` microseconds (1 .. 1000000).  The wait gives up, the kernel
 * records PA_ERR_TIMEOUT in the device status word and exits normally; the
 * CUDA context stays usable.  Used by tests of the failure path.
 */
int pa_selftest_timeout(int limit_us, void* stream);

/*
 * Limit of every device-side barrier wait, in milliseconds (1 .. 600000;
 * default 5000), for launches made after the call, process-wide.  A wait that
 * makes no progress for this long gives up and reports PA_ERR_TIMEOUT.  Raise
 * it where the GPU is time-sliced among many processes and a kernel may be
 * held off the GPU for long stretches.  Returns PA_OK or PA_ERR_INVALID_ARG.
 */
int pa_set_wait_limit_ms(int ms);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_ATTN_H_ */
