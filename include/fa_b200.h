/*
 * fa_b200.h -- C ABI of the B200 (sm_100a) fused exact-attention forward library.
 *
 * The library computes, for every batch b, query head hq and query row i,
 *
 *     O[b,hq,i,:] = sum_j softmax_j( scale * q_i . k_j  [+ causal mask] ) * v_j
 *     LSE[b,hq,i] = ln sum_j exp( scale * q_i . k_j )          (admissible j only)
 *
 * i.e. softmax(Q K^T / sqrt(d_k)) V from the page "FlashAttention (DE)", section
 * "Problematik der Standard-Attention", with the scale passed explicitly, plus the
 * per-row natural-log normaliser.  The N x N score matrix never reaches device memory:
 * Q/K/V are tiled through shared memory and tensor memory and an online softmax keeps a
 * running maximum and sum per row (same page, sections "Tiling und blockweise
 * Verarbeitung", "Online-Softmax-Berechnung" and "Zusammenfassen von Operationen in
 * einem CUDA-Kernel").  The result is exact up to floating-point rounding, as the
 * pages state for FlashAttention.
 *
 * Layout (all tensors contiguous, row-major, device memory of the current device):
 *   q : [B, Hq,  Nq, d]      k, v : [B, Hkv, Nk, d]
 *   o : [B, Hq,  Nq, d]      lse  : [B, Hq,  Nq]  (fp32)
 * Grouped-query / multi-query attention: Hq must be a multiple of Hkv and query head hq
 * reads K/V head hq / (Hq / Hkv) (consecutive query heads share a K/V head).
 * Causal masking admits key j for query i iff j <= i + (Nk - Nq): with Nq == Nk that is
 * j <= i, and otherwise the queries are taken as the last Nq positions of the Nk keys
 * (bottom-right alignment).  A query row with no admissible key (Nq > Nk) gets O = 0 and
 * LSE = -inf.
 *
 * Ownership: the caller allocates and owns every buffer.  The library keeps no pointer
 * after a call returns and allocates no device memory at call time, except fa_bwd, which
 * allocates and frees its scratch in stream order on the caller's stream (see there).
 * The library's static device memory -- the work counters below and fa_bwd_noalloc's
 * fixed 64 MiB scratch -- is part of its kernels' module: it is resident on every device
 * where the library's kernels are loaded, from the first call on that device until the
 * process exits, whichever entry points are used.
 *
 * Work distribution: the forward and backward kernels run one persistent CTA per SM (the
 * bf16 forward at head dim 256, and at 128 without the causal mask, one cluster of two CTAs
 * per two SMs, each pair sharing its tensor-core products), and the CTAs claim work units
 * from a counter of their launch.  The counters are 4096 pairs
 * of 32-bit words per device in the library's static device memory.  Every launch takes
 * the next pair (round-robin per device) and leaves it at zero when it ends.  So at most
 * 4096 of these launches may be in flight on one device at the same time; more, on
 * different streams, would share counters.  A launch captured into a CUDA graph keeps
 * the pair it was given at capture for every replay: a replay must not run at the same
 * time as any other call of this library on the same device (that call may hold the same
 * pair), or units are skipped or computed twice.
 *
 * Execution: every call validates its arguments on the host first; on a validation error
 * it returns without touching the GPU.  Otherwise it enqueues its kernels on `stream`
 * and returns immediately (asynchronous).  A device-side wait that gave up (see
 * fa_check_device_error) is reported by the next fa_check_device_error call.
 *
 * Thread safety: calls from several host threads are allowed.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream; 0 means the legacy default stream. */
typedef struct CUstream_st *fa_stream_t;

typedef enum fa_status {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,  /* null or misaligned pointer, bad size, bad scale, buffer
                                too small for the given shape or not device memory */
    FA_ERR_UNSUPPORTED = 2,  /* valid request outside what the kernels implement: head
                                dim not 64/128/256, GPU not sm_100, and the limits stated
                                at each entry point */
    FA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed (launch, attribute) */
    FA_ERR_TIMEOUT = 4       /* a bounded device-side wait gave up (see below) */
} fa_status;

typedef enum fa_dtype {
    FA_BF16 = 0,          /* q, k, v bf16 -> o bf16, lse fp32 */
    FA_BF16_OUT_F32 = 1,  /* q, k, v bf16 -> o fp32, lse fp32 */
    FA_E4M3 = 2           /* q, k, v OCP fp8 e4m3 -> o bf16, lse fp32; use fa_fwd_fp8 */
} fa_dtype;

/*
 * Fused attention forward, bf16 inputs, fp32 accumulation.
 *
 *   q, k, v  device pointers to bf16 tensors in the layout above (16-byte aligned)
 *   o        device pointer, bf16 (FA_BF16) or fp32 (FA_BF16_OUT_F32), [B,Hq,Nq,d]
 *   lse      device pointer, fp32 [B,Hq,Nq]: LSE = ln sum_j exp(scale * q_i . k_j)
 *   B, Hq, Hkv, Nq, Nk   >= 1; Hq % Hkv == 0
 *   d        head dimension, 64, 128 or 256
 *   scale    softmax scale (> 0, finite); callers normally pass 1/sqrt(d)
 *   causal   0 or 1
 *   dtype    FA_BF16 or FA_BF16_OUT_F32 (FA_E4M3 is rejected: use fa_fwd_fp8)
 *   stream   CUDA stream of the current device
 *
 * Returns FA_OK once the kernel is enqueued; FA_ERR_INVALID_ARG / FA_ERR_UNSUPPORTED
 * with nothing enqueued; FA_ERR_CUDA if the launch failed.
 */
fa_status fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                 int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                 fa_dtype dtype, fa_stream_t stream);

/*
 * fa_fwd for tensors that live in host memory.  The pages describe the kernel, whose
 * inputs already sit in GPU memory; this call is a transfer pipeline around it for
 * callers whose Q, K, V and results are in host memory.  The problem is cut into chunks of
 * consecutive K/V heads (flattened over the batch) together with the query heads that read
 * them; for every tensor a chunk is one contiguous byte range.  Chunk c's inputs are
 * copied host -> device on an internal stream while the kernel of chunk c-1 runs on
 * `stream` and the outputs of earlier chunks are copied device -> host on a second
 * internal stream, so with pinned host memory the copies in both directions overlap the
 * computation.  The result equals fa_fwd on the same data, bit for bit.
 *
 *   q_host, k_host, v_host   host pointers, bf16, layout as for fa_fwd; read
 *   o_host, lse_host         host pointers, written (o bf16 or fp32 as dtype, lse fp32)
 *   q_dev .. lse_dev         device buffers of fa_fwd's sizes and alignment, owned by the
 *                            caller; they hold the copies and the device-side results
 *   chunks                   number of chunks (an even split, clamped to B*Hkv); 0 lets
 *                            the library size them: as many K/V heads per chunk as fit
 *                            one wave of the kernel's work units, at least one
 *   other arguments as for fa_fwd (dtype FA_BF16 or FA_BF16_OUT_F32)
 *
 * Ordering: nothing touches the buffers before the work already enqueued on `stream` has
 * finished, and work enqueued on `stream` after this call starts only once every copy of
 * it has finished; the call returns once everything is enqueued (with pageable host
 * memory the CUDA runtime may block inside the copies).  The host buffers must stay valid
 * and unmodified until then.  The library allocates no memory per call; it keeps two
 * streams and four events per device, created on first use, and serialises the enqueueing
 * of concurrent calls on one device.  Returns FA_OK; FA_ERR_INVALID_ARG for a null host
 * pointer, chunks < 0 or any argument fa_fwd would reject, with nothing enqueued;
 * FA_ERR_CUDA if a copy or launch could not be enqueued (the caller's stream still waits
 * for what was).
 */
fa_status fa_fwd_host(const void *q_host, const void *k_host, const void *v_host,
                      void *o_host, float *lse_host, void *q_dev, void *k_dev, void *v_dev,
                      void *o_dev, float *lse_dev, int B, int Hq, int Hkv, int Nq, int Nk,
                      int d, float scale, int causal, fa_dtype dtype, int chunks,
                      fa_stream_t stream);

/*
 * fa_fwd with dropout on the attention weights, fused into the kernel: the page "Flash
 * Attention" (section "Zentrale technische Innovationen", the fusion bullet) lists dropout
 * among the operations fused with the softmax.  With P the attention weights of a row,
 *
 *     O_i = sum_j P_ij keep_ij v_j / (1 - thr/256),    thr = round(256 * dropout_p)
 *
 * and LSE as without dropout.  keep_ij = 1 iff byte (j mod 32), little-endian in the four
 * 64-bit words, of the Philox4x64-10 block (Salmon et al., SC'11) for counter
 * (j / 32, i, b*Hq + hq, 0) and key (seed, offset) is >= thr.  The dropout probability is
 * thus thr/256; the same (seed, offset) gives the same mask.
 *
 *   dropout_p   in [0, 1) (else FA_ERR_INVALID_ARG); rounded to a multiple of 1/256
 *   dtype       FA_BF16 or FA_BF16_OUT_F32;  d 64, 128 or 256
 *   other arguments as for fa_fwd
 */
fa_status fa_fwd_dropout(const void *q, const void *k, const void *v, void *o, float *lse,
                         int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                         int causal, float dropout_p, uint64_t seed, uint64_t offset,
                         fa_dtype dtype, fa_stream_t stream);

/*
 * Fused attention forward over a batch of sequences of different lengths, packed without
 * padding: the page "FlashAttention 4: Praxisleitfaden ..." (section "Kompatibilitaet und
 * aktueller Stand") describes variable sequence lengths as batching sequences of
 * different length without padding, addressed through cu_seqlens offsets.
 *
 *   q           bf16 [total_q, Hq, d]   (token-major: the Hq heads of a token adjacent)
 *   k, v        bf16 [total_k, Hkv, d]
 *   o           bf16 or fp32 (dtype) [total_q, Hq, d]
 *   lse         fp32 [Hq, total_q]
 *   cu_seqlens_q, cu_seqlens_k   device int32 arrays of B+1 entries: sequence b has
 *               query tokens cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 and key tokens
 *               cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1.  Entries must be non-decreasing,
 *               start at 0 and end at total_q / total_k.
 *   max_seqlen_q   at least the longest query sequence (work is planned for it)
 *   d           64, 128 or 256;  dtype FA_BF16 or FA_BF16_OUT_F32
 *
 * Each sequence is attended on its own; causal masking is per sequence, bottom-right
 * aligned as above.  The offsets are read on the device: wrong offsets give wrong results
 * but every load and store stays inside the tensors.  Errors as for fa_fwd.
 */
fa_status fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                        const int *cu_seqlens_q, const int *cu_seqlens_k, int B, int Hq,
                        int Hkv, int total_q, int total_k, int max_seqlen_q, int d,
                        float scale, int causal, fa_dtype dtype, fa_stream_t stream);

/*
 * Fused attention forward, fp8 (OCP e4m3) inputs with per-(batch, head) scales, fp32
 * accumulation, bf16 output.  FP8 on the tensor cores is the low-precision variant the
 * page "FlashAttention-3 (DE)" describes (section "Neue Hardwarefaehigkeiten der
 * Hopper-GPU (H100)", FP8 format).
 *
 * The real values are q = descale_q[b*Hq+hq] * e4m3(q8), k = descale_k[b*Hkv+hk] *
 * e4m3(k8), v = descale_v[b*Hkv+hk] * e4m3(v8).  The descale arrays are fp32 device
 * arrays of B*Hq, B*Hkv and B*Hkv entries.  The kernel rounds the softmax numerators P
 * to e4m3 before the P.V product (values in [0, 256]).
 *
 *   d must be 128.  Other arguments as for fa_fwd; o is bf16 [B,Hq,Nq,d].
 */
fa_status fa_fwd_fp8(const void *q, const void *k, const void *v, void *o, float *lse,
                     int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                     int causal, const float *descale_q, const float *descale_k,
                     const float *descale_v, fa_stream_t stream);

/*
 * Backward pass of the bf16 forward above: the gradients of O with respect to Q, K and V
 * for an upstream gradient dO.  The page "Flash Attention" (section "Zentrale technische
 * Innovationen", the recomputation bullet) states that FlashAttention does not keep the
 * attention matrix for the backward pass but computes it again; this call recomputes
 * P = exp(scale * Q K^T - LSE) tile by tile from Q, K and the forward's LSE and forms
 *
 *     dV = P^T dO,   dS = P o (dO V^T - D),   D_i = sum_t dO_it O_it,
 *     dQ = scale * dS K,   dK = scale * dS^T Q
 *
 * (o is the Hadamard product; D_i equals sum_j P_ij (dO V^T)_ij).  Under grouped heads
 * the dK and dV of a K/V head sum the contributions of the query heads that read it.
 *
 *   q, k, v     the forward's inputs, bf16, layout as for fa_fwd
 *   o, lse      the forward's outputs for these inputs (o bf16 [B,Hq,Nq,d], lse fp32)
 *   dout        bf16 [B,Hq,Nq,d], the gradient of the loss with respect to o
 *   dq          bf16 [B,Hq,Nq,d] out;  dk, dv  bf16 [B,Hkv,Nk,d] out
 *   B, Hq, Hkv, Nq, Nk, scale, causal   as for fa_fwd (the causal mask aligned at the
 *   bottom right); d must be 64 or 128.  Query rows that admit no key (causal, Nq > Nk:
 *   O = 0, LSE = -inf) get a zero dQ row and add nothing to dK and dV.
 *
 * All pointers 16-byte aligned (lse 4-byte).  The outputs must not overlap the inputs.
 * Scratch: the call allocates B*Hq*(Nq*d + 2*ceil(Nq/64)*64) * 4 bytes on `stream` (an
 * fp32 dQ accumulator and two per-row vectors) from a stream-ordered memory pool that the
 * library creates per device on first use, and frees it on the same stream.  The pool
 * keeps up to 4 GiB of freed scratch for later calls for the life of the process.  dQ is
 * summed with fp32 reduce-adds whose order varies, so its last bits may differ between
 * runs (dK and dV do not).  Enqueues a memset and three kernels.  Returns FA_OK once
 * enqueued; FA_ERR_INVALID_ARG / FA_ERR_UNSUPPORTED (d not 64 or 128, GPU not sm_100)
 * with nothing enqueued; FA_ERR_CUDA if the scratch allocation or a launch failed.
 */
fa_status fa_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
                 const float *lse, void *dq, void *dk, void *dv, int B, int Hq, int Hkv,
                 int Nq, int Nk, int d, float scale, int causal, fa_stream_t stream);

/*
 * fa_bwd without any allocation at call time.  The pages describe nothing like it: it is
 * an engineering variant for callers that cannot let the library allocate device memory
 * per call (a framework whose own caching allocator holds nearly all of the device's
 * memory, or a service that must keep a fixed footprint).  Arguments, results and errors
 * are those of fa_bwd, except for the scratch: instead of allocating it on `stream`, the
 * call uses one fixed 64 MiB buffer that the library holds per device.  The buffer is a
 * static device array of the library's module, so those 64 MiB are taken on every device
 * where the library's kernels are loaded, by any entry point, until the process exits.
 * The first fa_bwd_noalloc call on a device looks up the buffer's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.  A problem
 * whose scratch, B*Hq*(Nq*d + 2*ceil(Nq/64)*64) * 4 bytes (each part rounded up to 256
 * bytes), does not fit returns FA_ERR_UNSUPPORTED with nothing enqueued.  Every call
 * clears the dQ accumulator part of the buffer before using it.  Calls on the same stream
 * are ordered; calls that may overlap in time on the same device (other streams, other
 * host threads) share the buffer and race, so the caller must serialise them.
 */
fa_status fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                         const void *dout, const float *lse, void *dq, void *dk, void *dv,
                         int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                         int causal, fa_stream_t stream);

/*
 * Per-(batch, head) fp8-e4m3 quantisation of a bf16 tensor, optionally with incoherent
 * processing: the page "FlashAttention-3 (DE)", section "Niedrige Praezision (FP8) mit
 * reduziertem Quantisierungsfehler", multiplies the query and key vectors by a random
 * orthogonal (Hadamard) matrix before quantising them to FP8.  The matrix spreads large
 * entries over all coordinates and, being orthogonal, leaves Q K^T unchanged, so codes
 * made from rotated Q and K can be passed straight to fa_fwd_fp8.  Rotate Q and K with
 * the same signs; quantise V without rotation.
 *
 *   x        device pointer, bf16 [B, H, N, d] (16-byte aligned, finite values)
 *   signs    device pointer to d int8 entries, or NULL for no rotation.  An entry < 0
 *            stands for -1, any other for +1.  With signs every row is replaced by
 *            y = x diag(s) H / sqrt(d), H the Sylvester-Hadamard matrix of order d
 *            (H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]).
 *   x8       device pointer, e4m3 codes [B, H, N, d] (16-byte aligned); must not overlap
 *            x, signs or descale
 *   descale  device pointer, fp32 [B*H]: per slice amax = max |y|, descale = amax / 448,
 *            code = e4m3(y / descale) rounded to nearest even, so y ~ descale * e4m3(code).
 *            A slice of zeros gets descale 1 and zero codes.
 *   B, H, N  >= 1
 *   d        128 (the head dimension of fa_fwd_fp8)
 *
 * The call enqueues one kernel on `stream` (the CTAs that share a slice combine their
 * maxima on chip, so nothing is cleared beforehand).  Returns FA_OK once enqueued; FA_ERR_INVALID_ARG (null, misaligned or
 * undersized buffer, bad size) or FA_ERR_UNSUPPORTED (d != 128, GPU not sm_100) with
 * nothing enqueued; FA_ERR_CUDA if a launch failed.
 */
fa_status fa_quantize_e4m3(const void *x, const int8_t *signs, void *x8, float *descale,
                           int B, int H, int N, int d, fa_stream_t stream);

/*
 * Device-side failure report.  Every wait inside the kernels (on a shared-memory
 * mbarrier filled by a TMA copy or a tensor-core commit) is bounded in time; a wait
 * that runs out sets a device error word, makes the other warps of the CTA stop, drains
 * the CTA's copies in flight, frees its tensor memory and returns.  The outputs of such
 * a call are undefined.
 *
 * fa_check_device_error synchronises `stream`, reads and clears the error word of the
 * current device and returns FA_ERR_TIMEOUT if it was set (FA_ERR_CUDA if the
 * synchronisation itself failed), else FA_OK.
 */
fa_status fa_check_device_error(fa_stream_t stream);

/*
 * Statistics of the online softmax's lazy rescaling.  The page "FlashAttention 4:
 * Praxisleitfaden ...", section "Intelligenteres Online-Softmax-Rescaling in FA4", states
 * that rescaling the accumulator only when the running maximum has moved far (here: by
 * more than 8 in log2 units) needs about ten times fewer rescales than doing so whenever
 * it moves.  The CTA-pair kernel -- fa_fwd and fa_fwd_host in bf16 at d = 128 without
 * the causal mask and at d = 256 with or without it -- counts, per (query row, key block)
 * step, whether it rescaled, and whether the eager rule would have; the other kernel
 * instances count nothing.  Counters are per device and sum
 * over all launches (concurrent ones included) since the last reset.
 *
 * fa_rescale_stats synchronises `stream`, then writes the counters of the current device:
 *   steps   (query row, key block) steps processed (rows of the last partial unit
 *           included: a unit is 256 query rows, a key block 128 keys)
 *   lazy    rescales made (after the row's first admissible key)
 *   eager   rescales the eager rule would have made on the same rows
 * and clears them if `reset` is non-zero.  Returns FA_OK, FA_ERR_INVALID_ARG for a null
 * pointer, FA_ERR_CUDA if a CUDA call failed.
 */
fa_status fa_rescale_stats(fa_stream_t stream, unsigned long long *steps,
                           unsigned long long *lazy, unsigned long long *eager, int reset);

/*
 * Self-test of the failure path above, without faulting anything: launches one warp that
 * waits on a shared-memory mbarrier nothing ever arrives on, with a limit of timeout_us
 * microseconds (1 .. 1000000).  The wait runs out, the kernel records the time-out in the
 * device error word and returns; the next fa_check_device_error(stream) reports
 * FA_ERR_TIMEOUT and clears the word.  Returns FA_OK once launched, FA_ERR_INVALID_ARG
 * for an out-of-range timeout, FA_ERR_CUDA if the launch failed.
 */
fa_status fa_selftest_bounded_wait(int timeout_us, fa_stream_t stream);

/* Static English description of a status code. */
const char *fa_status_string(fa_status s);

/* Library version as major*10000 + minor*100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
