/*
 * fa.h -- C ABI of the fused, tiled attention for NVIDIA B200 (sm_100a): the
 * forward pass (with key windows or an additive score bias) and its gradients.
 *
 * The operation (sources: "FlashAttention 算子" article on mooersco.com, sections
 * "标准 Attention 的瓶颈在哪" and "昇腾NPU上的分块策略"):
 *
 *     O = softmax(scale * Q K^T  [with causal mask]) V
 *
 * computed block by block with an online softmax (running row maximum and row
 * sum, partial output rescaled when the maximum moves), so that the Nq x Nk
 * score and probability matrices never reach device memory.  The tensors are
 * the [batch, heads, sequence, head_dim] fp16 tensors of the PyTorch call on
 * that page ("通过 PyTorch 调用 FlashAttention"); head_dim is 64, 128 or 256
 * as that section lists; causal masking is its is_causal flag; grouped-query
 * and multi-query heads (Hkv < Hq) are those of section 六 of the
 * gitcode.csdn.net article.
 *
 * Conventions shared by every entry point below
 * ---------------------------------------------
 * Layout     q, o: [B, Hq, Nq, D]; k, v: [B, Hkv, Nk, D]; all contiguous
 *            (row-major, D fastest), all of one 16-bit dtype.  lse: float32
 *            [B, Hq, Nq], contiguous.
 * Memory     q, k, v, o and lse are DEVICE pointers on the current CUDA device.
 *            Each of q, k, v, o must be 16-byte aligned (tensor-memory-access
 *            descriptors require it); lse must be 4-byte aligned.  The caller
 *            owns every buffer; the library allocates no device memory and
 *            keeps no per-call state.  o and lse must not overlap q, k or v.
 * Heads      Hq must be a multiple of Hkv; query head h reads key/value head
 *            h / (Hq / Hkv) (contiguous groups).
 * Causal     causal != 0 keeps key j for query i iff j <= i (top-left
 *            alignment, as PyTorch's scaled_dot_product_attention(is_causal=True)).
 * Scale      any finite float, applied to the scores before the softmax; the
 *            pages use 1/sqrt(D).  scale = 0 gives the plain average of V.
 * LSE        lse[b,h,i] = ln sum_j exp(scale * q_i . k_j) over the visible keys
 *            (natural log, scale included).  lse may be NULL: then it is not
 *            written.
 * Stream     `stream` is a cudaStream_t (NULL = legacy default stream).  The
 *            call only enqueues work and returns; results are ready when the
 *            stream reaches that point.
 * Errors     every entry point returns FA_OK (0) or one of the fa_status codes
 *            below.  Argument errors are detected on the host before anything
 *            is enqueued; nothing is launched then.  Faults inside the kernel
 *            are not reported by the return value: a kernel wait that exceeds
 *            its time limit records FA_ERR_DEVICE_TIMEOUT in a device status
 *            word that fa_device_status() reads.
 * Threads    the entry points are thread-safe; per-device set-up (function
 *            attributes, driver entry point) happens once, on first use.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

enum fa_dtype { FA_FP16 = 0, FA_BF16 = 1 };

enum fa_status {
  FA_OK = 0,
  FA_ERR_NULL_POINTER = 1,         /* q, k, v or o is NULL                        */
  FA_ERR_MISALIGNED = 2,           /* q, k, v, o not 16-byte aligned; lse not 4    */
  FA_ERR_BAD_SHAPE = 3,            /* B, Hq, Hkv, Nq or Nk < 1, or sizes overflow  */
  FA_ERR_BAD_GROUPING = 4,         /* Hq % Hkv != 0                               */
  FA_ERR_UNSUPPORTED_HEAD_DIM = 5, /* D not in {64, 128, 256}                      */
  FA_ERR_BAD_SCALE = 6,            /* scale is NaN or infinite                     */
  FA_ERR_BAD_DTYPE = 7,            /* dtype not FA_FP16 or FA_BF16                 */
  FA_ERR_NO_DEVICE = 8,            /* no current CUDA device, or it is not sm_100  */
  FA_ERR_LAUNCH = 9,               /* the CUDA runtime refused the launch          */
  FA_ERR_DRIVER = 10,              /* tensor-map encoding via the driver failed    */
  FA_ERR_DEVICE_TIMEOUT = 11,      /* (device status) a kernel wait hit its limit  */
  FA_ERR_OVERLAP = 12,             /* o or lse overlaps q, k or v                  */
  FA_ERR_SCRATCH_TOO_SMALL = 13,   /* fa_fwd_noalloc: static scratch too small     */
  FA_ERR_BAD_WINDOW = 14,          /* fa_fwd_window: bound < -1, or causal + right > 0 */
  FA_ERR_BAD_WORKSPACE = 15,       /* fa_bwd, fa_fwd_unfused: workspace NULL, too small or misaligned */
  FA_ERR_LIBRARY = 16              /* fa_fwd_unfused: a cuBLAS call failed          */
};

/*
 * Fused attention forward (the operation above).
 *   q, k, v   device inputs (see Layout); read only.
 *   o         device output [B, Hq, Nq, D], same dtype as the inputs, rounded to
 *             nearest even from the fp32 result.
 *   lse       device output [B, Hq, Nq] float32, or NULL.
 *   B         batch size;  Hq, Hkv  query and key/value heads;
 *   Nq, Nk    query and key sequence lengths (any value >= 1; tails are masked);
 *   D         head_dim, one of 64, 128, 256;
 *   scale     score scale;  causal  0 or 1;
 *   stream    cudaStream_t to enqueue on;
 *   dtype     FA_FP16 or FA_BF16.
 */
int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
           int Hkv, int Nq, int Nk, int D, float scale, int causal, void *stream, int dtype);

/* fa_fwd with the dtype fixed (the fourteen-argument form). */
int fa_fwd_fp16(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                int Hkv, int Nq, int Nk, int D, float scale, int causal, void *stream);
int fa_fwd_bf16(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                int Hkv, int Nq, int Nk, int D, float scale, int causal, void *stream);

/*
 * fa_fwd with a caller-provided device workspace (no counterpart on the pages: it
 * exists for load balance on this device).  With a workspace, non-causal calls
 * take their work tiles from a counter in the workspace (dynamic schedule); a
 * call whose last round of tiles would keep at most half of the SMs busy gives
 * each of those tiles to two CTAs, one per half of the key blocks (from 24 key
 * blocks up); and a call with fewer work tiles than SMs (KV-cache decode: the
 * query heads of a GQA group share one tile when they fit its 128 rows) shares
 * the key blocks of all tiles out evenly over the SMs (stream-K).  Every part
 * leaves its un-normalised partial output in the workspace and the last to
 * finish merges them, in a fixed order.  Results agree with fa_fwd within
 * rounding (the order of the additions differs) and repeat bit for bit.
 *   workspace        device memory of at least fa_fwd_workspace_size(D) bytes,
 *                    256-byte aligned (else FA_ERR_MISALIGNED), zero-filled
 *                    before its first use.  Every call that completes leaves the
 *                    workspace's arrival counters at zero again, so one zero-fill
 *                    suffices.  Calls that may run concurrently need separate
 *                    workspaces.  After FA_ERR_DEVICE_TIMEOUT, zero it again.
 *                    NULL (or too small) gives exactly fa_fwd.
 *   workspace_bytes  its size.
 */
int fa_fwd_ws(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
              int Hkv, int Nq, int Nk, int D, float scale, int causal, void *stream, int dtype,
              void *workspace, size_t workspace_bytes);

/* Workspace bytes fa_fwd_ws needs on the current device for head_dim D (about 20 MB
 * on a 148-SM B200); 0 if D is unsupported or no device is current. */
size_t fa_fwd_workspace_size(int D);

/*
 * Attention with a key window (a mask beyond causal: the pages place the mask
 * step on the vector unit, and the scaled_dot_product_attention call of the
 * mooersco.com page takes an attn_mask).  Query i sees key j iff
 *     i - window_left <= j <= i + window_right      (0-based, top-left aligned),
 * a bound of -1 meaning no bound on that side; causal = 1 is window_right = 0
 * (window_right must then be -1 or 0).  A query row that sees no key (only
 * when Nq > Nk + window_left) gets O = 0 and LSE = -inf.  Key blocks wholly
 * outside a tile's windows are not read.  Other arguments, layout and errors
 * as fa_fwd_ws (the workspace is optional and only balances the schedule:
 * windowed calls are never split); FA_ERR_BAD_WINDOW for a bound below -1 or
 * a causal call with window_right > 0.  window_left = window_right = -1 gives
 * fa_fwd_ws's result within rounding.
 */
int fa_fwd_window(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                  int Hq, int Hkv, int Nq, int Nk, int D, float scale, int causal,
                  int window_left, int window_right, void *stream, int dtype, void *workspace,
                  size_t workspace_bytes);

/*
 * Attention with an additive score bias (a mask beyond causal: the mask step
 * the pages place on the vector unit, and the float attn_mask of the
 * scaled_dot_product_attention call on the mooersco.com page):
 *     O_i = sum_j softmax_j(scale q_i.k_j + bias[b, hq, i, j]) v_j,
 * with -inf in the bias removing a key (causal still applies when causal = 1).
 *   bias       device pointer, same dtype as q (fp16 / bf16), 16-byte aligned;
 *              element (b, hq, i, j) at bias + b * bias_stride_b +
 *              hq * bias_stride_h + i * bias_stride_q + j;
 *   strides    in elements, >= 0, multiples of 8 (else FA_ERR_MISALIGNED);
 *              a zero stride broadcasts that dimension (e.g. a key-padding
 *              mask [B, 1, 1, Nk] has bias_stride_h = bias_stride_q = 0).
 * A query row whose keys are all removed gets O = 0 and LSE = -inf.  LSE
 * includes the bias.  Bias tiles are staged through shared memory by TMA (one
 * 128 x 128 tile per key block, read once per query tile).  Other arguments,
 * layout and errors as fa_fwd; o and lse may not overlap the bias.
 */
int fa_fwd_bias(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                int Hkv, int Nq, int Nk, int D, float scale, int causal, const void *bias,
                long long bias_stride_b, long long bias_stride_h, long long bias_stride_q,
                void *stream, int dtype);

/*
 * fa_fwd_bias with a key window as well (both masks of the mask step at once):
 * key j is visible to query i iff i - window_left <= j <= i + window_right
 * (-1: no bound; causal = 1 adds j <= i) and its bias is not -inf; the visible
 * scores get the bias added as in fa_fwd_bias.  A row with no visible key gets
 * O = 0 and LSE = -inf.  Windowed calls run the 128-row-tile kernel, which
 * takes each tile's own key-block range.  Arguments, layout and errors as
 * fa_fwd_bias and fa_fwd_window (FA_ERR_BAD_WINDOW for a bound < -1, or
 * window_right > 0 with causal = 1); window_left = window_right = -1 is
 * fa_fwd_bias.
 */
int fa_fwd_bias_window(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                       int Hq, int Hkv, int Nq, int Nk, int D, float scale, int causal,
                       const void *bias, long long bias_stride_b, long long bias_stride_h,
                       long long bias_stride_q, int window_left, int window_right, void *stream,
                       int dtype);

/*
 * fa_fwd_bias_window with a caller workspace (as fa_fwd_ws: at least
 * fa_fwd_workspace_size(D) bytes, 256-byte aligned, zero-filled before first
 * use and left zeroed; NULL = fa_fwd_bias_window).  With it, bias launches
 * take work units from the dynamic schedule, and those with more than 128
 * query rows and no key window split the last round of tiles over two CTAs
 * (merged in a fixed order; a part in which the bias removed every key of a
 * row carries no weight).  The workspace may not overlap the bias
 * (FA_ERR_OVERLAP).  Other arguments and errors as fa_fwd_bias_window.
 */
int fa_fwd_bias_ws(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                   int Hkv, int Nq, int Nk, int D, float scale, int causal, const void *bias,
                   long long bias_stride_b, long long bias_stride_h, long long bias_stride_q,
                   int window_left, int window_right, void *stream, int dtype, void *workspace,
                   size_t workspace_bytes);

/*
 * Backward pass: the gradients of the attention above for an upstream gradient
 * dout (the pages mention only that training keeps gradients -- hwcomputing.
 * csdn.net page, section on standard attention; the operation is taken as the
 * exact gradient of O = softmax(scale Q K^T) V):
 *   P = exp(scale Q K^T - LSE), dV = P^T dO, dP = dO V^T, Delta = rowsum(dO * O),
 *   dS = P * (dP - Delta), dQ = scale dS K, dK = scale dS^T Q
 * (causal: keys j <= i as in the forward pass; GQA: dK, dV sum over the query
 * heads of each group).  P is recomputed from q, k and the forward pass's lse,
 * never stored.
 *   q, k, v, o  the forward pass's inputs and output (layout as fa_fwd);
 *   dout        [B, Hq, Nq, D] upstream gradient, same dtype;
 *   lse         [B, Hq, Nq] float32 from the forward pass (natural log);
 *   dq          [B, Hq, Nq, D];  dk, dv  [B, Hkv, Nk, D]  outputs, same dtype;
 *   workspace   device scratch of at least fa_bwd_workspace_size(B, Hq, Nq)
 *               bytes, 256-byte aligned, caller-owned (Delta and lse * log2 e,
 *               padded to 128-row blocks; no zero-fill needed); else
 *               FA_ERR_BAD_WORKSPACE / FA_ERR_MISALIGNED.
 * D must be 64, 128 or 256 (else FA_ERR_UNSUPPORTED_HEAD_DIM).  Outputs and
 * the workspace may not overlap any input or each other (FA_ERR_OVERLAP).
 * Kernels on `stream`: Delta, then dK and dV, then dQ (at D = 256 dV and dK
 * are two launches over 64-row query blocks, and dQ runs over 64-key blocks:
 * one CTA's tensor memory holds only one 256-column accumulator next to the
 * score blocks); asynchronous; deterministic (no atomics).  Other errors as
 * fa_fwd.
 */
int fa_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
           const float *lse, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Nq, int Nk,
           int D, float scale, int causal, void *stream, int dtype, void *workspace,
           size_t workspace_bytes);

/*
 * fa_bwd with a key window (the gradient of fa_fwd_window's operation): query
 * i sees keys i - window_left .. i + window_right (-1: no bound; causal = 1 is
 * window_right = 0, which must then be -1 or 0, else FA_ERR_BAD_WINDOW).  A
 * row that saw no key (its lse is -inf) contributes nothing: its dQ row is 0.
 * Key/query blocks wholly outside the windows are skipped.  Other arguments
 * and errors as fa_bwd; window_left = window_right = -1 is fa_bwd.
 */
int fa_bwd_window(const void *q, const void *k, const void *v, const void *o, const void *dout,
                  const float *lse, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Nq,
                  int Nk, int D, float scale, int causal, int window_left, int window_right,
                  void *stream, int dtype, void *workspace, size_t workspace_bytes);

/*
 * fa_bwd with an additive score bias (the gradient of fa_fwd_bias's operation
 * with respect to q, k and v; the bias is a given input and gets no gradient):
 * P = exp(scale Q K^T + bias - LSE) in every formula of fa_bwd, with lse from
 * fa_fwd_bias on the same bias.  Bias layout, strides and their errors as
 * fa_fwd_bias; causal as fa_bwd.  A row whose keys the bias removed entirely
 * (its lse is -inf) contributes nothing: its dQ row is 0.  Both kernels stage
 * each block pair's 128 x 128 bias tile through shared memory by TMA.  D must
 * be 64 or 128 (else FA_ERR_UNSUPPORTED_HEAD_DIM: at 256 the tile does not fit
 * beside the operands).  The outputs and the workspace may not overlap the
 * bias (FA_ERR_OVERLAP).  Other arguments and errors as fa_bwd.
 */
int fa_bwd_bias(const void *q, const void *k, const void *v, const void *o, const void *dout,
                const float *lse, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Nq,
                int Nk, int D, float scale, int causal, const void *bias, long long bias_stride_b,
                long long bias_stride_h, long long bias_stride_q, void *stream, int dtype,
                void *workspace, size_t workspace_bytes);

/*
 * fa_bwd_bias with a key window as well (the gradient of fa_fwd_bias_window's
 * operation): query i sees keys i - window_left .. i + window_right (-1: no
 * bound; causal = 1 is window_right = 0) and the bias enters P as in
 * fa_bwd_bias; query and key blocks wholly outside the windows are skipped.
 * A row with no visible key contributes nothing.  Arguments and errors as
 * fa_bwd_bias and fa_bwd_window; window_left = window_right = -1 is
 * fa_bwd_bias.
 */
int fa_bwd_bias_window(const void *q, const void *k, const void *v, const void *o,
                       const void *dout, const float *lse, void *dq, void *dk, void *dv, int B,
                       int Hq, int Hkv, int Nq, int Nk, int D, float scale, int causal,
                       const void *bias, long long bias_stride_b, long long bias_stride_h,
                       long long bias_stride_q, int window_left, int window_right, void *stream,
                       int dtype, void *workspace, size_t workspace_bytes);

/* Workspace bytes fa_bwd needs: 8 * B * Hq * (Nq rounded up to 128); 0 for bad sizes. */
size_t fa_bwd_workspace_size(int B, int Hq, int Nq);

/*
 * fa_fwd_ws for callers that cannot allocate device memory.  The pages have no
 * counterpart: this entry point exists for callers such as a serving engine
 * whose memory pool already owns all of the device's free memory, or a plug-in
 * interface that hands the library only its inputs and outputs -- there a
 * cudaMalloc would fail, or stall the device while the caller's stream is busy.
 * It takes exactly fa_fwd's arguments and allocates nothing (no cudaMalloc, no
 * cudaFree, no allocating library routine); the scratch of the split tail and
 * of stream-K decode launches is a file-scope device array of fa_fwd_noalloc_scratch_bytes() bytes (24 MiB) that
 * every GPU loading this library holds until the process exits.
 *   - Argument errors are returned before any CUDA call, as for fa_fwd.
 *   - The first call on each device looks up that array's device address
 *     (cudaGetSymbolAddress) with the device current; make that first call
 *     before any stream capture.  If the lookup fails the call returns
 *     FA_ERR_LAUNCH and launches nothing; the next call tries again.
 *   - Each call clears the array's arrival counters on `stream` before its
 *     kernel; all calls share the one array, so calls whose work overlaps on
 *     the GPU (other streams, other threads) race and must not be issued.
 *   - A problem whose split tail would need more scratch than the array holds
 *     returns FA_ERR_SCRATCH_TOO_SMALL and launches nothing (a stream-K launch
 *     uses fewer CTAs instead, or none of the split).
 * Results are bit-identical to fa_fwd_ws's with a workspace of
 * fa_fwd_workspace_size(D) bytes (the same split and the same fixed merge
 * order), except for a stream-K launch that one of the two scratch sizes cuts
 * to fewer CTAs than the other: those agree within rounding.
 */
int fa_fwd_noalloc(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                   int Hkv, int Nq, int Nk, int D, float scale, int causal, void *stream,
                   int dtype);

/* Size in bytes of fa_fwd_noalloc's static scratch array. */
size_t fa_fwd_noalloc_scratch_bytes(void);

/*
 * Standard attention in three steps through device memory -- the comparison
 * the pages make (mooersco.com article, "标准 Attention 的瓶颈在哪" and the table of
 * "跟标准 Attention 的性能差距有多大"; gitcode.csdn.net article, section 二): S =
 * scale Q K^T is written out (fp32), a row-softmax kernel reads it and writes P
 * (rounded to the input dtype) and the LSE, and O = P V reads P back.  The two
 * products are cuBLAS batched GEMMs with fp32 accumulation; the softmax is this
 * library's kernel.  It exists to measure what the fused kernel saves (time,
 * device memory, DRAM traffic); it is not the fast path.
 *   Arguments, layout, causal, scale and LSE as fa_fwd; D in {64, 128, 256}.
 *   workspace  device buffer of at least fa_fwd_unfused_workspace_size(B, Hq, Nq, Nk)
 *              bytes, 256-byte aligned, caller-owned (holds S and P: 6 bytes per
 *              score); FA_ERR_BAD_WORKSPACE otherwise.
 *   Errors     as fa_fwd, plus FA_ERR_LIBRARY if creating the cuBLAS handle (once
 *              per device, on the first call; it allocates cuBLAS's own device
 *              memory) or a cuBLAS call fails.
 *   Results agree with fa_fwd's within the rounding of P (both round P to the
 *   input dtype, at different points).
 */
int fa_fwd_unfused(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                   int Hkv, int Nq, int Nk, int D, float scale, int causal, void *stream,
                   int dtype, void *workspace, size_t workspace_bytes);

/* Workspace bytes fa_fwd_unfused needs: 256-aligned 4 + 2 bytes per score (B * Hq * Nq * Nk);
 * 0 for bad sizes. */
size_t fa_fwd_unfused_workspace_size(int B, int Hq, int Nq, int Nk);

/* Process-wide cap on the CTAs (one per SM) a launch uses; 0, the default, means
 * every SM.  Useful to leave SMs to concurrent work.  Returns the previous cap,
 * or FA_ERR_BAD_SHAPE for n < 0. */
int fa_set_max_ctas(int n);

/* Human-readable text for a status code (static storage; never NULL). */
const char *fa_status_string(int status);

/*
 * Device status word of the current device: FA_OK, or FA_ERR_DEVICE_TIMEOUT if
 * a kernel of this library gave up on a wait since the last reset.  Synchronises
 * the device.  reset != 0 clears the word after reading it.  Returns a negative
 * value if the word cannot be read (no device).
 */
int fa_device_status(int reset);

/*
 * Diagnostic companion of fa_device_status: where the first timed-out wait
 * happened since the last reset, packed as
 *   CTA index << 48 | warp << 40 | shared-memory address of the mbarrier << 8 | phase parity
 * (0 if none).  Synchronises the device.  Returns FA_OK, FA_ERR_NULL_POINTER or
 * FA_ERR_NO_DEVICE.
 */
int fa_device_timeout_site(unsigned long long *site);

/*
 * Diagnostic: y[i] = 2^x[i] computed the way the softmax computes the share of
 * its exponentials that it moves from the MUFU unit to the FMA pipe (no
 * counterpart on the pages; it exists so tests can check that approximation):
 * round-to-nearest range reduction and a cubic minimax polynomial with p(0) = 1,
 * max relative error 1.02e-4 for -125 <= x < 128, exact at integer x; inputs
 * below -125 give ~2^-125.
 * x, y: device float arrays of n elements.  Asynchronous on `stream`.
 */
int fa_debug_exp2_fma(const float *x, float *y, int n, void *stream);

/*
 * Diagnostic for the failure detection of the kernels' waits (no counterpart on
 * the pages): enqueues one warp that runs the same bounded mbarrier wait as the
 * attention kernels on a barrier nothing ever arrives on.  After the wait limit
 * (about 1 s) it records FA_ERR_DEVICE_TIMEOUT in the device status word and the
 * site in fa_device_timeout_site, and returns; nothing hangs or faults.  Reset
 * the status word (fa_device_status(1)) afterwards.
 */
int fa_debug_wait_timeout(void *stream);

/* Number of 256-row work tiles (128-row at D = 256) of the two-query-tile
 * kernel for these sizes; 0 for invalid arguments.  Host only; used to size
 * tests.  (Launches with at most 128 query rows, key windows, or fewer of these
 * tiles than half the CTAs run 128-row tiles instead.) */
long long fa_fwd_num_tiles(int B, int Hq, int Nq, int D);

#ifdef __cplusplus
}
#endif
#endif /* FA_H_ */
