/*
 * ss2d.h -- C ABI of the B200 (sm_100a) SS2D library.
 *
 * The library computes the forward pass of the 2D selective scan (SS2D) used
 * by VMamba, and the 1D selective scan with one or two directions used by
 * Vision Mamba (Vim), and the backward pass of both (ss2d_backward,
 * selective_scan_bwd, below):
 *
 *   cross_scan   "Vision Mamba" (dileepadev tutorial), section "The 2D
 *                Challenge: Adapting SSMs to Images", CrossScanModule; and
 *                "VMamba架构解析" (mhpn.cn), section 1, cross_scan: an H x W
 *                map is read in four orders, stacked as
 *                  k = 0  row-major                     p = l
 *                  k = 1  row-major reversed            p = L-1-l
 *                  k = 2  column-major (l = w*H + h)    p = h*W + w
 *                  k = 3  column-major reversed
 *                where p = h*W + w is the pixel visited at scan step l.
 *   selective scan  "Vision Mamba" (dileepadev), section "Background: State
 *                Space Models and Mamba", SelectiveSSM; the recurrence is the
 *                discrete system of "Vision Mamba: Efficient Visual
 *                Representation Learning with Bidirectional State Space
 *                Model" (aipaper.cc), section 4.1.  Per direction k and
 *                channel d (row kd = k*D + d of the parameters):
 *                  A[n]  = -exp(A_log[kd, n])
 *                  dt_l  = softplus(delta[b,k,d,l] + delta_bias[kd])
 *                  h_l[n] = exp(dt_l*A[n]) * h_{l-1}[n] + dt_l*Bs[b,k,n,l]*u_l,
 *                           h_{-1} = 0, state held in float32
 *                  Y_k[l] = sum_n Cs[b,k,n,l]*h_l[n] + Dskip[kd]*u_l
 *                with u_l = x[b, d, p(l)].
 *   cross_merge  same CrossScanModule: each Y_k is put back in pixel order
 *                and the directions are summed, always in the order
 *                ((Y_0 + Y_1) + Y_2) + Y_3, so results are deterministic.
 *   1D variant   Vim block ("Vision Mamba ..." summary, section 4.3): a
 *                forward scan (k = 0) and a scan of the reversed sequence
 *                (k = 1, whose output is flipped back), added.
 *
 * Memory: every pointer is either a DEVICE pointer (memory of the current
 * CUDA device, or managed memory) or a HOST pointer; all pointers of one call
 * must be of the same kind.
 *   - device pointers: the call is asynchronous on `stream` and returns after
 *     enqueueing.  Scratch for the per-direction partial outputs (K = 4, or
 *     K = 2 with N > 16: 4*B*K*D*L bytes) and, when sequences are split into chunks, for the
 *     chunk states (68*B*K*D*(chunks-1) bytes) is taken from a stream-ordered
 *     pool on `stream` and returned on `stream`.  Nothing is synchronised.
 *   - host pointers (pageable or pinned): the call copies the inputs to the
 *     current device, runs the device path, copies y back and synchronises
 *     `stream` before returning.  Device buffers come from the same pool.
 *     With more than 16 MB of input the batch goes in slices of whole
 *     elements (up to 8) through two copy streams of the library's own, so
 *     that copies in, kernels and copies out overlap (pinned buffers are
 *     needed for the overlap); every slice keeps the whole call's chunk
 *     plan, so y is bit for bit the device path's.  The extra streams are
 *     ordered after `stream`'s earlier work and joined back into it.
 * The caller owns every buffer; the library keeps no pointer after a call.
 * Inputs are never written.  y must not overlap any input.
 *
 * Layouts (contiguous, C order):
 *   x          (B, D, H, W)   dtype   (u of the 1D call: (B, D, L))
 *   delta      (B, K, D, L)   dtype   raw delta, in direction k's SCAN order
 *   Bs, Cs     (B, K, N, L)   dtype   in direction k's SCAN order
 *   A_log      (K*D, N)       float32
 *   Dskip      (K*D)          float32
 *   delta_bias (K*D)          float32
 *   y          (B, D, H, W) / (B, D, L)  float32, pixel order, overwritten
 * where L = H*W.  Every pointer must be 16-byte aligned.  Limits: B <= 65535,
 * L < 2^31.
 *
 * Precision: dtype is the storage type of x, delta, Bs and Cs; all
 * arithmetic and the state are float32.
 *
 * Errors: every entry point returns an ss2d_status; nothing else crosses
 * the ABI.  A status below zero means nothing was enqueued, except
 * SS2D_ERR_CUDA, which reports a CUDA error seen while enqueueing or (host
 * path) while running; ss2d_last_error() then gives CUDA's message for the
 * calling thread.  Sizes of zero (B, D, H or W) are valid and do nothing.
 * The functions hold no global mutable state besides the per-thread error
 * text and are safe to call from several threads.
 */
#ifndef SS2D_B200_H
#define SS2D_B200_H

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SS2D_OK = 0,
    SS2D_ERR_NULL = -1,   /* a required pointer is NULL                      */
    SS2D_ERR_SHAPE = -2,  /* a size is negative, or a product overflows     */
    SS2D_ERR_DTYPE = -3,  /* dtype is not one of ss2d_dtype                  */
    SS2D_ERR_K = -4,      /* K not in {1,2,4} (2D) or {1,2} (1D)             */
    SS2D_ERR_N = -5,      /* N not in 1..64 (1..16 for ss2d_forward_timed) */
    SS2D_ERR_ALIGN = -6,  /* a pointer is not 16-byte aligned                */
    SS2D_ERR_ALLOC = -7,  /* device memory for scratch or staging ran out    */
    SS2D_ERR_CUDA = -8,   /* a CUDA call failed; see ss2d_last_error()       */
    SS2D_ERR_PTR = -9,    /* host and device pointers mixed in one call      */
    SS2D_ERR_VARIANT = -10, /* unknown kernel variant (ss2d_forward_ex)      */
    SS2D_ERR_SCRATCH = -11  /* needs more scratch than ss2d_forward_noalloc's
                               fixed buffer holds                             */
} ss2d_status;

typedef enum {
    SS2D_F32 = 0,   /* x, delta, Bs, Cs stored as float32  */
    SS2D_BF16 = 1,  /* x, delta, Bs, Cs stored as bfloat16 */
    SS2D_F16 = 2    /* x, delta, Bs, Cs stored as IEEE float16 (the FP16 path of
                       "VMamba架构解析", section 2; the state stays float32) */
} ss2d_dtype;

/* SS2D forward: cross_scan -> selective scan of each direction -> cross_merge.
 * K = 4 is the SS2D of the pages; K = 2 (directions 0 and 1 only) and K = 1
 * (row-major only) are also accepted.  N in 1..64: the states of a channel
 * never interact, so more than 16 run as groups of 16 states one after the
 * other, each adding its C.h terms to the output (the skip term once); the
 * pages use N = 16 and mention d_state 8 ("VMamba架构解析", section 5).
 * K = 2 with N <= 16: the scan pass does the cross_merge itself -- y is
 * zeroed on `stream`, then both directions add their outputs into it with
 * float atomic adds; two terms give the same bits in either order, so y is
 * exactly y_0 + y_1 as the merge kernel would sum it.
 * `stream` is a cudaStream_t (NULL = the legacy default stream). */
int ss2d_forward(const void *x, const void *delta, const float *A_log,
                 const void *Bs, const void *Cs, const float *Dskip,
                 const float *delta_bias, float *y,
                 int B, int D, int H, int W, int N, int K, int dtype,
                 void *stream);

/* 1D selective scan, Vim's bidirectional case: u (B, D, L); K = 1 (forward
 * only) or K = 2 (forward plus the reversed sequence, flipped back, added).
 * Direction 1 reads u from the end (u[L-1-l] at step l); its delta, Bs and
 * Cs rows are in that reversed scan order.  Other arguments as ss2d_forward. */
int selective_scan_fwd(const void *u, const void *delta, const float *A_log,
                       const void *Bs, const void *Cs, const float *Dskip,
                       const float *delta_bias, float *y,
                       int B, int D, int L, int N, int K, int dtype,
                       void *stream);

/* cross_scan + selective scan WITHOUT cross_merge: writes each direction's
 * output, in PIXEL order, to y_dir (B, K, D, H, W) float32 (for the 1D call
 * with two_d = 0: (B, K, D, L), direction 1 flipped back to sequence order).
 * This is what the tutorial's CrossScanModule concatenates before its output
 * projection.  Device pointers only (SS2D_ERR_PTR otherwise); asynchronous
 * on `stream`; scratch from the same stream-ordered pool as ss2d_forward
 * (the scan-order rows, then a copy kernel puts each direction in pixel
 * order).  variant as in ss2d_forward_ex. */
int ss2d_scan_directions(const void *x, const void *delta, const float *A_log,
                         const void *Bs, const void *Cs, const float *Dskip,
                         const float *delta_bias, float *y_dir,
                         int B, int D, int H, int W, int N, int K, int dtype,
                         int two_d, void *stream, int variant);

/* Gated forward: as ss2d_forward / selective_scan_fwd, then y = SiLU(z) * y
 * pointwise, SiLU(z) = z / (1 + e^-z) -- the output gate of the Vim block
 * ("Vision Mamba ..." summary, section 4.3: each direction's output is
 * multiplied by SiLU(z) before the directions are added; the same z for all
 * directions, so the gate is applied once to the fixed-order sum) and of the
 * tutorial's SelectiveSSM ("Vision Mamba" (dileepadev), section "Background:
 * State Space Models and Mamba").  z has the layout and dtype of x (u).
 * Device pointers only (SS2D_ERR_PTR otherwise); asynchronous on `stream`;
 * the gate runs inside the cross_merge kernel, which every gated call
 * launches (also for K = 1). */
int ss2d_forward_gated(const void *x, const void *delta, const float *A_log,
                       const void *Bs, const void *Cs, const float *Dskip,
                       const float *delta_bias, const void *z, float *y,
                       int B, int D, int H, int W, int N, int K, int dtype,
                       void *stream);
int selective_scan_fwd_gated(const void *u, const void *delta, const float *A_log,
                             const void *Bs, const void *Cs, const float *Dskip,
                             const float *delta_bias, const void *z, float *y,
                             int B, int D, int L, int N, int K, int dtype,
                             void *stream);

/* As ss2d_forward_ex / selective_scan_fwd_ex, and also the final states:
 * h_last (B,K,D,N) float32 receives, for every direction k and channel d,
 * the state h after the last step of direction k's scan order (the state a
 * scan continued past the end of the sequence would start from; the Vim
 * summary's section 4.4 keeps states on chip and writes only outputs, so
 * this is the one state a caller can get back).  Device pointers only
 * (host pointers: SS2D_ERR_PTR); h_last null: SS2D_ERR_NULL. */
int ss2d_forward_final_state(const void *x, const void *delta, const float *A_log,
                             const void *Bs, const void *Cs, const float *Dskip,
                             const float *delta_bias, float *y, float *h_last,
                             int B, int D, int H, int W, int N, int K, int dtype,
                             void *stream, int variant);
int selective_scan_fwd_final_state(const void *u, const void *delta, const float *A_log,
                                   const void *Bs, const void *Cs, const float *Dskip,
                                   const float *delta_bias, float *y, float *h_last,
                                   int B, int D, int L, int N, int K, int dtype,
                                   void *stream, int variant);

/* Backward of ss2d_forward / selective_scan_fwd: the gradients of
 * sum(dy * y) with respect to every input ("Vision Mamba ..." summary,
 * section 4.4: the backward recomputes the scan from the inputs instead of
 * reading stored states; here from chunk entry states every 16 steps).
 *   dy          float32, the layout of y (and of x / u)
 *   dx / du     float32, the layout of x / u
 *   ddelta      float32 (B,K,D,L), scan order, like delta
 *   dA_log      float32 (K*D,N)      dBs, dCs  float32 (B,K,N,L)
 *   dDskip      float32 (K*D)        ddelta_bias float32 (K*D)
 * Every output is overwritten.  The inputs are those of the forward call
 * (same dtype, layouts, K and N rules); all pointers are device pointers of
 * the current device, 16-byte aligned (host pointers: SS2D_ERR_PTR).
 * Asynchronous on `stream`; scratch comes from the library's stream-ordered
 * pool.  The parameter gradients are summed over the batch and the
 * sequence in a fixed order, so repeated calls give identical results.
 * dx sums the directions' du as the forward's cross_merge sums y (K = 2
 * with N <= 16: dx zeroed, then both directions added into it with float
 * atomic adds, the same bits in either order).
 * With B, H*W or L zero the parameter gradients are set to zero. */
int ss2d_backward(const void *x, const void *delta, const float *A_log,
                  const void *Bs, const void *Cs, const float *Dskip,
                  const float *delta_bias, const float *dy,
                  float *dx, float *ddelta, float *dA_log, float *dBs, float *dCs,
                  float *dDskip, float *ddelta_bias,
                  int B, int D, int H, int W, int N, int K, int dtype, void *stream);
int selective_scan_bwd(const void *u, const void *delta, const float *A_log,
                       const void *Bs, const void *Cs, const float *Dskip,
                       const float *delta_bias, const float *dy,
                       float *du, float *ddelta, float *dA_log, float *dBs, float *dCs,
                       float *dDskip, float *ddelta_bias,
                       int B, int D, int L, int N, int K, int dtype, void *stream);

/* As ss2d_forward, with an explicit kernel variant (index into the table
 * that ss2d_variant_name() describes; -1 = the library's own choice for the
 * shape).  Every variant computes the same result up to float32 rounding
 * order; the choice only changes how the work is laid out on the GPU. */
int ss2d_forward_ex(const void *x, const void *delta, const float *A_log,
                    const void *Bs, const void *Cs, const float *Dskip,
                    const float *delta_bias, float *y,
                    int B, int D, int H, int W, int N, int K, int dtype,
                    void *stream, int variant);

/* As selective_scan_fwd, with an explicit kernel variant (see above). */
int selective_scan_fwd_ex(const void *u, const void *delta, const float *A_log,
                          const void *Bs, const void *Cs, const float *Dskip,
                          const float *delta_bias, float *y,
                          int B, int D, int L, int N, int K, int dtype,
                          void *stream, int variant);

/* How a call with this shape and variant (-1 = the library's choice) is
 * executed: steps per chunk, chunks per sequence, and kernel launches per
 * call (1 scan pass, or state pass + carry + scan pass when the sequence is
 * chunked, once per group of 16 states; plus one cross_merge launch when
 * K = 4, or K = 2 with N > 16; K = 2 with N <= 16 merges in the scan pass
 * after a memset of y, which is not counted).  Host only. */
int ss2d_plan(int two_d, int B, int D, int H, int W, int N, int K, int variant,
              int *chunk_len, int *num_chunks, int *launches);

/* Measurement helper: runs one ss2d_forward (two_d = 1) or
 * selective_scan_fwd (two_d = 0) call on device pointers, recording CUDA
 * events on `stream` around each of its kernel launches, synchronises the
 * stream and writes the device time of each launch in milliseconds to
 * launch_ms[0..3] in the order [chunk state pass, carry, scan pass,
 * cross_merge]; a launch the call does not make gets -1 (K = 2 with
 * N <= 16: cross_merge is the empty interval after the scan pass, which
 * merges itself).  Blocking. */
int ss2d_forward_timed(const void *x, const void *delta, const float *A_log,
                       const void *Bs, const void *Cs, const float *Dskip,
                       const float *delta_bias, float *y,
                       int B, int D, int H, int W, int N, int K, int dtype,
                       int two_d, void *stream, int variant, float *launch_ms);

/* Number of kernel variants, and a static description of variant i
 * ("" for an index out of range). */
int ss2d_num_variants(void);
const char *ss2d_variant_name(int i);

/* The variant ss2d_forward / selective_scan_fwd would pick for this shape
 * (two_d = 1 for ss2d_forward, 0 for the 1D call; H = 1, W = L for 1D). */
int ss2d_pick_variant(int two_d, int B, int D, int H, int W, int N, int K);

/* Size in bytes of the fixed device scratch buffer of ss2d_forward_noalloc
 * (96 MiB): enough for the VMamba-T stage-1 SS2D layer, B = 8, D = 192,
 * 56 x 56, K = 4. */
#define SS2D_NOALLOC_SCRATCH_BYTES (96u * 1024u * 1024u)

/* ss2d_forward that allocates no memory.  There is no counterpart in the
 * papers: the entry point exists for callers that cannot let a library
 * allocate device memory once they run -- programs whose own caching
 * allocator has reserved (nearly) all device memory, latency-bound loops in
 * which a growing pool would call into the driver, processes held to a fixed
 * device footprint.  Its scratch (the per-direction rows and chunk states
 * ss2d_forward takes from its pool: 4*B*K*D*H*W bytes when K = 4 or
 * K = 2 with N > 16 (K = 2 with N <= 16 adds into y instead), plus
 * 68*B*K*D*(chunks-1) bytes when ss2d_plan reports chunks > 1, each rounded
 * up to 256) lives in one statically sized device buffer of
 * SS2D_NOALLOC_SCRATCH_BYTES per device, part of the library's device image.
 *   - Same arguments, layouts, results and limits as ss2d_forward, DEVICE
 *     pointers only (SS2D_ERR_PTR otherwise); asynchronous on `stream`.
 *   - A problem whose scratch would not fit returns SS2D_ERR_SCRATCH before
 *     anything is enqueued; ss2d_last_error() then gives the bytes needed.
 *   - Every call looks the buffer's address up on the current device
 *     (cudaGetSymbolAddress) and keeps nothing between calls, so a device
 *     reset between calls is safe.  The first call on a device loads the
 *     module that holds the buffer, which is when its memory is reserved;
 *     make this first call on each device before any stream capture begins.
 *   - Nothing in the buffer has to start at zero: every word a call reads is
 *     written earlier in the same call.
 *   - One buffer per device: calls on one device whose work can overlap in
 *     time (other streams, other host threads) race on it and give wrong
 *     results.  Serialise them: one stream, or streams ordered by events. */
int ss2d_forward_noalloc(const void *x, const void *delta, const float *A_log,
                         const void *Bs, const void *Cs, const float *Dskip,
                         const float *delta_bias, float *y,
                         int B, int D, int H, int W, int N, int K, int dtype,
                         void *stream);

/* ---- the fused front (conv1d + SiLU + x_proj + dt_proj) -----------------
 *
 * "Vision Mamba" (dileepadev tutorial), section "Background: State Space
 * Models and Mamba", SelectiveSSM.forward; "Vision Mamba ..." summary,
 * section 4.3 (the Vim block: every direction its own conv1d and
 * projections, direction 1 on the sequence reversed).  For direction k
 * (K = 1: forward only; K = 2: forward and reversed), batch element b and
 * step l of the direction's own order s (s[l] = x[b, l] for k = 0,
 * x[b, L-1-l] for k = 1):
 *   c[l, d]   = conv_b[k, d] + sum_{j<4} conv_w[k, d, j] * s[l-3+j, d]
 *               (causal depthwise conv1d of width 4, zeros before l = 0)
 *   u[l, d]   = SiLU(c[l, d]) = c / (1 + exp(-c))
 *   x_dbl[l]  = W_x[k] u[l]     (x_proj, D -> 1 + 2N, no bias) =
 *               (dt_raw[l], B[0..N-1, l], C[0..N-1, l])
 *   delta     = w_dt[k, d] * dt_raw[l]   (dt_proj, a Linear from 1 to D;
 *               its bias is the scan's delta_bias)
 * then the selective scan of every direction over its own u, delta, B, C
 * (as selective_scan_fwd, with A_log, Dskip, delta_bias rows k*D + d) and
 * y = Y_0 + Y_1 flipped back.  x_proj runs on the tensor cores (tcgen05)
 * with bfloat16 operands -- u and W_x rounded to nearest even -- and a
 * float32 accumulator; u is kept for the scan in the input dtype (for
 * bfloat16 input the x_proj operand blocks are that copy), dt_raw, B and C
 * in float32; no (D, L) delta array is ever written.  K = 2 with N <= 16:
 * y is zeroed and both directions add into it (two terms, the same bits in
 * either order) instead of a merge launch.
 *
 * Layouts (contiguous, C order; all pointers DEVICE memory of the current
 * device, 16-byte aligned):
 *   x       (B, L, D)  dtype    the input branch, channels last
 *   conv_w  (K, D, 4)  float32  taps, oldest step first
 *   conv_b  (K, D)     float32
 *   W_x     (K, 1 + 2N, D) float32   x_proj weight (row 0: dt, then B, then C)
 *   w_dt    (K, D)     float32  dt_proj weight
 *   A_log   (K*D, N), Dskip (K*D), delta_bias (K*D)  float32, as selective_scan_fwd
 *   y       (B, D, L)  float32, overwritten
 * K in {1, 2}, N in 1..64, dtype any ss2d_dtype; B * K * ceil(L / 128) *
 * ceil(D / 64) at most 2^31 - 1 (SS2D_ERR_SHAPE otherwise).  Scratch (u,
 * dt_raw, B, C with rows padded to a multiple of 8 steps, the x_proj
 * operand blocks, and the scan's scratch) comes from the stream-ordered
 * pool on `stream`; asynchronous.  A tensor-core
 * completion wait that runs out of time (2 s) is recorded for
 * ss2d_check_waits(); the call's y is then not valid. */
int selective_scan_fwd_front(const void *x, const float *conv_w, const float *conv_b,
                             const float *W_x, const float *w_dt, const float *A_log,
                             const float *Dskip, const float *delta_bias, float *y,
                             int B, int D, int L, int N, int K, int dtype, void *stream);

/* selective_scan_fwd_front that also synchronises `stream` and returns the
 * device time of its launches in launch_ms[0..2] (milliseconds, CUDA events
 * on `stream`): the front kernel, the scan passes, cross_merge (-1 when not
 * launched, K = 1; K = 2 with N <= 16 merges inside the scan pass, after a
 * memset of y that the second figure includes, and the third is the empty
 * interval after it).  For benchmarks. */
int selective_scan_fwd_front_timed(const void *x, const float *conv_w, const float *conv_b,
                                   const float *W_x, const float *w_dt, const float *A_log,
                                   const float *Dskip, const float *delta_bias, float *y,
                                   int B, int D, int L, int N, int K, int dtype, void *stream,
                                   float *launch_ms);

/* The front alone (same definition and layouts as selective_scan_fwd_front),
 * for callers that run their own scan: writes u (B, K, D, L) in the input
 * dtype and dt_raw (B, K, L), Bs, Cs (B, K, N, L) float32, each in its
 * direction's scan order.  L must be a multiple of 8 (SS2D_ERR_SHAPE
 * otherwise).  Device pointers only; asynchronous. */
int ss2d_front_project(const void *x, const float *conv_w, const float *conv_b,
                       const float *W_x, void *u, float *dt_raw, float *Bs, float *Cs,
                       int B, int D, int L, int N, int K, int dtype, void *stream);

/* Bounded waits.  The kernels that wait on an mbarrier (the front's
 * tensor-core completion) give up after a time limit instead of spinning
 * forever; they then record the fault in a device word and finish without
 * writing their outputs, so the CUDA context stays usable.  This call reads
 * that word on the current device (a blocking copy: call it after the
 * stream work it is meant to check), clears it, and returns SS2D_ERR_CUDA
 * with a description in ss2d_last_error() if a wait ran out, SS2D_OK
 * otherwise. */
int ss2d_check_waits(void);

/* Enqueue a kernel whose one wait can never complete (an mbarrier that
 * nothing arrives on), with a limit of limit_us microseconds (1..10^6): it
 * gives up, records the fault and returns; ss2d_check_waits() then reports
 * it.  A check of the time-out path itself. */
int ss2d_wait_selftest(int limit_us, void *stream);

/* Static text for a status code. */
const char *ss2d_status_string(int status);

/* CUDA's message for the last SS2D_ERR_CUDA / SS2D_ERR_ALLOC seen on the
 * calling thread, or the scratch bytes of the last SS2D_ERR_SCRATCH ("" if
 * none). */
const char *ss2d_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SS2D_B200_H */
