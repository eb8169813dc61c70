/*
 * la.h -- C ABI of the B200 causal linear attention library (libla.so).
 *
 * Causal linear attention, for every batch b and head h independently:
 *
 *     y_i = phi(q_i) S_i / (phi(q_i) . z_i),
 *     S_i = sum_{j<=i} phi(k_j) v_j^T   [F x Dv],   z_i = sum_{j<=i} phi(k_j)   [F]
 *
 * ("Simple linear attention language models balance the recall-throughput
 * tradeoff", Knowl 3: the masked parallel form for y_i and the recurrent
 * updates of s_i and z_i; "Transformers are RNNs", abstract: the
 * associativity that makes the cost linear in N.)  The sum includes j = i and
 * the denominator has no epsilon.
 *
 * Feature maps (phi : R^dqk -> R^F):
 *   LA_FMAP_ELU1    phi(x)_a = x_a + 1 if x_a > 0 else exp(x_a); F = dqk
 *                   (the elu(x)+1 map of "Transformers are RNNs", alpha = 1).
 *   LA_FMAP_TAYLOR2 phi(x) = [1 | x / dqk^(1/4) | x_a x_b / (sqrt(2) sqrt(dqk))],
 *                   second block row-major in (a, b); F = 1 + dqk + dqk^2.
 *                   phi(q).phi(k) = 1 + q.k/sqrt(dqk) + (q.k)^2/(2 dqk)
 *                   (BASED page, Knowl 3, second-order Taylor map with the
 *                   scaling inside phi; 273 features for dqk = 16, Knowl 5).
 *   LA_FMAP_TAYLOR2_SYM the same map with each pair of equal second-order
 *                   features (a,b), (b,a) folded into one:
 *                   phi(x) = [1 | x / dqk^(1/4) | x_a^2 / (sqrt(2) sqrt(dqk)) for
 *                   each a | x_a x_b / sqrt(dqk) for a < b, row-major];
 *                   F = 1 + 2 dqk + dqk (dqk - 1) / 2 (153 for dqk = 16, the
 *                   count in the BASED page's state-size expression
 *                   (d+1)(1 + 3d'/2 + d'^2/2), Knowl 7).  phi(q).phi(k) is the
 *                   same as for TAYLOR2, so o, den and gradients are the same;
 *                   only the state S, z is smaller: its pair row (a,b) holds
 *                   (S[a,b] + S[b,a]) / sqrt(2) of the TAYLOR2 state.  A decode
 *                   step moves 44 % fewer state bytes.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates or frees device memory and never synchronises, except
 *    la_get_device_status.  Work is enqueued on `stream` (a cudaStream_t,
 *    passed as void*; NULL is the legacy default stream) and runs
 *    asynchronously.  The tensor-core forward kernels and the decode kernels
 *    are launched with programmatic stream serialization: each waits for the
 *    kernel before it in the stream to complete before it touches memory,
 *    and lets the kernel after it be scheduled while it drains.  A kernel of
 *    the caller that follows one of these calls and is itself launched with
 *    programmatic stream serialization must wait for its prerequisite grid
 *    (griddepcontrol.wait) before it reads this call's results, as that
 *    launch attribute requires of every kernel.
 *  - Layouts are dense row-major: q, k [B,H,N,dqk]; v, o [B,H,N,dv];
 *    gradients like their primal; den [B,H,N] fp32; state S [B,H,F,dv] fp32
 *    and z [B,H,F] fp32 with the feature order above and no padding.
 *  - dtype selects the element type of q, k, v, o, dout, dq, dk, dv and of the
 *    decode q, k, v, y: LA_F32 (float) or LA_BF16 (bfloat16).  State, den and
 *    all accumulation are fp32.
 *  - Pointers must be 16-byte aligned (z and den need only 4-byte alignment).
 *  - Argument errors are returned synchronously, before anything is launched:
 *    LA_ERR_INVALID_ARG (null required pointer, non-positive size, overflow,
 *    misalignment, workspace too small, or a first tensor operand that is not
 *    memory of the calling thread's current device -- another device's
 *    memory or pageable host memory; the kernels run on the current device)
 *    or LA_ERR_UNSUPPORTED (a valid
 *    combination this build has no kernel for).  A failed launch returns
 *    LA_ERR_CUDA.  Errors detected on the device (a bounded wait that ran out,
 *    a failed device-side check) are recorded in a per-device status word and
 *    reported by la_get_device_status.
 *  - Results are deterministic: the same call on the same inputs gives the
 *    same bits.
 *  - Supported sizes: dqk in [1,128] for ELU1 and [1,16] for the Taylor maps;
 *    dv in [1,128]; N >= 1; B*H*N*max(dqk,dv) < 2^31 elements.  The fast
 *    tensor-core paths cover bf16 with (ELU1, dqk = dv in {64,128}) and
 *    (TAYLOR2 or TAYLOR2_SYM, dqk = 16, dv = 64); other valid combinations run
 *    on exact fp32 CUDA-core kernels.
 */
#ifndef LA_H
#define LA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LA_API __attribute__((visibility("default")))
#else
#define LA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { LA_FMAP_ELU1 = 0, LA_FMAP_TAYLOR2 = 1, LA_FMAP_TAYLOR2_SYM = 2 } la_fmap;
typedef enum { LA_F32 = 0, LA_BF16 = 1 } la_dtype;
typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = 1,
    LA_ERR_UNSUPPORTED = 2,
    LA_ERR_CUDA = 3,
    LA_ERR_TIMEOUT = 4,      /* a bounded device-side wait ran out          */
    LA_ERR_DEVICE_CHECK = 5, /* a device-side bounds/consistency check failed */
    LA_ERR_SCRATCH_LIMIT = 6 /* la_forward_noalloc: sizes need more than its built-in scratch */
} la_status;

/* Library version as 10000*major + 100*minor + patch. */
LA_API int la_version(void);

/* Human-readable name of a status code (static string, never NULL). */
LA_API const char *la_status_string(int status);

/* Feature dimension F of a feature map: dqk for ELU1, 1 + dqk + dqk^2 for
 * TAYLOR2 (BASED page, Knowl 5: 273 for dqk = 16), 1 + 2 dqk + dqk (dqk-1)/2
 * for TAYLOR2_SYM (153 for dqk = 16).  Returns -1 for an unknown map or
 * dqk < 1. */
LA_API int64_t la_feature_dim(int fmap, int dqk);

/* Bytes of device workspace la_forward needs for these sizes (0 if none).
 * The workspace carries what one launch of the call hands to the next: for
 * the bf16 elu dqk = dv = 64 forward, the phi(K) tiles, a state snapshot per
 * 128-token chunk and two partial sums per block; for the other tensor-core
 * shapes, when a long sequence is split across thread blocks, one state
 * increment per segment.  The caller allocates it.  Its contents need not be
 * initialised: every value a call reads from it was written earlier in the
 * same call.  Calls that may run at the same time need separate workspaces.
 * Returns 0 also for invalid arguments. */
LA_API size_t la_forward_workspace_bytes(int B, int H, int N, int dqk, int dv, int fmap, int dtype);

/* Bytes of device workspace la_backward needs: den_i and dden_i per token
 * (fp32), plus, when a sequence is split across thread blocks, one S and one
 * R increment per segment.  Same rules as la_forward_workspace_bytes. */
LA_API size_t la_backward_workspace_bytes(int B, int H, int N, int dqk, int dv, int fmap, int dtype);

/* Causal linear attention forward (prefill / training forward).
 * BASED page, Knowl 3 (parallel form for y_i) computed chunk by chunk as in
 * Knowl 5 (a masked quadratic term inside each chunk plus the product with
 * the state accumulated over earlier chunks), starting from a zero state.
 *   q, k      [B,H,N,dqk] dtype, read
 *   v         [B,H,N,dv]  dtype, read
 *   o         [B,H,N,dv]  dtype, written (y_i, rounded to nearest even for bf16)
 *   s_out     [B,H,F,dv]  fp32, nullable: final state S_N (Knowl 5: the
 *             prefill may write its final state for generation)
 *   z_out     [B,H,F]     fp32, nullable: final z_N
 *   den_out   [B,H,N]     fp32, nullable: den_i = phi(q_i).z_i
 *   workspace, workspace_bytes: at least la_forward_workspace_bytes(...)
 *             bytes of device memory (may be NULL when that is 0).
 * Outputs must not overlap inputs. */
LA_API la_status la_forward(const void *q, const void *k, const void *v, void *o,
                     float *s_out, float *z_out, float *den_out,
                     void *workspace, size_t workspace_bytes,
                     int B, int H, int N, int dqk, int dv, int fmap, int dtype,
                     void *stream);

/* la_forward starting from a given state instead of zero: resumes a prefill
 * (chunked prompt processing) from the state a previous la_forward,
 * la_forward_from_state or la_decode_step left.
 *
 *   S_i = S0 + sum_{j<=i} phi(k_j) v_j^T,   z_i = z0 + sum_{j<=i} phi(k_j),
 *   y_i = phi(q_i) S_i / phi(q_i) . z_i
 *
 * (the recurrence of the BASED page, Knowl 3, with s_0 = S0 and z_0 = z0;
 * running a sequence in two calls gives the outputs and final state of one
 * call over the whole sequence.)
 *   s_in [B,H,F,dv] fp32, z_in [B,H,F] fp32: S0 and z0 per (b, h), in the
 *          layout of s_out / z_out; read only.  Required (NULL is
 *          LA_ERR_INVALID_ARG) and must not overlap s_out or z_out
 *          (LA_ERR_INVALID_ARG).  For the Taylor map the state pairs
 *          rows (a, b) and (b, a) of the second-order block: any state this
 *          library returns has them equal, and the outputs depend only on
 *          their sum; the returned state keeps any difference between them
 *          unchanged.
 * Every other argument, the workspace size (la_forward_workspace_bytes) and
 * the errors are those of la_forward. */
LA_API la_status la_forward_from_state(const void *q, const void *k, const void *v, void *o,
                                       const float *s_in, const float *z_in,
                                       float *s_out, float *z_out, float *den_out,
                                       void *workspace, size_t workspace_bytes,
                                       int B, int H, int N, int dqk, int dv, int fmap, int dtype,
                                       void *stream);

/* Bytes of device workspace la_forward_varlen needs for nseq sequences of at
 * most max_seqlen tokens (0 if none); the rules of la_forward_workspace_bytes. */
LA_API size_t la_forward_varlen_workspace_bytes(int nseq, int H, int max_seqlen, int dqk, int dv,
                                                int fmap, int dtype);

/* Forward over a batch of sequences of different lengths, packed along the
 * token axis without padding.  Each sequence is its own causal recurrence
 * (BASED page, Knowl 3, one state per sequence and head), started from zero
 * or from s_in; no state crosses from one sequence to the next.  It is
 * la_forward (or la_forward_from_state) on B = 1, N = T with the state reset at
 * every sequence boundary.
 *   q, k        [H, T, dqk] dtype, read; v [H, T, dv] dtype, read
 *   o           [H, T, dv]  dtype, written
 *   cu_seqlens  [nseq + 1] int32, DEVICE memory, read: sequence n holds tokens
 *               cu_seqlens[n] .. cu_seqlens[n+1] - 1 of every head;
 *               0 = cu_seqlens[0] <= cu_seqlens[1] <= ... <= cu_seqlens[nseq] = T.
 *               Empty sequences are allowed (their final state is their
 *               starting state).
 *   max_seqlen  a bound on every sequence's length, >= 1; a bound above T is
 *               taken as T (it sizes the grid and the workspace, which
 *               la_forward_varlen_workspace_bytes(nseq, H, min(max_seqlen, T),
 *               ...) gives; a tight bound is fastest)
 *   s_in, z_in  [nseq, H, F, dv], [nseq, H, F] fp32, nullable (both or neither):
 *               the state entering each sequence; must not overlap s_out/z_out
 *   s_out, z_out [nseq, H, F, dv], [nseq, H, F] fp32, nullable: final states
 *   den_out     [H, T] fp32, nullable
 *   workspace   at least la_forward_varlen_workspace_bytes(...) bytes
 * The lengths live on the device, so they are checked there: a sequence with
 * cu_seqlens[n] < 0, a decreasing pair, an end beyond T or a length above
 * max_seqlen writes nothing and sets LA_ERR_DEVICE_CHECK in the device
 * status word.  Host-side argument errors are those of la_forward.  The
 * bf16 shapes with a tensor-core forward use it (the elu d = 64 shape takes
 * the one-launch chunked kernel rather than the split forward); every other
 * combination runs on the exact fp32 CUDA-core kernel. */
LA_API la_status la_forward_varlen(const void *q, const void *k, const void *v, void *o,
                                   const int32_t *cu_seqlens, int nseq, int max_seqlen, int T,
                                   const float *s_in, const float *z_in,
                                   float *s_out, float *z_out, float *den_out,
                                   void *workspace, size_t workspace_bytes,
                                   int H, int dqk, int dv, int fmap, int dtype, void *stream);

/* Gated (decayed) causal linear attention: a scalar forget gate per token,
 * a_t = exp(g_t), multiplies the state before the token is added:
 *
 *   S_t = a_t S_{t-1} + phi(k_t) v_t^T,   z_t = a_t z_{t-1} + phi(k_t),
 *   y_t = phi(q_t) S_t / phi(q_t) . z_t
 *
 * (the gated update C_t = F_t C_{t-1} + k_t v_t^T and the scalar-times-
 * identity state matrix a_t I of the reader comments on the 'Transformers
 * are RNNs' discussion page; the input-dependent decay of the BASED page,
 * Knowl 10).  The pages give no normaliser for the gated form; the same gate
 * decays z, so y_t is the mean of v_1..v_t weighted by
 * (a_{j+1} ... a_t) phi(q_t).phi(k_j).  With g = 0 everywhere this is
 * la_forward / la_forward_from_state.
 *   log_decay  [B,H,N] fp32, read: g_t = log a_t.  Gates are forget gates,
 *              g_t <= 0 (a_t in [0, 1]); -inf forgets everything before t.
 *              Positive g is computed by the same formulas but can overflow.
 *   s_in, z_in nullable (both or neither): the state entering each slice.
 *              (For a Taylor start state, the difference between the paired
 *              rows (a, b) and (b, a) decays with the gates like the rest of
 *              the state.)
 * The other arguments, layouts and errors are those of la_forward_from_state.
 * The bf16 shapes with a tensor-core forward run on it (long sequences split
 * into segments whose increments and summed gates go through the workspace,
 * la_forward_decay_workspace_bytes); there a gate below e^-80 counts as
 * e^-80, which is zero next to any surviving term in fp32.  Every other
 * combination runs on the exact fp32 CUDA-core forward, which takes -inf as
 * it is. */
LA_API size_t la_forward_decay_workspace_bytes(int B, int H, int N, int dqk, int dv, int fmap, int dtype);

LA_API la_status la_forward_decay(const void *q, const void *k, const void *v, const float *log_decay,
                                  void *o, const float *s_in, const float *z_in,
                                  float *s_out, float *z_out, float *den_out,
                                  void *workspace, size_t workspace_bytes,
                                  int B, int H, int N, int dqk, int dv, int fmap, int dtype,
                                  void *stream);

/* Gradients of la_forward_decay (from a zero state) for an upstream gradient
 * dout: dq, dk, dv as in la_backward, and dlog_decay [B,H,N] fp32 = dL/dg_t.
 * The weights of each output row sum to one, so
 *     dL/dg_l = sum over the pairs j < l <= i of w_ij dL/dw_ij
 *             = -sum_{j>=l} phi(k_j) . dL/dphi(k_j),
 * a suffix sum of per-key terms that the reverse-order pass produces.  bf16
 * with a tensor-core shape (elu dqk = dv in {64, 128}; either Taylor map with
 * dqk = 16, dv = 64) runs on the tensor-core backward with the gates inside
 * each chunk's weights (a gate below e^-80 counts as e^-80, as in the
 * forward) and a final suffix-sum kernel for dlog_decay; every other
 * combination runs on the exact fp32 CUDA-core backward.  Workspace:
 * la_backward_decay_workspace_bytes (its contents need no initialisation). */
LA_API size_t la_backward_decay_workspace_bytes(int B, int H, int N, int dqk, int dv, int fmap, int dtype);

LA_API la_status la_backward_decay(const void *q, const void *k, const void *v, const float *log_decay,
                                   const void *dout, void *dq, void *dk, void *dv, float *dlog_decay,
                                   void *workspace, size_t workspace_bytes,
                                   int B, int H, int N, int dqk, int dv_dim, int fmap, int dtype,
                                   void *stream);

/* One gated decode step: S = a S + phi(k) v^T, z = a z + phi(k), then y as in
 * la_decode_step, with a = exp(log_decay[b,h]) per head (log_decay [B,H]
 * fp32, read).  Arguments and errors otherwise those of la_decode_step. */
LA_API la_status la_decode_step_decay(const void *q, const void *k, const void *v, const float *log_decay,
                                      void *y, float *s, float *z, int B, int H, int dqk, int dv,
                                      int fmap, int dtype, void *stream);

/* Causal sliding-window softmax attention, BASED's local exact mixer
 * (BASED page, Knowl 4): query i attends only to keys max(0, i-w+1) .. i,
 *
 *     o_i = sum_j softmax_j(s_ij) v_j,   s_ij = q_i . k_j / sqrt(dqk)
 *
 * (the pages give no scale; the standard 1/sqrt(dqk) of scaled dot-product
 * attention is used).
 *   q, k [B,H,N,dqk], v, o [B,H,N,dv] dtype; lse_out [B,H,N] fp32 nullable:
 *   log sum_j exp(s_ij) over the window.
 *   window  w >= 1 (up to 1024).  bf16 with dqk = dv = 64 and w a multiple of
 *   16 up to 128 (Knowl 4: widths that are multiples of 16, generally no
 *   larger than 128) runs on the tensor cores; every other combination on an
 *   exact fp32 CUDA-core kernel.
 * Errors: LA_ERR_INVALID_ARG for a size below 1, an unknown dtype or more
 * than 2^31 elements in one tensor; LA_ERR_UNSUPPORTED for dqk or dv above
 * 128 or w above 1024.  The cache and decode calls below check the same. */
LA_API la_status la_swa_forward(const void *q, const void *k, const void *v, void *o, float *lse_out,
                                int B, int H, int N, int dqk, int dv, int window, int dtype,
                                void *stream);

/* la_kernel_plan for the sliding-window calls: decode = 0 for
 * la_swa_forward, 1 for la_swa_decode_step (N ignored).  Same output rules. */
LA_API int la_swa_kernel_plan(int decode, int B, int H, int N, int dqk, int dv, int window, int dtype,
                              char *buf, size_t buflen);

/* The w-token key/value cache of sliding-window generation (Knowl 4):
 * k_cache [B,H,w,dqk], v_cache [B,H,w,dv] of dtype; token t of a sequence
 * lives in slot t mod w.  la_swa_cache_fill copies the last min(N, w) tokens
 * of a prefill's k, v [B,H,N,*] into their slots. */
LA_API la_status la_swa_cache_fill(const void *k, const void *v, void *k_cache, void *v_cache,
                                   int B, int H, int N, int dqk, int dv, int window, int dtype,
                                   void *stream);

/* One sliding-window decode step (Knowl 5, the sliding-window generation
 * kernel): for each (b,h), store the new k, v [B,H,*] in slot pos[b] mod w
 * of the cache, then y [B,H,dv] = softmax attention of q over the
 * min(pos[b] + 1, w) cached tokens.  pos [B] int32, DEVICE memory, read: the
 * number of tokens sequence b held before this one; the caller advances it.
 * A negative pos[b] writes nothing for that sequence and sets
 * LA_ERR_DEVICE_CHECK in the device status word. */
LA_API la_status la_swa_decode_step(const void *q, const void *k, const void *v, void *y,
                                    void *k_cache, void *v_cache, const int32_t *pos,
                                    int B, int H, int dqk, int dv, int window, int dtype, void *stream);

/* la_forward for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this entry point; it is an interface
 * convenience.  la_forward may need a workspace (la_forward_workspace_bytes)
 * that the caller allocates.  Some callers have no device allocator to call:
 * a plugin running inside a host program that owns every device allocation
 * and hands out none, or a service that keeps a fixed device footprint and
 * forbids allocating on its serving path.  This variant takes the same
 * inputs and outputs as la_forward but no workspace: it uses a scratch
 * array of LA_NOALLOC_SCRATCH_BYTES (32 MiB) compiled into the library as a
 * static device array, which every GPU that loads the library holds until
 * the process exits.  It never calls cudaMalloc, cudaFree or any allocating
 * library routine.
 *   - Sizes whose workspace would exceed the scratch are rejected with
 *     LA_ERR_SCRATCH_LIMIT before anything is launched (for example elu
 *     dqk = dv = 64 with B*H = 32 and N = 16384 needs 48 MB).
 *   - The first call on a device looks up the scratch array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.  The address is kept for the life of the
 *     process: after cudaDeviceReset on a device the array goes with the old
 *     context, and this entry point must not be called on that device again
 *     in the same process.
 *   - All calls share the one array and it keeps the last call's contents.
 *     Nothing in it needs to start at zero (each call writes every value it
 *     later reads), but calls whose executions overlap on the GPU (on
 *     different streams, or from different host threads) race on it and
 *     give wrong results: serialise them.
 * Other arguments, outputs and errors are those of la_forward. */
#define LA_NOALLOC_SCRATCH_BYTES (32u << 20)
LA_API la_status la_forward_noalloc(const void *q, const void *k, const void *v, void *o,
                                    float *s_out, float *z_out, float *den_out,
                                    int B, int H, int N, int dqk, int dv, int fmap, int dtype,
                                    void *stream);

/* Gradients of the forward with respect to q, k and v for an upstream
 * gradient dout.  The pages give no backward pass; this is the derivative
 * of the Knowl 3 parallel form: with den_i = phi(q_i).z_i,
 * y_i = phi(q_i) S_i / den_i, g_i = dout_i / den_i and dden_i = -g_i . y_i,
 * a forward-order scan of (S, z) gives dphi(q_i) = S_i g_i + z_i dden_i, and
 * a reverse-order scan of R_j = sum_{i>=j} phi(q_i) g_i^T and
 * r_j = sum_{i>=j} phi(q_i) dden_i gives dphi(k_j) = R_j v_j + r_j and
 * dv_j = R_j^T phi(k_j); dq, dk then pass through the Jacobian of phi.
 * y_i and den_i are recomputed in fp32 inside the call rather than taken
 * from a rounded forward output: dq is a small difference of large terms
 * (sum_j a_ij (v_j - y_i) = 0), so a bf16-rounded y would be amplified.
 *   q, k, dout, v  as in la_forward (dout like o), read
 *   dq, dk    [B,H,N,dqk] dtype, written
 *   dv        [B,H,N,dv]  dtype, written
 *   workspace, workspace_bytes: at least la_backward_workspace_bytes(...)
 *             bytes of device memory (per-token den_i and dden_i, fp32). */
LA_API la_status la_backward(const void *q, const void *k, const void *v, const void *dout,
                             void *dq, void *dk, void *dv,
                             void *workspace, size_t workspace_bytes,
                             int B, int H, int N, int dqk, int dvdim, int fmap, int dtype,
                             void *stream);

/* One recurrent decode step for B*H heads (BASED page, Knowl 3 recurrent
 * form; Knowl 5 generation kernel): S += phi(k) v^T, z += phi(k),
 * y = phi(q) S / phi(q).z using the UPDATED state.
 *   q, k  [B,H,dqk] dtype, read;  v [B,H,dv] dtype, read
 *   y     [B,H,dv]  dtype, written
 *   s     [B,H,F,dv] fp32, read and updated in place
 *   z     [B,H,F]    fp32, read and updated in place
 * The state is read once and written once per call. */
LA_API la_status la_decode_step(const void *q, const void *k, const void *v, void *y,
                         float *s, float *z,
                         int B, int H, int dqk, int dv, int fmap, int dtype,
                         void *stream);

/* Materialise phi for `rows` input vectors: x [rows,dqk] -> phi [rows,F],
 * both of `dtype` (fp32 arithmetic, rounded once for bf16).  A test and
 * baseline helper; the attention kernels compute phi on chip instead. */
LA_API la_status la_feature_map(const void *x, void *phi, int64_t rows, int dqk, int fmap,
                         int dtype, void *stream);

/* Which kernels a call would launch, without launching anything (for
 * launch accounting in benchmarks and tests).  op: 0 = la_forward,
 * 1 = la_backward, 2 = la_decode_step, 3 = la_forward_varlen (B = nseq,
 * N = max_seqlen), 4 = la_forward_decay, 5 = la_backward_decay for the
 * tensor-core shapes.  Writes a comma-separated list of
 * kernel names (truncated to buflen-1 characters, NUL-terminated) to buf
 * when buf is non-NULL, and returns the number of kernel launches the call
 * makes, or -1 for arguments the call itself would reject.  The gated
 * calls outside this list launch fixed kernels: la_decode_step_decay the
 * one op 2 reports for its shape, la_backward_decay on the other shapes one
 * bwd_simt_kernel. */
LA_API int la_kernel_plan(int op, int B, int H, int N, int dqk, int dv, int fmap, int dtype,
                          char *buf, size_t buflen);

/* Synchronise `stream`, then read and clear the calling device's status
 * word.  Returns LA_OK, LA_ERR_TIMEOUT or LA_ERR_DEVICE_CHECK for errors
 * recorded by kernels since the last call, or LA_ERR_CUDA if the
 * synchronisation itself failed. */
LA_API la_status la_get_device_status(void *stream);

/* Self-test of the device-side failure path.  Launches one block that waits
 * on a shared-memory mbarrier nothing ever arrives on, through the same
 * bounded wait every tensor-core kernel uses, with its limit set to
 * `wait_us` microseconds instead of the kernels' 2 s.  The wait runs out,
 * the block records the timeout in the status word and returns, so the
 * context stays usable: the next la_get_device_status on this device returns
 * LA_ERR_TIMEOUT, the one after it LA_OK.  wait_us must lie in [1, 2000000];
 * other values return LA_ERR_INVALID_ARG before any launch. */
LA_API la_status la_selftest_bounded_wait(unsigned int wait_us, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LA_H */
