/*
 * libgdn2 -- Gated DeltaNet-2 recurrence on NVIDIA B200 (sm_100a).
 *
 * The recurrence ("Gated DeltaNet-2: Decoupling Erase and Write in Linear
 * Attention", iplexlaw.co.kr analysis, section "Independent decisions on two
 * axes"), per batch item b, head h and token t, with state S in R^{d_k x d_v}:
 *
 *     Sbar = diag(alpha_t) S_{t-1}        channel-wise decay of the key rows
 *     e    = b_t (.) k_t                  erase vector (key channels)
 *     z    = w_t (.) v_t                  write vector (value channels)
 *     r    = Sbar^T e                     old read at the erase address
 *     S_t  = Sbar + k_t (z - r)^T         delta write
 *     o_t  = S_t^T q_t                    output from the state after this token's update
 *
 * The prefill entry points (gdn2_chunk_fwd and its packed, segmented and
 * from-logits forms) and the decode step compute exactly this, in the two
 * execution modes the pages describe ("Token processing and parallel training":
 * chunkwise WY with 64-token chunks for training/prefill; the mindpattern.ai
 * DeltaNet trail: a fused recurrent mode for decode, with identical
 * mathematics).  gdn2_chunk_bwd gives the gradients of the prefill.
 *
 * Conventions shared by every call
 *   - All pointers are DEVICE pointers, 16-byte aligned, to dense row-major
 *     tensors.  The library allocates nothing and keeps no pointer after return.
 *   - Per-token tensors have layout [B][T][H][d] (decode: [B][H][d]).  q, k are
 *     d_k wide, v and o are d_v wide; alpha and b are d_k wide; w is d_v wide.
 *   - States are FP32 [B][H][d_k][d_v]: row i is key channel i.
 *   - q, k, v and o share the element type `dt` (BF16 or FP32).  Gates (alpha,
 *     b, w) and states are always FP32.  Accumulation is FP32.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous on that stream and never synchronise the device.
 *   - Supported head sizes: d_k, d_v in {64, 128}.  Other sizes return
 *     GDN2_ERR_UNSUPPORTED.
 *   - Preconditions (documented, not checked on the device): 0 <= alpha <= 1;
 *     b and w are not clamped (the pages ablate an erase gate in [0, 2]).
 *     Every alpha in [0, 1] is supported, however strong the decay: the
 *     prefill shortens a chunk wherever the decay accumulated inside it would
 *     leave the FP32 range of its factors.  Values of alpha below 2^-64 are
 *     computed as 2^-64 (a decayed state row then keeps less than 2^-64 of its
 *     old value instead of less than that; the difference is below FP32
 *     rounding of any quantity of the size of the state).
 *   - Errors: argument problems are detected on the host before any launch and
 *     return GDN2_ERR_INVALID_ARG / GDN2_ERR_UNSUPPORTED with nothing enqueued.
 *     A failed launch returns GDN2_ERR_CUDA; gdn2_last_error() describes it.
 *     Kernels never trap.
 */
#ifndef GDN2_H_
#define GDN2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN2_OK = 0,
    GDN2_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, negative size, aliasing not allowed */
    GDN2_ERR_UNSUPPORTED = 2,  /* head size or dtype the library does not implement */
    GDN2_ERR_CUDA = 3          /* a CUDA runtime call or kernel launch failed */
} gdn2_status;

typedef enum {
    GDN2_BF16 = 0,  /* q, k, v, o are bfloat16 */
    GDN2_FP32 = 1   /* q, k, v, o are float32  */
} gdn2_dtype;

/*
 * Chunkwise prefill ("Token processing and parallel training": 64-token blocks;
 * the per-channel decay accumulated inside a block is folded into the erase-side
 * and key-side factors, leaving one unit-triangular system and matrix products
 * per block; decay, state and the triangular system in FP32).
 *
 *   q, k      [B][T][H][d_k]  dt            read
 *   v         [B][T][H][d_v]  dt            read
 *   alpha, b  [B][T][H][d_k]  float         read
 *   w         [B][T][H][d_v]  float         read
 *   S0        [B][H][d_k][d_v] float        read; NULL means a zero initial state
 *   o         [B][T][H][d_v]  dt            written (o_t of every token)
 *   S_T       [B][H][d_k][d_v] float        written (state after token T-1); may be
 *                                           NULL, and may alias S0 (in-place chaining)
 *
 * T may be any value >= 0 (the last chunk may be partial; chunking restarts at
 * t = 0 in every call, which does not change the result).  T = 0 writes S_T = S0.
 * B = 0 or H = 0 is a no-op.  o must not overlap any input.
 * BF16 with d_k = d_v = 128 runs on the tcgen05 tensor-core path; every other
 * combination runs an FP32 CUDA-core path with the same mathematics.
 */
gdn2_status gdn2_chunk_fwd(const void *q, const void *k, const void *v,
                           const float *alpha, const float *b, const float *w,
                           const float *S0, void *o, float *S_T,
                           int B, int T, int H, int d_k, int d_v,
                           gdn2_dtype dt, void *stream);

/*
 * Chunkwise prefill of a packed batch of N variable-length sequences (the same
 * recurrence per sequence; chunking restarts at every sequence start).
 *
 *   q, k      [T_total][H][d_k]  dt          read (sequence n is rows cu_seqlens[n]
 *   v         [T_total][H][d_v]  dt          .. cu_seqlens[n+1] - 1 of every tensor)
 *   alpha, b  [T_total][H][d_k]  float       read
 *   w         [T_total][H][d_v]  float       read
 *   cu_seqlens [N + 1] int32     DEVICE      read: 0 = cu[0] <= cu[1] <= ... <= cu[N] =
 *                                            T_total.  Not checked on the host (it lives
 *                                            on the device); the kernels clamp every
 *                                            offset into [0, T_total], so a bad table
 *                                            never reads or writes outside the buffers.
 *   S0        [N][H][d_k][d_v]   float       read; NULL means zero initial states
 *   o         [T_total][H][d_v]  dt          written
 *   S_T       [N][H][d_k][d_v]   float       written (state after each sequence's last
 *                                            token; S0 for an empty sequence); may be
 *                                            NULL, and may alias S0
 *
 * Equivalent to one gdn2_chunk_fwd per sequence, in one launch (and bit for bit
 * identical to those calls).  N = 0 or H = 0 is a no-op.
 */
gdn2_status gdn2_chunk_fwd_varlen(const void *q, const void *k, const void *v,
                                  const float *alpha, const float *b, const float *w,
                                  const int32_t *cu_seqlens, int N,
                                  const float *S0, void *o, float *S_T,
                                  int T_total, int H, int d_k, int d_v,
                                  gdn2_dtype dt, void *stream);

/*
 * Chunkwise prefill of B sequences of T tokens, with each sequence cut into P
 * segments processed in parallel — for few long sequences, where the plain call
 * runs one serial chain per (sequence, head).  Same arguments and result as
 * gdn2_chunk_fwd (up to rounding: the state crosses segment boundaries through
 * an FP32 matrix product instead of the chunk loop).
 *
 * The recurrence is affine in the state ("Independent decisions on two axes":
 * S_t = (I - k_t e_t^T) diag(alpha_t) S_{t-1} + k_t z_t^T), so over a segment
 * S_end = M S_start + C, with C the end state from a zero start and M the end
 * state from the identity with z = 0.  The call runs the chunk kernel over
 * segments 0 .. P-2 twice (C and M), chains S_start(s+1) = M_s S_start(s) + C_s,
 * then runs every segment from its start state: about three times the
 * sequential work on up to 3 P times as many SMs.
 *
 *   segments   0: chosen from the shape and the current device's SM count (1 —
 *              the plain call — unless fewer chunk steps per SM result);
 *              n >= 1: n segments (capped at the number of 64-token chunks).
 *              Segments are whole chunks long, the last one shorter.
 *   workspace  DEVICE, caller-owned, 256-byte aligned, at least
 *              gdn2_chunk_fwd_segmented_workspace_size(B, T, H, d_k, d_v,
 *              segments) bytes (0 when the call resolves to one segment, in
 *              which case workspace may be NULL); contents on entry do not
 *              matter; must not overlap any argument.
 *
 * More than one segment needs BF16 with d_k = d_v = 128 (the tensor-core path):
 * GDN2_ERR_UNSUPPORTED otherwise (segments = 0 or 1 run the plain call for any
 * supported shape).  A workspace that is NULL, misaligned or too small is
 * GDN2_ERR_INVALID_ARG.  Five launches on the stream; nothing is allocated.
 * The workspace must stay untouched until the stream reaches the end of the call.
 */
gdn2_status gdn2_chunk_fwd_segmented(const void *q, const void *k, const void *v,
                                     const float *alpha, const float *b, const float *w,
                                     const float *S0, void *o, float *S_T,
                                     int B, int T, int H, int d_k, int d_v,
                                     gdn2_dtype dt, int segments,
                                     void *workspace, size_t workspace_bytes,
                                     void *stream);

/* Workspace bytes of gdn2_chunk_fwd_segmented for these arguments (segments = 0
 * resolves against the current device; 0 if there is none or the call needs no
 * workspace).  Host-only, no device memory touched. */
size_t gdn2_chunk_fwd_segmented_workspace_size(int B, int T, int H, int d_k, int d_v,
                                               int segments);

/* The number of segments gdn2_chunk_fwd_segmented would use (BF16 assumed;
 * 1 means the plain call).  Host-only. */
int gdn2_chunk_fwd_segments(int B, int T, int H, int d_k, int d_v, int segments);

/*
 * Chunkwise prefill from pre-activation logits, with the input preparation fused
 * into the tensor-core kernel ("Token processing and parallel training": the query
 * and key paths end in SiLU and L2 normalisation, the value path in SiLU;
 * "Independent decisions on two axes": the erase and write gates are sigmoids of
 * their own projections).  Per token and head, inside the kernel:
 *   q = silu(xq) / ||silu(xq)||_2,  k = silu(xk) / ||silu(xk)||_2  (a zero row stays zero)
 *   v = silu(xv),  alpha = exp(-softplus(xa)) = 1 / (1 + e^xa),  b = sigmoid(xb),  w = sigmoid(xw)
 * then the recurrence of gdn2_chunk_fwd (alpha's parameterisation is this
 * library's reading: the paper does not give it).  Every input is BF16, which
 * cuts the bytes read per token and head from 2,304 (BF16 q, k, v and FP32
 * gates) to 1,536.  The activations and the norm are computed in FP32 from the
 * BF16 logits; nothing is rounded back to BF16 on the way.
 *
 *   xq, xk, xa, xb  [B][T][H][128]  BF16   read
 *   xv, xw          [B][T][H][128]  BF16   read
 *   S0, o, S_T      as in gdn2_chunk_fwd (o BF16)
 *
 * d_k = d_v = 128 only (GDN2_ERR_UNSUPPORTED otherwise).  T = 0 writes S_T = S0;
 * B = 0 or H = 0 is a no-op; o must not overlap any input.
 */
gdn2_status gdn2_chunk_fwd_logits(const void *xq, const void *xk, const void *xv,
                                  const void *xa, const void *xb, const void *xw,
                                  const float *S0, void *o, float *S_T,
                                  int B, int T, int H, int d_k, int d_v, void *stream);

/*
 * Output epilogue ("Token processing and parallel training": after the recurrent
 * update, RMS normalisation and a separate output gate, distinct from the write
 * gate, come before the output projection).  Per (token, head) row of d_v
 * channels, in one pass:
 *   y = o / sqrt(mean_j(o_j^2) + eps) * weight * sigmoid(g)
 * The paper names the two steps without their form; this library's readings are
 * a norm over one head's channels with a per-channel weight, and a sigmoid gate.
 *
 *   o, g     [B][T][H][d_v]  dt      read (o: the recurrence's output; g: gate logits)
 *   weight   [d_v]           float   read
 *   y        [B][T][H][d_v]  dt      written; may alias o exactly (in place)
 *
 * d_v 64 or 128; eps finite and >= 0.  FP32 arithmetic, output rounded to dt.
 */
gdn2_status gdn2_output_gate(const void *o, const void *g, const float *weight, float eps, void *y,
                             int B, int T, int H, int d_v, gdn2_dtype dt, void *stream);

/*
 * Chunkwise backward ("Token processing and parallel training": training goes
 * through the chunkwise form, so its gradient carries the channel-wise decay and
 * the separate erase and write gates through every per-block factor).  Computes
 * the gradient of a scalar loss with respect to every input of gdn2_chunk_fwd,
 * given the loss's gradients with respect to its outputs.  FP32 arithmetic on
 * CUDA cores; the decay factors are exponentials of differences of cumulative
 * log-decays, so no factor leaves the FP32 range for any alpha in (0, 1].
 *
 *   q, k, v, alpha, b, w, S0   as in gdn2_chunk_fwd (B sequences of T tokens)   read
 *   dO        [B][T][H][d_v]  dt            read (dLoss/do)
 *   dST       [B][H][d_k][d_v] float        read (dLoss/dS_T); NULL means zero
 *   dq, dk    [B][T][H][d_k]  dt            written
 *   dv        [B][T][H][d_v]  dt            written
 *   dalpha, db [B][T][H][d_k] float         written
 *   dw        [B][T][H][d_v]  float         written
 *   dS0       [B][H][d_k][d_v] float        written; may be NULL
 *   workspace device buffer of at least gdn2_chunk_bwd_workspace_size(...)
 *             bytes, 16-byte aligned, owned by the caller; its contents on
 *             entry do not matter and are overwritten.
 *
 * The forward pass is recomputed inside (the states at chunk boundaries go to
 * the workspace), so nothing from gdn2_chunk_fwd needs to be kept.  alpha is
 * differentiated at max(alpha, 2^-64), the value the prefill computes with;
 * dalpha divides by that value.  Supported: d_k, d_v in {64, 128}, BF16 or FP32,
 * B * H <= 65535 (GDN2_ERR_UNSUPPORTED beyond).
 * T = 0, B = 0 or H = 0: nothing is read; dS0 = dST (zero if dST is NULL).
 * No output may overlap an input, another output or the workspace.
 */
gdn2_status gdn2_chunk_bwd(const void *q, const void *k, const void *v,
                           const float *alpha, const float *b, const float *w,
                           const float *S0, const void *dO, const float *dST,
                           void *dq, void *dk, void *dv,
                           float *dalpha, float *db, float *dw, float *dS0,
                           void *workspace, size_t workspace_bytes,
                           int B, int T, int H, int d_k, int d_v,
                           gdn2_dtype dt, void *stream);

/* Bytes of workspace gdn2_chunk_bwd needs for these sizes (0 if unsupported). */
size_t gdn2_chunk_bwd_workspace_size(int B, int T, int H, int d_k, int d_v);

/*
 * gdn2_chunk_bwd for callers that cannot allocate device memory (no counterpart
 * in the paper: an interface for code that runs inside another runtime's memory
 * manager or a fixed memory budget, or on a host path where cudaMalloc/cudaFree
 * would synchronise the device).  Same arguments and results as gdn2_chunk_bwd
 * without the workspace, which is a fixed 32 MiB array in the library's own
 * device memory, reserved on every GPU that loads the library until the process
 * exits.  Allocates nothing.
 *
 * Sizes whose gdn2_chunk_bwd_workspace_size exceeds 32 MiB are rejected with
 * GDN2_ERR_INVALID_ARG (gdn2_last_error says so).  The first call on a device
 * looks up the array's device address there (cudaGetSymbolAddress); make that
 * first call before any stream capture on that device.  Every call shares the
 * array: calls whose kernels may overlap on the GPU (other streams, other host
 * threads, without ordering) race on it.  Nothing in it needs clearing between
 * calls.
 */
gdn2_status gdn2_chunk_bwd_noalloc(const void *q, const void *k, const void *v,
                                   const float *alpha, const float *b, const float *w,
                                   const float *S0, const void *dO, const float *dST,
                                   void *dq, void *dk, void *dv,
                                   float *dalpha, float *db, float *dw, float *dS0,
                                   int B, int T, int H, int d_k, int d_v,
                                   gdn2_dtype dt, void *stream);

/*
 * Fused single-token decode step (the recurrent mode; the same mathematics with
 * T = 1, updating the state in place).
 *
 *   q, k      [B][H][d_k]  dt     read
 *   v         [B][H][d_v]  dt     read
 *   alpha, b  [B][H][d_k]  float  read
 *   w         [B][H][d_v]  float  read
 *   S         [B][H][d_k][d_v] float   read and overwritten with S_t
 *   o         [B][H][d_v]  dt     written
 *
 * Memory-bound: each call reads and writes every state once.  B = 0 or H = 0 is
 * a no-op.  o must not overlap S or any input.
 */
gdn2_status gdn2_recurrent_step(const void *q, const void *k, const void *v,
                                const float *alpha, const float *b, const float *w,
                                float *S, void *o,
                                int B, int H, int d_k, int d_v,
                                gdn2_dtype dt, void *stream);

/* Human-readable name of a status code (static string). */
const char *gdn2_status_string(gdn2_status s);

/* Text of the last GDN2_ERR_CUDA / argument error seen by this thread (static
 * thread-local buffer, valid until the next call on the same thread). */
const char *gdn2_last_error(void);

/* Device-side failure flag of the current device (synchronous; call between
 * launches).  *code = 0 when every kernel finished normally; nonzero when a
 * bounded wait inside a kernel gave up (the kernel then skipped its remaining
 * work, released its resources and returned; outputs of that call are
 * undefined).  clear != 0 resets the flag. */
gdn2_status gdn2_device_error(unsigned int *code, int clear);

/* Test hook for the kernels' failure handling.  Every wait inside the
 * tensor-core prefill kernel gives up after `cycles` SM clock cycles (default 4e9, about 2 s at the B200's
 * clock), after which the kernel raises the device-side failure flag (see
 * gdn2_device_error), skips its remaining work, waits for its in-flight
 * tensor-core operations, releases its Tensor Memory and returns.  A tiny
 * value makes the next launches fail on purpose; cycles <= 0 restores the
 * default.  Process-wide; takes effect at the next launch. */
gdn2_status gdn2_set_wait_limit(long long cycles);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int gdn2_version(void);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* GDN2_H_ */
