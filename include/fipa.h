/*
 * fipa.h -- C ABI of the fused Invariant Point Attention forward (B200, sm_100a).
 *
 * The operation is the IPA aggregation core defined on the BioTorch problem
 * page "Invariant point attention (IPA)", section "Required behavior":
 * frames applied to every query/key/value point, the logit
 *
 *   L_ijh = q_ih.k_jh / sqrt(3D) + pair_bias_ijh / sqrt(3)
 *           - 1/2 softplus(point_w_raw_h) sqrt(2/(27P)) sum_p |T_i q_ihp - T_j k_jhp|^2,
 *
 * the mask rule (key j permitted iff mask_i && mask_j && pair_mask_ij), a
 * stable softmax over j (all-zero row for an empty neighbourhood), the
 * scalar / pair / global-point aggregation, the inverse frame transform of
 * the aggregated points, the point-length features, the head-major feature
 * concatenation and the affine output projection (zero update for an empty
 * neighbourhood).
 *
 * The pair representation is given in the factorised form of "Flash
 * Invariant Point Attention" (FlashIPA): z_ij[c] = sum_r z1[i,r,c] z2[j,r,c]
 * with factors of shape (B, L, r, d); the per-head pair logit is its
 * projection pair_bias_ijh = sum_c z_ij[c] Wb[c,h], and the aggregated pair
 * value is sum_j a_hij z_ij.  No B x N x N tensor is written to device
 * memory by the forward (except the optional attention output).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers on the handle's device, owned
 *     by the caller, contiguous row-major, aligned to their element size
 *     (the workspace to 256 bytes).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - Entry points return a status; they never abort, throw or trap.  A call
 *     that fails validation launches nothing.  fipa_last_error() gives a
 *     one-line reason for the handle's most recent failure.
 *   - fipa_forward allocates nothing and does not synchronise; its kernels run
 *     asynchronously on `stream`.  One handle must not be used by two streams
 *     at the same time (its status word is shared).
 */
#ifndef FIPA_H
#define FIPA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FIPA_OK = 0,
  FIPA_ERR_INVALID_ARG = 1,     /* null / misaligned pointer, non-positive dim, bad enum */
  FIPA_ERR_UNSUPPORTED = 2,     /* valid request outside what this build implements      */
  FIPA_ERR_WORKSPACE = 3,       /* workspace pointer NULL or smaller than required        */
  FIPA_ERR_CUDA = 4,            /* a CUDA runtime/driver call failed (see last_error)     */
  FIPA_ERR_DEVICE_TIMEOUT = 5,  /* a bounded device-side wait expired (read by sync_status) */
  FIPA_ERR_INTERNAL = 6
} fipa_status;

/* dtype of ALL floating inputs ("all floating tensors are finite with common
 * dtype", Required behavior).  Outputs are float32 in both modes. */
typedef enum { FIPA_F32 = 0, FIPA_BF16 = 1 } fipa_dtype;

/* Problem sizes; every field must be > 0 ("All dimensions ... are positive").
 * F = H * (Dv + 4 Q + Cz) is derived. */
typedef struct {
  int B;     /* batch                                  */
  int N;     /* residues per sample (padded length)    */
  int H;     /* heads                                  */
  int D;     /* scalar query/key channels              */
  int Dv;    /* scalar value channels                  */
  int P;     /* query/key points per head              */
  int Q;     /* value points per head                  */
  int Cz;    /* pair channels (factor width d)         */
  int R;     /* pair factor rank r                     */
  int Cout;  /* output channels of w_out               */
} fipa_dims;

typedef struct fipa_handle fipa_handle;

/* Create a handle on CUDA device `device`.  `max_dims` may be NULL; if given,
 * later calls with any dim larger than it fail with FIPA_ERR_INVALID_ARG.
 * Allocates a few bytes of device memory for the status word (the only
 * allocation the library makes).  *out is NULL on failure.
 * Environment read here, once per handle:
 *   FIPA_WAIT_TIMEOUT_MS=<ms>  budget of every bounded device wait (default 2000)
 *   FIPA_PAIR_SPLIT=0          bfloat16 mode: pair-bias operand as one fp16 half
 *                              instead of hi + lo (faster; errors near the bf16
 *                              tolerance, so off by default)
 *   FIPA_VALUE_BUFFER=0|1|2    bfloat16 mode: each key tile's value chunks land
 *                              in a buffer of their own (the u lo chunks of the
 *                              query tile then stream with the keys); 1 (default)
 *                              from 8 key tiles per sample up, 2 wherever it
 *                              fits, 0 never
 *   FIPA_RING_STAGES=2..8      tuning: cap the shared-memory ring stages of the
 *                              core and backward kernels (default: as many as fit)
 *   FIPA_TRACE_CTA=<n>         debug trace of one core CTA (see fipa_trace_copy) */
fipa_status fipa_create(fipa_handle** out, const fipa_dims* max_dims,
                        fipa_dtype dtype, int device);

/* Bytes of device workspace fipa_forward needs for `dims` (O(B*N), no N^2
 * term).  Pure host arithmetic; no CUDA call. */
fipa_status fipa_workspace_size(const fipa_handle* h, const fipa_dims* dims,
                                size_t* bytes);

/* Fused IPA forward.
 *   q, k        [B,N,H,D]            scalar queries / keys (projected)
 *   v           [B,N,H,Dv]           scalar values
 *   q_pts,k_pts [B,N,H,P,3]          LOCAL query / key points
 *   v_pts       [B,N,H,Q,3]          LOCAL value points
 *   rot         [B,N,3,3]            proper rotations, column-vector convention
 *   trans       [B,N,3]              translations: T_i(x) = rot_i @ x + trans_i
 *   z1, z2      [B,N,R,Cz]           pair factors, z_ij[c] = sum_r z1[i,r,c] z2[j,r,c]
 *   Wb          [Cz,H]               per-head projection of the pair representation
 *   point_w_raw [H]                  raw distance weight (softplus applied inside)
 *   (all of the above: float32 or bfloat16 as fixed at fipa_create)
 *   mask        [B,N]   uint8        1 = valid residue
 *   pair_mask   [B,N,N] uint8 or NULL (NULL = all pairs allowed)
 *   w_out       [F,Cout], b_out [Cout]  (input dtype)
 *   eps         > 0, used only inside the output point-length square root
 * Outputs (float32, written for every row including padded / empty ones):
 *   out_update        [B,N,Cout]     zero for an empty neighbourhood
 *   out_local_points  [B,N,H,Q,3]    zero for an empty neighbourhood
 *   out_attention     [B,H,N,N] or NULL: the normalised attention, recomputed
 *                     by a separate validation kernel (O(N^2) memory and time)
 *   out_lse           [B,H,N] or NULL: natural-log logsumexp of the permitted
 *                     logits of each row, -inf for an empty neighbourhood
 * workspace: device buffer of >= fipa_workspace_size() bytes, 256-byte aligned,
 * contents undefined on entry and exit. */
fipa_status fipa_forward(fipa_handle* h,
                         const void* q, const void* k, const void* v,
                         const void* q_pts, const void* k_pts, const void* v_pts,
                         const void* rot, const void* trans,
                         const void* z1, const void* z2, const void* Wb,
                         const void* point_w_raw,
                         const uint8_t* mask, const uint8_t* pair_mask,
                         const void* w_out, const void* b_out, double eps,
                         const fipa_dims* dims,
                         float* out_update, float* out_local_points,
                         float* out_attention, float* out_lse,
                         void* workspace, size_t workspace_bytes,
                         void* stream);

/* The forward for query rows [row_begin, row_end) of every sample: the same
 * arguments and outputs as fipa_forward, restricted to those rows.  Each
 * output row depends on its own query and on all keys of its sample (page
 * "Invariant point attention (IPA)", Required behavior: the softmax runs over
 * every permitted key j of row i), so disjoint ranges, on one GPU or one per
 * GPU, together give exactly the full forward, bit for bit.  Every key is still
 * lifted (the prologue's O(N) work is repeated by each range); the fused core,
 * the output projection and the optional attention output run only for the
 * range's rows.  Rows outside the range are not written, in any output.
 *   row_begin   multiple of 128 (the query tile), 0 <= row_begin < row_end
 *   row_end     multiple of 128, or N; row_end <= N
 * Anything else returns FIPA_ERR_INVALID_ARG before any launch. */
fipa_status fipa_forward_rows(fipa_handle* h,
                              const void* q, const void* k, const void* v,
                              const void* q_pts, const void* k_pts, const void* v_pts,
                              const void* rot, const void* trans,
                              const void* z1, const void* z2, const void* Wb,
                              const void* point_w_raw,
                              const uint8_t* mask, const uint8_t* pair_mask,
                              const void* w_out, const void* b_out, double eps,
                              const fipa_dims* dims, int row_begin, int row_end,
                              float* out_update, float* out_local_points,
                              float* out_attention, float* out_lse,
                              void* workspace, size_t workspace_bytes,
                              void* stream);

/* Allocation-free forward.  No counterpart on the method's pages: this entry
 * point exists for callers that cannot allocate device memory where they call
 * the forward: a plugin whose host framework owns every device allocation
 * through its own pool and gives the plugin none, or a latency-bound caller
 * that may not call cudaMalloc at run time (it can synchronise the device, and
 * it can fail under memory pressure in the middle of a step).  Such callers
 * can create neither a workspace nor a handle (fipa_create allocates the
 * handle's status word), so this call takes neither.
 *
 * Scratch: one fixed device array of FIPA_NOALLOC_SCRATCH_BYTES (32 MiB)
 * inside the library, held by every GPU that loads the library until the
 * process exits.  Problems whose fipa_workspace_size exceeds it are rejected
 * with FIPA_ERR_WORKSPACE before anything is launched.  The call makes no
 * cudaMalloc / cudaFree and calls no allocating routine.
 *
 * Device: every pointer and `stream` must belong to the CURRENT device (the
 * call looks up the scratch of the current device); q or out_update on
 * another device returns FIPA_ERR_INVALID_ARG before any launch.
 *
 * Set-up: the first call on each device looks up the array's device address
 * with cudaGetSymbolAddress and reads FIPA_WAIT_TIMEOUT_MS (as fipa_create
 * does); a device that is not sm_100 returns FIPA_ERR_UNSUPPORTED there.
 *
 * Sharing: every call uses the same array and leaves its contents behind, so
 * calls whose kernels could overlap on the GPU (different streams without
 * ordering between them) race; order them on one stream or with events.
 * Nothing in the array needs clearing between calls: every kernel writes all
 * of what a later kernel of the same call reads.
 *
 * Arguments and outputs are those of fipa_forward (no attention output); the
 * kernels run asynchronously on `stream`.  A bounded device-side wait that
 * expires (which only a faulty device or build can cause) leaves the outputs
 * undefined and is not reported by this call. */
#define FIPA_NOALLOC_SCRATCH_BYTES (32u << 20)
fipa_status fipa_forward_noalloc(fipa_dtype dtype,
                                 const void* q, const void* k, const void* v,
                                 const void* q_pts, const void* k_pts, const void* v_pts,
                                 const void* rot, const void* trans,
                                 const void* z1, const void* z2, const void* Wb,
                                 const void* point_w_raw,
                                 const uint8_t* mask, const uint8_t* pair_mask,
                                 const void* w_out, const void* b_out, double eps,
                                 const fipa_dims* dims,
                                 float* out_update, float* out_local_points, float* out_lse,
                                 void* stream);

/* Gradients of the backward pass: float32 device buffers, each with the layout
 * of the input it belongs to.  Every element is written. */
typedef struct {
  float* q;            /* [B,N,H,D]   */
  float* k;            /* [B,N,H,D]   */
  float* v;            /* [B,N,H,Dv]  */
  float* q_pts;        /* [B,N,H,P,3] */
  float* k_pts;        /* [B,N,H,P,3] */
  float* v_pts;        /* [B,N,H,Q,3] */
  float* rot;          /* [B,N,3,3]   */
  float* trans;        /* [B,N,3]     */
  float* z1;           /* [B,N,R,Cz]  */
  float* z2;           /* [B,N,R,Cz]  */
  float* Wb;           /* [Cz,H]      */
  float* point_w_raw;  /* [H]         */
  float* w_out;        /* [F,Cout]    */
  float* b_out;        /* [Cout]      */
} fipa_grads;

/* Bytes of device workspace fipa_backward needs for `dims` (O(B*N): the
 * recompute's workspace plus the backward's per-residue buffers).  Pure host
 * arithmetic.  FIPA_ERR_UNSUPPORTED for widths beyond the backward kernels'
 * tensor-memory or shared-memory budget. */
fipa_status fipa_backward_workspace_size(const fipa_handle* h, const fipa_dims* dims,
                                         size_t* bytes);

/* Backward pass (training).  The page "Invariant point attention (IPA)",
 * section "Starter code", grades the full suite "including gradients"; this
 * computes them: the gradient of <d_update, update> + <d_local_points,
 * local_points> with respect to every floating input of fipa_forward (masks
 * are not differentiated), written to `grads`.
 *   inputs            exactly those of the fipa_forward call being differentiated
 *   d_update          [B,N,Cout] float32 cotangent of update
 *   d_local_points    [B,N,H,Q,3] float32 cotangent of local_points, or NULL (zero)
 *   grads             float32 outputs (fipa_grads), caller-owned device buffers
 *   workspace         >= fipa_backward_workspace_size() bytes, 256-byte aligned
 * The call recomputes the forward it needs (the lift and the fused core, which
 * also keeps the normalised aggregates of every row) inside the workspace, so
 * it needs no state from an earlier fipa_forward.  Rows with an empty
 * neighbourhood have constant (zero) outputs and pass no gradient back.
 * The attention products run on fp16 tensor-core operands with fp32
 * accumulation, for bfloat16 and float32 inputs alike (float32 inputs are
 * recomputed in the bfloat16 lifted layout); the two dense products of the
 * output projection (d_update w_out^T and features^T d_update) take every
 * float32 operand as a bfloat16 hi + lo pair (about 2^-17 relative).  The
 * gradients' normwise error is of the order of 1e-3.  Allocates nothing, does not synchronise; kernels run on `stream`.
 * Deterministic: every sum is taken in a fixed order. */
fipa_status fipa_backward(fipa_handle* h,
                          const void* q, const void* k, const void* v,
                          const void* q_pts, const void* k_pts, const void* v_pts,
                          const void* rot, const void* trans,
                          const void* z1, const void* z2, const void* Wb,
                          const void* point_w_raw,
                          const uint8_t* mask, const uint8_t* pair_mask,
                          const void* w_out, const void* b_out, double eps,
                          const fipa_dims* dims,
                          const float* d_update, const float* d_local_points,
                          const fipa_grads* grads,
                          void* workspace, size_t workspace_bytes,
                          void* stream);

/* Training without the recompute: fipa_forward_train is fipa_forward (no
 * attention output) that also keeps, in a workspace of
 * fipa_backward_workspace_size() bytes, the state the backward needs (the
 * lifted rows, the row statistics and the normalised aggregates of every row);
 * fipa_backward_saved then takes the gradients from that state instead of
 * recomputing the lift and the fused core.  Same arguments as fipa_forward /
 * fipa_backward.  The workspace must not be written between the two calls, and
 * both must get the same inputs and dims (not checked: the backward would use
 * stale state).  The gradients equal fipa_backward's bit for bit.  bfloat16
 * inputs only (FIPA_ERR_UNSUPPORTED otherwise). */
fipa_status fipa_forward_train(fipa_handle* h,
                               const void* q, const void* k, const void* v,
                               const void* q_pts, const void* k_pts, const void* v_pts,
                               const void* rot, const void* trans,
                               const void* z1, const void* z2, const void* Wb,
                               const void* point_w_raw,
                               const uint8_t* mask, const uint8_t* pair_mask,
                               const void* w_out, const void* b_out, double eps,
                               const fipa_dims* dims,
                               float* out_update, float* out_local_points, float* out_lse,
                               void* workspace, size_t workspace_bytes, void* stream);
fipa_status fipa_backward_saved(fipa_handle* h,
                                const void* q, const void* k, const void* v,
                                const void* q_pts, const void* k_pts, const void* v_pts,
                                const void* rot, const void* trans,
                                const void* z1, const void* z2, const void* Wb,
                                const void* point_w_raw,
                                const uint8_t* mask, const uint8_t* pair_mask,
                                const void* w_out, const void* b_out, double eps,
                                const fipa_dims* dims,
                                const float* d_update, const float* d_local_points,
                                const fipa_grads* grads,
                                void* workspace, size_t workspace_bytes,
                                void* stream);

/* Device time in milliseconds of each stage of the most recent fipa_backward
 * or fipa_backward_saved recorded with stage timing on (fipa_enable_stage_timing),
 * in launch order: [0] recompute (lift and fused core; about 0 when saved), [1] cotangent preparation (d_update @
 * w_out^T and the per-residue dO rows), [2] q-side kernel (dS, dQhat), [3]
 * k-side kernel (dKhat, dVhat, dz2), [4] chain rule through frames and
 * factors and the weight gradients.  Waits for that call's last event. */
#define FIPA_BWD_STAGES 5
fipa_status fipa_backward_stage_times(fipa_handle* h, float* ms, int n);

/* The IPA layer around the core (float32 handle).  The page "Invariant point
 * attention (IPA)" (Required behavior) defines the core as starting after the
 * input projections and ending before any residual or frame update, and asks
 * not to invent weights; this layer applies the plainest forms of those steps
 * with every weight supplied by the caller:
 *   X = s @ W_in + b_in                      s [B,N,Cs], W_in [Cs,Din], b_in [Din]
 *       split in order into q [H,D], k [H,D], v [H,Dv], q_pts [H,P,3],
 *       k_pts [H,P,3], v_pts [H,Q,3], z1 [R,Cz], z2 [R,Cz] (row-major blocks),
 *       Din = H(2D + Dv) + 3H(2P + Q) + 2 R Cz
 *   the fused core with rot, trans, masks, Wb, point_w_raw, w_out [F,Cs], b_out [Cs]
 *   s' = s + update                          -> out_s [B,N,Cs]
 *   [b c d tx ty tz] = s' @ W_bb + b_bb      W_bb [Cs,6], b_bb [6]
 *   R' = R R(q), q = (1,b,c,d)/|(1,b,c,d)|;  t' = R (tx,ty,tz) + t
 *                                            -> out_rot [B,N,3,3], out_trans [B,N,3]
 *   (a masked residue keeps its frame), and the core's local points.
 * dims->Cout must equal Cs.  All pointers float32 device buffers except the
 * masks; workspace >= fipa_layer_workspace_size() bytes, 256-byte aligned.
 * FIPA_ERR_UNSUPPORTED with a bfloat16 handle.  Allocates nothing; runs on
 * `stream`. */
fipa_status fipa_layer_workspace_size(const fipa_handle* h, const fipa_dims* dims, size_t* bytes);
fipa_status fipa_ipa_layer(fipa_handle* h, const float* s, const float* W_in, const float* b_in,
                           const float* rot, const float* trans, const uint8_t* mask,
                           const uint8_t* pair_mask, const float* Wb, const float* point_w_raw,
                           const float* w_out, const float* b_out, const float* W_bb,
                           const float* b_bb, double eps, const fipa_dims* dims,
                           float* out_s, float* out_rot, float* out_trans, float* out_local_points,
                           void* workspace, size_t workspace_bytes, void* stream);

/* k-nearest-neighbour distogram features ("Flash Invariant Point Attention",
 * rebuttal answer 6: keep the k nearest neighbours of each residue,
 * (B, L, k, n_bins), instead of the (B, L, L, n_bins) distogram; found
 * block-wise, without an L x L matrix).
 *   trans       [B,N,3]  frame translations (float32 or bfloat16 as `dtype`)
 *   mask        [B,N]    uint8, 1 = valid residue
 *   k           1..32 neighbours per residue (the pages use 20)
 *   edges       [n_bins - 1] float32, ascending; the bin of a distance d is the
 *               number of edges e <= d (NULL allowed when n_bins == 1)
 * Outputs (device, caller-owned):
 *   out_idx     [B,N,k] int32   neighbour residue indices, nearest first; the
 *               neighbours of i are the valid residues of its sample, i itself
 *               included; ties in distance go to the smaller index
 *   out_dist    [B,N,k] float32 distances (+inf for an empty slot)
 *   out_bin     [B,N,k] int32   distogram bins (-1 for an empty slot)
 *   out_onehot  [B,N,k,n_bins] float32 one-hot bins, or NULL
 * A masked residue has no neighbours (all slots empty); a sample with fewer
 * than k valid residues leaves the remaining slots empty.  The order is decided
 * on the squared distance ((dx dx) + (dy dy)) + (dz dz), each operation rounded
 * to float32.  No handle: every pointer belongs to the current device.
 * Allocates nothing; runs on `stream`.  FIPA_ERR_UNSUPPORTED for k > 32 or
 * B > 65535. */
fipa_status fipa_knn_distogram(fipa_dtype dtype, const void* trans, const uint8_t* mask,
                               int B, int N, int k, const float* edges, int n_bins,
                               int32_t* out_idx, float* out_dist, int32_t* out_bin,
                               float* out_onehot, void* stream);

/* Wait for `stream`, then read and clear the handle's device status word.
 * Returns FIPA_ERR_DEVICE_TIMEOUT if a kernel gave up on a bounded wait since
 * the last call, FIPA_ERR_CUDA if the stream reports an error, else FIPA_OK. */
fipa_status fipa_sync_status(fipa_handle* h, void* stream);

/* Failure-path self-test.  Launches on `stream` one CTA whose bounded wait on
 * an mbarrier that nothing completes runs out after `timeout_ms` (1..10000):
 * the kernel records FIPA_ERR_DEVICE_TIMEOUT in the handle's status word and
 * returns, exactly as a real wait of any library kernel would, without a
 * fault or a hang; the next fipa_sync_status reports it and clears the word.
 * Returns FIPA_ERR_INVALID_ARG for a null handle or an out-of-range timeout. */
fipa_status fipa_selftest_timeout(fipa_handle* h, unsigned timeout_ms, void* stream);

/* Profiling aid (stage timing).  With `enable` nonzero, later fipa_forward
 * calls on this handle record a CUDA event before and after each of their
 * kernels on the call's stream; the events are created here, so fipa_forward
 * still allocates nothing.  `enable` = 0 turns recording off and frees them.
 * fipa_backward calls record their own stage events the same way.
 * A CUDA graph captured from a timed call records into these events on every
 * replay: release such a graph before turning timing off. */
fipa_status fipa_enable_stage_timing(fipa_handle* h, int enable);

/* Device time in milliseconds of each stage of the most recent fipa_forward
 * recorded with stage timing on, in launch order: [0] prologue (output-weight
 * preparation, group origins and lifted rows), [1] fused attention core with
 * the feature epilogue, [2] output projection, [3] attention output (0 when
 * not requested).  Each interval spans one kernel launch between two event
 * records.  Waits for that call's last event.  `n` = capacity of `ms` (up to
 * FIPA_STAGES values are written). */
#define FIPA_STAGES 4
fipa_status fipa_stage_times(fipa_handle* h, float* ms, int n);

/* Debug tracing.  When the environment variable FIPA_TRACE_CTA=<n> is set at
 * fipa_create, the handle owns a small device buffer and the fused core's CTA
 * number n (linear block index) logs (event id, SM clock) pairs per warp role
 * during every fipa_forward.  fipa_trace_copy waits for `stream` and copies the
 * log: 4 roles (0 TMA producer, 1 MMA issuer, 2 softmax lane 0, 3 key-term
 * warps) x FIPA_TRACE_CAP entries x {event, clock}, int64, -1 = unused.
 * Returns FIPA_ERR_INVALID_ARG if tracing is off or `n_values` is too small. */
#define FIPA_TRACE_CAP 4096
fipa_status fipa_trace_copy(fipa_handle* h, int64_t* host, size_t n_values, void* stream);

/* Number of kernels one fipa_forward with these dims launches (plus one when
 * the attention output is requested).  Pure host arithmetic. */
fipa_status fipa_kernel_count(const fipa_handle* h, const fipa_dims* dims, int with_attention,
                              int* count);

/* Static description of a status code. */
const char* fipa_status_string(fipa_status s);

/* One-line reason for the handle's most recent failure ("" if none).
 * The string is owned by the handle and valid until its next call. */
const char* fipa_last_error(const fipa_handle* h);

/* Release the handle and its status word.  NULL is accepted. */
fipa_status fipa_destroy(fipa_handle* h);

#ifdef __cplusplus
}
#endif
#endif /* FIPA_H */
