/*
 * gdn2.h -- C ABI of the B200 (sm_100a) Gated DeltaNet-2 forward operator.
 *
 * The operator is the Gated Delta Rule-2 recurrence.  Per (sequence, head),
 * for t = 1..T (page "Gated DeltaNet-2：将擦除与写入分开", iplexlaw blog,
 * section "在两个维度上独立控制"):
 *
 *     e_t = b_t * k_t                   erase vector, key channels
 *     z_t = w_t * v_t                   write vector, value channels
 *     Sbar = diag(alpha_t) S_{t-1}      channel-wise decay on the key axis
 *     r_t = Sbar^T e_t                  read along the erase vector
 *     S_t = Sbar + k_t (z_t - r_t)^T
 *     o_t = scale * S_t^T q_t           the query reads the updated state
 *
 * with alpha_t = exp(log_alpha_t).  The state S is dk x dv (row = key channel,
 * column = value channel).  gdn2_chunk_fwd evaluates the recurrence in the
 * 64-token chunkwise WY form (same page, section "词元路径与并行训练": 64-token
 * chunks, cumulative channel-wise decay folded into the erase factors, an
 * in-chunk triangular solve plus dense products, fp32 for the decay, the state
 * and the solve).  Results equal the token recurrence up to rounding.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers.   Every tensor argument is a DEVICE pointer owned by the caller,
 *             16-byte aligned and densely packed in the layout given below.
 *             The library allocates no memory and never synchronises a
 *             stream; all work is enqueued on `stream` (0 = legacy default).
 * Layouts.    Token-major.  q, k, log_alpha, b : [B, T, H, dk];
 *             v, w, out : [B, T, H, dv]; states h0, hT : [N, H, dk, dv] fp32
 *             with N = B (dense) or N = num_seqs (packed).
 * Precision.  q, k, v and out are fp32 (GDN2_IO_F32) or bf16 (GDN2_IO_BF16);
 *             log_alpha, b, w, h0, hT and state are always fp32.  The decay,
 *             the state and the triangular solve are computed in fp32.
 * Packing.    With cu_seqlens != NULL the batch is one packed row (B must be
 *             1, T = total tokens) holding num_seqs sequences; sequence n
 *             covers tokens [cu_seqlens[n], cu_seqlens[n+1]).  cu_seqlens is
 *             an int32 device array of num_seqs + 1 entries, starting at 0,
 *             non-decreasing and ending at T.  Chunks start at each sequence's
 *             first token, so a sequence's result does not depend on what it
 *             is packed with (bitwise).
 * Shapes.     dk and dv are each 64 or 128; H >= 1; B >= 1; T >= 0.
 * Errors.     Returned as gdn2_status, never thrown; the library never exits,
 *             aborts or traps.  A returned GDN2_OK means the host-side checks
 *             passed and the launches were accepted.  cu_seqlens lives on the
 *             device, so its contents are checked on the device: a bad array
 *             leaves the outputs unspecified and stores GDN2_ERR_SEQLENS in the
 *             workspace status word (see gdn2_workspace_layout).
 */
#ifndef GDN2_H_
#define GDN2_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define GDN2_API __attribute__((visibility("default")))
#else
#define GDN2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gdn2_status {
  GDN2_OK = 0,
  GDN2_ERR_NULL = 1,          /* a required pointer is NULL                       */
  GDN2_ERR_SHAPE = 2,         /* unsupported or inconsistent sizes                */
  GDN2_ERR_DTYPE = 3,         /* unknown gdn2_io_dtype                            */
  GDN2_ERR_ALIGN = 4,         /* a pointer is not 16-byte aligned                 */
  GDN2_ERR_SEQLENS = 5,       /* cu_seqlens is malformed (device status word)     */
  GDN2_ERR_WORKSPACE = 6,     /* workspace missing or smaller than required       */
  GDN2_ERR_CUDA = 7,          /* a CUDA runtime call or launch failed             */
  GDN2_ERR_DEVICE_TIMEOUT = 8,/* a bounded device-side wait gave up               */
  GDN2_ERR_UNSUPPORTED = 9    /* the current device is not sm_100 (B200 class)    */
} gdn2_status;

typedef enum gdn2_io_dtype {
  GDN2_IO_F32 = 0,   /* q, k, v, out in fp32 (correctness mode)                  */
  GDN2_IO_BF16 = 1   /* q, k, v, out in bf16 (the fast path)                    */
} gdn2_io_dtype;

/* Problem description.  `workspace` is a caller-owned device buffer of at
 * least gdn2_workspace_size(desc) bytes, 256-byte aligned; its contents on
 * entry do not matter and are overwritten. */
typedef struct gdn2_desc {
  int B;                   /* batch size (1 when packed)                         */
  int T;                   /* tokens per sequence, or total tokens when packed   */
  int H;                   /* heads                                              */
  int dk;                  /* key dimension, 64 or 128                           */
  int dv;                  /* value dimension, 64 or 128                         */
  int num_seqs;            /* packed: sequences in the row (>= 1, with         */
                           /* cu_seqlens); dense: must be 0                     */
  gdn2_io_dtype io;        /* dtype of q, k, v, out                              */
  void* workspace;         /* device scratch, caller-owned                       */
  size_t workspace_bytes;  /* its size in bytes                                  */
} gdn2_desc;

/* Where the per-chunk factors live inside the workspace, so that callers
 * (and tests) can inspect what gdn2_chunk_prep produced.  All offsets are in
 * bytes from `workspace`.  Factor tensors are indexed [max_chunks, H, ...] in
 * the element size `factor_elem_bytes` (4 = fp32 for GDN2_IO_F32, 2 = bf16 for
 * GDN2_IO_BF16); rows past a chunk's last token are zero.  Chunk c of
 * sequence n has global index chunk_offsets[n] + c (int32 array of N + 1
 * entries); gamma_last is [max_chunks, H, dk] fp32.
 *
 * Two factor sets exist.  Both hold Q_eff, O_part and gamma_last.
 *  factor_set 0 ("WY", fp32 I/O and dk = 64): W, U~ and Kbar, with which the
 *    walk computes U = U~ - W S and S' = diag(gamma) S + Kbar^T U.
 *  factor_set 1 ("affine", bf16 I/O with dk = 128): the chunk's affine state
 *    map, Mp = Kbar^T W [dk, dk] and Nc = Kbar^T U~ [dk, dv], so that
 *    S' = diag(gamma) S - Mp S + Nc (one matrix product per chunk).  In this
 *    set Mp and Q_eff are stored with their columns divided by colscale
 *    ([., H, dk] fp32, exp of the in-chunk cumulative log-decay at token 32,
 *    1 for chunks from the exact kernel): the factors are Mp diag(colscale)
 *    and Q_eff diag(colscale).
 * Tensors of the other set have zero size. */
typedef struct gdn2_ws_layout {
  size_t total_bytes;
  int max_chunks;            /* upper bound on chunks: T_total/64 + N            */
  int factor_elem_bytes;
  int factor_set;            /* 0 = WY, 1 = affine (see above)                   */
  int reserved;
  size_t off_W;              /* W     = T E~           [., H, 64, dk]   set 0    */
  size_t off_Ut;             /* U~    = T Z            [., H, 64, dv]   set 0    */
  size_t off_Kbar;           /* Kbar  = k exp(g_n - g) [., H, 64, dk]   set 0    */
  size_t off_Qeff;           /* Q_eff = Q~ - P W       [., H, 64, dk]            */
  size_t off_Opart;          /* O_part= P U~           [., H, 64, dv]            */
  size_t off_gamma_last;     /* exp(g_n)               [., H, dk] fp32           */
  size_t off_Mp;             /* Mp    = Kbar^T W       [., H, dk, dk]   set 1    */
  size_t off_Nc;             /* Nc    = Kbar^T U~      [., H, dk, dv]   set 1    */
  size_t off_chunk_offsets;  /* int32 [N + 1]                                    */
  size_t off_status;         /* int32 status word (a gdn2_status value)          */
  size_t off_fix;            /* int32 [1 + max_chunks * H]: chunks whose decay   */
                             /* is too steep for the tensor-core prep, redone    */
                             /* exactly ([0] = count, then chunk * H + head)     */
  size_t off_sync;           /* int32 [2 + max_chunks * H] (set 1): [0] next     */
                             /* prep task, [1] walk redo flag, then one ready    */
                             /* flag per (chunk, head) for the fused prep + walk */
                             /* (0 = not yet, 2 = factors written, 3 = handed    */
                             /* back for the exact redo)                         */
  size_t off_colscale;       /* column scale of Mp, Q_eff [., H, dk] fp32 set 1 */
} gdn2_ws_layout;

/* Bytes of workspace gdn2_chunk_fwd needs for `desc` (0 if desc is invalid).
 * num_seqs > 0 describes a packed call (cu_seqlens given), 0 a dense one. */
GDN2_API size_t gdn2_workspace_size(const gdn2_desc* desc);

/* Fill *layout for `desc`.  Host-only, no CUDA call. */
GDN2_API gdn2_status gdn2_workspace_layout(const gdn2_desc* desc, gdn2_ws_layout* layout);

/* Chunkwise forward pass: O and the final state.
 *   q, k       : [B, T, H, dk]  io dtype
 *   v          : [B, T, H, dv]  io dtype
 *   log_alpha  : [B, T, H, dk]  fp32, log of the channel-wise decay (<= 0)
 *   b          : [B, T, H, dk]  fp32 erase gate (key channels)
 *   w          : [B, T, H, dv]  fp32 write gate (value channels)
 *   scale      : output scale (the usual choice dk^-1/2 is the caller's)
 *   h0         : [N, H, dk, dv] fp32 initial state, or NULL for zeros
 *   cu_seqlens : int32 [num_seqs + 1] (device) or NULL for B dense sequences
 *   out        : [B, T, H, dv]  io dtype
 *   hT         : [N, H, dk, dv] fp32 final state, or NULL to skip; may alias h0
 * Asynchronous on `stream`.  For bf16 I/O with dk = 128, when the walk needs
 * at most (SM count - 32) CTAs (sequences x H x dv/64), the prep and the walk
 * run in one launch and the walk takes each chunk's factors as soon as they
 * are written (gdn2_chunk_fused, a cooperative launch: all its CTAs are
 * resident at once, or it is not launched); otherwise, or when the
 * cooperative launch is refused (fewer SMs available than the device has),
 * it runs gdn2_chunk_prep then gdn2_chunk_walk.  Both orders compute the same
 * values. */
GDN2_API gdn2_status gdn2_chunk_fwd(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                           const float* log_alpha, const float* b, const float* w, float scale,
                           const float* h0, const int32_t* cu_seqlens, void* out, float* hT,
                           cudaStream_t stream);

/* Stage 1 of gdn2_chunk_fwd: gate preparation and the intra-chunk WY factors
 * of every (chunk, head), written to the workspace (layout above).  Depends
 * only on the inputs of each chunk, not on any state. */
GDN2_API gdn2_status gdn2_chunk_prep(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                            const float* log_alpha, const float* b, const float* w,
                            const int32_t* cu_seqlens, cudaStream_t stream);

/* Stage 2 of gdn2_chunk_fwd: the inter-chunk state walk and the outputs,
 * reading the factors gdn2_chunk_prep left in the workspace.  If
 * chunk_states is not NULL it receives the state at the START of every chunk,
 * [max_chunks, H, dk, dv] fp32 indexed by global chunk index (diagnostics). */
GDN2_API gdn2_status gdn2_chunk_walk(const gdn2_desc* desc, float scale, const float* h0,
                            const int32_t* cu_seqlens, void* out, float* hT,
                            float* chunk_states, cudaStream_t stream);

/* The bookkeeping every chunked call starts with: chunk offsets of the
 * sequences (from cu_seqlens on the device), the status word, and the lists
 * and flags of the affine path, all in the workspace.  gdn2_chunk_fwd and
 * gdn2_chunk_prep run it themselves; gdn2_chunk_fused needs it first. */
GDN2_API gdn2_status gdn2_chunk_plan(const gdn2_desc* desc, const int32_t* cu_seqlens, cudaStream_t stream);

/* The single launch of gdn2_chunk_fwd's fused path (see there), without the
 * plan before it or the exact redo after it of chunks whose decay is too steep
 * for the tensor-core prep; call gdn2_chunk_plan first.  A call then gives the
 * full result unless such a chunk exists, which gdn2_chunk_fwd handles.
 * Returns GDN2_ERR_UNSUPPORTED when the problem does not take the fused path
 * (not bf16 with dk = 128, or the walk needs too many CTAs) or when the
 * cooperative launch cannot make every CTA resident at once. */
GDN2_API gdn2_status gdn2_chunk_fused(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                             const float* log_alpha, const float* b, const float* w, float scale,
                             const float* h0, const int32_t* cu_seqlens, void* out, float* hT,
                             cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Two-level chunk scan (state passing between ranges of a sequence).
 *
 * Over any range of tokens the recurrence is affine in the state: the state at
 * the end of the range is Phi S_start + Psi, with Phi (dk x dk) the product of
 * the per-token linear parts (I - k_t e_t^T) diag(alpha_t) and Psi (dk x dv)
 * the state the range reaches from zero (page "Gated DeltaNet-2：将擦除与写入分开",
 * section "在两个维度上独立控制", applied token after token).  Maps of
 * consecutive ranges compose: (Phi2 Phi1, Phi2 Psi1 + Psi2).  The walk over a
 * long sequence is a chain of T/64 dependent chunk steps; splitting it into
 * segments of L chunks turns it into (1) every segment's map, in parallel,
 * (2) a short fp32 scan of the maps that gives each segment its start state,
 * (3) every segment's walk with outputs, in parallel.  Ranks that each hold a
 * range of one long sequence pass state the same way: each computes its
 * range's map (gdn2_state_map), the maps of the earlier ranges give its start
 * state, and it runs gdn2_chunk_fwd from there.
 * Affine factor set only (bf16 I/O with dk = 128); GDN2_ERR_UNSUPPORTED
 * otherwise.
 * ------------------------------------------------------------------------ */

/* Workspace bytes of gdn2_chunk_fwd_segmented: gdn2_workspace_size(desc) plus
 * the segments, their maps and start states (0 if desc is invalid or not the
 * affine set).  segment_chunks = L, the chunks per segment; 0 chooses
 * max(8, ceil(chunks per sequence / 4)) (from desc alone). */
GDN2_API size_t gdn2_segmented_workspace_size(const gdn2_desc* desc, int segment_chunks);

/* gdn2_chunk_fwd through the two-level chunk scan (arguments and results as
 * there; desc->workspace holds gdn2_segmented_workspace_size(desc,
 * segment_chunks) bytes).  Each sequence is split into segments of
 * segment_chunks 64-token chunks (0: see above); the outputs equal
 * gdn2_chunk_fwd's up to rounding (the start state of a segment is the fp32
 * product of the earlier segments' maps instead of a chunk-by-chunk walk).
 * Asynchronous on `stream`. */
GDN2_API gdn2_status gdn2_chunk_fwd_segmented(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                                              const float* log_alpha, const float* b, const float* w, float scale,
                                              const float* h0, const int32_t* cu_seqlens, void* out, float* hT,
                                              int segment_chunks, cudaStream_t stream);

/* The affine state map of every sequence of the call (the whole range of its
 * tokens): phi [N, H, dk, dk] and psi [N, H, dk, dv], fp32, device, so that
 * the final state from a start state S is phi S + psi.  q is needed by the
 * chunk preparation it shares with gdn2_chunk_fwd; the workspace is
 * gdn2_workspace_size(desc) bytes.  An empty sequence (or a malformed
 * cu_seqlens, reported in the status word) gives the identity map.
 * Asynchronous on `stream`. */
GDN2_API gdn2_status gdn2_state_map(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                                    const float* log_alpha, const float* b, const float* w,
                                    const int32_t* cu_seqlens, float* phi, float* psi, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Token path around the operator (page "Gated DeltaNet-2：将擦除与写入分开",
 * section "词元路径与并行训练"): q and k pass through a short causal
 * convolution, SiLU and L2 normalisation, v through the convolution and SiLU;
 * the operator's output passes through RMS normalisation and an output gate of
 * its own.  The linear projections before and after need trained weights and
 * stay with the caller.  Readings where the pages are silent: depthwise
 * convolution over the H*d channels of a projection, causal inside each
 * sequence (tokens before its first count as zero), width conv_width (1..8);
 * eps = 1e-6 in both norms; the gate is sigmoid(g).
 * ------------------------------------------------------------------------ */

/* q = l2norm(silu(conv(q_raw))), k = l2norm(silu(conv(k_raw))),
 * v = silu(conv(v_raw)), per token and head.
 *   q_raw, k_raw, q, k : [B, T, H, dk] io dtype;  v_raw, v : [B, T, H, dv]
 *   conv_q, conv_k     : [H * dk, conv_width] fp32, tap i weighs token t - i
 *   conv_v             : [H * dv, conv_width] fp32
 *   cu_seqlens         : as for gdn2_chunk_fwd (sequence starts reset the
 *                        convolution), or NULL for B dense sequences.  It is
 *                        not validated here (there is no status word): a
 *                        malformed array gives unspecified outputs, but
 *                        every access stays inside the buffers above and
 *                        its num_seqs + 1 entries.
 * desc: B, T, H, dk, dv, num_seqs and io as for gdn2_chunk_fwd (the workspace
 * is not used).  Outputs must not overlap the inputs.  Device pointers,
 * 16-byte aligned.  Asynchronous on `stream`.
 * Errors (before any launch): GDN2_ERR_NULL, _DTYPE, _SHAPE (dims, num_seqs
 * against cu_seqlens, conv_width outside 1..8), _ALIGN; _UNSUPPORTED without
 * an sm_100 device. */
GDN2_API gdn2_status gdn2_token_prologue(const gdn2_desc* desc, const void* q_raw, const void* k_raw,
                                         const void* v_raw, const float* conv_q, const float* conv_k,
                                         const float* conv_v, int conv_width, const int32_t* cu_seqlens, void* q,
                                         void* k, void* v, cudaStream_t stream);

/* out = rmsnorm(o) * norm_weight * sigmoid(gate), per token and head, the norm
 * over the dv channels of a head.
 *   o, gate, out : [B, T, H, dv] io dtype (out may be o);  norm_weight : [dv] fp32
 * desc: B, T, H, dk, dv, io (the rest is not used).  Asynchronous on `stream`.
 * Errors (before any launch): GDN2_ERR_NULL, _DTYPE, _SHAPE, _ALIGN (every
 * pointer 16-byte aligned); _UNSUPPORTED without an sm_100 device. */
GDN2_API gdn2_status gdn2_token_epilogue(const gdn2_desc* desc, const void* o, const void* gate,
                                         const float* norm_weight, void* out, cudaStream_t stream);

/* gdn2_chunk_walk with the walk taking each chunk only once its ready flag in
 * the workspace (off_sync, the flags gdn2_chunk_fused's prep raises) reads 2,
 * and with every bounded device-side wait limited to wait_budget_ns (0 = the
 * default of 2 s).  For tests and diagnostics of the fused path's hand-off: a
 * walk whose flags nobody raises ends after the limit with
 * GDN2_ERR_DEVICE_TIMEOUT in the workspace status word and its outputs
 * unspecified, instead of hanging.  Affine factor set only (bf16 I/O with
 * dk = 128); GDN2_ERR_UNSUPPORTED otherwise.  Asynchronous on `stream`. */
GDN2_API gdn2_status gdn2_chunk_walk_flagged(const gdn2_desc* desc, float scale, const float* h0,
                                             const int32_t* cu_seqlens, void* out, float* hT,
                                             unsigned long long wait_budget_ns, cudaStream_t stream);

/* Bytes of workspace gdn2_chunk_bwd needs for `desc` (0 if desc is invalid):
 * a status word, the fp32 chunk factors of the forward (W, U~, Kbar, Q_eff,
 * O_part, gamma_n, the chunk map), T and P of every (chunk, head), three fp32
 * dk x dv matrices per (chunk, head) (the forward state at the chunk's start,
 * the gradient reaching its end, and the outputs' share scale Q_eff^T dO of
 * the gradient reaching its start), and two fp32 64 x dv tiles per (chunk,
 * head) (U = U~ - W S0 and Kbar times the gradient at its end). */
GDN2_API size_t gdn2_backward_workspace_size(const gdn2_desc* desc);

/* Gradients of gdn2_chunk_fwd's outputs: given dO (the gradient of out) and
 * dhT (of hT), the gradients of every input, through the 64-token chunk form
 * (page "Gated DeltaNet-2：将擦除与写入分开", section "词元路径与并行训练":
 * the operator is trained chunk by chunk, its gradients flowing through the
 * gated keys and values; the update is the one of section "在两个维度上独立控制"),
 * fp32 on the CUDA cores for both I/O types:
 *   1. the chunk factors, T = (I + A)^-1 and P are recomputed in fp32;
 *   2. the forward state at every chunk start is recomputed, and
 *   3. beside it (the two walks are independent) the chunks are walked in
 *      reverse: the gradient reaching a chunk's start state is
 *      dS0 = gamma_n dS1 - W^T (Kbar dS1) + scale Q_eff^T dO, the last term
 *      formed for every chunk before the walk
 *      (dS1 of a sequence's last chunk is dhT; dh0 is dS0 of its first);
 *   4. every (chunk, head) then gives its tokens' gradients from its start
 *      state, the gradient at its end and dO, independently of the others.
 * desc, q, k, v, log_alpha, b, w, scale, h0, cu_seqlens: as for
 *   gdn2_chunk_fwd (the same call's inputs); desc->workspace holds at least
 *   gdn2_backward_workspace_size(desc) bytes, 256-byte aligned;
 * dO  : [B, T, H, dv] io dtype;  dhT : [N, H, dk, dv] fp32, NULL = zero;
 * dq, dk, dlog_alpha, db : [B, T, H, dk] fp32;  dv, dw : [B, T, H, dv] fp32;
 * dh0 : [N, H, dk, dv] fp32 (the gradient of h0, also when h0 is NULL).
 * Every gradient is written (for packed rows the call clears them on
 * `stream` first).  Device pointers, 16-byte aligned, owned by the caller.
 * A malformed cu_seqlens sets GDN2_ERR_SEQLENS in the workspace's first
 * int32 and leaves every gradient zero; nothing outside the arrays is
 * touched.  Asynchronous on `stream`. */
GDN2_API gdn2_status gdn2_chunk_bwd(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                                    const float* log_alpha, const float* b, const float* w, float scale,
                                    const float* h0, const int32_t* cu_seqlens, const void* dO, const float* dhT,
                                    float* dq, float* dk, float* dv, float* dlog_alpha, float* db, float* dw,
                                    float* dh0, cudaStream_t stream);

/* One decode token for a batch of states, updated in place.
 * desc: B = batch, H, dk, dv, io (T, num_seqs and the workspace are ignored).
 *   q, k, log_alpha, b : [B, H, dk]   (q, k in io dtype; the rest fp32)
 *   v, w               : [B, H, dv]   (v in io dtype; w fp32)
 *   state              : [B, H, dk, dv] fp32, read and overwritten
 *   out                : [B, H, dv]   io dtype
 * Same recurrence as gdn2_chunk_fwd with T = 1 (constant-memory decoding,
 * page "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention",
 * cere-bro blog, section "TL;DR"). */
GDN2_API gdn2_status gdn2_recurrent_step(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                                const float* log_alpha, const float* b, const float* w, float scale,
                                float* state, void* out, cudaStream_t stream);

/* Size of the library's own device scratch used by gdn2_chunk_fwd_noalloc. */
#define GDN2_NOALLOC_SCRATCH_BYTES (32u << 20)

/* gdn2_chunk_fwd without a caller-provided workspace (the paper has no
 * counterpart: this is a deployment convenience, not part of the method).
 *
 * Some callers cannot allocate device memory at the point where they run the
 * operator: a plugin inside a host framework that owns every device
 * allocation, code running while a CUDA graph is being captured (where
 * cudaMalloc is not allowed), or a latency-critical path that must not risk
 * the implicit device synchronisation an allocation can cause.  This entry
 * point takes the same arguments as gdn2_chunk_fwd and ignores
 * desc->workspace / workspace_bytes; the scratch is a fixed array of
 * GDN2_NOALLOC_SCRATCH_BYTES that lives inside the library's device image.
 * Every GPU that loads the library holds that array until the process exits.
 *
 *  - Limit: if gdn2_workspace_size(desc) exceeds GDN2_NOALLOC_SCRATCH_BYTES
 *    the call returns GDN2_ERR_WORKSPACE and launches nothing; use
 *    gdn2_chunk_fwd with your own workspace for such sizes.
 *  - Set-up: every call looks up the array's device address on the current
 *    device (cudaGetSymbolAddress, a host-side query).  The first call on a
 *    device may load the library's device code there, so make that first
 *    call outside any stream capture.
 *  - Sharing: all calls use the same array and it keeps the last call's
 *    contents (nothing in it needs to start at zero).  Calls whose work
 *    overlaps on the GPU (other streams, other host threads) race on it:
 *    order them on one stream or use gdn2_chunk_fwd.
 *  - Device-side errors (a malformed cu_seqlens, a bounded wait that gave
 *    up) land in a status word inside the array, as they do in a workspace;
 *    gdn2_noalloc_status copies it out.
 * It calls no cudaMalloc, cudaFree or allocating library routine. */
GDN2_API gdn2_status gdn2_chunk_fwd_noalloc(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                                            const float* log_alpha, const float* b, const float* w, float scale,
                                            const float* h0, const int32_t* cu_seqlens, void* out, float* hT,
                                            cudaStream_t stream);

/* The status word the last gdn2_chunk_fwd_noalloc call for the same `desc`
 * left in the library's scratch (GDN2_OK, or an error found on the device:
 * GDN2_ERR_SEQLENS, GDN2_ERR_DEVICE_TIMEOUT), copied into the caller's
 * device int32 *status (16-byte aligned) on `stream`, so it is read after that
 * call's work when both are on one stream.  desc must describe the same
 * problem (num_seqs > 0 for a packed call); its workspace fields are ignored.
 * Returns GDN2_ERR_WORKSPACE for problems the no-alloc call rejects.  It
 * allocates nothing. */
GDN2_API gdn2_status gdn2_noalloc_status(const gdn2_desc* desc, int32_t* status, cudaStream_t stream);

/* Static description of a status code. */
GDN2_API const char* gdn2_status_string(gdn2_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
GDN2_API int gdn2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN2_H_ */
