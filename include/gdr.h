/*
 * gdr.h -- C ABI of libgdr, the gated delta rule forward for NVIDIA B200 (sm_100a).
 *
 * The operation (Gated DeltaNet-2 Q&A page, Q3 "update equation"; Gated DeltaNet-2
 * Review §3-1; Gated DeltaNet explainer, "Mechanism" for the read-out):
 *
 *     S_t = (I - k_t (b_t . k_t)^T) diag(exp(g_t)) S_{t-1} + k_t (w_t . v_t)^T
 *     o_t = S_t^T q_t
 *
 * per sequence and head, with state S in R^{dk x dv} (fp32), channel-wise log-decay
 * g_t in R^{dk} (fp32), erase gate b_t in [0,1]^{dk} and write gate w_t in [0,1]^{dv}.
 * The tied modes are the reductions named on the same Q3: KDA (b = w = beta * 1) and
 * Gated DeltaNet (additionally a scalar decay, S_t = alpha_t (I - beta_t k k^T)
 * S_{t-1} + beta_t k v^T with alpha_t = exp(g_t)).  The gate-ablation variants of the
 * Gated DeltaNet-2 Review (§5, "Gate ablation") keep one gate channel-wise and make the
 * other a per-token scalar: b-only (channel erase b, scalar write w) and w-only (scalar
 * erase b, channel write w).  The "expanded erase range" variant of the same table is
 * b in [0, 2], which every mode accepts as input values.
 *
 * Common conventions
 *   - Every pointer is a DEVICE pointer on the current CUDA device; the caller owns
 *     every buffer.  The library allocates no device memory and keeps no state
 *     between calls.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream) and the call returns without synchronising.  Arguments are
 *     validated on the host first: on any error nothing is launched.
 *   - Layouts are row-major and contiguous:
 *       q, k   [B, H, T, dk]          v, o   [B, H, T, dv]
 *       g_log  [B, H, T, dk] fp32     (GDR_MODE_GDN: [B, H, T])
 *       b      [B, H, T, dk]          (KDA, GDN: beta [B, H, T]; w-only: [B, H, T])
 *       w      [B, H, T, dv]          (KDA, GDN: ignored, may be NULL; b-only: [B, H, T])
 *       S0,S_T [B, H, dk, dv] fp32
 *   - q, k, v, b, w, o have the element type `dtype`; g_log and states are fp32.
 *   - Every pointer must be 16-byte aligned (GDR_ERR_ALIGN otherwise).
 *   - Supported sizes: dk, dv in {16, 32, 64, 128}; chunk in {16, 32, 64}; any
 *     T >= 0; B, H >= 0.  Sizes are int; B*H*T*max(dk,dv) must fit in int64.
 *   - The decay is meant to forget: g_log <= 0.  Positive values are computed as
 *     written but can overflow fp32 over long chunks.
 */
#ifndef GDR_H
#define GDR_H

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDR_OK = 0,
    GDR_ERR_NULL = -1,     /* a required pointer is NULL */
    GDR_ERR_DIM = -2,      /* unsupported size (dk, dv, chunk) or negative B, H, T, N */
    GDR_ERR_MODE = -3,     /* unknown gdr_mode_t */
    GDR_ERR_DTYPE = -4,    /* unknown gdr_dtype_t */
    GDR_ERR_ALIGN = -5,    /* a pointer is not 16-byte aligned */
    GDR_ERR_CUDA = -6,     /* a CUDA launch or attribute call failed */
    GDR_ERR_TIMEOUT = -7,  /* a bounded device-side wait gave up (tensor-core path) */
    GDR_ERR_WORKSPACE = -8,/* workspace missing, misaligned or smaller than required */
    GDR_ERR_VALUE = -9,    /* a scalar argument is out of range (eps, b_range, layout) */
    GDR_ERR_BOUNDS = -10   /* debug build only: an in-kernel bounds check failed */
} gdr_status_t;

typedef enum {
    GDR_MODE_GDN2 = 0,     /* Gated DeltaNet-2: g [dk], b [dk], w [dv] per token */
    GDR_MODE_KDA = 1,      /* KDA: g [dk], beta per token in b; w ignored */
    GDR_MODE_GDN = 2,      /* Gated DeltaNet: scalar g, beta per token in b; w ignored */
    GDR_MODE_BONLY = 3,    /* b-only variant: g [dk], b [dk], scalar write w per token */
    GDR_MODE_WONLY = 4     /* w-only variant: g [dk], scalar erase b per token, w [dv] */
} gdr_mode_t;

typedef enum {
    GDR_F32 = 0,           /* q, k, v, b, w, o are float */
    GDR_BF16 = 1           /* q, k, v, b, w, o are bfloat16 */
} gdr_dtype_t;

typedef enum {
    GDR_LAYOUT_BHTD = 0,   /* head-major:  [B, H, T, D] (scalar gates [B, H, T]) */
    GDR_LAYOUT_BTHD = 1    /* token-major: [B, T, H, D] (scalar gates [B, T, H]), as the
                              projections of a token-mixer block produce them */
} gdr_layout_t;

/*
 * gdr_chunk_fwd -- chunkwise-parallel forward over whole sequences.
 *
 * Computes o_t for t = 0..T-1 and the final state S_T from the initial state S0 by
 * the chunkwise WY form of the recurrence (Gated DeltaNet-2 Q&A page, Q4; Gated
 * DeltaNet-2 Review §3-2.5): within a chunk of `chunk` tokens the cumulative
 * channel-wise decay is absorbed into the rank-one erase factor, the token
 * interactions become dense products, and only the state crosses chunk borders.
 * The result equals the sequential recurrence up to rounding.
 *
 *   S0   NULL = zero initial state.
 *   S_T  NULL = do not write the final state.  S_T may equal S0 (in-place update).
 *   o    [B,H,T,dv], written for every t.  Must not overlap any input.
 *   T == 0 writes S_T = S0 (or zeros) and nothing else.
 *
 * Paths: dtype == GDR_BF16 with dk == dv == 128 and chunk == 64 runs on the
 * tcgen05 tensor cores (bf16 operands, fp32 accumulation and state); every other
 * case runs the fp32 CUDA-core kernel.  Returns GDR_OK once the work is enqueued.
 * A bounded wait that expired inside the tensor-core kernel of an earlier call is
 * reported as GDR_ERR_TIMEOUT by gdr_last_device_error().
 */
gdr_status_t gdr_chunk_fwd(const void *q, const void *k, const void *v, const float *g_log,
                           const void *b, const void *w, const float *S0, void *o, float *S_T,
                           int B, int H, int T, int dk, int dv, int chunk, gdr_mode_t mode,
                           gdr_dtype_t dtype, void *stream);

/*
 * Sequence split for long sequences with few sequence-heads.
 *
 * The recurrence is affine in the state: over a segment of the sequence,
 * S_end = M S_start + S_local, with M (dk x dk) the product of the segment's per-token
 * transitions (I - k (b.k)^T) diag(exp g) and S_local the end state reached from a zero
 * start (Gated DeltaNet-2 Q&A page, Q3 update equation; only the state crosses chunk
 * borders, Gated DeltaNet-2 Review §3-2.5).  gdr_chunk_fwd_split cuts every sequence into
 * `nseg` segments of whole chunks and runs, on the stream, three kernels: (1) the end
 * states S_local and the transitions M of the segments, all segments in parallel;
 * (2) the chain S_start(s+1) = M_s S_start(s) + S_local(s) in fp32; (3) the forward of
 * every segment from its own S_start, again in parallel.  Results equal gdr_chunk_fwd up
 * to rounding; the work is about twice as large, the parallelism nseg times larger.
 *
 * Only the tensor-core shape is split (bf16, dk = dv = 128, chunk 64); for any other
 * shape nseg must be 1.  nseg is clamped to the number of chunks and, after rounding
 * segments to whole chunks, may shrink.  nseg == 1 is exactly gdr_chunk_fwd (no
 * workspace needed).  The workspace is caller-owned device memory of at least
 * gdr_chunk_fwd_split_workspace(B, H, dk, dv, nseg) bytes, 16-byte aligned; its
 * contents are scratch and need no initialisation.  S_T may equal S0.
 */

/* Recommended segment count for this device and problem (1 = do not split). */
int gdr_chunk_fwd_split_segments(int B, int H, int T, int dk, int dv, int chunk, gdr_dtype_t dtype);

/* Workspace bytes needed by gdr_chunk_fwd_split (0 for invalid arguments). */
unsigned long long gdr_chunk_fwd_split_workspace(int B, int H, int dk, int dv, int nseg);

/* As gdr_chunk_fwd, with the sequence cut into nseg segments (see above).
 * Returns GDR_ERR_WORKSPACE if nseg > 1 needs a workspace that is missing, misaligned or
 * smaller than gdr_chunk_fwd_split_workspace(). */
gdr_status_t gdr_chunk_fwd_split(const void *q, const void *k, const void *v, const float *g_log,
                                 const void *b, const void *w, const float *S0, void *o,
                                 float *S_T, int B, int H, int T, int dk, int dv, int chunk,
                                 gdr_mode_t mode, gdr_dtype_t dtype, int nseg, void *workspace,
                                 unsigned long long workspace_bytes, void *stream);

/*
 * Two-phase forward for few sequence-heads.
 *
 * The chunkwise WY form splits every chunk's work into a part that does not depend on the
 * state and one that does (Gated DeltaNet-2 Review §3-2.5, "Chunkwise WY training": the
 * WY factors W = T (decayed, b-scaled K) and U = T (w.V) with T = (I + A)^-1 are built
 * inside a chunk, and only the state S crosses chunk borders).  gdr_chunk_fwd_two_phase
 * runs them as separate phases on the stream:
 *   (1) for every chunk of every sequence-head at once: the chunk-local cumulative decay,
 *       A, T, W and U, the decayed queries Qg and keys Kb and the lower-triangular P; each
 *       chunk's record goes to the workspace (73 KB per chunk, bf16 tiles);
 *   (2) the recurrence over the records: per sequence-head (or per segment, when nseg >
 *       1, chained exactly as gdr_chunk_fwd_split chains them) E = U - W S,
 *       O = Qg S + P E, S' = diag(exp gamma_C) (S + Kb^T E).
 * Phase one fills the GPU however few sequence-heads there are, and phase two's per-chunk
 * chain is two tensor-core round trips.  It pays for that with memory traffic (each record
 * is written once and read once per state pass), so it wins when the sequence-heads are
 * fewer than the SMs; gdr_chunk_fwd_two_phase_segments says when.  Results equal
 * gdr_chunk_fwd up to rounding (W and U are rounded to bf16 as operands).
 *
 * Shape: bf16, dk = dv = 128, chunk 64, head-major [B, H, T, D] as gdr_chunk_fwd (other
 * shapes: GDR_ERR_DIM).  The workspace is caller-owned device memory of at least
 * gdr_chunk_fwd_two_phase_workspace(B, H, T, dk, dv, chunk, nseg) bytes, 16-byte aligned;
 * its contents are scratch and need no initialisation.  nseg is clamped and rounded to
 * whole chunks as in gdr_chunk_fwd_split.  S_T may equal S0.  Errors: those of
 * gdr_chunk_fwd_split, GDR_ERR_WORKSPACE for a missing, misaligned or short workspace.
 * Bounded device waits report GDR_ERR_TIMEOUT through gdr_last_device_error().
 */

/* Segment count for phase two of the two-phase forward on this device and problem, or 0
 * when the fused kernel (gdr_chunk_fwd / gdr_chunk_fwd_split) is expected to be faster. */
int gdr_chunk_fwd_two_phase_segments(int B, int H, int T, int dk, int dv, int chunk, gdr_dtype_t dtype);

/* Workspace bytes needed by gdr_chunk_fwd_two_phase (0 for invalid arguments). */
unsigned long long gdr_chunk_fwd_two_phase_workspace(int B, int H, int T, int dk, int dv, int chunk, int nseg);

gdr_status_t gdr_chunk_fwd_two_phase(const void *q, const void *k, const void *v, const float *g_log,
                                     const void *b, const void *w, const float *S0, void *o,
                                     float *S_T, int B, int H, int T, int dk, int dv, int chunk,
                                     gdr_mode_t mode, gdr_dtype_t dtype, int nseg, void *workspace,
                                     unsigned long long workspace_bytes, void *stream);

/*
 * gdr_chunk_fwd_split_noalloc -- gdr_chunk_fwd_split without a caller workspace.
 *
 * The pages have no counterpart to this entry point; it exists for callers that cannot
 * allocate device memory: plugins whose host framework owns every device allocation,
 * and latency-critical loops where a cudaMalloc, which may synchronise the device, is
 * not acceptable.  Its workspace is a fixed 24 MiB array inside the library (every GPU
 * that loads the library holds it until the process exits); the call itself allocates
 * nothing.  Arguments and results are those of gdr_chunk_fwd_split.
 *
 *   - Limit: the split's workspace, gdr_chunk_fwd_split_workspace(B, H, dk, dv, nseg),
 *     must fit in 24 MiB (e.g. B*H*nseg <= 128 at dk = dv = 128); larger requests
 *     return GDR_ERR_WORKSPACE before anything is launched.
 *   - Arguments are checked first, exactly as gdr_chunk_fwd_split checks them; a call
 *     that needs no workspace (one segment, or no sequence-head) runs unsplit and never
 *     touches the array.
 *   - The array's device address belongs to the CUDA context that loaded the library's
 *     module.  A call made outside a stream capture looks it up afresh in the current
 *     context (so calls after a cudaDeviceReset, or in another context, use the right
 *     one); a call made while its stream is being captured makes no lookup and uses the
 *     address the last uncaptured call in the same context found, so make at least one
 *     call in each context before any stream capture begins (else GDR_ERR_CUDA).
 *   - Every call shares the one array, which keeps the previous call's contents; the
 *     split reads only what the same call wrote, so nothing needs clearing.  Calls
 *     that overlap on the GPU (for example on two streams) race on the array and must
 *     be serialised by the caller.
 */
gdr_status_t gdr_chunk_fwd_split_noalloc(const void *q, const void *k, const void *v,
                                         const float *g_log, const void *b, const void *w,
                                         const float *S0, void *o, float *S_T, int B, int H,
                                         int T, int dk, int dv, int chunk, gdr_mode_t mode,
                                         gdr_dtype_t dtype, int nseg, void *stream);

/*
 * Sequence split across GPUs (one state hand-off per segment).
 *
 * Only the state crosses chunk borders (Gated DeltaNet-2 Review §3-2.5, "Chunkwise WY
 * training"), and the recurrence is affine in it: over a segment of the sequence,
 * S_end = M S_start + S_local (Gated DeltaNet-2 Q&A page, Q3 update equation).  R holders
 * (ranks, one per GPU) each take one contiguous range of the tokens of every
 * sequence-head, in order.  Holder r computes its segment's maps, the holders exchange
 * them (one all-gather, done by the caller's communication library), each chains them to
 * its own start state and runs gdr_chunk_fwd on its range from that state: it owns o of
 * its range, and the last holder's end state is S_T.  The Python binding's
 * chunk_fwd_seqpar does all of this over torch.distributed.
 *
 * gdr_chunk_fwd_segment_maps -- the maps of one segment held on its own.
 *   q .. w        the segment's tokens, laid out as for gdr_chunk_fwd with T = its length
 *   S0            start state of the segment if known (holder 0: the sequence's S0), else
 *                 NULL: S_local is then the end state reached from a zero state
 *   S_local       [B,H,dk,dv] fp32 (written): the end state reached from S0
 *   M             [B,H,dk,dk] fp32 (written) or NULL: the segment's transition map, the
 *                 end state reached from the identity with the write term (w.v) dropped;
 *                 holders 1 .. R-2 need it, holders 0 and R-1 do not
 * bf16 with dk = dv = 128 and chunk 64 only (else GDR_ERR_DIM); T >= 1.  Asynchronous on
 * `stream`; the caller owns every buffer.
 */
gdr_status_t gdr_chunk_fwd_segment_maps(const void *q, const void *k, const void *v, const float *g_log,
                                        const void *b, const void *w, const float *S0, float *S_local,
                                        float *M, int B, int H, int T, int dk, int dv, int chunk,
                                        gdr_mode_t mode, gdr_dtype_t dtype, void *stream);

/*
 * gdr_chain_segment_states -- the start state of holder r from every holder's maps.
 *   M_all         [R][B,H,dk,dk] fp32: the gathered transition maps (entries of holders 0
 *                 and R-1 are not read; may be NULL when r < 2)
 *   S_local_all   [R][B,H,dk,dv] fp32: the gathered end states, holder 0's from S0 (may be
 *                 NULL when r = 0)
 *   S0            [B,H,dk,dv] fp32 or NULL (zero): the sequence's start state, read when r = 0
 *   S_start       [B,H,dk,dv] fp32 (written)
 * r = 0: S_start = S0; r >= 1: S = S_local_all[0], then S <- M_all[i] S + S_local_all[i] for
 * i = 1 .. r-1, in fp32 on the GPU.  dk = dv = 128; 0 <= r < R.
 */
gdr_status_t gdr_chain_segment_states(const float *M_all, const float *S_local_all, const float *S0,
                                      float *S_start, int R, int r, int B, int H, int dk, int dv, void *stream);

/*
 * gdr_decode_step -- one-token recurrent update for N sequences x H heads.
 *
 * The recurrent form used for constant-memory decoding (Gated DeltaNet-2 Q&A page,
 * introduction; Gated DeltaNet-2 Review §3-2.1): S <- update(S) in place and
 * o = S_new^T q.  Layout is the forward's with T = 1 and N in place of B:
 * q, k [N,H,dk]; v, o [N,H,dv]; g_log [N,H,dk] (GDN: [N,H]); b [N,H,dk]
 * (KDA, GDN: beta [N,H]); w [N,H,dv]; S [N,H,dk,dv] fp32, read and written.
 * o must not overlap S or any input.  Runs on CUDA cores (bandwidth-bound).
 */
gdr_status_t gdr_decode_step(const void *q, const void *k, const void *v, const float *g_log,
                             const void *b, const void *w, float *S, void *o, int N, int H,
                             int dk, int dv, gdr_mode_t mode, gdr_dtype_t dtype, void *stream);

/*
 * gdr_mixer_fwd -- the recurrence inside its token-mixer block, fused into one kernel.
 *
 * The block around the recurrence (Gated DeltaNet-2 Review §4-3, engineering notes):
 * the q and k paths end in an L2 normalisation, the decay branch is a log-decay
 * projection kept in fp32, the erase and write gates are their own projections through
 * a sigmoid, and the recurrent output is RMS-normalised and multiplied by a SiLU output
 * gate.  This call takes the raw projections and returns the gated output:
 *
 *     q_t <- q_t / sqrt(|q_t|^2 + 1e-6)        k_t <- k_t / sqrt(|k_t|^2 + 1e-6)
 *     g_t  = -softplus(xg_t)                    (natural-log decay, <= 0)
 *     b_t  = b_range * sigmoid(xb_t)            w_t = sigmoid(xw_t)
 *     o_t  = the forward of gdr_chunk_fwd on (q, k, v, g, b, w) from S0
 *     y_t  = o_t / sqrt(mean_v o_t[v]^2 + eps) * norm_weight * z_t * sigmoid(z_t)
 *
 * In the tied modes (KDA, GDN) xb holds the raw beta, beta = b_range * sigmoid(xb) is
 * both gates, and xw is ignored (may be NULL).  b-only: xw [.., T] is the raw scalar
 * write gate; w-only: xb [.., T] is the raw scalar erase gate.  b_range = 2 is the
 * expanded erase range b in [0, 2]; the write gate is never scaled except as beta.
 *
 *   layout       GDR_LAYOUT_BHTD: every per-token tensor is [B, H, T, D] (scalar gates
 *                [B, H, T]); GDR_LAYOUT_BTHD: [B, T, H, D] (scalar gates [B, T, H]).
 *                q, k, xb (per channel) have D = dk; v, xw (per channel), z, y have
 *                D = dv; xg has D = dk (GDN: a scalar).
 *   xg           fp32 pre-activation decay.  q, k, v, xb, xw, z, y: bf16.
 *   norm_weight  fp32 [dv], shared by the heads.
 *   S0, S_T      fp32 [B, H, dk, dv] as in gdr_chunk_fwd (NULL: zero / not written).
 *   eps          > 0 and finite; b_range >= 0 and finite (else GDR_ERR_VALUE).
 *   y            must not overlap any input.
 *
 * Supported: dtype GDR_BF16, dk = dv = 128, chunk = 64 (the tcgen05 kernel); other
 * sizes return GDR_ERR_DIM, GDR_F32 returns GDR_ERR_DTYPE.  Every pointer 16-byte
 * aligned.  T == 0 writes S_T = S0 (or zeros).  Asynchronous on `stream`; validation
 * first, as for every entry point.
 */
gdr_status_t gdr_mixer_fwd(const void *q, const void *k, const void *v, const float *xg,
                           const void *xb, const void *xw, const void *z,
                           const float *norm_weight, const float *S0, void *y, float *S_T,
                           int B, int H, int T, int dk, int dv, int chunk, gdr_mode_t mode,
                           gdr_dtype_t dtype, gdr_layout_t layout, float b_range, float eps,
                           void *stream);

/*
 * gdr_chunk_bwd -- the gate-aware backward of gdr_chunk_fwd.
 *
 * Gradients of L = sum_t <o_t, dO_t> + <S_T, dS_T> with respect to q, k, v, g_log, b, w
 * and S0, for the forward of gdr_chunk_fwd on the same inputs (the pages' training path
 * runs the chunkwise WY algorithm with a gate-aware backward: Gated DeltaNet-2 Review
 * §4-3; Gated DeltaNet-2 Q&A page, Q4).  The backward differentiates the chunkwise form:
 * it recomputes the states at every 64-token boundary, walks the chunks backwards for the
 * state gradient, then forms every chunk's input gradients in parallel.  For bf16 with
 * dk = dv = 128 all three run on the tcgen05 tensor cores (bf16 operands, fp32
 * accumulation), 64-token chunks; a chunk whose cumulative decay exceeds e^-60 is done in
 * fp32 on CUDA cores with exact per-pair decays, as is everything for other shapes (32-token
 * chunks).  Equal to the adjoint of the sequential recurrence up to rounding.
 *
 *   dO      [B,H,T,dv], element type `dtype`.       dS_T  fp32 [B,H,dk,dv] or NULL (= 0).
 *   dq, dk  [B,H,T,dk]; dv [B,H,T,dv]; db, dw shaped like b, w; all of type `dtype`.
 *           Tied and scalar modes receive the summed gradient of the shared parameter
 *           (KDA, GDN: d beta = sum_c db + sum_v dw in db; b-only: the scalar write gate's
 *           gradient in dw; w-only: the scalar erase gate's in db).  dw may be NULL in KDA
 *           and GDN.
 *   dg      fp32, shaped like g_log.                 dS0   fp32 [B,H,dk,dv] or NULL.
 *   workspace  caller-owned device memory of at least gdr_chunk_bwd_workspace(B, H, T, dk,
 *           dv) bytes, 16-byte aligned (GDR_ERR_WORKSPACE otherwise); scratch, no
 *           initialisation needed.  Outputs must not overlap inputs or the workspace.
 *   Sizes as gdr_chunk_fwd (dk, dv in {16, 32, 64, 128}); T == 0 writes dS0 = dS_T (or 0).
 */
unsigned long long gdr_chunk_bwd_workspace(int B, int H, int T, int dk, int dv);

gdr_status_t gdr_chunk_bwd(const void *q, const void *k, const void *v, const float *g_log,
                           const void *b, const void *w, const float *S0, const void *dO,
                           const float *dS_T, void *dq, void *dk_, void *dv_, float *dg,
                           void *db, void *dw, float *dS0, int B, int H, int T, int dk, int dv,
                           gdr_mode_t mode, gdr_dtype_t dtype, void *workspace,
                           unsigned long long workspace_bytes, void *stream);

/*
 * gdr_last_device_error -- read and clear the device-side error word.
 *
 * Synchronises `stream`, then returns GDR_ERR_TIMEOUT if a bounded wait inside a
 * tensor-core kernel or the streaming decode kernel gave up since the last call
 * (the kernel then skipped its remaining work, drained its own copies and released
 * its tensor memory), GDR_ERR_CUDA if the stream reports a CUDA error, else GDR_OK.
 */
gdr_status_t gdr_last_device_error(void *stream);

/*
 * The debug build (libgdr_debug.so, compiled with -DGDR_DEBUG; the pages have no
 * counterpart).  Its kernels check that every bulk copy's source range, every clamped tail
 * load, every output row and every workspace or checkpoint slot they touch lies inside the
 * extents the call's arguments imply; a failed check skips the access and records its site
 * (no trap), gdr_last_device_error() then returns GDR_ERR_BOUNDS and
 * gdr_debug_bounds_site() the site (1xx tensor-core forward, 2xx decode, 3xx tensor-core
 * backward, 4xx CUDA-core backward, 5xx split chaining, 6xx CUDA-core forward).  It stands
 * in for a memory sanitizer, which is not available; results are identical otherwise.
 * gdr_debug_build() is 1 in that library and 0 in the release build, where the bounds
 * site is always 0.
 */
int gdr_debug_build(void);
int gdr_debug_bounds_site(void);

/*
 * gdr_test_set_first_wait_limit -- test hook for the bounded-wait expiry path.  The pages
 * have no counterpart to it.
 *
 * polls != 0: in every call enqueued afterwards, the first mbarrier wait of each CTA of the
 * tensor-core forward (its state group's wait for the first chunk's operands), of the
 * streaming decode kernel (its first state copy) and of the tensor-core per-chunk backward
 * kernel (its raw input copies) gives up after `polls` non-blocking polls instead of the
 * normal bound of 2^24.  The producer is then merely still working, so the expiry path
 * (abort flag, drain of the kernel's own copies and tensor-core work, TMEM released)
 * runs for real and gdr_last_device_error() reports GDR_ERR_TIMEOUT; the outputs of such a
 * call are unspecified.  polls = 0 (the default) restores the normal bound.  Host-side
 * state of the library, not thread-safe; for tests only.
 */
void gdr_test_set_first_wait_limit(unsigned polls);

/* Human-readable name of a status code (static storage, never NULL). */
const char *gdr_status_string(gdr_status_t status);

#ifdef __cplusplus
}
#endif
#endif /* GDR_H */
