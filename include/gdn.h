/*
 * gdn.h -- C-ABI of libgdn: the gated delta-rule recurrence on one NVIDIA B200 (sm_100a).
 *
 * The operation, per (sequence, head), with state S in R^{dk x dv}:
 *
 *     S_t = a_t (I - b_t k_t k_t^T) S_{t-1} + b_t k_t v_t^T,     o_t = S_t^T q_t
 *
 * with a_t = exp(log_alpha_t) in [0, 1] (data-dependent forget gate) and b_t = beta_t in [0, 2].
 * Sources:
 *   - Sykra README, "Architectural Highlights": Gated DeltaNet layers trained chunk-parallel
 *     through the WY / unit-triangular transform (a triangular solve per chunk, the rest as
 *     matrix products); a data-dependent forget gate a_t; generation as an O(d^2) update of a
 *     fixed d x d state.  Also its "Computational Complexity" table (O(N d) training, O(d^2)
 *     per decode step).
 *   - DeltaPhase README, section 1 "Extended Householder Beta Range": beta in (0, 2), beta = 2 an
 *     exact Householder reflection; "Fast Triangular Solve": an exact O(C^2) per-chunk solve.
 *   - DeltaPhase README, section 2: the delta rule as read-out -> error -> rank-one update.
 * Readings taken where the pages are silent: the read-out uses the post-update state; there is
 * no 1/sqrt(dk) query scale; a_t and b_t are scalars per (token, head); the library does not
 * normalise q or k.
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is a DEVICE pointer owned by the caller (the exception:
 *     gdn_chunk_fwd_host, which takes host buffers).  The library allocates no memory, keeps no
 *     state between calls and may be called from several host threads (the exceptions:
 *     gdn_chunk_fwd_noalloc owns a fixed scratch array per device; gdn_chunk_fwd_host keeps two
 *     copy streams and a few events per device, made on its first call).
 *   - Calls are asynchronous: they validate on the host, enqueue kernels on `stream` (a
 *     cudaStream_t; NULL = the legacy default stream) and return.  Errors found on the host are
 *     returned before anything is enqueued, so a failed call writes nothing.
 *   - Element type of q, k, v and out: `dtype` (GDN_DTYPE_BF16 or GDN_DTYPE_F32).  Gates
 *     (log_alpha, beta) and states (S0, S_final, S_inout) are always fp32.
 *   - All tensors are contiguous row-major; every pointer must be 16-byte aligned.
 *   - Return value: GDN_OK (0) or a negative GDN_ERR_* code; gdn_last_error() then gives a
 *     one-line reason (per host thread).
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum gdn_status {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARGUMENT = -1, /* null required pointer, bad size, misaligned pointer      */
    GDN_ERR_UNSUPPORTED = -2,      /* head size, chunk or dtype outside an entry's support      */
    GDN_ERR_WORKSPACE = -3,        /* workspace NULL or smaller than the query function says   */
    GDN_ERR_CUDA = -4,             /* a CUDA launch or driver call failed (see gdn_last_error) */
    GDN_ERR_TIMEOUT = -5           /* reserved: a bounded device-side wait ran out             */
};

enum gdn_dtype {
    GDN_DTYPE_F32 = 0,
    GDN_DTYPE_BF16 = 1
};

/*
 * gdn_chunk_fwd -- prefill / training forward of the recurrence over whole sequences, computed
 * chunk by chunk in the WY / UT-transform form (Sykra README, "Architectural Highlights";
 * DeltaPhase README, section 1 "Fast Triangular Solve").  Per chunk of C = `chunk` tokens:
 *     A = strictly_lower(diag(b) (Gam o K K^T)),  T = (I + A)^{-1},
 *     W = T diag(b gam) K,  U~ = T diag(b) V,  U = U~ - W S,
 *     O = diag(gam) Q S + lower_incl(Gam o Q K^T) U,  S <- gam_C S + (diag(lam) K)^T U,
 * where gam, lam, Gam are the products of a_j from the chunk start / to the chunk end / between
 * two tokens.  The result equals the sequential recurrence up to rounding.
 *
 * Layouts
 *   dense  (cu_seqlens == NULL): q,k [B,T,H,dk]; v,out [B,T,H,dv]; log_alpha,beta [B,T,H]
 *   varlen (cu_seqlens != NULL): B = number of sequences, T = total tokens; q,k [T,H,dk];
 *          v,out [T,H,dv]; log_alpha,beta [T,H]; cu_seqlens: DEVICE int32 [B+1], cu[0] = 0,
 *          cu[B] = T, non-decreasing (contents are not checked: malformed offsets are undefined
 *          behaviour).  Sequence s owns tokens cu[s] .. cu[s+1]-1 and is chunked from its own
 *          first token; a sequence of length 0 gets S_final = S0 and no outputs.
 *   S0, S_final: [B,H,dk,dv] fp32.  S0 == NULL: zero initial state.  S_final == NULL: not
 *          written.  S_final == S0 (same pointer) is allowed (in-place carry); no other
 *          overlap between any output and any input is allowed.
 * Arguments
 *   B >= 1, T >= 0 (T == 0 only with cu_seqlens), H >= 1; dk, dv in {64, 128, 256}; chunk in
 *   {64, 128}.  Paths: dk, dv in {64, 128} at chunk 64 run the fused kernels (bf16: tcgen05;
 *   fp32: CUDA cores), and bf16 at dv = 256 runs there as two 128-column blocks (value columns do
 *   not interact); key head size 256, chunk 128 and fp32 at dv = 256 run the general path
 *   (gdn_chunk_general.cu: fp32 on CUDA cores, the chunk factors through the workspace).
 *   log_alpha <= 0 expected (-inf allowed: an exact reset); positive values are accepted but
 *   may overflow.  beta in [0, 2].
 *   workspace / workspace_bytes: device scratch of at least gdn_chunk_fwd_workspace_bytes(...)
 *   bytes, 256-byte aligned (may be NULL when that function returns 0).  Its contents on entry
 *   do not matter; calls that share a workspace must not overlap in time.
 */
GDN_API int gdn_chunk_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                  const float *beta, const float *S0, void *out, float *S_final, int B, int T,
                  int H, int dk, int dv, int chunk, const int32_t *cu_seqlens, int dtype,
                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_chunk_fwd_fused -- gdn_chunk_fwd with its input prologue fused into the kernel: q_raw and
 * k_raw are the unnormalised projections, and a_raw, b_raw the raw gate projections, so the
 * separate passes that would normalise and activate them (one read and one write of q, k and
 * the gates in HBM) are not needed.  Per (token, head), in fp32 inside the kernel:
 *     q = q_raw / sqrt(|q_raw|^2 + 1e-6),   k likewise   (rounded to bf16 for the MMAs)
 *     log_alpha = -a_scale * softplus(a_raw)   (a_raw = +inf: an exact reset)
 *     beta      =  b_scale * sigmoid(b_raw)    (DeltaPhase README, section 1 "Extended
 *                                               Householder Beta Range": beta = 2 sigmoid(W_beta x))
 * after which the operation is exactly gdn_chunk_fwd's (Sykra README, "Architectural
 * Highlights": data-dependent forget gate alpha_t in (0, 1]).  Layouts, S0 / S_final, varlen,
 * workspace (query gdn_chunk_fwd_workspace_bytes with the same sizes) and asynchrony as for
 * gdn_chunk_fwd; a_raw, b_raw [tokens, H] fp32.  dtype must be GDN_DTYPE_BF16 (else
 * GDN_ERR_UNSUPPORTED); a_scale must be finite and >= 0 and b_scale in [0, 2] (else
 * GDN_ERR_INVALID_ARGUMENT).
 */
GDN_API int gdn_chunk_fwd_fused(const void *q_raw, const void *k_raw, const void *v, const float *a_raw,
                                const float *b_raw, const float *S0, void *out, float *S_final, int B,
                                int T, int H, int dk, int dv, int chunk, const int32_t *cu_seqlens,
                                int dtype, float a_scale, float b_scale, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * gdn_chunk_fwd_gva -- gdn_chunk_fwd with grouped value heads: Hv value heads share Hk q/k heads
 * (Hv a multiple of Hk), value head h reading q/k head h / (Hv / Hk), as grouped-query attention
 * shares key/value heads among query heads (Sykra README, "Architectural Highlights": GQA).
 * Gates, values, outputs and states are per value head:
 *   q,k [B,T,Hk,dk] (varlen [T,Hk,dk]); v,out [B,T,Hv,dv]; log_alpha,beta [B,T,Hv];
 *   S0, S_final [B,Hv,dk,dv].
 * Everything else (dtypes, varlen, workspace, in-place carry, errors) as gdn_chunk_fwd; query the
 * workspace with H = Hv.  Hk = Hv is gdn_chunk_fwd.
 */
GDN_API int gdn_chunk_fwd_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                              const float *beta, const float *S0, void *out, float *S_final, int B, int T,
                              int Hk, int Hv, int dk, int dv, int chunk, const int32_t *cu_seqlens,
                              int dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_chunk_fwd_workspace_bytes -- device scratch that gdn_chunk_fwd needs for these sizes
 * (varlen: non-zero when cu_seqlens will be passed).  Returns 0 when no scratch is needed and
 * (size_t)-1 for arguments gdn_chunk_fwd would reject.
 *   Scratch is needed only by the segment scan: dense bf16 calls whose B*H (sequence, head)
 *   chains number at most half the SMs of the CURRENT device and whose sequences span at least
 *   32 chunks are cut into segments, each segment's state map S -> M S + S_loc is computed in
 *   parallel, the maps are scanned per chain, and the outputs are recomputed per segment.  The
 *   scratch then holds, per segment and head, S_loc and the entry state (dk x dv fp32 each), M
 *   (dk x dk fp32) and a segment offset table; it is at most about 3 * (SM count) * dk * dv * 4
 *   bytes.  Query with the device current that the call will run on.
 */
GDN_API size_t gdn_chunk_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int varlen,
                                     int dtype);

/*
 * gdn_chunk_fwd_noalloc -- gdn_chunk_fwd without a workspace argument: the scratch of the segment
 * scan (see gdn_chunk_fwd_workspace_bytes) comes from a fixed 32 MiB array of device memory that
 * the library owns, one per device.  The pages that define the operation have no counterpart of
 * this entry point; it exists for callers that cannot provide device scratch (a serving runtime
 * that has reserved its device memory up front and admits no call-time allocation, or a C host
 * program without a device allocator).  Arguments, layouts and results are those of
 * gdn_chunk_fwd.
 *   - Every argument is checked on the host first, as gdn_chunk_fwd checks it; a rejected call
 *     touches no device state.  Sizes that need no scratch (enough chains to fill the device:
 *     gdn_chunk_fwd_workspace_bytes returns 0) run as gdn_chunk_fwd without a workspace and never
 *     touch the array.
 *   - Every call that needs scratch looks up the array's address in the current context.  The
 *     first such call on a device also loads the module that holds it; make that first call
 *     before any stream capture on that device.
 *   - Footprint: the array takes 32 MiB of device memory on every device where its module is
 *     loaded -- with CUDA's default lazy module loading, from the first gdn_chunk_fwd_noalloc
 *     call on that device that needs scratch; with CUDA_MODULE_LOADING=EAGER, from the CUDA
 *     runtime's initialisation of the device -- until the process exits.  Callers that reserve
 *     device memory up front should budget for it.
 *   - Calls on the same device must not overlap in time (two streams, two host threads): they
 *     share the one array.  Nothing in it needs to start at zero.
 *   - Sizes whose scratch would exceed 32 MiB return GDN_ERR_WORKSPACE (about 3 * SMs * dk * dv
 *     * 4 bytes are needed at most: 29.1 MB for dk = dv = 128 on 148 SMs).
 */
GDN_API int gdn_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *log_alpha,
                                  const float *beta, const float *S0, void *out, float *S_final, int B,
                                  int T, int H, int dk, int dv, int chunk, const int32_t *cu_seqlens,
                                  int dtype, void *stream);

/*
 * gdn_chunk_fwd_host -- gdn_chunk_fwd from and to HOST buffers: q, k, v, log_alpha, beta, S0 (may
 * be NULL), cu_seqlens (may be NULL) are read from host memory and out, S_final (may be NULL) are
 * written to host memory, in gdn_chunk_fwd's layouts; the arithmetic is gdn_chunk_fwd's.  The
 * batch is cut into at most 4 parts of whole sequences (varlen: about equal token counts); each
 * part's inputs are copied up on a side stream, the part runs on `stream` once they have arrived,
 * and its outputs are copied down on a second side stream, so copies in both directions overlap
 * each other and the compute.  Host buffers in page-locked memory (cudaHostAlloc, or a pinned
 * torch tensor) make the copies asynchronous; pageable buffers work, with the copies serialised.
 * `workspace`: DEVICE memory of gdn_chunk_fwd_host_workspace_bytes(...) bytes, 256-byte
 * aligned, holding device copies of every input and output and the device entry's own scratch.
 * Asynchronous like every entry: the outputs are in host memory once `stream` has completed (the
 * side streams are joined back into it), and the host input buffers must stay unchanged until
 * then.  cu_seqlens is read on the host during the call (it decides the parts) and must run from
 * 0 to T without decreasing.  Errors as gdn_chunk_fwd; GDN_ERR_CUDA if the copy streams cannot be
 * made.  Nothing in the pages corresponds to this entry: it is the host-memory interface a
 * serving process without device tensors of its own would call.
 */
GDN_API int gdn_chunk_fwd_host(const void *q, const void *k, const void *v, const float *log_alpha,
                               const float *beta, const float *S0, void *out, float *S_final, int B, int T,
                               int H, int dk, int dv, int chunk, const int32_t *cu_seqlens, int dtype,
                               void *workspace, size_t workspace_bytes, void *stream);

/* Device workspace gdn_chunk_fwd_host needs for these sizes; (size_t)-1 for sizes it rejects. */
GDN_API size_t gdn_chunk_fwd_host_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int varlen,
                                                  int dtype);

/*
 * gdn_phase_fwd -- the complex-phase delta memory (DeltaPhase README, section 2 "Complex Phase
 * Matrix Delta Memory" in its gated-decay form; keys e^{s dt} with Re s <= 0 as in section 5).
 * Per (sequence, head) a complex state M in C^{dv x dk}; per token t, with complex key K_t and
 * query Q_t (dk), real value V_t (dv) and scalars lam_t = exp(log_lam_t), beta_t:
 *     e_t = V_t - (1/dk) Re(M_{t-1} conj K_t)          (read-out before the update)
 *     M_t = lam_t M_{t-1} + beta_t e_t K_t^T
 *     o_t = (1/dk) Re(M_t conj Q_t)                     (reading: the query reads the new state)
 * Layouts (dense [B, T, ...] or packed with cu_seqlens, as gdn_chunk_fwd):
 *     K, Q [.., H, dk, 2] fp32 (re, im pairs); v, out [.., H, dv] in dtype;
 *     log_lam, beta [.., H] fp32; M0, M_final [B, H, dv, dk, 2] fp32 (re, im), either may be NULL.
 * log_lam must be finite (lam > 0): the computation runs the real gated delta rule at head size
 * 2 dk with a = lam and b = beta / lam (see gdn_phase.cu), on the tcgen05 kernel for bf16 (at
 * dk = 32, dv = 64 with the conversion of K, Q, beta and V inside it) and the fp32 CUDA-core
 * kernel for fp32.  dk in {32, 64}, dv in {64, 128}, or 256 with bf16.  Workspace:
 * gdn_phase_fwd_workspace_bytes(...) bytes of device memory, 256-byte aligned.  Errors as
 * gdn_chunk_fwd (the library's own scratch only is written before a late CUDA error).
 */
GDN_API int gdn_phase_fwd(const float *K, const float *Q, const void *v, const float *log_lam, const float *beta,
                          const float *M0, void *out, float *M_final, int B, int T, int H, int dk, int dv,
                          const int32_t *cu_seqlens, int dtype, void *workspace, size_t workspace_bytes,
                          void *stream);

/* Workspace gdn_phase_fwd needs for these sizes; (size_t)-1 for sizes it rejects. */
GDN_API size_t gdn_phase_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, int varlen, int dtype);

/*
 * gdn_phase_rowdecay_fwd -- the complex-phase delta memory with one decay per output row of the
 * state, the Laplace core's diag(r_t) (DeltaPhase README, section 5 "Delta-Laplace Phase Memory
 * Core", "Exact Chunkwise-Parallel Scan"; the delta steps of section 2).  Row j of M (value
 * channel j) decays by its own r_t,j = exp(log_r_t,j):
 *     e_t,j = V_t,j - (1/dk) Re(M_{t-1}[j] . conj K_t)
 *     M_t[j] = r_t,j M_{t-1}[j] + beta_t e_t,j K_t
 *     o_t,j = (1/dk) Re(M_t[j] . conj Q_t)
 * Layouts as gdn_phase_fwd, with log_r [.., H, dv] fp32 (one decay per token, head and channel,
 * finite) in place of log_lam.  dk in {32, 64} complex, any dv in 1 .. 4096, B and H up to 65535,
 * dtype bf16 or fp32 for v and out (fp32-level arithmetic: the products shared by the channels
 * run on the tensor cores as three tf32 products of hi / lo splits, about 2^-21 relative).  No
 * workspace.  It runs in chunks of 32 tokens (gdn_phase_rowdecay.cu).  Errors as gdn_chunk_fwd; a
 * device-side wait that runs out is reported by gdn_device_status; M0 == M_final (in-place carry)
 * is allowed.
 */
GDN_API int gdn_phase_rowdecay_fwd(const float *K, const float *Q, const void *v, const float *log_r,
                                   const float *beta, const float *M0, void *out, float *M_final, int B, int T,
                                   int H, int dk, int dv, const int32_t *cu_seqlens, int dtype, void *stream);

/*
 * gdn_phase_bwd -- gradients of gdn_phase_fwd for dk = 32 complex (64 real) and dv in {64, 128, 256}:
 * given the forward's inputs, dout = dL/dout (dtype) and dM_final = dL/dM_final ((re, im) pairs,
 * NULL: zero), it writes fp32
 *     dK, dQ [.., H, 32, 2] (d/dRe, d/dIm pairs), dv [.., H, dv], dlog_lam, dbeta [.., H],
 *     dM0 [B, H, dv, 32, 2] (NULL: not written).
 * The fp32 backward of the real recurrence runs on the map gdn_phase_fwd uses (see gdn_phase.cu),
 * followed by its chain rule.  Workspace: gdn_phase_bwd_workspace_bytes(...), 256-byte aligned.
 */
GDN_API int gdn_phase_bwd(const float *K, const float *Q, const void *v, const float *log_lam, const float *beta,
                          const float *M0, const void *dout, const float *dM_final, float *dK, float *dQ,
                          float *dv_out, float *dlog_lam, float *dbeta, float *dM0, int B, int T, int H, int dk,
                          int dv, const int32_t *cu_seqlens, int dtype, void *workspace, size_t workspace_bytes,
                          void *stream);

/* Workspace gdn_phase_bwd needs for these sizes; (size_t)-1 for sizes it rejects. */
GDN_API size_t gdn_phase_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, int varlen);

/*
 * gdn_chunk_bwd -- gradients of gdn_chunk_fwd (the training path; Sykra README, "Architectural
 * Highlights": chunk-parallel training through the WY / unit triangular transform), for
 * dk in {64, 128}, dv in {64, 128, 256} and chunk = 64.  Given the forward's inputs (same layouts,
 * dtype for q, k, v and dout) and dout = dL/dout, dS_final = dL/dS_final (NULL: zero), it writes
 *     dq, dk [.., H, dk], dv [.., H, dv], dlog_alpha, dbeta [.., H]   (fp32, always)
 *     dS0 [B, H, dk, dv] fp32 (NULL: not written)
 * dk = 128 runs the key dimension as two 64-column blocks (sums of block products; the chunk
 * transition M as four 64 x 64 blocks).
 * A value head of dv = 64 VS columns runs as VS heads of 64 columns that share q, k and the gates
 * (value columns never interact); their dq, dk, dlog_alpha and dbeta are summed.
 * Computed from the chunk form with fp32-level accuracy: the 64 x 64 products run on the tensor
 * cores as three tf32 products (x = hi + lo; a b ~ hi hi + hi lo + lo hi), everything else in
 * fp32.  Every chunk's state map
 * S' = M S + Bm and gradient map dS = M^T dS' + (Q^T diag(gam) - W^T P^T) dO are formed in
 * parallel, two scans over each sequence's chunks give the entry states and exit gradients, and
 * every chunk's input gradients are then formed in parallel.  log_alpha = -inf (an exact reset)
 * gets dlog_alpha = 0.  Workspace: gdn_chunk_bwd_workspace_bytes(...) bytes, 256-byte aligned
 * (eight 16 KB matrices per chunk, head and 64-column value block, sixteen at dk = 128, plus
 * the partial q/k and gate gradients when dv > 64).  Errors as gdn_chunk_fwd; other head sizes return
 * GDN_ERR_UNSUPPORTED.
 */
GDN_API int gdn_chunk_bwd(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, const float *S0, const void *dout, const float *dS_final,
                          float *dq, float *dk, float *dv, float *dlog_alpha, float *dbeta, float *dS0,
                          int B, int T, int H, int dk_, int dv_, int chunk, const int32_t *cu_seqlens,
                          int dtype, void *workspace, size_t workspace_bytes, void *stream);

/* Workspace gdn_chunk_bwd needs for these sizes; (size_t)-1 for sizes it rejects. */
GDN_API size_t gdn_chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int varlen);

/*
 * gdn_chunk_bwd_gva -- gdn_chunk_bwd with grouped value heads (see gdn_chunk_fwd_gva): q, k
 * [.., Hk, dk]; v, dout [.., Hv, dv]; gates [.., Hv]; states [B, Hv, dk, dv]; value head h reads
 * q/k head h / (Hv / Hk).  dq, dk [.., Hk, 64] are the sums over each q/k head's Hv / Hk value
 * heads; dv, dlog_alpha, dbeta, dS0 stay per value head.  Workspace:
 * gdn_chunk_bwd_gva_workspace_bytes(...) (gdn_chunk_bwd's plus per-value-head dq and dk).
 */
GDN_API int gdn_chunk_bwd_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                              const float *beta, const float *S0, const void *dout, const float *dS_final,
                              float *dq, float *dk, float *dv, float *dlog_alpha, float *dbeta, float *dS0, int B,
                              int T, int Hk, int Hv, int dk_, int dv_, int chunk, const int32_t *cu_seqlens,
                              int dtype, void *workspace, size_t workspace_bytes, void *stream);

/* Workspace gdn_chunk_bwd_gva needs for these sizes; (size_t)-1 for sizes it rejects. */
GDN_API size_t gdn_chunk_bwd_gva_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv, int chunk,
                                                 int varlen);

/*
 * gdn_chunk_bwd_fused -- gradients of gdn_chunk_fwd_fused with respect to its RAW inputs: given
 * q_raw, k_raw, v (dtype), a_raw, b_raw (fp32), S0, a_scale, b_scale as passed to the forward,
 * dout = dL/dout (dtype) and dS_final = dL/dS_final (NULL: zero), it writes fp32
 *     dq_raw, dk_raw [.., H, 64], dv [.., H, dv], da_raw, db_raw [.., H], dS0 (NULL: not written).
 * The prologue (rows divided by sqrt(|x|^2 + 1e-6), log alpha = -a_scale softplus(a),
 * beta = b_scale sigmoid(b)) is formed again in fp32, the recurrence's backward runs in fp32 on
 * it (as gdn_chunk_bwd with fp32 inputs), and the chain rule through the prologue follows:
 * dx = (dq - q (q . dq)) / |x|_eps, da = -a_scale sigmoid(a) dlog_alpha (0 at a = +inf),
 * db = b_scale sigmoid(b) (1 - sigmoid(b)) dbeta.  dk = 64, dv in {64, 128, 256}, chunk = 64.  Workspace:
 * gdn_chunk_bwd_fused_workspace_bytes(...) bytes of device memory, 256-byte aligned.  Errors as
 * gdn_chunk_bwd; a_scale must be finite and >= 0, b_scale in [0, 2].
 */
GDN_API int gdn_chunk_bwd_fused(const void *q_raw, const void *k_raw, const void *v, const float *a_raw,
                                const float *b_raw, const float *S0, const void *dout, const float *dS_final,
                                float *dq_raw, float *dk_raw, float *dv, float *da_raw, float *db_raw, float *dS0,
                                int B, int T, int H, int dk, int dv_, int chunk, const int32_t *cu_seqlens,
                                int dtype, float a_scale, float b_scale, void *workspace, size_t workspace_bytes,
                                void *stream);

/* Workspace gdn_chunk_bwd_fused needs for these sizes; (size_t)-1 for sizes it rejects. */
GDN_API size_t gdn_chunk_bwd_fused_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int varlen);

/*
 * gdn_decode_step -- one generation step: every (n, h) state takes exactly one token, in place
 * (Sykra README, "Architectural Highlights" and "Computational Complexity": an O(d^2) update of
 * a fixed d x d state per token).  With r = S^T k, s = S^T q (both from the state before the
 * step):
 *     u   = b (v - a r)
 *     out = a s + (k . q) u
 *     S  <- a S + k u^T
 *   q,k [N,H,dk]; v,out [N,H,dv] in dtype; log_alpha,beta [N,H] fp32; S_inout [N,H,dk,dv] fp32,
 *   read and overwritten.  N >= 1, H >= 1, dk, dv in {64, 128, 256} (dv = 256 runs as two
 *   128-column blocks per state, and dk = 256 as dv / 64 blocks of 64 columns).  No overlap
 *   between S_inout and the other arguments.
 */
GDN_API int gdn_decode_step(const void *q, const void *k, const void *v, const float *log_alpha,
                    const float *beta, float *S_inout, void *out, int N, int H, int dk, int dv,
                    int dtype, void *stream);

/*
 * gdn_decode_step_fused -- gdn_decode_step from raw projections, the prologue of
 * gdn_chunk_fwd_fused formed inside the step (one launch; the state is still read and written
 * once): q_raw, k_raw [N,H,dk] in dtype are divided by sqrt(|x|^2 + 1e-6) over their dk elements,
 * a_raw, b_raw [N,H] fp32 become log alpha = -a_scale softplus(a) (a = +inf: an exact reset) and
 * beta = b_scale sigmoid(b); v, out, S_inout and the head sizes as gdn_decode_step.  a_scale must
 * be finite and >= 0, b_scale in [0, 2] (GDN_ERR_INVALID_ARGUMENT otherwise).
 */
GDN_API int gdn_decode_step_fused(const void *q_raw, const void *k_raw, const void *v, const float *a_raw,
                                  const float *b_raw, float *S_inout, void *out, int N, int H, int dk, int dv,
                                  int dtype, float a_scale, float b_scale, void *stream);

/*
 * gdn_decode_step_gva -- gdn_decode_step with grouped value heads (see gdn_chunk_fwd_gva):
 * q,k [N,Hk,dk]; v,out [N,Hv,dv]; log_alpha,beta [N,Hv]; S_inout [N,Hv,dk,dv]; state (n, h)
 * reads q/k head h / (Hv / Hk) of sequence n.
 */
GDN_API int gdn_decode_step_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                                const float *beta, float *S_inout, void *out, int N, int Hk, int Hv,
                                int dk, int dv, int dtype, void *stream);

/*
 * gdn_device_status -- synchronise `stream`, then report whether any kernel of this library
 * recorded a device-side failure since the previous call (a bounded wait on an mbarrier that ran
 * out, after which the kernel stopped issuing work and returned): GDN_ERR_TIMEOUT if so, GDN_OK
 * if not, GDN_ERR_CUDA if the synchronisation itself failed.  The record is per device and is
 * cleared by this call.
 *   - After GDN_ERR_TIMEOUT the outputs of every call enqueued since the previous status check
 *     are undefined (the kernel that gave up skipped the rest of its work, and tensor-core or
 *     copy operations it had already issued may have finished after it stopped waiting for
 *     them).  Discard those results and run the calls again.  Only a wait that ran out is
 *     recorded -- no memory access is made out of bounds -- so the context itself stays usable;
 *     a caller that cannot tell why a wait ran out (a wait runs out only when an operation did
 *     not complete within 2 s) should synchronise, check for CUDA errors, and recreate the
 *     context if any is reported.
 */
GDN_API int gdn_device_status(void *stream);

/*
 * gdn_selftest_wait_timeout -- exercise the failure path of the bounded waits: enqueues on `stream`
 * one kernel whose wait on an mbarrier that nothing arrives on runs out after limit_ms (1..2000)
 * milliseconds; the kernel records it in the device error word the other kernels use and returns.
 * The next gdn_device_status(stream) then reports GDN_ERR_TIMEOUT (and clears the record); the
 * context stays usable.  Nothing is faulted or hung: the wait is bounded.  The pages have no
 * counterpart of it; it exists for the library's own failure-detection test.
 */
GDN_API int gdn_selftest_wait_timeout(int limit_ms, void *stream);

/* Static text for a status code. */
GDN_API const char *gdn_status_string(int status);

/* One-line reason for the last failed call on this host thread ("" when none). */
GDN_API const char *gdn_last_error(void);

/* Library version string. */
GDN_API const char *gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
