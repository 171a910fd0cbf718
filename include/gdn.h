/*
 * gdn.h -- C ABI of libgdn: the gated delta rule forward pass and decode step
 * on NVIDIA B200 (sm_100a).
 *
 * The operation ("Gated Delta Networks: Improving Mamba2 with Delta Rule";
 * recurrence on the phantomic12 "gated-deltanet" page, mechanism paragraph,
 * and the dmarx anthology LIT-137, "Standing in the anthology"; readout on the
 * portpowered "Gated DeltaNet" page, "How It Works"):
 *
 *     S_t = S_{t-1} (alpha_t (I - beta_t k_t k_t^T)) + beta_t v_t k_t^T
 *     o_t = S_t q_t                      (read after the write at t)
 *
 * with S_t a d_v x d_k matrix per (sequence, head), alpha_t = exp(g_t).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller. The library
 *     allocates no memory and frees none.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream) and return once work is enqueued.
 *   - Inputs are never modified, except `state` in gdn_decode_step.
 *   - Outputs are undefined when a call returns an error.
 *   - Row-major layouts:
 *       q, k   [B, T, H, d_k]      v, o   [B, T, H, d_v]
 *       g, beta [B, T, H] fp32      (g = log alpha; any finite value; beta is
 *                                    not clamped, so beta in (0, 2) -- the
 *                                    negative-eigenvalue extension -- works)
 *       states [N, H, d_k, d_v] fp32 with state[n][h][j][i] = S_{i j}
 *       (the memory holds S^T, d_v contiguous).
 *   - dtype selects the type of q, k, v and o: GDN_BF16 or GDN_F32.
 *   - No C++ exceptions cross the ABI. Host-side checks return an error code
 *     and launch nothing.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define GDN_OK                 0
#define GDN_ERR_INVALID_ARG    1  /* null required pointer, bad size, misaligned pointer, bad cu_seqlens */
#define GDN_ERR_UNSUPPORTED    2  /* valid but not implemented: d_k or d_v > 128, chunk not in {16,32,64} */
#define GDN_ERR_WORKSPACE      3  /* workspace missing or smaller than gdn_chunk_fwd_workspace_size() */
#define GDN_ERR_CUDA           4  /* a CUDA runtime/driver call or kernel launch failed */
#define GDN_ERR_DEVICE_TIMEOUT 5  /* a bounded device-side wait expired (reported by gdn_get_status) */
#define GDN_ERR_DEVICE_BOUNDS  6  /* bounds-checked builds only (-DGDN_CHECKS=1): a kernel computed a
                                     global-memory index outside its buffer and skipped the access
                                     (reported by gdn_get_status) */

/* Element types of q, k, v, o. */
#define GDN_BF16 0
#define GDN_F32  1

/* Chunked-forward implementations (gdn_chunk_fwd_path). */
#define GDN_PATH_TCGEN05 1   /* bf16, d_k = d_v = 128, chunk = 64: tensor-core kernels */
#define GDN_PATH_SIMT    2   /* everything else with d <= 128: fp32 CUDA-core kernel */

/*
 * gdn_chunk_fwd_workspace_size -- bytes of device workspace gdn_chunk_fwd needs.
 *
 * An upper bound that does not depend on the contents of cu_seqlens: for
 * packed sequences (num_seqs > 0) it assumes the worst case of
 * (T + num_seqs * (chunk - 1)) / chunk chunks. Returns 0 for invalid sizes.
 * The workspace must be 256-byte aligned; its contents need no initialisation.
 * Sized for the current CUDA device: with few long sequences the tensor-core
 * path splits the state scan into segments (gdn_chunk_fwd_scan_segments) and
 * needs three fp32 states per segment and head more.
 */
size_t gdn_chunk_fwd_workspace_size(int B, int T, int H, int d_k, int d_v, int num_seqs,
                                    int chunk, int dtype);

/*
 * gdn_chunk_fwd -- the whole-sequence forward pass, computed chunkwise.
 *
 * Algorithm: the chunkwise-parallel WY representation / UT transform extended
 * to carry the decay gate (phantomic12 page, mechanism paragraph; LIT-137,
 * "Standing in the anthology"; SOTA-135, "Source"). Per chunk of `chunk`
 * tokens: Gamma = cumsum(g); A = strictly-lower beta (K K^T .* exp(Gamma_r -
 * Gamma_s)); T = (I + A)^-1; W = T diag(beta exp(Gamma)) K; U = T diag(beta) V;
 * V_new = U - W S^T; O = diag(exp(Gamma)) Q S^T + (Q K^T .* M) V_new with the
 * diagonal included in M; S <- exp(Gamma_last) S + V_new^T diag(exp(Gamma_last
 * - Gamma)) K. The result equals the token recurrence up to rounding.
 *
 *   q, k, v, o      see layouts above; 16-byte aligned.
 *   g, beta         [B, T, H] fp32, 4-byte aligned.
 *   initial_state   [N, H, d_k, d_v] fp32 or NULL (zero state); 16-byte aligned.
 *   cu_seqlens      NULL, or int32 [num_seqs + 1] device array of packed
 *                   sequence boundaries: cu[0] = 0, non-decreasing,
 *                   cu[num_seqs] = T; requires B == 1. Sequence n covers
 *                   tokens [cu[n], cu[n+1]), starts from initial_state[n] and
 *                   ends in final_state[n]; no state flows between sequences.
 *                   Its contents are checked on the device; a violation is
 *                   reported as GDN_ERR_INVALID_ARG by gdn_get_status and no
 *                   output is written.
 *   N               num_seqs with cu_seqlens, otherwise B.
 *   chunk           tokens per chunk: 64 for the tensor-core path; 16, 32 or
 *                   64 for the CUDA-core path. Chunks start at each
 *                   sequence's first token; the last one may be partial.
 *   final_state     [N, H, d_k, d_v] fp32 or NULL (not written).
 *   workspace       device scratch of at least gdn_chunk_fwd_workspace_size()
 *                   bytes, 256-byte aligned, not used by any concurrent call.
 *   stream          cudaStream_t as void*.
 *
 * Returns GDN_OK once all kernels are enqueued. Path: GDN_PATH_TCGEN05 for
 * dtype GDN_BF16 with d_k = d_v = 128 and chunk = 64, GDN_PATH_SIMT otherwise.
 */
int gdn_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                  const float *beta, const float *initial_state, const int32_t *cu_seqlens,
                  int B, int T, int H, int d_k, int d_v, int num_seqs, int chunk, int dtype,
                  void *o, float *final_state, void *workspace, size_t workspace_bytes,
                  void *stream);

/*
 * gdn_chunk_fwd_simt -- same contract as gdn_chunk_fwd, but always runs the
 * fp32 CUDA-core kernel (the path fp32 inputs and general head sizes take).
 * Useful to cross-check the tensor-core path on the same bf16 inputs.
 */
int gdn_chunk_fwd_simt(const void *q, const void *k, const void *v, const float *g,
                       const float *beta, const float *initial_state, const int32_t *cu_seqlens,
                       int B, int T, int H, int d_k, int d_v, int num_seqs, int chunk, int dtype,
                       void *o, float *final_state, void *workspace, size_t workspace_bytes,
                       void *stream);

/*
 * gdn_chunk_fwd_noalloc -- gdn_chunk_fwd without a caller-supplied workspace.
 *
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory: code running while a CUDA graph is
 * being captured, plugins inside engines that own all device memory and
 * offer no allocation hook, and latency-critical paths that cannot afford
 * cudaMalloc's implicit synchronisation. It allocates nothing: its scratch is
 * a fixed 64 MiB array built into the library, which every GPU that loads
 * the library keeps reserved until the process exits.
 *
 *   Arguments, layouts and results are those of gdn_chunk_fwd, minus
 *   workspace / workspace_bytes.
 *   Returns GDN_ERR_WORKSPACE (and launches nothing) when these sizes need
 *   more than 64 MiB of scratch, i.e. gdn_chunk_fwd_workspace_size(...) >
 *   64 MiB -- roughly 2,000 (chunk, head) pairs on the tensor-core path.
 *   That size is evaluated against the current device's SM count (the
 *   segmented scan's layout depends on it); the check launches nothing.
 *   The first call on a device looks up the array's device address (once per
 *   device, thread-safe); make that first call before any stream capture.
 *   The address stays cached for the process: after cudaDeviceReset it is
 *   stale, and this entry point must not be called again.
 *   All calls on a device share the array and it keeps the last call's
 *   contents, so calls that overlap on the GPU (different streams, no
 *   ordering between them) race and produce undefined results; serialise
 *   them. Device-side errors (bad cu_seqlens contents, an expired bounded
 *   wait) are recorded only in that internal scratch and are not reported by
 *   gdn_get_status; check cu_seqlens on the host when using this variant.
 */
int gdn_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *initial_state,
                          const int32_t *cu_seqlens, int B, int T, int H, int d_k, int d_v,
                          int num_seqs, int chunk, int dtype, void *o, float *final_state,
                          void *stream);

/* 1 if this library was built with device-side bounds checks (-DGDN_CHECKS=1),
 * else 0. In a checked build the tensor-core chunked forward pass (chunk map,
 * prep, state scan, segment composition) compares every plain global-memory
 * index with the extent of its buffer before the access; an index outside it
 * skips the access and records GDN_ERR_DEVICE_BOUNDS for gdn_get_status. (TMA
 * copies need no check: the hardware clips them to the tensor map.) It is
 * the stand-in for a memory checker when none is available; it is slower and
 * not meant for production. */
int gdn_checked_build(void);

/* Which implementation gdn_chunk_fwd and gdn_kda_chunk_fwd would run for
 * these sizes (GDN_PATH_TCGEN05 or GDN_PATH_SIMT), or a negative value if
 * unsupported. */
int gdn_chunk_fwd_path(int d_k, int d_v, int chunk, int dtype);

/*
 * gdn_chunk_fwd_scan_segments -- into how many segments per sequence the
 * tensor-core path splits its sequential state scan, on a device with `sms`
 * streaming multiprocessors (1 = no split). Pure host arithmetic.
 *
 * The chunk-to-chunk state map S -> S (gamma_last I - W^T D K) + U^T D K is
 * affine in S, so a sequence's chain of chunks can run as segments: every
 * segment from S = 0 and, with V = 0, from S = I (its map S -> S P + H), a
 * short fp32 composition of the start states, and every segment again from
 * its start state. This is a reading of the pages' parallel-over-chunks
 * training algorithm (phantomic12 page, mechanism paragraph), not a step they
 * print. Used only for equal-length sequences (no cu_seqlens) when the three
 * passes take at most 70 % of the chunk periods of one plain pass.
 */
int gdn_chunk_fwd_scan_segments(int B, int T, int H, int d_k, int d_v, int num_seqs, int chunk,
                                int dtype, int sms);

/*
 * gdn_decode_step -- one recurrent token for N*H independent states, in place.
 *
 * Per (n, h) (one step of the recurrence above; constant-size state, no KV
 * cache: phantomic12 page, mechanism paragraph):
 *     alpha = exp(g); x = S k; y = S q; u = beta (v - alpha x)
 *     S <- alpha S + u k^T;  o = S q = alpha y + (k . q) u
 *
 *   q, k   [N, H, d_k]   v, o  [N, H, d_v]   (dtype), 16-byte aligned
 *   g, beta [N, H] fp32
 *   state  [N, H, d_k, d_v] fp32, read and overwritten; 16-byte aligned.
 * Supports d_k <= 128, d_v <= 128 with d_v a multiple of 4.
 */
int gdn_decode_step(const void *q, const void *k, const void *v, const float *g,
                    const float *beta, float *state, void *o, int N, int H, int d_k,
                    int d_v, int dtype, void *stream);

/*
 * Channel-wise gate (the Kimi Delta Attention variant, named as the
 * recurrence's successor on the dmarx anthology LIT-137 page, "Standing in the
 * anthology", and on SOTA-135, "Sequence": the scalar decay becomes one decay
 * per d_k channel). With alpha_t a d_k vector, diag(alpha_t) stands where the
 * scalar stood:
 *
 *     S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = S_t q_t
 *
 * g = log alpha is then fp32 [B, T, H, d_k] (chunked) or [N, H, d_k] (decode),
 * 4-byte aligned; everything else is as for the scalar gate. The pages give no
 * equations for the variant; this reading is the plain substitution.
 */

/* Bytes of workspace gdn_kda_chunk_fwd needs (same rules as
 * gdn_chunk_fwd_workspace_size); 0 for invalid sizes. */
size_t gdn_kda_chunk_fwd_workspace_size(int B, int T, int H, int d_k, int d_v, int num_seqs,
                                        int chunk, int dtype);

/*
 * gdn_kda_chunk_fwd -- the whole-sequence forward pass with the channel-wise
 * gate, chunkwise. Per chunk, Gamma = cumsum(g) per channel and the decay
 * moves inside the dot products:
 *   A_rs = beta_r sum_j k_rj k_sj exp(Gamma_rj - Gamma_sj) (s < r); T = (I + A)^-1
 *   W = T diag(beta) (K .* exp(Gamma)); U = T diag(beta) V; V_new = U - W S^T
 *   P_rs = sum_j q_rj k_sj exp(Gamma_rj - Gamma_sj) (s <= r)
 *   O = (Q .* exp(Gamma)) S^T + P V_new
 *   S <- S diag(exp(Gamma_last)) + V_new^T (K .* exp(Gamma_last - Gamma))
 * bf16 with d_k = d_v = 128 and chunk = 64 runs on the tensor-core kernels:
 * A and P come from warp-level bf16 tensor-core tiles of operands scaled
 * against the first row b of each 16-row block, e^(Gamma_r - Gamma_b) and
 * e^(Gamma_b - Gamma_s), which factor the decay exactly; the rest is the
 * scalar gate's chunk pipeline with Q .* exp(Gamma) and a per-channel state
 * decay. Those scalings need e^(15 max|g|) to fit fp32, i.e. |g| < 5.9 per
 * token and channel (alpha > 0.0028); the fp32 CUDA-core kernel (every other
 * size and dtype) has no such bound. Arguments, layouts, ownership and errors
 * as gdn_chunk_fwd, except g: [B, T, H, d_k] fp32. Supports d_k, d_v <= 128
 * and chunk 16, 32 or 64.
 */
int gdn_kda_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                      const float *beta, const float *initial_state, const int32_t *cu_seqlens,
                      int B, int T, int H, int d_k, int d_v, int num_seqs, int chunk, int dtype,
                      void *o, float *final_state, void *workspace, size_t workspace_bytes,
                      void *stream);

/*
 * gdn_kda_decode_step -- one token with the channel-wise gate for N*H states,
 * in place. Per (n, h), with a = exp(g) [d_k]:
 *     x = S diag(a) k; y = S diag(a) q; u = beta (v - x)
 *     S <- S diag(a) + u k^T;  o = S q = y + (k . q) u
 * Arguments as gdn_decode_step, except g: [N, H, d_k] fp32.
 */
int gdn_kda_decode_step(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, float *state, void *o, int N, int H, int d_k,
                        int d_v, int dtype, void *stream);

/*
 * Backward pass (gradients of gdn_chunk_fwd, scalar gate). The pages call the
 * chunkwise algorithm a training algorithm (phantomic12 page, mechanism
 * paragraph) but give no gradients; they follow by reverse-mode
 * differentiation of the recurrence. For the loss
 *     L = sum(d_o * o) + sum(d_final_state * final_state)
 * with G = dL/dS_t, x_t = S_{t-1} k_t, u_t = beta_t (v_t - alpha_t x_t), going
 * backwards over t:
 *     G += d_o_t q_t^T;  dq_t = S_t^T d_o_t
 *     Gk = G k_t;  dv_t = beta_t Gk;  dbeta_t = Gk . (v_t - alpha_t x_t)
 *     dg_t = alpha_t (<G, S_{t-1}> - beta_t Gk . x_t)
 *     dk_t = G^T u_t - alpha_t beta_t S_{t-1}^T Gk
 *     G <- alpha_t (G - beta_t Gk k_t^T)
 * and d_initial_state = G at each sequence's start.
 */

/* Bytes of workspace gdn_chunk_bwd needs for these sizes and dtype; 0 for
 * invalid sizes. The chunkwise tensor-core backward (bf16, d_k = d_v = 128)
 * needs the forward pass's gdn_chunk_fwd workspace (one scan segment) plus,
 * per (chunk, head), two bf16 128 x 128 states (64 KB): O(T / 64 d^2). Every
 * other size and dtype runs the token-level backward; see
 * gdn_chunk_bwd_exact_workspace_size. */
size_t gdn_chunk_bwd_workspace_size(int B, int T, int H, int d_k, int d_v, int num_seqs,
                                    int dtype);

/* Bytes of workspace gdn_chunk_bwd_exact needs: 256 + B*T*H*(128*128 + d_v)*4
 * (every token's S_{t-1} in a 128 x 128 fp32 block, and S_{t-1} k_t), rounded
 * up; 0 for invalid sizes. */
size_t gdn_chunk_bwd_exact_workspace_size(int B, int T, int H, int d_k, int d_v, int num_seqs);

/*
 * gdn_chunk_bwd -- gradients of the forward pass for the loss above.
 *
 *   q, k, v, g, beta, initial_state, cu_seqlens, B, T, H, d_k, d_v, num_seqs,
 *   dtype              as for gdn_chunk_fwd (the forward inputs).
 *   d_o                [B, T, H, d_v] (dtype), 16-byte aligned: dL/do.
 *   d_final_state      [N, H, d_k, d_v] fp32 (S^T storage) or NULL (zero).
 *   dq, dk             [B, T, H, d_k] fp32 outputs.
 *   dv                 [B, T, H, d_v] fp32 output.
 *   dg, dbeta          [B, T, H] fp32 outputs (dg = dL/d(log alpha)).
 *   d_initial_state    [N, H, d_k, d_v] fp32 output (also when
 *                      initial_state is NULL: the gradient at a zero state).
 *   workspace          >= gdn_chunk_bwd_workspace_size() bytes, 256-byte
 *                      aligned, not shared with a concurrent call.
 * Supports d_k <= 128 and d_v <= 128 with d_v a multiple of 4; dq, dk, dv
 * 8-byte aligned. bf16 with d_k = d_v = 128 runs the chunkwise backward on
 * the tensor cores (64-token chunks; the derivation is in the header of the
 * kernels' source): the forward pass again, its scan also keeping every
 * chunk's entering state S_c (bf16); a reverse scan over the chunks, two CTAs
 * per (sequence, head), of dS_c = gamma_last dS_{c+1} - dX^T W +
 * (gamma dO)^T Q, keeping each chunk's dS_{c+1} (bf16); and one kernel over
 * all (chunk, head) units for dq, dk, dv, dg, dbeta. gdn_chunk_fwd_save and
 * gdn_chunk_bwd_saved split the same work for a training step (below). bf16 operands, fp32
 * accumulation: its parity bar is the bf16 tolerance. Every other size and
 * dtype runs gdn_chunk_bwd_exact. Bad cu_seqlens contents are reported by
 * gdn_get_status (GDN_ERR_INVALID_ARG); the affected sequences are not
 * computed.
 */
int gdn_chunk_bwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                  const float *initial_state, const int32_t *cu_seqlens, const void *d_o,
                  const float *d_final_state, int B, int T, int H, int d_k, int d_v,
                  int num_seqs, int dtype, float *dq, float *dk, float *dv, float *dg,
                  float *dbeta, float *d_initial_state, void *workspace,
                  size_t workspace_bytes, void *stream);

/*
 * gdn_chunk_fwd_save -- the forward pass of a training step: gdn_chunk_fwd
 * (same arguments and outputs, 64-token chunks) that also leaves in
 * `workspace` what the chunkwise backward would otherwise recompute: the
 * chunk map, the prep tiles (-W, (D K)^T, T diag(beta), P, the decay
 * factors) and every chunk's entering state S_c (bf16). The pages present the
 * chunkwise algorithm for training (phantomic12 page, mechanism paragraph);
 * keeping the forward's intermediates for the backward is this library's
 * reading of that use.
 *   workspace          >= gdn_chunk_bwd_workspace_size() bytes for the same
 *                      sizes, 256-byte aligned; owned by the caller and handed
 *                      unchanged to gdn_chunk_bwd_saved.
 * Tensor-core path only (bf16, d_k = d_v = 128): GDN_ERR_UNSUPPORTED
 * otherwise. The state scan always runs as one pass per (sequence, head) here
 * (gdn_chunk_fwd may split long sequences into segments), so o and
 * final_state are those of that pass.
 */
int gdn_chunk_fwd_save(const void *q, const void *k, const void *v, const float *g,
                       const float *beta, const float *initial_state, const int32_t *cu_seqlens,
                       int B, int T, int H, int d_k, int d_v, int num_seqs, int dtype, void *o,
                       float *final_state, void *workspace, size_t workspace_bytes,
                       void *stream);

/*
 * gdn_chunk_bwd_saved -- gdn_chunk_bwd (same arguments and outputs) for a
 * workspace that gdn_chunk_fwd_save filled from the same q, k, v, g, beta,
 * initial_state, cu_seqlens and sizes on this stream: the forward replay is
 * skipped and only the reverse chain and the per-unit kernel run. The
 * workspace's saved part is read, not changed (the call may be repeated for
 * another d_o); its scratch part takes each chunk's dS_{c+1}, so two calls
 * on one workspace must not overlap on the GPU. Tensor-core path only:
 * GDN_ERR_UNSUPPORTED otherwise. The
 * kernels trust the saved chunk table: a workspace that gdn_chunk_fwd_save
 * did not fill for these inputs is undefined behaviour.
 */
int gdn_chunk_bwd_saved(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, const float *initial_state,
                        const int32_t *cu_seqlens, const void *d_o, const float *d_final_state,
                        int B, int T, int H, int d_k, int d_v, int num_seqs, int dtype,
                        float *dq, float *dk, float *dv, float *dg, float *dbeta,
                        float *d_initial_state, void *workspace, size_t workspace_bytes,
                        void *stream);

/*
 * gdn_chunk_bwd_exact -- the same gradients by the token-level recurrence in
 * fp32, for every supported size and dtype (bf16 inputs are upcast exactly):
 * a forward replay that stores every S_{t-1} (gdn_chunk_bwd_exact_workspace_size
 * bytes, O(T d^2)), then the reverse sweep. Arguments as gdn_chunk_bwd.
 */
int gdn_chunk_bwd_exact(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, const float *initial_state,
                        const int32_t *cu_seqlens, const void *d_o, const float *d_final_state,
                        int B, int T, int H, int d_k, int d_v, int num_seqs, int dtype,
                        float *dq, float *dk, float *dv, float *dg, float *dbeta,
                        float *d_initial_state, void *workspace, size_t workspace_bytes,
                        void *stream);

/*
 * gdn_selftest_wait_timeout -- device self-test of the bounded waits (the
 * pages have no counterpart; it tests this library's failure handling).
 *
 * Launches, on `stream`, one small kernel that waits on a barrier nothing
 * ever completes, with the same bounded wait (about 1 s of SM clock) that the
 * chunked-forward kernels use. The wait must give up: afterwards
 * gdn_get_status(workspace, stream) returns GDN_ERR_DEVICE_TIMEOUT (and clears
 * the error word), and the context stays usable. `workspace`: caller-owned
 * device memory of at least 256 bytes, 256-byte aligned; its first 256 bytes
 * are overwritten. Returns GDN_OK once launched, GDN_ERR_WORKSPACE or
 * GDN_ERR_CUDA otherwise.
 */
int gdn_selftest_wait_timeout(void *workspace, void *stream);

/*
 * gdn_get_status -- synchronises `stream`, then reports the first error seen:
 * GDN_ERR_CUDA for a failed kernel, or the code a gdn_chunk_fwd kernel left in
 * `workspace` (GDN_ERR_DEVICE_TIMEOUT, GDN_ERR_INVALID_ARG for bad
 * cu_seqlens). Clears the device error word. `workspace` may be NULL.
 */
int gdn_get_status(void *workspace, void *stream);

/*
 * gdn_set_profile_events -- optional timing hook for benchmarks and profilers.
 *
 * When set (non-NULL cudaEvent_t handles passed as void*), every later
 * gdn_chunk_fwd / gdn_chunk_fwd_simt call records them on its stream:
 *   ev_start   before the chunk-map kernel,
 *   ev_prep    before the per-chunk preparation kernel (tensor-core path;
 *              the CUDA-core path records it right before its one kernel),
 *   ev_scan    before the sequential scan/output kernel (CUDA-core path: same
 *              point as ev_prep),
 *   ev_end     after the last kernel.
 * Pass four NULLs to stop. Process-wide setting, not thread-safe; the caller
 * owns the events. Returns GDN_OK, or GDN_ERR_INVALID_ARG if only some of the
 * four are NULL.
 */
int gdn_set_profile_events(void *ev_start, void *ev_prep, void *ev_scan, void *ev_end);

/* Human-readable name of a status code (static string). */
const char *gdn_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
