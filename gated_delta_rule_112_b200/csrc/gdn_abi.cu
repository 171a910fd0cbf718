// Host side of the C ABI declared in include/gdn.h: argument validation,
// workspace sizing, dispatch to the kernels and status reporting. Nothing
// here allocates device memory.
#include <cstdio>

#include "bwd_internal.cuh"
#include "gdn_internal.cuh"

using namespace gdn;

namespace gdn {

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms;
}

ProfileEvents g_profile = {nullptr, nullptr, nullptr, nullptr};
}

namespace {

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool tc_path(int dk, int dv, int chunk, int dtype) {
  return dtype == GDN_BF16 && dk == 128 && dv == 128 && chunk == 64;
}

// Shared checks of gdn_chunk_fwd / gdn_chunk_fwd_simt.
int check_chunk_args(const void *q, const void *k, const void *v, const float *g,
                     const float *beta, const float *s0, const int32_t *cu, int B, int T, int H,
                     int dk, int dv, int num_seqs, int chunk, int dtype, const void *o,
                     const float *sN, const void *ws) {
  if (dtype != GDN_BF16 && dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
  if (B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1) return GDN_ERR_INVALID_ARG;
  if (cu && (B != 1 || num_seqs < 1)) return GDN_ERR_INVALID_ARG;
  if (!cu && num_seqs != 0) return GDN_ERR_INVALID_ARG;
  if (int64_t(B) * T * H * (dk > dv ? dk : dv) >= (int64_t(1) << 31)) return GDN_ERR_UNSUPPORTED;
  if (dk > 128 || dv > 128) return GDN_ERR_UNSUPPORTED;
  if (chunk != 16 && chunk != 32 && chunk != 64) return GDN_ERR_UNSUPPORTED;
  if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_INVALID_ARG;
  if (!ws) return GDN_ERR_WORKSPACE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(g, 4) || !aligned(beta, 4) || !aligned(s0, 16) || !aligned(sN, 16) ||
      !aligned(cu, 4))
    return GDN_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return GDN_ERR_WORKSPACE;
  return GDN_OK;
}

// force_simt: the CUDA-core kernel even where the tensor-core path applies.
// channel_gate: g is [B, T, H, d_k] (one log-decay per d_k channel); the
// CUDA-core kernel is the only path for it.
int run_chunk(bool force_simt, bool channel_gate, const void *q, const void *k, const void *v,
              const float *g, const float *beta, const float *s0, const int32_t *cu, int B,
              int T, int H, int dk, int dv, int num_seqs, int chunk, int dtype, void *o,
              float *sN, void *ws, size_t ws_bytes, void *stream) {
  int rc = check_chunk_args(q, k, v, g, beta, s0, cu, B, T, H, dk, dv, num_seqs, chunk, dtype,
                            o, sN, ws);
  if (rc != GDN_OK) return rc;
  // bf16 with d_k = d_v = 128 and 64-token chunks runs on the tensor-core
  // kernels for both gates; everything else on the CUDA-core kernel.
  const bool tc = !force_simt && tc_path(dk, dv, chunk, dtype);
  const int segs = scan_segments(B, T, H, cu ? num_seqs : 0, chunk, tc, device_sms());
  const WsLayout L = ws_layout(B, T, H, cu ? num_seqs : 0, chunk, tc, segs, tc && channel_gate);
  if (ws_bytes < L.total) return GDN_ERR_WORKSPACE;
  const int N = cu ? num_seqs : B;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  prof_record(g_profile.start, s);
  cudaError_t e = launch_chunk_map(cu, B, T, cu ? num_seqs : 0, chunk, ws, L, s);
  if (e != cudaSuccess) return GDN_ERR_CUDA;
  if (tc) {
    e = launch_chunk_tc(q, k, v, g, beta, s0, B, T, H, N, o, sN, ws, L, s);
  } else {
    prof_record(g_profile.prep, s);
    prof_record(g_profile.scan, s);
    e = launch_chunk_simt(q, k, v, g, beta, s0, cu, B, T, H, dk, dv, N, chunk, dtype, o, sN,
                          static_cast<uint32_t *>(ws), s, channel_gate);
  }
  prof_record(g_profile.end, s);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t gdn_chunk_fwd_workspace_size(int B, int T, int H, int d_k, int d_v, int num_seqs,
                                    int chunk, int dtype) {
  if (B < 1 || T < 0 || H < 1 || d_k < 1 || d_v < 1 || num_seqs < 0) return 0;
  if (chunk != 16 && chunk != 32 && chunk != 64) return 0;
  const bool tc = tc_path(d_k, d_v, chunk, dtype);
  return ws_layout(B, T, H, num_seqs, chunk, tc,
                   scan_segments(B, T, H, num_seqs, chunk, tc, device_sms()))
      .total;
}

int gdn_chunk_fwd_scan_segments(int B, int T, int H, int d_k, int d_v, int num_seqs, int chunk,
                                int dtype, int sms) {
  if (B < 0 || T < 0 || H < 0 || num_seqs < 0 || sms < 0) return 1;
  return scan_segments(B, T, H, num_seqs, chunk, tc_path(d_k, d_v, chunk, dtype), sms);
}

int gdn_chunk_fwd_path(int d_k, int d_v, int chunk, int dtype) {
  if (d_k < 1 || d_v < 1 || d_k > 128 || d_v > 128) return -1;
  if (chunk != 16 && chunk != 32 && chunk != 64) return -1;
  if (dtype != GDN_BF16 && dtype != GDN_F32) return -1;
  return tc_path(d_k, d_v, chunk, dtype) ? GDN_PATH_TCGEN05 : GDN_PATH_SIMT;
}

int gdn_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                  const float *beta, const float *initial_state, const int32_t *cu_seqlens,
                  int B, int T, int H, int d_k, int d_v, int num_seqs, int chunk, int dtype,
                  void *o, float *final_state, void *workspace, size_t workspace_bytes,
                  void *stream) {
  return run_chunk(false, false, q, k, v, g, beta, initial_state, cu_seqlens, B, T, H, d_k,
                   d_v, num_seqs, chunk, dtype, o, final_state, workspace, workspace_bytes,
                   stream);
}

int gdn_chunk_fwd_simt(const void *q, const void *k, const void *v, const float *g,
                       const float *beta, const float *initial_state, const int32_t *cu_seqlens,
                       int B, int T, int H, int d_k, int d_v, int num_seqs, int chunk, int dtype,
                       void *o, float *final_state, void *workspace, size_t workspace_bytes,
                       void *stream) {
  return run_chunk(true, false, q, k, v, g, beta, initial_state, cu_seqlens, B, T, H, d_k,
                   d_v, num_seqs, chunk, dtype, o, final_state, workspace, workspace_bytes,
                   stream);
}

size_t gdn_kda_chunk_fwd_workspace_size(int B, int T, int H, int d_k, int d_v, int num_seqs,
                                        int chunk, int dtype) {
  if (B < 1 || T < 0 || H < 1 || d_k < 1 || d_v < 1 || num_seqs < 0) return 0;
  if (chunk != 16 && chunk != 32 && chunk != 64) return 0;
  const bool tc = tc_path(d_k, d_v, chunk, dtype);
  const int segs = scan_segments(B, T, H, num_seqs, chunk, tc, device_sms());
  return ws_layout(B, T, H, num_seqs, chunk, tc, segs, tc).total;
}

int gdn_kda_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                      const float *beta, const float *initial_state, const int32_t *cu_seqlens,
                      int B, int T, int H, int d_k, int d_v, int num_seqs, int chunk, int dtype,
                      void *o, float *final_state, void *workspace, size_t workspace_bytes,
                      void *stream) {
  return run_chunk(false, true, q, k, v, g, beta, initial_state, cu_seqlens, B, T, H, d_k, d_v,
                   num_seqs, chunk, dtype, o, final_state, workspace, workspace_bytes, stream);
}

namespace {
int run_decode(bool channel_gate, const void *q, const void *k, const void *v, const float *g,
               const float *beta, float *state, void *o, int N, int H, int d_k, int d_v,
               int dtype, void *stream) {
  if (dtype != GDN_BF16 && dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
  if (N < 1 || H < 1 || d_k < 1 || d_v < 1) return GDN_ERR_INVALID_ARG;
  if (d_k > 128 || d_v > 128 || (d_v % 4) != 0) return GDN_ERR_UNSUPPORTED;
  if (int64_t(N) * H >= (int64_t(1) << 31)) return GDN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !g || !beta || !state || !o) return GDN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(state, 16) || !aligned(g, 4) || !aligned(beta, 4))
    return GDN_ERR_INVALID_ARG;
  cudaError_t e = launch_decode(q, k, v, g, beta, state, o, N, H, d_k, d_v, dtype,
                                static_cast<cudaStream_t>(stream), channel_gate);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
}  // namespace

int gdn_decode_step(const void *q, const void *k, const void *v, const float *g,
                    const float *beta, float *state, void *o, int N, int H, int d_k, int d_v,
                    int dtype, void *stream) {
  return run_decode(false, q, k, v, g, beta, state, o, N, H, d_k, d_v, dtype, stream);
}

int gdn_kda_decode_step(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, float *state, void *o, int N, int H, int d_k,
                        int d_v, int dtype, void *stream) {
  return run_decode(true, q, k, v, g, beta, state, o, N, H, d_k, d_v, dtype, stream);
}

size_t gdn_chunk_bwd_exact_workspace_size(int B, int T, int H, int d_k, int d_v, int num_seqs) {
  if (B < 1 || T < 0 || H < 1 || d_k < 1 || d_v < 1 || num_seqs < 0) return 0;
  return bwd_layout(B, T, H, d_k, d_v).total;
}

size_t gdn_chunk_bwd_workspace_size(int B, int T, int H, int d_k, int d_v, int num_seqs,
                                    int dtype) {
  if (B < 1 || T < 0 || H < 1 || d_k < 1 || d_v < 1 || num_seqs < 0) return 0;
  if (tc_path(d_k, d_v, 64, dtype)) return bwd_tc_layout(B, T, H, num_seqs).total;
  return bwd_layout(B, T, H, d_k, d_v).total;
}

}  // extern "C"

namespace {

// saved: the workspace holds a gdn_chunk_fwd_save pass over the same inputs
// (tensor-core path only), so the forward replay is skipped.
int run_bwd(bool exact, bool saved, const void *q, const void *k, const void *v, const float *g,
            const float *beta, const float *initial_state, const int32_t *cu_seqlens,
            const void *d_o, const float *d_final_state, int B, int T, int H, int d_k, int d_v,
            int num_seqs, int dtype, float *dq, float *dk, float *dv, float *dg, float *dbeta,
            float *d_initial_state, void *workspace, size_t workspace_bytes, void *stream) {
  if (dtype != GDN_BF16 && dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
  if (B < 1 || T < 0 || H < 1 || d_k < 1 || d_v < 1) return GDN_ERR_INVALID_ARG;
  if (cu_seqlens && (B != 1 || num_seqs < 1)) return GDN_ERR_INVALID_ARG;
  if (!cu_seqlens && num_seqs != 0) return GDN_ERR_INVALID_ARG;
  if (d_k > 128 || d_v > 128 || (d_v % 4) != 0) return GDN_ERR_UNSUPPORTED;
  if (int64_t(B) * T * H * (d_k > d_v ? d_k : d_v) >= (int64_t(1) << 31)) return GDN_ERR_UNSUPPORTED;
  if (!d_initial_state) return GDN_ERR_INVALID_ARG;
  if (T > 0 && (!q || !k || !v || !g || !beta || !d_o || !dq || !dk || !dv || !dg || !dbeta))
    return GDN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(d_o, 16) ||
      !aligned(g, 4) || !aligned(beta, 4) || !aligned(initial_state, 16) ||
      !aligned(d_final_state, 16) || !aligned(d_initial_state, 16) || !aligned(dq, 8) ||
      !aligned(dk, 8) || !aligned(dv, 8) || !aligned(dg, 4) || !aligned(dbeta, 4) ||
      !aligned(cu_seqlens, 4))
    return GDN_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256)) return GDN_ERR_WORKSPACE;
  const int N = cu_seqlens ? num_seqs : B;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (saved && !tc_path(d_k, d_v, 64, dtype)) return GDN_ERR_UNSUPPORTED;
  if (!exact && tc_path(d_k, d_v, 64, dtype)) {
    const BwdTcLayout L = bwd_tc_layout(B, T, H, cu_seqlens ? num_seqs : 0);
    if (workspace_bytes < L.total) return GDN_ERR_WORKSPACE;
    if (T == 0) {
      // no tokens: the initial-state gradient is the final-state gradient
      const size_t bytes = size_t(N) * H * 128 * 128 * sizeof(float);
      e = d_final_state ? cudaMemcpyAsync(d_initial_state, d_final_state, bytes,
                                          cudaMemcpyDeviceToDevice, s)
                        : cudaMemsetAsync(d_initial_state, 0, bytes, s);
      if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, 256, s);
    } else {
      e = launch_bwd_tc(q, k, v, g, beta, initial_state, cu_seqlens, d_o, d_final_state, N, B,
                        T, H, cu_seqlens ? num_seqs : 0, dq, dk, dv, dg, dbeta,
                        d_initial_state, workspace, L, s, !saved);
    }
  } else {
    const BwdLayout L = bwd_layout(B, T, H, d_k, d_v);
    if (workspace_bytes < L.total) return GDN_ERR_WORKSPACE;
    e = launch_bwd(q, k, v, g, beta, initial_state, cu_seqlens, d_o, d_final_state, N, B, T, H,
                   d_k, d_v, dtype, dq, dk, dv, dg, dbeta, d_initial_state, workspace, L, s);
  }
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

extern "C" {

int gdn_chunk_bwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                  const float *initial_state, const int32_t *cu_seqlens, const void *d_o,
                  const float *d_final_state, int B, int T, int H, int d_k, int d_v,
                  int num_seqs, int dtype, float *dq, float *dk, float *dv, float *dg,
                  float *dbeta, float *d_initial_state, void *workspace,
                  size_t workspace_bytes, void *stream) {
  return run_bwd(false, false, q, k, v, g, beta, initial_state, cu_seqlens, d_o, d_final_state,
                 B, T, H, d_k, d_v, num_seqs, dtype, dq, dk, dv, dg, dbeta, d_initial_state,
                 workspace, workspace_bytes, stream);
}

int gdn_chunk_bwd_saved(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, const float *initial_state,
                        const int32_t *cu_seqlens, const void *d_o, const float *d_final_state,
                        int B, int T, int H, int d_k, int d_v, int num_seqs, int dtype,
                        float *dq, float *dk, float *dv, float *dg, float *dbeta,
                        float *d_initial_state, void *workspace, size_t workspace_bytes,
                        void *stream) {
  return run_bwd(false, true, q, k, v, g, beta, initial_state, cu_seqlens, d_o, d_final_state,
                 B, T, H, d_k, d_v, num_seqs, dtype, dq, dk, dv, dg, dbeta, d_initial_state,
                 workspace, workspace_bytes, stream);
}

int gdn_chunk_fwd_save(const void *q, const void *k, const void *v, const float *g,
                       const float *beta, const float *initial_state, const int32_t *cu_seqlens,
                       int B, int T, int H, int d_k, int d_v, int num_seqs, int dtype, void *o,
                       float *final_state, void *workspace, size_t workspace_bytes,
                       void *stream) {
  int rc = check_chunk_args(q, k, v, g, beta, initial_state, cu_seqlens, B, T, H, d_k, d_v,
                            num_seqs, 64, dtype, o, final_state, workspace);
  if (rc != GDN_OK) return rc;
  if (!tc_path(d_k, d_v, 64, dtype)) return GDN_ERR_UNSUPPORTED;
  const int ns = cu_seqlens ? num_seqs : 0;
  const BwdTcLayout L = bwd_tc_layout(B, T, H, ns);
  if (workspace_bytes < L.total) return GDN_ERR_WORKSPACE;
  const int N = cu_seqlens ? num_seqs : B;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_chunk_map(cu_seqlens, B, T, ns, 64, workspace, L.fwd, s);
  if (e == cudaSuccess) {
    __nv_bfloat16 *sc =
        reinterpret_cast<__nv_bfloat16 *>(static_cast<char *>(workspace) + L.s_chunks);
    e = launch_chunk_tc(q, k, v, g, beta, initial_state, B, T, H, N, o, final_state, workspace,
                        L.fwd, s, sc);
  }
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

int gdn_chunk_bwd_exact(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, const float *initial_state,
                        const int32_t *cu_seqlens, const void *d_o, const float *d_final_state,
                        int B, int T, int H, int d_k, int d_v, int num_seqs, int dtype,
                        float *dq, float *dk, float *dv, float *dg, float *dbeta,
                        float *d_initial_state, void *workspace, size_t workspace_bytes,
                        void *stream) {
  return run_bwd(true, false, q, k, v, g, beta, initial_state, cu_seqlens, d_o, d_final_state,
                 B, T, H, d_k, d_v, num_seqs, dtype, dq, dk, dv, dg, dbeta, d_initial_state,
                 workspace, workspace_bytes, stream);
}

int gdn_get_status(void *workspace, void *stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
  if (!workspace) return GDN_OK;
  uint32_t err = 0;
  if (cudaMemcpy(&err, workspace, sizeof(err), cudaMemcpyDeviceToHost) != cudaSuccess)
    return GDN_ERR_CUDA;
  if (err) {
    const uint32_t zero = 0;
    if (cudaMemcpy(workspace, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return GDN_ERR_CUDA;
  }
  if (err & kErrTimeout) return GDN_ERR_DEVICE_TIMEOUT;
  if (err & kErrBounds) return GDN_ERR_DEVICE_BOUNDS;
  if (err & kErrLayout) return GDN_ERR_CUDA;
  if (err & kErrBadSeqlens) return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

int gdn_set_profile_events(void *ev_start, void *ev_prep, void *ev_scan, void *ev_end) {
  const int nulls = !ev_start + !ev_prep + !ev_scan + !ev_end;
  if (nulls != 0 && nulls != 4) return GDN_ERR_INVALID_ARG;
  g_profile.start = static_cast<cudaEvent_t>(ev_start);
  g_profile.prep = static_cast<cudaEvent_t>(ev_prep);
  g_profile.scan = static_cast<cudaEvent_t>(ev_scan);
  g_profile.end = static_cast<cudaEvent_t>(ev_end);
  return GDN_OK;
}

int gdn_checked_build(void) { return GDN_CHECKS ? 1 : 0; }

const char *gdn_status_string(int status) {
  switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
    case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
    case GDN_ERR_DEVICE_TIMEOUT: return "GDN_ERR_DEVICE_TIMEOUT";
    case GDN_ERR_DEVICE_BOUNDS: return "GDN_ERR_DEVICE_BOUNDS";
    default: return "GDN_ERR_UNKNOWN";
  }
}

}  // extern "C"
