// Internal declarations of the backward pass (host ABI layer and kernels).
#pragma once
#include "gdn_internal.cuh"

namespace gdn {

// Workspace of the backward pass: the 256 B control block, then S_{t-1}
// before every token (fp32, one 128 x 128 block per (token, head) in the
// kernels' own slot order, whatever d_k, d_v <= 128) and x_t = S_{t-1} k_t
// (fp32 [B*T][H][d_v]).
struct BwdLayout {
  size_t s_prev, x, total;
};
inline BwdLayout bwd_layout(int B, int T, int H, int dk, int dv) {
  (void)dk;
  BwdLayout L{};
  const size_t rows = size_t(B) * size_t(T) * size_t(H);
  L.s_prev = 256;
  L.x = align_up(L.s_prev + rows * size_t(128 * 128) * sizeof(float), 256);
  L.total = align_up(L.x + rows * size_t(dv) * sizeof(float), 256);
  return L;
}

// Workspace of the chunkwise backward pass on the tensor cores (bf16,
// d_k = d_v = 128, 64-token chunks): the forward pass's layout (one segment:
// chunk table, prep tiles -W, (D K)^T, T diag(beta), P and the decay
// factors), then per (chunk, head) unit the state entering the chunk (bf16,
// in the state scan's store order: the 16-byte piece of columns 8 p .. 8 p + 7
// of row i at piece index p * 128 + i) and the gradient with respect to the
// state leaving it (bf16 [d_v][d_k]): O(T / 64 d^2) in all.
struct BwdTcLayout {
  WsLayout fwd;
  size_t s_chunks, gprime, total;
};
inline BwdTcLayout bwd_tc_layout(int B, int T, int H, int num_seqs) {
  BwdTcLayout L{};
  L.fwd = ws_layout(B, T, H, num_seqs, 64, true, 1, false);
  const size_t units = size_t(L.fwd.max_chunks) * size_t(H);
  L.s_chunks = L.fwd.total;
  L.gprime = align_up(L.s_chunks + units * 128 * 128 * 2, 1024);
  L.total = align_up(L.gprime + units * 128 * 128 * 2, 1024);
  return L;
}

// The chunkwise backward's kernels. replay = false: ws already holds the
// chunk map, the prep tiles and the chunk states of a forward pass over the
// same inputs (gdn_chunk_fwd_save), so only the reverse chain and the unit
// kernel run.
cudaError_t launch_bwd_tc(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *s0, const int32_t *cu,
                          const void *d_o, const float *d_sN, int N, int B, int T, int H,
                          int num_seqs, float *dq, float *dkk, float *dvv, float *dg,
                          float *dbeta, float *ds0, void *ws, const BwdTcLayout &L,
                          cudaStream_t s, bool replay = true);

cudaError_t launch_bwd(const void *q, const void *k, const void *v, const float *g,
                       const float *beta, const float *s0, const int32_t *cu, const void *d_o,
                       const float *d_sN, int N, int B, int T, int H, int dk, int dv, int dtype,
                       float *dq, float *dkk, float *dvv, float *dg, float *dbeta, float *ds0,
                       void *ws, const BwdLayout &L, cudaStream_t s);

}  // namespace gdn
