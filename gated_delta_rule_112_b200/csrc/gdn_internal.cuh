// Internal declarations shared by the host ABI layer and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "gdn.h"  // public C ABI (include/, on the -I path)

namespace gdn {

// Device error bits (stored in the first word of the workspace).
constexpr uint32_t kErrBadSeqlens = 1u;
constexpr uint32_t kErrTimeout = 2u;
constexpr uint32_t kErrLayout = 4u;   // shared-memory window not 1024-byte aligned

// One chunk of one sequence (shared by all heads).
struct ChunkInfo {
  int32_t seq;    // sequence index n
  int32_t cidx;   // chunk index within the sequence
  int32_t row0;   // first token row in the flattened [B*T] token axis
  int32_t len;    // valid tokens in this chunk (1..chunk)
};

// Workspace layout. Offsets are in bytes from the (256-byte aligned) base.
//   [0, 256)       control block: word 0 = device error bits, word 1 = total chunks
//   chunk table    ChunkInfo[max_chunks]
//   seq_first      int32[N + 1]  global index of each sequence's first chunk
//   tensor-core path only, per (chunk, head) unit u = chunk * H + h:
//   w              bf16 [units][64][d_k = 128]   -W of the chunk (rows = tokens)
//   kt             bf16 [units][d_k = 128][64]   (D K)^T, D = diag(exp(Gamma_last - Gamma))
//   tb             bf16 [units][64][64]          T diag(beta) of the chunk (UT transform)
//   pm             bf16 [units][64][64]          (Q K^T) .* decay mask, diagonal included
//   gam            fp32 [units][128]             exp(Gamma_c) (64), then exp(Gamma_last - Gamma_s) (64)
struct WsLayout {
  size_t chunk_table, seq_first, w, kt, tb, pm, gam, total;
  int max_chunks;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline int max_chunks_for(int B, int T, int num_seqs, int chunk) {
  if (num_seqs > 0) return int((int64_t(T) + int64_t(num_seqs) * (chunk - 1)) / chunk);
  return int(int64_t(B) * ((int64_t(T) + chunk - 1) / chunk));
}

inline WsLayout ws_layout(int B, int T, int H, int num_seqs, int chunk, bool tc) {
  WsLayout L{};
  const int N = num_seqs > 0 ? num_seqs : B;
  L.max_chunks = max_chunks_for(B, T, num_seqs, chunk);
  size_t off = 256;
  L.chunk_table = off;
  off = align_up(off + sizeof(ChunkInfo) * size_t(L.max_chunks > 0 ? L.max_chunks : 1), 256);
  L.seq_first = off;
  off = align_up(off + sizeof(int32_t) * size_t(N + 1), 1024);
  if (tc) {
    const size_t units = size_t(L.max_chunks) * H;
    L.w = off;   off = align_up(off + units * 64 * 128 * 2, 1024);
    L.kt = off;  off = align_up(off + units * 128 * 64 * 2, 1024);
    L.tb = off;  off = align_up(off + units * 64 * 64 * 2, 1024);
    L.pm = off;  off = align_up(off + units * 64 * 64 * 2, 1024);
    L.gam = off; off = align_up(off + units * 128 * 4, 1024);
  }
  L.total = off;
  return L;
}

// Optional events recorded around the chunked-forward kernels (see
// gdn_set_profile_events). All null when profiling is off.
struct ProfileEvents {
  cudaEvent_t start, prep, scan, end;
};
extern ProfileEvents g_profile;
inline void prof_record(cudaEvent_t e, cudaStream_t s) {
  if (e) cudaEventRecord(e, s);
}

// Kernel launchers (defined in the .cu files; return a cudaError_t).
cudaError_t launch_chunk_map(const int32_t *cu_seqlens, int B, int T, int num_seqs, int chunk,
                             void *ws, const WsLayout &L, cudaStream_t s);
cudaError_t launch_chunk_simt(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *s0, const int32_t *cu, int B,
                              int T, int H, int dk, int dv, int N, int chunk, int dtype, void *o,
                              float *sN, uint32_t *err, cudaStream_t s);
cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *s0, int B, int T, int H, int N,
                            void *o, float *sN, void *ws, const WsLayout &L, cudaStream_t s);
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float *state, void *o, int N, int H, int dk, int dv,
                          int dtype, cudaStream_t s);

}  // namespace gdn
