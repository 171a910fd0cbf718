// Internal declarations shared by the host ABI layer and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gdn.h"  // public C ABI (include/, on the -I path)

namespace gdn {

// Device error bits (stored in the first word of the workspace).
constexpr uint32_t kErrBadSeqlens = 1u;
constexpr uint32_t kErrTimeout = 2u;
constexpr uint32_t kErrLayout = 4u;   // shared-memory window not 1024-byte aligned
constexpr uint32_t kErrBounds = 8u;   // checked builds: an index outside its buffer (access skipped)

// Bounds checks of plain global-memory accesses, compiled in with
// -DGDN_CHECKS=1 (gdn_checked_build() == 1). GDN_IN_BOUNDS(err, idx, extent)
// is true when 0 <= idx < extent; otherwise it records kErrBounds in *err
// (and, the first time, the source line in err[2] and the index in err[3])
// and is false, so the caller skips the access. Without GDN_CHECKS it is the
// constant true and costs nothing.
#ifndef GDN_CHECKS
#define GDN_CHECKS 0
#endif
#ifdef __CUDACC__
__device__ __forceinline__ bool gdn_bounds_fail(uint32_t *err, long long idx, int line) {
  if (err && !(atomicOr(err, kErrBounds) & kErrBounds)) {
    err[2] = uint32_t(line);
    err[3] = uint32_t(idx);
  }
  return false;
}
#if GDN_CHECKS
#define GDN_IN_BOUNDS(err, idx, extent)                                                   \
  ((static_cast<long long>(idx) >= 0 && static_cast<long long>(idx) < static_cast<long long>(extent)) \
       ? true                                                                            \
       : ::gdn::gdn_bounds_fail((err), static_cast<long long>(idx), __LINE__))
#else
#define GDN_IN_BOUNDS(err, idx, extent) true
#endif
#endif

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
//                  channel-wise gate: fp32 [units][256]: 1 (64), unused (64), then the
//                  per-channel state decay exp(Gamma_last,j) (128)
//   qt             channel-wise gate only: bf16 [units][64][d_k]  Q .* exp(Gamma)
//   tensor-core path with a segmented state scan (segs > 1, see scan_segments):
//   seg_first      int32[B * segs + 1]  first chunk of each segment
//   hbuf, pbuf     fp32 [B * segs][H][d_k][d_v]  each segment's state from S = 0,
//                  and its transition (the state from S = I with V = 0)
//   sstart         fp32 [B * segs][H][d_k][d_v]  each segment's true start state
struct WsLayout {
  size_t chunk_table, seq_first, w, kt, tb, pm, gam, qt, seg_first, hbuf, pbuf, sstart, total;
  int max_chunks, segs;
  bool kda;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline int max_chunks_for(int B, int T, int num_seqs, int chunk) {
  if (num_seqs > 0) return int((int64_t(T) + int64_t(num_seqs) * (chunk - 1)) / chunk);
  return int(int64_t(B) * ((int64_t(T) + chunk - 1) / chunk));
}

// Segments per sequence for the tensor-core state scan. The scan is a chain
// of dependent chunks per (sequence, head), one CTA each; with few chains and
// many chunks most SMs idle. Split into G segments, the chain runs as three
// passes of T / G chunks: every segment from S = 0 and, with V = 0, from
// S = I (its affine map S -> S P_g + H_g), a short fp32 composition of the
// segments' start states, and every segment again from its true start. G is
// chosen by counting chunk periods on `sms` SMs (one CTA per SM); 1 means one
// plain pass. Only for B sequences of equal length (no cu_seqlens).
constexpr int kMaxScanSegments = 16;
inline int scan_segments(int B, int T, int H, int num_seqs, int chunk, bool tc, int sms) {
  if (!tc || num_seqs > 0 || B <= 0 || T <= 0 || H <= 0 || sms <= 0) return 1;
  const long long cps = (int64_t(T) + chunk - 1) / chunk;
  const long long chains = int64_t(B) * H;
  auto waves = [&](long long ctas) { return (ctas + sms - 1) / sms; };
  const long long plain = waves(chains) * cps;
  int best = 1;
  long long best_cost = plain;
  for (int G = 2; G <= kMaxScanSegments && G <= cps; ++G) {
    const long long len = (cps + G - 1) / G;
    const long long g = (cps + len - 1) / len;            // non-empty segments
    // + 8 chunk periods for the composition kernel and the extra launches
    const long long cost = (waves(2 * chains * g) + waves(chains * g)) * len + 8;
    if (cost < best_cost) {
      best_cost = cost;
      best = int(g);
    }
  }
  return (best > 1 && best_cost * 10 <= plain * 7) ? best : 1;   // at least 30 % faster
}

inline WsLayout ws_layout(int B, int T, int H, int num_seqs, int chunk, bool tc, int segs = 1,
                          bool kda = false) {
  WsLayout L{};
  L.kda = kda;
  const int N = num_seqs > 0 ? num_seqs : B;
  L.max_chunks = max_chunks_for(B, T, num_seqs, chunk);
  L.segs = segs;
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
    L.gam = off; off = align_up(off + units * (kda ? 256 : 128) * 4, 1024);
    if (kda) {
      L.qt = off;  off = align_up(off + units * 64 * 128 * 2, 1024);
    }
    if (segs > 1) {
      const size_t nseg = size_t(B) * segs;
      const size_t states = nseg * H * 128 * 128 * sizeof(float);
      L.seg_first = off; off = align_up(off + sizeof(int32_t) * (nseg + 1), 1024);
      L.hbuf = off;      off = align_up(off + states, 1024);
      L.pbuf = off;      off = align_up(off + states, 1024);
      L.sstart = off;    off = align_up(off + states, 1024);
    }
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
// Tensor maps (host side) for TMA loads, 128-byte swizzle where noted:
// tokens [rows, H, 128] bf16 with a 64 x 1 x 64 box (swizzled), and a 2-D
// [rows, inner] map with a (box_inner, box_rows) box. False when the driver's
// encoder is unavailable or rejects the map.
bool map_tokens(CUtensorMap *m, const void *base, long long rows, int H);
bool map_2d(CUtensorMap *m, const void *base, CUtensorMapDataType t, int esize, long long rows,
            int inner, int box_inner, int box_rows, CUtensorMapSwizzle sw);

cudaError_t launch_chunk_map(const int32_t *cu_seqlens, int B, int T, int num_seqs, int chunk,
                             void *ws, const WsLayout &L, cudaStream_t s);
// Streaming multiprocessors of the current device (0 if it cannot be read).
int device_sms();
cudaError_t launch_chunk_simt(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *s0, const int32_t *cu, int B,
                              int T, int H, int dk, int dv, int N, int chunk, int dtype, void *o,
                              float *sN, uint32_t *err, cudaStream_t s, bool channel_gate);
// s_chunks: see the state scan (backward pass only; requires L.segs == 1).
cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *s0, int B, int T, int H, int N,
                            void *o, float *sN, void *ws, const WsLayout &L, cudaStream_t s,
                            __nv_bfloat16 *s_chunks = nullptr);
// channel_gate: g is [N, H, d_k] (one log-decay per d_k channel), else [N, H].
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float *state, void *o, int N, int H, int dk, int dv,
                          int dtype, cudaStream_t s, bool channel_gate);

}  // namespace gdn
