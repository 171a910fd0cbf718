// Chunk bookkeeping shared by both chunked-forward paths: the chunk map that
// validates cu_seqlens and lists every (sequence, chunk) of the batch. Chunks
// start at each sequence's first token and the last one of a sequence may be
// partial (the chunkwise algorithm of "Gated Delta Networks", phantomic12
// page, mechanism paragraph, applied per sequence).
#include "gdn_internal.cuh"

namespace gdn {
namespace {

// ---------------------------------------------------------------------------
// Chunk map: validates cu_seqlens and lists every (sequence, chunk).
// One CTA of 1024 threads; thread t owns a contiguous range of sequences.
__global__ void __launch_bounds__(1024) gdn_chunk_map_kernel(
    const int32_t *__restrict__ cu, int B, int T, int num_seqs, int chunk,
    uint32_t *__restrict__ ctrl, ChunkInfo *__restrict__ table,
    int32_t *__restrict__ seq_first, int max_chunks, int segs, int32_t *__restrict__ seg_first) {
  // The kernels launched after this one may start their prologues now; they
  // wait for this grid before reading what it writes.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int N = num_seqs > 0 ? num_seqs : B;
  const int tid = threadIdx.x;
  if (!cu) {
    // B sequences of T tokens: every entry has a closed form.
    const int cps = (T + chunk - 1) / chunk;
    const int total = B * cps;
    for (int idx = tid; idx < total; idx += blockDim.x) {
      const int n = idx / cps, c = idx - n * cps;
      ChunkInfo ci;
      ci.seq = n;
      ci.cidx = c;
      ci.row0 = n * T + c * chunk;
      ci.len = min(chunk, T - c * chunk);
      if (GDN_IN_BOUNDS(ctrl, idx, max_chunks)) table[idx] = ci;
    }
    for (int n = tid; n <= N; n += blockDim.x)
      if (GDN_IN_BOUNDS(ctrl, n, N + 1)) seq_first[n] = n * cps;
    if (segs > 1) {
      // segment g of sequence n: chunks [n cps + g len, min(n cps + (g + 1) len, (n + 1) cps))
      const int len = (cps + segs - 1) / segs;
      for (int e = tid; e <= N * segs; e += blockDim.x) {
        const int n = e / segs, gi = e - n * segs;
        if (GDN_IN_BOUNDS(ctrl, e, N * segs + 1))
          seg_first[e] = (n >= N) ? N * cps : n * cps + min(gi * len, cps);
      }
    }
    if (tid == 0) {
      ctrl[0] = 0;
      ctrl[1] = uint32_t(total);
    }
    return;
  }
  __shared__ int32_t scan[1024];
  __shared__ int bad;
  if (tid == 0) bad = 0;
  __syncthreads();
  const int per = (N + 1023) / 1024;
  const int n0 = min(N, tid * per), n1 = min(N, n0 + per);
  int32_t local = 0;
  for (int n = n0; n < n1; ++n) {
    const int a = GDN_IN_BOUNDS(ctrl, n + 1, N + 1) ? cu[n] : 0;
    const int b = GDN_IN_BOUNDS(ctrl, n + 1, N + 1) ? cu[n + 1] : 0;
    if ((n == 0 && a != 0) || b < a || (n == N - 1 && b != T)) bad = 1;
    const int len = b - a;
    if (len > 0) local += (len + chunk - 1) / chunk;
  }
  scan[tid] = local;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const int32_t add = tid >= off ? scan[tid - off] : 0;
    __syncthreads();
    scan[tid] += add;
    __syncthreads();
  }
  const int32_t total = scan[1023];
  if (bad || total > max_chunks) {
    if (tid == 0) {
      ctrl[0] = kErrBadSeqlens;
      ctrl[1] = 0;
    }
    return;
  }
  int32_t first = scan[tid] - local;
  for (int n = n0; n < n1; ++n) {
    const bool ok = GDN_IN_BOUNDS(ctrl, n + 1, N + 1);
    const int row0 = ok ? cu[n] : 0;
    const int len = ok ? cu[n + 1] - row0 : 0;
    if (ok) seq_first[n] = first;
    for (int c = 0; c * chunk < len; ++c) {
      ChunkInfo ci;
      ci.seq = n;
      ci.cidx = c;
      ci.row0 = row0 + c * chunk;
      ci.len = min(chunk, len - c * chunk);
      if (GDN_IN_BOUNDS(ctrl, first + c, max_chunks)) table[first + c] = ci;
    }
    if (len > 0) first += (len + chunk - 1) / chunk;
  }
  if (tid == 1023) seq_first[N] = total;
  if (tid == 0) {
    ctrl[0] = 0;
    ctrl[1] = uint32_t(total);
  }
}

}  // namespace

cudaError_t launch_chunk_map(const int32_t *cu_seqlens, int B, int T, int num_seqs, int chunk,
                             void *ws, const WsLayout &L, cudaStream_t s) {
  char *base = static_cast<char *>(ws);
  // The kernel writes the control block itself (error word, chunk count).
  gdn_chunk_map_kernel<<<1, 1024, 0, s>>>(
      cu_seqlens, B, T, num_seqs, chunk, reinterpret_cast<uint32_t *>(base),
      reinterpret_cast<ChunkInfo *>(base + L.chunk_table),
      reinterpret_cast<int32_t *>(base + L.seq_first), L.max_chunks, L.segs,
      L.segs > 1 ? reinterpret_cast<int32_t *>(base + L.seg_first) : nullptr);
  return cudaGetLastError();
}

}  // namespace gdn
