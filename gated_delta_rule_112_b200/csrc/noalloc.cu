// gdn_chunk_fwd_noalloc: the chunked forward pass for callers that cannot
// allocate device memory.
//
// Some callers have no way to provide the scratch buffer gdn_chunk_fwd needs:
// code running while a CUDA graph is being captured (where cudaMalloc is not
// allowed), plugins inside engines that own every byte of device memory and
// expose no allocation hook, and latency-critical paths that must not pay for
// cudaMalloc's implicit device synchronisation. This entry point uses a
// fixed-size scratch array that is part of the library itself instead.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library keeps kNoAllocScratchBytes of device memory reserved for it until
// the process exits. Its device address is looked up once per device (under a
// mutex) with cudaGetSymbolAddress; in host code the array's name is only a
// host-side stand-in and must never be handed to a kernel. The looked-up
// address is cached for the life of the process: after cudaDeviceReset it is
// stale and this entry point must not be called again. All calls on a device
// share the one array, and it keeps whatever the last call left there.
#include <mutex>

#include "gdn_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;   // 64 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void *g_scratch_addr[kMaxDevices] = {};
std::mutex g_setup_mutex;

}  // namespace

extern "C" int gdn_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                     const float *g, const float *beta,
                                     const float *initial_state, const int32_t *cu_seqlens,
                                     int B, int T, int H, int d_k, int d_v, int num_seqs,
                                     int chunk, int dtype, void *o, float *final_state,
                                     void *stream) {
  // Size check first. It launches nothing, but the size depends on the current
  // device's SM count (the segmented scan's layout does), which it queries.
  const size_t need =
      gdn_chunk_fwd_workspace_size(B, T, H, d_k, d_v, num_seqs, chunk, dtype);
  if (need > kNoAllocScratchBytes) return GDN_ERR_WORKSPACE;

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDN_ERR_CUDA;
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
      void *p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return GDN_ERR_CUDA;
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }
  // gdn_chunk_fwd validates every argument, and its first kernel writes the
  // control block (the device error word and the chunk count) before the
  // kernels that read it run; all other scratch contents are written before
  // they are read.
  return gdn_chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, B, T, H, d_k, d_v,
                       num_seqs, chunk, dtype, o, final_state, scratch, kNoAllocScratchBytes,
                       stream);
}
