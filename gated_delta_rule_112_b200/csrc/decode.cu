// Single-token recurrent step of the gated delta rule, in place on the fp32
// state ("Gated Delta Networks", phantomic12 page, mechanism paragraph: a
// fixed-size state per head and no KV cache, so a decode step reads and
// writes exactly that state once).
//
// Per (n, h), with the state held transposed in memory (st[j][i] = S_ij):
//   x_i = sum_j st[j][i] k_j      y_i = sum_j st[j][i] q_j
//   u_i = beta (v_i - alpha x_i)
//   st[j][i] <- alpha st[j][i] + u_i k_j
//   o_i = alpha y_i + (k . q) u_i     (= S_t q, read after the write)
//
// Channel-wise gate (the Kimi Delta Attention variant: dmarx anthology
// LIT-137, "Standing in the anthology"; SOTA-135, "Sequence"): alpha_j per d_k
// channel j, S_t = S_{t-1} diag(alpha)(I - beta k k^T) + beta v k^T, so
//   x_i = sum_j st[j][i] alpha_j k_j    y_i = sum_j st[j][i] alpha_j q_j
//   u_i = beta (v_i - x_i)    st[j][i] <- alpha_j st[j][i] + u_i k_j
//   o_i = y_i + (k . q) u_i
//
// One CTA per state (256 threads = 8 warps). Lane t owns columns 4t..4t+3
// (one 16-byte vector per row, so a warp reads a 512-byte row contiguously),
// warp w owns rows w, w+8, w+16, ... The whole 64 KB state sits in registers
// between the read and the write, so HBM sees exactly one read and one write
// of it. Loads and stores use the streaming cache hint: the full state set is
// far larger than L2 and is not reused within a step.
#include "gdn_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kMaxRowsPerWarp = 128 / kDecWarps;  // 16

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

template <typename T, bool KDA>
__global__ void __launch_bounds__(kDecThreads, 2)
    gdn_decode_kernel(const T *__restrict__ q, const T *__restrict__ k,
                      const T *__restrict__ v, const float *__restrict__ g,
                      const float *__restrict__ beta, float *__restrict__ state,
                      T *__restrict__ o, int dk, int dv) {
  __shared__ float ks[128], qs[128], us[128], as[128];
  __shared__ float xpart[kDecWarps][128], ypart[kDecWarps][128];
  __shared__ float kq_s;

  const int unit = blockIdx.x;  // n * H + h
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float *st = state + size_t(unit) * dk * dv;

  // Issue the state loads first so they are in flight while q, k, v arrive.
  const int col = lane * 4;
  const bool col_ok = col < dv;
  float4 S[kMaxRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kMaxRowsPerWarp; ++r) {
    const int j = warp + r * kDecWarps;
    if (col_ok && j < dk)
      S[r] = __ldcs(reinterpret_cast<const float4 *>(st + size_t(j) * dv + col));
    else
      S[r] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (tid < dk) {
    ks[tid] = to_f32(k[size_t(unit) * dk + tid]);
    qs[tid] = to_f32(q[size_t(unit) * dk + tid]);
    if (KDA) as[tid] = expf(g[size_t(unit) * dk + tid]);
  }
  __syncthreads();
  if (warp == 0) {  // k . q
    float acc = 0.f;
    for (int j = lane; j < dk; j += 32) acc += ks[j] * qs[j];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) kq_s = acc;
  }
  // Partial x = S k and y = S q over this warp's rows.
  float4 xp = make_float4(0.f, 0.f, 0.f, 0.f), yp = xp;
#pragma unroll
  for (int r = 0; r < kMaxRowsPerWarp; ++r) {
    const int j = warp + r * kDecWarps;
    const float aj = KDA && j < dk ? as[j] : 1.f;
    const float kj = j < dk ? aj * ks[j] : 0.f, qj = j < dk ? aj * qs[j] : 0.f;
    xp.x += S[r].x * kj; xp.y += S[r].y * kj; xp.z += S[r].z * kj; xp.w += S[r].w * kj;
    yp.x += S[r].x * qj; yp.y += S[r].y * qj; yp.z += S[r].z * qj; yp.w += S[r].w * qj;
  }
  if (col_ok) {
    *reinterpret_cast<float4 *>(&xpart[warp][col]) = xp;
    *reinterpret_cast<float4 *>(&ypart[warp][col]) = yp;
  }
  __syncthreads();
  // scalar gate: alpha multiplies x and y here; channel gate: already inside them
  const float alpha = KDA ? 1.f : expf(g[unit]);
  const float b = beta[unit];
  if (tid < dv) {
    float x = 0.f, y = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) { x += xpart[w][tid]; y += ypart[w][tid]; }
    const float u = b * (to_f32(v[size_t(unit) * dv + tid]) - alpha * x);
    us[tid] = u;
    o[size_t(unit) * dv + tid] = from_f32<T>(alpha * y + kq_s * u);
  }
  __syncthreads();
  if (col_ok) {
    const float4 u4 = *reinterpret_cast<const float4 *>(&us[col]);
#pragma unroll
    for (int r = 0; r < kMaxRowsPerWarp; ++r) {
      const int j = warp + r * kDecWarps;
      if (j < dk) {
        const float kj = ks[j], aj = KDA ? as[j] : alpha;
        float4 n;
        n.x = aj * S[r].x + u4.x * kj;
        n.y = aj * S[r].y + u4.y * kj;
        n.z = aj * S[r].z + u4.z * kj;
        n.w = aj * S[r].w + u4.w * kj;
        __stcs(reinterpret_cast<float4 *>(st + size_t(j) * dv + col), n);
      }
    }
  }
}

template <bool KDA>
void launch_decode_t(const void *q, const void *k, const void *v, const float *g,
                     const float *beta, float *state, void *o, unsigned units, int dk, int dv,
                     int dtype, cudaStream_t s) {
  if (dtype == GDN_BF16)
    gdn_decode_kernel<__nv_bfloat16, KDA><<<units, kDecThreads, 0, s>>>(
        static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
        static_cast<const __nv_bfloat16 *>(v), g, beta, state,
        static_cast<__nv_bfloat16 *>(o), dk, dv);
  else
    gdn_decode_kernel<float, KDA><<<units, kDecThreads, 0, s>>>(
        static_cast<const float *>(q), static_cast<const float *>(k),
        static_cast<const float *>(v), g, beta, state, static_cast<float *>(o), dk, dv);
}

}  // namespace

cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float *state, void *o, int N, int H, int dk, int dv,
                          int dtype, cudaStream_t s, bool channel_gate) {
  const unsigned units = unsigned(N) * unsigned(H);
  if (channel_gate)
    launch_decode_t<true>(q, k, v, g, beta, state, o, units, dk, dv, dtype, s);
  else
    launch_decode_t<false>(q, k, v, g, beta, state, o, units, dk, dv, dtype, s);
  return cudaGetLastError();
}

}  // namespace gdn
