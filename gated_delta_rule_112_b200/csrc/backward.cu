// Gradients of the gated delta rule forward pass (scalar gate) for a loss with
// dL/do = d_o and dL/dS_final = d_final_state.
//
// The pages describe the chunkwise algorithm as a training algorithm
// ("Gated Delta Networks", phantomic12 page, mechanism paragraph) but give no
// gradients. They follow by reverse-mode differentiation of the recurrence
// S_t = alpha_t S_{t-1} + u_t k_t^T, u_t = beta_t (v_t - alpha_t S_{t-1} k_t),
// o_t = S_t q_t. With G = dL/dS_t (all later tokens already folded in),
// going backwards over t:
//   G += do_t q_t^T
//   dq_t = S_t^T do_t = alpha S_{t-1}^T do_t + k_t (u_t . do_t)
//   Gk = G k_t;  dv_t = beta Gk;  dbeta_t = Gk . (v_t - alpha x_t)   (x_t = S_{t-1} k_t)
//   dg_t = alpha (<G, S_{t-1}> - beta Gk . x_t)
//   dk_t = G^T u_t - alpha beta S_{t-1}^T Gk
//   G <- alpha (G - beta Gk k_t^T)                                     (= dL/dS_{t-1})
// and dL/dS_0 = G at the sequence start.
//
// Two kernels, one CTA per (sequence, head), 256 threads, the 128 x 128 fp32
// state in registers with the decode kernel's layout (warp w owns rows
// j = w, w+8, ...; lane l owns columns 4l..4l+3 of the S^T storage st[j][i]):
//   gdn_bwd_replay_kernel  runs the recurrence forward and streams every
//                          S_{t-1} (64 KB) and x_t to the workspace;
//   gdn_bwd_kernel         walks the tokens backwards with G in registers,
//                          S_{t-1} of the next token prefetched into shared
//                          memory with cp.async while the current one is used.
// This trades O(T d^2) workspace and HBM traffic for simplicity; the states
// could instead be recomputed per chunk from chunk-boundary states.
#include "bwd_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdWarps = kBwdThreads / 32;
constexpr int kRows = 128 / kBwdWarps;   // 16 rows of the state per warp

template <typename Elt>
__device__ __forceinline__ float ldf(const Elt *p);
template <>
__device__ __forceinline__ float ldf<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// Sums v[r] over the 32 lanes for 16 rows at once: at each butterfly step a
// lane keeps half of its rows and adds the partner's copy of them, so after
// 8 + 4 + 2 + 1 exchanges and a last one with lane ^ 1, lane L holds the sum
// for row L >> 1 (16 shuffles instead of 16 separate five-shuffle sums).
__device__ __forceinline__ float warp_rows16_sum(float (&v)[16], int lane) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool hi = lane & 16;
    const float keep = hi ? v[i + 8] : v[i], send = hi ? v[i] : v[i + 8];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool hi = lane & 8;
    const float keep = hi ? v[i + 4] : v[i], send = hi ? v[i] : v[i + 4];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool hi = lane & 4;
    const float keep = hi ? v[i + 2] : v[i], send = hi ? v[i] : v[i + 2];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  {
    const bool hi = lane & 2;
    const float keep = hi ? v[1] : v[0], send = hi ? v[0] : v[1];
    v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}

// Token range [t0, t1) of sequence n in the flattened B*T token axis. Returns
// false (and records the error) for cu_seqlens entries that leave that range.
__device__ __forceinline__ bool seq_range(const int32_t *cu, int n, int N, int B, int T, int &t0,
                                         int &t1, uint32_t *ctrl) {
  if (!cu) {
    t0 = n * T;
    t1 = t0 + T;
    return true;
  }
  t0 = cu[n];
  t1 = cu[n + 1];
  const bool ok = 0 <= t0 && t0 <= t1 && t1 <= B * T && (n > 0 || t0 == 0) &&
                  (n < N - 1 || t1 == B * T);
  if (!ok) atomicOr(ctrl, kErrBadSeqlens);
  return ok;
}

template <typename Elt>
__global__ void __launch_bounds__(kBwdThreads, 1) gdn_bwd_replay_kernel(
    const Elt *__restrict__ k, const Elt *__restrict__ v, const float *__restrict__ g,
    const float *__restrict__ beta, const float *__restrict__ s0, const int32_t *__restrict__ cu,
    int N, int B, int T, int H, int dk, int dv, float *__restrict__ s_prev,
    float *__restrict__ x_out, uint32_t *__restrict__ ctrl) {
  // ks alternates between two buffers by token parity: a thread may write the
  // next token's key while slower threads still read this one's in the update.
  __shared__ float ksb[2][128], us[128];
  __shared__ float xpart[kBwdWarps][128];
  const int n = blockIdx.x / H, h = blockIdx.x - n * H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int t0, t1;
  if (!seq_range(cu, n, N, B, T, t0, t1, ctrl)) return;
  const int col = 4 * lane;
  const bool col_ok = col < dv;
  const size_t SS = size_t(dk) * dv;

  float4 S[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int j = warp + r * kBwdWarps;
    S[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (s0 && col_ok && j < dk)
      S[r] = *reinterpret_cast<const float4 *>(s0 + (size_t(n) * H + h) * SS + size_t(j) * dv + col);
  }
  for (int t = t0; t < t1; ++t) {
    const size_t row = size_t(t) * H + h;
    float *dst = s_prev + row * SS;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int j = warp + r * kBwdWarps;
      if (col_ok && j < dk) __stcs(reinterpret_cast<float4 *>(dst + size_t(j) * dv + col), S[r]);
    }
    float *ks = ksb[(t - t0) & 1];
    if (tid < dk) ks[tid] = ldf(k + row * dk + tid);
    __syncthreads();
    float4 xp = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int j = warp + r * kBwdWarps;
      const float kj = j < dk ? ks[j] : 0.f;
      xp.x += S[r].x * kj; xp.y += S[r].y * kj; xp.z += S[r].z * kj; xp.w += S[r].w * kj;
    }
    if (col_ok) *reinterpret_cast<float4 *>(&xpart[warp][col]) = xp;
    __syncthreads();
    const float alpha = expf(g[row]), b = beta[row];
    if (tid < dv) {
      float x = 0.f;
#pragma unroll
      for (int w = 0; w < kBwdWarps; ++w) x += xpart[w][tid];
      x_out[row * dv + tid] = x;
      us[tid] = b * (ldf(v + row * dv + tid) - alpha * x);
    }
    __syncthreads();
    if (col_ok) {
      const float4 u4 = *reinterpret_cast<const float4 *>(&us[col]);
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const int j = warp + r * kBwdWarps;
        const float kj = j < dk ? ks[j] : 0.f;
        S[r].x = alpha * S[r].x + u4.x * kj;
        S[r].y = alpha * S[r].y + u4.y * kj;
        S[r].z = alpha * S[r].z + u4.z * kj;
        S[r].w = alpha * S[r].w + u4.w * kj;
      }
    }
    // us and xpart are rewritten at the next token only after its first
    // barrier, which every thread reaches after finishing this update.
  }
}

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void *gptr) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(gptr) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Shared memory of gdn_bwd_kernel: two 64 KB stages of S_{t-1} (rows of dv
// floats, the global layout), then the per-token vectors.
constexpr uint32_t kStage = 128 * 128 * 4;

template <typename Elt>
__global__ void __launch_bounds__(kBwdThreads, 1) gdn_bwd_kernel(
    const Elt *__restrict__ q, const Elt *__restrict__ k, const Elt *__restrict__ v,
    const float *__restrict__ g, const float *__restrict__ beta, const int32_t *__restrict__ cu,
    const Elt *__restrict__ d_o, const float *__restrict__ d_sN, int N, int B, int T, int H, int dk,
    int dv, const float *__restrict__ s_prev, const float *__restrict__ x_in,
    float *__restrict__ dq, float *__restrict__ dkk, float *__restrict__ dvv,
    float *__restrict__ dg, float *__restrict__ dbeta, float *__restrict__ ds0,
    uint32_t *__restrict__ ctrl) {
  extern __shared__ __align__(16) uint8_t smem[];
  float *stage = reinterpret_cast<float *>(smem);              // [2][128][128]
  float *ks = stage + 2 * 128 * 128, *qs = ks + 128, *dos = qs + 128, *us = dos + 128;
  float *xs = us + 128, *rs = xs + 128, *gks = rs + 128;
  float *gkpart = gks + 128;                                   // [kBwdWarps][128]
  float *red = gkpart + kBwdWarps * 128;                       // [3][kBwdWarps]
  const int n = blockIdx.x / H, h = blockIdx.x - n * H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int t0, t1;
  if (!seq_range(cu, n, N, B, T, t0, t1, ctrl)) return;
  const int col = 4 * lane;
  const bool col_ok = col < dv;
  const size_t SS = size_t(dk) * dv;

  float4 G[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int j = warp + r * kBwdWarps;
    G[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (d_sN && col_ok && j < dk)
      G[r] = *reinterpret_cast<const float4 *>(d_sN + (size_t(n) * H + h) * SS + size_t(j) * dv +
                                               col);
  }
  // Each thread copies exactly the 16-byte slots it later reads, so its own
  // cp.async completion is all the ordering it needs.
  auto prefetch = [&](int t, int buf) {
    const float *src = s_prev + (size_t(t) * H + h) * SS;
    float *dst = stage + buf * 128 * 128;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int j = warp + r * kBwdWarps;
      if (col_ok && j < dk)
        cp_async16(smem_u32(dst + j * 128 + col), src + size_t(j) * dv + col);
    }
    cp_async_commit();
  };
  if (t1 > t0) prefetch(t1 - 1, 0);
  int buf = 0;
  for (int t = t1 - 1; t >= t0; --t, buf ^= 1) {
    const size_t row = size_t(t) * H + h;
    const float alpha = expf(g[row]), b = beta[row];
    if (tid < dk) {
      ks[tid] = ldf(k + row * dk + tid);
      qs[tid] = ldf(q + row * dk + tid);
    }
    if (tid < dv) {
      const float x = x_in[row * dv + tid], r = ldf(v + row * dv + tid) - alpha * x;
      xs[tid] = x;
      rs[tid] = r;
      us[tid] = b * r;
      dos[tid] = ldf(d_o + row * dv + tid);
    }
    cp_async_wait_all();
    float4 S[kRows];
    const float *cur = stage + buf * 128 * 128;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int j = warp + r * kBwdWarps;
      S[r] = (col_ok && j < dk) ? *reinterpret_cast<const float4 *>(cur + j * 128 + col)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (t > t0) prefetch(t - 1, buf ^ 1);
    __syncthreads();                                           // (A) token vectors ready
    const float4 do4 = col_ok ? *reinterpret_cast<const float4 *>(&dos[col])
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 u4 = col_ok ? *reinterpret_cast<const float4 *>(&us[col])
                             : make_float4(0.f, 0.f, 0.f, 0.f);
    const float udo = warp_sum(dot4(u4, do4));                 // u . do (a warp spans all columns)
    float4 gk = make_float4(0.f, 0.f, 0.f, 0.f);
    float gs = 0.f;
    float part[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int j = warp + r * kBwdWarps;
      const float kj = j < dk ? ks[j] : 0.f, qj = j < dk ? qs[j] : 0.f;
      // G += do q^T
      G[r].x += do4.x * qj; G[r].y += do4.y * qj; G[r].z += do4.z * qj; G[r].w += do4.w * qj;
      gk.x += G[r].x * kj; gk.y += G[r].y * kj; gk.z += G[r].z * kj; gk.w += G[r].w * kj;
      gs += dot4(G[r], S[r]);
      part[r] = dot4(S[r], do4);                               // (S_{t-1}^T do)_j, this lane's columns
    }
    {  // dq_j = alpha (S_{t-1}^T do)_j + k_j (u . do); lanes 2m, 2m+1 hold row j = warp + 8m
      const float sdo = warp_rows16_sum(part, lane);
      const int j = warp + kBwdWarps * (lane >> 1);
      if ((lane & 1) == 0 && j < dk) dq[row * dk + j] = alpha * sdo + ks[j] * udo;
    }
    if (col_ok) *reinterpret_cast<float4 *>(&gkpart[warp * 128 + col]) = gk;
    gs = warp_sum(gs);
    if (lane == 0) red[warp] = gs;
    __syncthreads();                                           // (B) partials of G k
    if (warp < 4) {   // threads 0-127 own one column i of d_v <= 128 each
      const int i = tid;
      float s = 0.f;
      if (i < dv) {
#pragma unroll
        for (int w = 0; w < kBwdWarps; ++w) s += gkpart[w * 128 + i];
        gks[i] = s;
        dvv[row * dv + i] = b * s;
      }
      const float db = warp_sum(i < dv ? s * rs[i] : 0.f);
      const float gx = warp_sum(i < dv ? s * xs[i] : 0.f);
      if (lane == 0) {
        red[kBwdWarps + warp] = db;
        red[2 * kBwdWarps + warp] = gx;
      }
    }
    __syncthreads();                                           // (C) G k and the sums
    if (tid == 0) {
      float gsum = 0.f, db = 0.f, gx = 0.f;
#pragma unroll
      for (int w = 0; w < kBwdWarps; ++w) gsum += red[w];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        db += red[kBwdWarps + w];
        gx += red[2 * kBwdWarps + w];
      }
      dbeta[row] = db;
      dg[row] = alpha * (gsum - b * gx);
    }
    const float4 gk4 = col_ok ? *reinterpret_cast<const float4 *>(&gks[col])
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    const float ab = alpha * b;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int j = warp + r * kBwdWarps;
      const float kj = j < dk ? ks[j] : 0.f;
      // dk_j = (G^T u)_j - alpha beta (S_{t-1}^T Gk)_j, this lane's columns
      part[r] = dot4(G[r], u4) - ab * dot4(S[r], gk4);
      // G <- alpha (G - beta Gk k^T)
      G[r].x = alpha * (G[r].x - b * gk4.x * kj);
      G[r].y = alpha * (G[r].y - b * gk4.y * kj);
      G[r].z = alpha * (G[r].z - b * gk4.z * kj);
      G[r].w = alpha * (G[r].w - b * gk4.w * kj);
    }
    {
      const float d = warp_rows16_sum(part, lane);
      const int j = warp + kBwdWarps * (lane >> 1);
      if ((lane & 1) == 0 && j < dk) dkk[row * dk + j] = d;
    }
    __syncthreads();                                           // (D) vectors free for t - 1
  }
  cp_async_wait_all();
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int j = warp + r * kBwdWarps;
    if (col_ok && j < dk)
      *reinterpret_cast<float4 *>(ds0 + (size_t(n) * H + h) * SS + size_t(j) * dv + col) = G[r];
  }
}

constexpr size_t kBwdSmem = 2 * size_t(kStage) + (7 * 128 + kBwdWarps * 128 + 3 * kBwdWarps) * 4;

template <typename Elt>
cudaError_t launch_bwd_t(const void *q, const void *k, const void *v, const float *g,
                         const float *beta, const float *s0, const int32_t *cu, const void *d_o,
                         const float *d_sN, int N, int B, int T, int H, int dk, int dv,
                         float *dq, float *dkk, float *dvv, float *dg, float *dbeta, float *ds0,
                         void *ws, const BwdLayout &L, cudaStream_t s) {
  char *base = static_cast<char *>(ws);
  uint32_t *ctrl = reinterpret_cast<uint32_t *>(base);
  float *sp = reinterpret_cast<float *>(base + L.s_prev);
  float *xo = reinterpret_cast<float *>(base + L.x);
  const unsigned units = unsigned(N) * unsigned(H);
  gdn_bwd_replay_kernel<Elt><<<units, kBwdThreads, 0, s>>>(
      static_cast<const Elt *>(k), static_cast<const Elt *>(v), g, beta, s0, cu, N, B, T, H, dk, dv,
      sp, xo, ctrl);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  auto kern = gdn_bwd_kernel<Elt>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kBwdSmem));
  if (e != cudaSuccess) return e;
  kern<<<units, kBwdThreads, kBwdSmem, s>>>(
      static_cast<const Elt *>(q), static_cast<const Elt *>(k), static_cast<const Elt *>(v), g, beta,
      cu, static_cast<const Elt *>(d_o), d_sN, N, B, T, H, dk, dv, sp, xo, dq, dkk, dvv, dg, dbeta,
      ds0, ctrl);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd(const void *q, const void *k, const void *v, const float *g,
                       const float *beta, const float *s0, const int32_t *cu, const void *d_o,
                       const float *d_sN, int N, int B, int T, int H, int dk, int dv, int dtype,
                       float *dq, float *dkk, float *dvv, float *dg, float *dbeta, float *ds0,
                       void *ws, const BwdLayout &L, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, s);   // control block: error word
  if (e != cudaSuccess) return e;
  if (dtype == GDN_BF16)
    return launch_bwd_t<__nv_bfloat16>(q, k, v, g, beta, s0, cu, d_o, d_sN, N, B, T, H, dk, dv,
                                       dq, dkk, dvv, dg, dbeta, ds0, ws, L, s);
  return launch_bwd_t<float>(q, k, v, g, beta, s0, cu, d_o, d_sN, N, B, T, H, dk, dv, dq, dkk,
                             dvv, dg, dbeta, ds0, ws, L, s);
}

}  // namespace gdn
