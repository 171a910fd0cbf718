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
// Every d_v row of S evolves on its own (S_i <- alpha S_i + u_i k^T, u_i
// depends on S_i only), and so does every d_v column of G. Both kernels
// therefore give each warp 16 d_v columns and all 128 d_k rows of the state
// (S^T storage st[j][i]: lane l owns rows 4l..4l+3, 64 fp32 registers), so
// every reduction over d_k stays inside a warp:
//   gdn_bwd_replay_kernel  runs the recurrence forward and streams every
//                          S_{t-1} (64 KB, in the warps' own slot order) and
//                          x_t to the workspace; no barrier at all, the warps
//                          never wait on each other, so a (sequence, head)
//                          runs as two CTAs of 4 warps;
//   gdn_bwd_kernel         walks the tokens backwards with G in registers,
//                          S_{t-1} of the next token prefetched into shared
//                          memory with cp.async and the next token's vectors
//                          staged by the whole CTA; one barrier per token,
//                          where the 8 warps' partial dq, dk, dbeta and dg
//                          (sums over their columns) are added up.
// This trades O(T d^2) workspace and HBM traffic for simplicity; the states
// could instead be recomputed per chunk from chunk-boundary states.
#include "bwd_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdWarps = kBwdThreads / 32;
constexpr int kCols = 16;   // d_v columns per warp (8 warps x 16 = 128)
// The replay's warps never wait on each other, so each (sequence, head) runs
// as two CTAs of 4 warps (64 columns each): twice the SMs streaming states.
constexpr int kReplayWarps = 4;

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

// Sums v[c] over the 32 lanes for 16 columns at once: at each butterfly step a
// lane keeps half of its columns and adds the partner's copy of them, so after
// 8 + 4 + 2 + 1 exchanges and a last one with lane ^ 1, lane L holds the sum
// for column L >> 1 (16 shuffles instead of 16 separate five-shuffle sums).
__device__ __forceinline__ float warp_cols16_sum(float (&v)[16], int lane) {
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

// The lane's 4 x 16 block of a [d_k][d_v] fp32 state (rows j0.., columns c0..)
// to and from registers; entries outside d_k x d_v read as zero and are not
// written (d_v is a multiple of 4).
__device__ __forceinline__ void load_block(float (&X)[4][kCols], const float *src, int j0, int c0,
                                           int dk, int dv) {
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + a < dk && c0 + 4 * m < dv)
        x = *reinterpret_cast<const float4 *>(src + size_t(j0 + a) * dv + c0 + 4 * m);
      X[a][4 * m] = x.x; X[a][4 * m + 1] = x.y; X[a][4 * m + 2] = x.z; X[a][4 * m + 3] = x.w;
    }
}

// Position of a lane's float4 (column group w, row a of the lane, float4 m of
// the warp's 16 columns) inside one token's 128 x 128 block of the workspace.
// Consecutive lanes hold consecutive 16-byte slots, so every warp-wide store
// or load of S_{t-1} moves 512 contiguous bytes.
__device__ __forceinline__ int slot(int w, int a, int m, int lane) {
  return (((w * 4 + a) * 4 + m) * 32 + lane) * 4;
}
constexpr int kBlockWords = 128 * 128;   // one token's S_{t-1} in the workspace

template <bool kStreaming>
__device__ __forceinline__ void store_block(const float (&X)[4][kCols], float *dst, int j0, int c0,
                                            int dk, int dv) {
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int m = 0; m < 4; ++m)
      if (j0 + a < dk && c0 + 4 * m < dv) {
        const float4 x = make_float4(X[a][4 * m], X[a][4 * m + 1], X[a][4 * m + 2],
                                     X[a][4 * m + 3]);
        float4 *p = reinterpret_cast<float4 *>(dst + size_t(j0 + a) * dv + c0 + 4 * m);
        if (kStreaming) __stcs(p, x);
        else *p = x;
      }
}

template <typename Elt>
__global__ void __launch_bounds__(kReplayWarps * 32) gdn_bwd_replay_kernel(
    const Elt *__restrict__ k, const Elt *__restrict__ v, const float *__restrict__ g,
    const float *__restrict__ beta, const float *__restrict__ s0, const int32_t *__restrict__ cu,
    int N, int B, int T, int H, int dk, int dv, float *__restrict__ s_prev,
    float *__restrict__ x_out, uint32_t *__restrict__ ctrl) {
  const int n = blockIdx.x / H, h = blockIdx.x - n * H;
  const int lane = threadIdx.x & 31;
  const int warp = blockIdx.y * kReplayWarps + (threadIdx.x >> 5);   // column group 0..7
  int t0, t1;
  if (!seq_range(cu, n, N, B, T, t0, t1, ctrl)) return;
  const int c0 = warp * kCols, j0 = 4 * lane, cc = lane >> 1;
  if (c0 >= dv) return;   // this kernel has no barrier: an idle warp may leave
  const size_t SS = size_t(dk) * dv;
  const bool col_ok = c0 + cc < dv;

  float S[4][kCols];
  if (s0) load_block(S, s0 + (size_t(n) * H + h) * SS, j0, c0, dk, dv);
  else
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < kCols; ++c) S[a][c] = 0.f;

  // this lane's inputs of one token: k at its 4 rows, v at column c0 + (lane >> 1)
  float kn[4], vn = 0.f, an = 0.f, bn = 0.f;
  auto fetch = [&](int t) {
    const size_t row = size_t(t) * H + h;
#pragma unroll
    for (int a = 0; a < 4; ++a) kn[a] = j0 + a < dk ? ldf(k + row * dk + j0 + a) : 0.f;
    vn = col_ok ? ldf(v + row * dv + c0 + cc) : 0.f;
    an = g[row];
    bn = beta[row];
  };
  if (t1 > t0) fetch(t0);
  for (int t = t0; t < t1; ++t) {
    const size_t row = size_t(t) * H + h;
    float kt[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) kt[a] = kn[a];
    const float vt = vn, alpha = expf(an), b = bn;
    if (t + 1 < t1) fetch(t + 1);   // the next token's loads overlap this one
    {
      float *dst = s_prev + row * kBlockWords;
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int m = 0; m < 4; ++m)
          if (j0 + a < dk && c0 + 4 * m < dv)
            __stcs(reinterpret_cast<float4 *>(dst + slot(warp, a, m, lane)),
                   make_float4(S[a][4 * m], S[a][4 * m + 1], S[a][4 * m + 2], S[a][4 * m + 3]));
    }
    float xp[kCols];
#pragma unroll
    for (int c = 0; c < kCols; ++c)
      xp[c] = S[0][c] * kt[0] + S[1][c] * kt[1] + S[2][c] * kt[2] + S[3][c] * kt[3];
    const float x = warp_cols16_sum(xp, lane);   // x at column c0 + (lane >> 1)
    if ((lane & 1) == 0 && col_ok) x_out[row * dv + c0 + cc] = x;
    const float uc = b * (vt - alpha * x);
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      const float u = __shfl_sync(0xffffffffu, uc, 2 * c);
#pragma unroll
      for (int a = 0; a < 4; ++a) S[a][c] = alpha * S[a][c] + u * kt[a];
    }
  }
}

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void *gptr) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(gptr) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Shared memory of gdn_bwd_kernel (fp32 words): two 64 KB stages of S_{t-1}
// (rows of 128), then per token parity the staged vectors k, q, d_o, x, u, r
// (128 each) and alpha, beta; the warps' partial dq and dk ([8][128] each);
// and their partial dbeta, gx = Gk . x and <G, S_{t-1}> ([8][4]).
constexpr int kStageWords = 128 * 128;
constexpr int kVecWords = 6 * 128 + 2;
constexpr int kPartWords = 2 * kBwdWarps * 128;
constexpr int kRedWords = kBwdWarps * 4;
constexpr size_t kBwdSmem =
    size_t(2 * kStageWords + 2 * kVecWords + 2 * kPartWords + 2 * kRedWords) * 4;

template <typename Elt>
__global__ void __launch_bounds__(kBwdThreads, 1) gdn_bwd_kernel(
    const Elt *__restrict__ q, const Elt *__restrict__ k, const Elt *__restrict__ v,
    const float *__restrict__ g, const float *__restrict__ beta, const int32_t *__restrict__ cu,
    const Elt *__restrict__ d_o, const float *__restrict__ d_sN, int N, int B, int T, int H, int dk,
    int dv, const float *__restrict__ s_prev, const float *__restrict__ x_in,
    float *__restrict__ dq, float *__restrict__ dkk, float *__restrict__ dvv,
    float *__restrict__ dg, float *__restrict__ dbeta, float *__restrict__ ds0,
    uint32_t *__restrict__ ctrl) {
  extern __shared__ __align__(16) float smf[];
  float *stage = smf;                                  // [2][128][128]
  float *vec = stage + 2 * kStageWords;                // [2][kVecWords]
  float *part = vec + 2 * kVecWords;                   // [2][2][8][128]
  float *red = part + 2 * kPartWords;                  // [2][8][4]
  const int n = blockIdx.x / H, h = blockIdx.x - n * H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int t0, t1;
  if (!seq_range(cu, n, N, B, T, t0, t1, ctrl)) return;   // uniform over the CTA
  const int c0 = warp * kCols, j0 = 4 * lane, cc = lane >> 1;
  const size_t SS = size_t(dk) * dv;

  // Warps without columns (d_v < 128) contribute zero partials.
  for (int e = tid; e < 2 * kPartWords + 2 * kRedWords; e += kBwdThreads) part[e] = 0.f;

  float G[4][kCols];
  if (d_sN) load_block(G, d_sN + (size_t(n) * H + h) * SS, j0, c0, dk, dv);
  else
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < kCols; ++c) G[a][c] = 0.f;

  auto prefetch_state = [&](int t, int buf) {
    const float *src = s_prev + (size_t(t) * H + h) * kBlockWords;
    float *dst = stage + buf * kStageWords;
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int m = 0; m < 4; ++m)
        if (j0 + a < dk && c0 + 4 * m < dv) {
          const int o = slot(warp, a, m, lane);
          cp_async16(smem_u32(dst + o), src + o);
        }
    cp_async_commit();
  };
  // Staging of one token's vectors: thread tid < 128 owns index tid of k and q,
  // thread 128 + i owns column i of d_o, x, u and r; thread 0 also alpha, beta.
  float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f, ra = 0.f, rb = 0.f;
  auto fetch_vec = [&](int t) {
    const size_t row = size_t(t) * H + h;
    if (tid < 128) {
      r0 = tid < dk ? ldf(k + row * dk + tid) : 0.f;
      r1 = tid < dk ? ldf(q + row * dk + tid) : 0.f;
    } else {
      const int i = tid - 128;
      r0 = i < dv ? ldf(d_o + row * dv + i) : 0.f;
      r1 = i < dv ? x_in[row * dv + i] : 0.f;
      r2 = i < dv ? ldf(v + row * dv + i) : 0.f;
    }
    ra = g[row];
    rb = beta[row];
  };
  auto put_vec = [&](int buf) {
    float *V = vec + buf * kVecWords;
    const float alpha = expf(ra);
    if (tid < 128) {
      V[tid] = r0;                 // k
      V[128 + tid] = r1;           // q
    } else {
      const int i = tid - 128;
      const float r = r2 - alpha * r1;
      V[256 + i] = r0;             // d_o
      V[384 + i] = r1;             // x
      V[512 + i] = rb * r;         // u = beta (v - alpha x)
      V[640 + i] = r;              // r = v - alpha x
    }
    if (tid == 0) {
      V[768] = alpha;
      V[769] = rb;
    }
    (void)r3;
  };

  if (t1 > t0) {
    prefetch_state(t1 - 1, 0);
    fetch_vec(t1 - 1);
    put_vec(0);
  }
  __syncthreads();
  int p = 0;
  for (int t = t1 - 1; t >= t0; --t, p ^= 1) {
    const size_t row = size_t(t) * H + h;
    if (t > t0) fetch_vec(t - 1);                      // lands while this token computes
    cp_async_wait_all();
    float S[4][kCols];
    {
      const float *cur = stage + p * kStageWords;
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
          if (j0 + a < dk && c0 + 4 * m < dv)
            x = *reinterpret_cast<const float4 *>(cur + slot(warp, a, m, lane));
          S[a][4 * m] = x.x; S[a][4 * m + 1] = x.y; S[a][4 * m + 2] = x.z; S[a][4 * m + 3] = x.w;
        }
    }
    if (t > t0) prefetch_state(t - 1, p ^ 1);
    const float *V = vec + p * kVecWords;
    const float alpha = V[768], b = V[769], ab = alpha * b;
    float kt[4], qt[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      kt[a] = V[j0 + a];
      qt[a] = V[128 + j0 + a];
    }
    // G += d_o q^T; partial G k, <G, S_{t-1}>, S_{t-1}^T d_o and u . d_o over this warp's columns
    float gkp[kCols], dqp[4] = {0.f, 0.f, 0.f, 0.f}, gsp = 0.f, udo = 0.f;
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      const float d = V[256 + c0 + c], u = V[512 + c0 + c];
      udo += u * d;
      float acc = 0.f;
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        G[a][c] += d * qt[a];
        acc += G[a][c] * kt[a];
        gsp += G[a][c] * S[a][c];
        dqp[a] += S[a][c] * d;
      }
      gkp[c] = acc;
    }
    const float gk_own = warp_cols16_sum(gkp, lane);   // Gk at column c0 + (lane >> 1)
    if ((lane & 1) == 0 && c0 + cc < dv) dvv[row * dv + c0 + cc] = b * gk_own;
    gsp = warp_sum(gsp);
    float* P = part + p * kPartWords;
    {
      // dq_j partial = alpha (S_{t-1}^T d_o)_j + k_j (u . d_o), over this warp's columns
      const float4 w4 = make_float4(alpha * dqp[0] + kt[0] * udo, alpha * dqp[1] + kt[1] * udo,
                                    alpha * dqp[2] + kt[2] * udo, alpha * dqp[3] + kt[3] * udo);
      *reinterpret_cast<float4 *>(P + warp * 128 + j0) = w4;
    }
    float dkp[4] = {0.f, 0.f, 0.f, 0.f}, dbp = 0.f, gxp = 0.f;
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      const float gk = __shfl_sync(0xffffffffu, gk_own, 2 * c);
      const float u = V[512 + c0 + c];
      dbp += gk * V[640 + c0 + c];
      gxp += gk * V[384 + c0 + c];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        // dk_j partial = (G^T u)_j - alpha beta (S_{t-1}^T Gk)_j
        dkp[a] += G[a][c] * u - ab * S[a][c] * gk;
        // G <- alpha (G - beta Gk k^T)
        G[a][c] = alpha * (G[a][c] - b * gk * kt[a]);
      }
    }
    *reinterpret_cast<float4 *>(P + kBwdWarps * 128 + warp * 128 + j0) =
        make_float4(dkp[0], dkp[1], dkp[2], dkp[3]);
    float *R = red + p * kRedWords;
    if (lane == 0) {
      R[warp * 4 + 0] = dbp;   // identical on every lane: sums over the warp's columns
      R[warp * 4 + 1] = gxp;
      R[warp * 4 + 2] = gsp;
    }
    if (t > t0) put_vec(p ^ 1);
    __syncthreads();   // partials of token t and the vectors of token t - 1 are in place
    if (tid < 128) {
      if (tid < dk) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kBwdWarps; ++w) s += P[w * 128 + tid];
        dq[row * dk + tid] = s;
      }
    } else if (tid - 128 < dk) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kBwdWarps; ++w) s += P[kBwdWarps * 128 + w * 128 + tid - 128];
      dkk[row * dk + tid - 128] = s;
    }
    if (tid == 0) {
      float db = 0.f, gx = 0.f, gs = 0.f;
#pragma unroll
      for (int w = 0; w < kBwdWarps; ++w) {
        db += R[w * 4 + 0];
        gx += R[w * 4 + 1];
        gs += R[w * 4 + 2];
      }
      dbeta[row] = db;
      dg[row] = alpha * (gs - b * gx);
    }
  }
  cp_async_wait_all();
  store_block<false>(G, ds0 + (size_t(n) * H + h) * SS, j0, c0, dk, dv);
}

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
  const dim3 rgrid(units, (dv + kReplayWarps * kCols - 1) / (kReplayWarps * kCols));
  gdn_bwd_replay_kernel<Elt><<<rgrid, kReplayWarps * 32, 0, s>>>(
      static_cast<const Elt *>(k), static_cast<const Elt *>(v), g, beta, s0, cu, N, B, T, H, dk,
      dv, sp, xo, ctrl);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  auto kern = gdn_bwd_kernel<Elt>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kBwdSmem));
  if (e != cudaSuccess) return e;
  kern<<<units, kBwdThreads, kBwdSmem, s>>>(
      static_cast<const Elt *>(q), static_cast<const Elt *>(k), static_cast<const Elt *>(v), g,
      beta, cu, static_cast<const Elt *>(d_o), d_sN, N, B, T, H, dk, dv, sp, xo, dq, dkk, dvv, dg,
      dbeta, ds0, ctrl);
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
