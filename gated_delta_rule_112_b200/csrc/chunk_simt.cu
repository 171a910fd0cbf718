// The fp32 CUDA-core implementation of the chunkwise WY / UT-transform forward pass
// ("Gated Delta Networks", phantomic12 page, mechanism paragraph; LIT-137,
// "Standing in the anthology": the WY-based chunkwise algorithm extended to
// carry the gate). This path serves fp32 inputs (where fp32 accuracy is
// required end to end) and head sizes the tensor-core path does not cover.
//
// Per chunk (rows r, s < C; Gamma = inclusive cumsum of g inside the chunk):
//   A_rs = beta_r exp(Gamma_r - Gamma_s) k_r.k_s  (s < r)     T = (I + A)^-1
//   W = T diag(beta exp(Gamma)) K        U = T diag(beta) V     V_new = U - W S^T
//   O = diag(exp(Gamma)) Q S^T + (Q K^T .* M) V_new,  M_rs = exp(Gamma_r - Gamma_s), s <= r
//   S <- exp(Gamma_last) S + V_new^T diag(exp(Gamma_last - Gamma)) K
// Rows past a sequence's end are treated as k = q = v = 0, beta = g = 0,
// which leaves S unchanged; their outputs are not written.
//
// Channel-wise gate (the Kimi Delta Attention variant: dmarx anthology
// LIT-137, "Standing in the anthology"; SOTA-135, "Sequence"), g = log alpha
// per (token, head, d_k channel), S_t = S_{t-1} diag(alpha_t)(I - beta_t k_t
// k_t^T) + beta_t v_t k_t^T. Gamma is then a cumsum per channel and the decay
// moves inside the dot products:
//   A_rs = beta_r sum_j k_rj k_sj exp(Gamma_rj - Gamma_sj)  (s < r)
//   P_rs = sum_j q_rj k_sj exp(Gamma_rj - Gamma_sj)         (s <= r)
//   W = T diag(beta) (K .* exp(Gamma)),  O = (Q .* exp(Gamma)) S^T + P V_new
//   S <- S diag(exp(Gamma_last)) + V_new^T (K .* exp(Gamma_last - Gamma))
// Every exponent is a difference of cumulative sums over the tokens in
// between, so with alpha <= 1 no factor exceeds 1.
#include "gdn_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

template <typename T>
__device__ __forceinline__ float ld_f32(const T *p);
template <>
__device__ __forceinline__ float ld_f32<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ld_f32<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}
template <typename T>
__device__ __forceinline__ void st_from_f32(T *p, float x);
template <>
__device__ __forceinline__ void st_from_f32<float>(float *p, float x) { *p = x; }
template <>
__device__ __forceinline__ void st_from_f32<__nv_bfloat16>(__nv_bfloat16 *p, float x) {
  *p = __float2bfloat16_rn(x);
}

constexpr int kSimtThreads = 256;
constexpr int kDvt = 32;  // d_v columns per CTA
// The channel-wise gate runs with 16 warps: its CTA (219 KB of shared
// memory) is alone on its SM, and the extra warps hide the latency of the
// per-channel exponentials.
template <bool KDA>
constexpr int simt_threads() { return KDA ? 512 : kSimtThreads; }

// 2^x on the special-function unit (PTX ex2.approx, flush-to-zero).
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// fp32 chunked forward. Grid (N, H, ceil(d_v / 32)); one CTA walks all chunks
// of one sequence for one head and one 32-column slice of d_v, carrying its
// slice of the state in shared memory. KDA: channel-wise gate (g [rows, H, d_k]).
template <int C, typename T, bool KDA>
__global__ void __launch_bounds__(simt_threads<KDA>()) gdn_chunk_simt_kernel(
    const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
    const float *__restrict__ g, const float *__restrict__ beta, const float *__restrict__ s0,
    int H, int dk, int dv, T *__restrict__ o, float *__restrict__ sN,
    const uint32_t *__restrict__ ctrl, const ChunkInfo *__restrict__ table,
    const int32_t *__restrict__ seq_first) {
  extern __shared__ float sm[];
  constexpr int kThr = simt_threads<KDA>();
  if (ctrl[0] & kErrBadSeqlens) return;
  const int n = blockIdx.x, h = blockIdx.y, i0 = blockIdx.z * kDvt;
  const int tid = threadIdx.x;
  const int dkp = dk + 1;
  float *Ks = sm;                        // [C][dkp]
  float *Qs = Ks + C * dkp;              // [C][dkp]
  float *Ws = Qs + C * dkp;              // [C][dkp]
  float *Vs = Ws + C * dkp;              // [C][kDvt]
  float *Us = Vs + C * kDvt;             // [C][kDvt]
  float *Vn = Us + C * kDvt;             // [C][kDvt]
  float *Ss = Vn + C * kDvt;             // [dk][kDvt]  S^T slice: Ss[j][i'] = S[i0+i'][j]
  float *As = Ss + dk * kDvt;            // [C][C+1]
  float *Ts = As + C * (C + 1);          // [C][C+1]
  float *Ps = Ts + C * (C + 1);          // [C][C+1]
  float *Gm = Ps + C * (C + 1);          // [C] Gamma
  float *Bt = Gm + C;                    // [C] beta
  float *Ga = Bt + C;                    // [C] exp(Gamma)
  float *Dd = Ga + C;                    // [C] exp(Gamma_last - Gamma)
  // KDA only: per-channel Gamma log2(e), then K .* exp(Gamma); and Gamma_last
  // log2(e) per channel (exponentials as 2^x on the special-function unit)
  float *Gk = Dd + C;                    // [C][dkp]
  float *Gl = Gk + C * dkp;              // [dk]

  // Initial state slice.
  for (int e = tid; e < dk * kDvt; e += kThr) {
    const int j = e / kDvt, ii = e % kDvt;
    float x = 0.f;
    if (s0 && i0 + ii < dv) x = s0[((size_t(n) * H + h) * dk + j) * dv + i0 + ii];
    Ss[e] = x;
  }
  const int c_begin = seq_first[n], c_end = seq_first[n + 1];
  for (int cg = c_begin; cg < c_end; ++cg) {
    const ChunkInfo ci = table[cg];
    const int L = ci.len;
    __syncthreads();
    // 1. load the chunk (rows >= L as zeros)
    for (int e = tid; e < C * dk; e += kThr) {
      const int r = e / dk, j = e % dk;
      float kv = 0.f, qv = 0.f;
      if (r < L) {
        const size_t off = (size_t(ci.row0 + r) * H + h) * dk + j;
        kv = ld_f32(k + off);
        qv = ld_f32(q + off);
      }
      Ks[r * dkp + j] = kv;
      Qs[r * dkp + j] = qv;
    }
    for (int e = tid; e < C * kDvt; e += kThr) {
      const int r = e / kDvt, ii = e % kDvt;
      float vv = 0.f;
      if (r < L && i0 + ii < dv) vv = ld_f32(v + (size_t(ci.row0 + r) * H + h) * dv + i0 + ii);
      Vs[e] = vv;
    }
    if (tid < C) {
      const bool ok = tid < L;
      if (!KDA) Gm[tid] = ok ? g[size_t(ci.row0 + tid) * H + h] : 0.f;
      Bt[tid] = ok ? beta[size_t(ci.row0 + tid) * H + h] : 0.f;
    }
    if (KDA) {
      for (int e = tid; e < C * dk; e += kThr) {
        const int r = e / dk, j = e % dk;
        Gk[r * dkp + j] = r < L ? g[(size_t(ci.row0 + r) * H + h) * dk + j] : 0.f;
      }
    }
    __syncthreads();
    // 2. cumulative log-gate and the decay factors
    if (!KDA && tid == 0) {
      float acc = 0.f;
      for (int r = 0; r < C; ++r) { acc += Gm[r]; Gm[r] = acc; }
    }
    if (KDA && tid < dk) {   // one channel per thread
      constexpr float kLog2e = 1.4426950408889634f;
      float acc = 0.f;
      for (int r = 0; r < C; ++r) { acc += Gk[r * dkp + tid]; Gk[r * dkp + tid] = acc * kLog2e; }
      Gl[tid] = acc * kLog2e;
    }
    __syncthreads();
    if (!KDA && tid < C) {
      Ga[tid] = expf(Gm[tid]);
      Dd[tid] = expf(Gm[C - 1] - Gm[tid]);
    }
    // 3. A (strictly lower) and P = (Q K^T) .* M (diagonal included)
    if (KDA) {
      // One thread per 2 x 2 block of (r, s) pairs: every loaded row element is
      // used twice. Pair (r0, s1) of a diagonal block lies above the diagonal
      // and is skipped before its exponent is formed (it could overflow).
      constexpr int Cb = C / 2;
      for (int e = tid; e < Cb * Cb; e += kThr) {
        const int R = e / Cb, Sb = e % Cb;
        const int r0 = 2 * R, r1 = r0 + 1, s0 = 2 * Sb, s1 = s0 + 1;
        float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
        float p00 = 0.f, p01 = 0.f, p10 = 0.f, p11 = 0.f;
        if (Sb <= R) {
          const bool v01 = s1 <= r0;
          for (int j = 0; j < dk; ++j) {
            const float gr0 = Gk[r0 * dkp + j], gr1 = Gk[r1 * dkp + j];
            const float gs0 = Gk[s0 * dkp + j], gs1 = Gk[s1 * dkp + j];
            const float ks0 = Ks[s0 * dkp + j], ks1 = Ks[s1 * dkp + j];
            const float kr0 = Ks[r0 * dkp + j], kr1 = Ks[r1 * dkp + j];
            const float qr0 = Qs[r0 * dkp + j], qr1 = Qs[r1 * dkp + j];
            const float e00 = ks0 * ex2_fast(gr0 - gs0);
            const float e01 = v01 ? ks1 * ex2_fast(gr0 - gs1) : 0.f;
            const float e10 = ks0 * ex2_fast(gr1 - gs0);
            const float e11 = ks1 * ex2_fast(gr1 - gs1);
            a00 += kr0 * e00; p00 += qr0 * e00;
            a01 += kr0 * e01; p01 += qr0 * e01;
            a10 += kr1 * e10; p10 += qr1 * e10;
            a11 += kr1 * e11; p11 += qr1 * e11;
          }
        }
        As[r0 * (C + 1) + s0] = s0 < r0 ? Bt[r0] * a00 : 0.f;
        As[r0 * (C + 1) + s1] = s1 < r0 ? Bt[r0] * a01 : 0.f;
        As[r1 * (C + 1) + s0] = s0 < r1 ? Bt[r1] * a10 : 0.f;
        As[r1 * (C + 1) + s1] = s1 < r1 ? Bt[r1] * a11 : 0.f;
        Ps[r0 * (C + 1) + s0] = s0 <= r0 ? p00 : 0.f;
        Ps[r0 * (C + 1) + s1] = s1 <= r0 ? p01 : 0.f;
        Ps[r1 * (C + 1) + s0] = s0 <= r1 ? p10 : 0.f;
        Ps[r1 * (C + 1) + s1] = s1 <= r1 ? p11 : 0.f;
      }
    }
    for (int e = tid; !KDA && e < C * C; e += kThr) {
      const int r = e / C, s = e % C;
      float a = 0.f, p = 0.f;
      if (s <= r) {
        float dkk = 0.f, dqk = 0.f;
        {
          for (int j = 0; j < dk; ++j) {
            const float ksj = Ks[s * dkp + j];
            dkk += Ks[r * dkp + j] * ksj;
            dqk += Qs[r * dkp + j] * ksj;
          }
          const float decay = expf(Gm[r] - Gm[s]);
          if (s < r) a = Bt[r] * decay * dkk;
          p = decay * dqk;
        }
      }
      As[r * (C + 1) + s] = a;
      Ps[r * (C + 1) + s] = p;
    }
    __syncthreads();
    if (KDA) {
      // K and Q now enter only with their decays: Gk <- K .* exp(Gamma) (for W),
      // Ks <- K .* exp(Gamma_last - Gamma) (state update), Qs <- Q .* exp(Gamma).
      for (int e = tid; e < C * dk; e += kThr) {
        const int r = e / dk, j = e % dk;
        const float gam = Gk[r * dkp + j], kv = Ks[r * dkp + j], eg = ex2_fast(gam);
        Gk[r * dkp + j] = kv * eg;
        Ks[r * dkp + j] = kv * ex2_fast(Gl[j] - gam);
        Qs[r * dkp + j] *= eg;
      }
    }
    // 4. T = (I + A)^-1 by forward substitution; thread s owns column s.
    if (tid < C) {
      const int s = tid;
      for (int r = 0; r < C; ++r) Ts[r * (C + 1) + s] = (r == s) ? 1.f : 0.f;
      for (int r = s + 1; r < C; ++r) {
        float acc = 0.f;
        for (int m = s; m < r; ++m) acc += As[r * (C + 1) + m] * Ts[m * (C + 1) + s];
        Ts[r * (C + 1) + s] = -acc;
      }
    }
    __syncthreads();
    // 5. W = T diag(beta gamma) K, U = T diag(beta) V
    for (int e = tid; e < C * dk; e += kThr) {
      const int r = e / dk, j = e % dk;
      float acc = 0.f;
      if (KDA)
        for (int s = 0; s <= r; ++s) acc += Ts[r * (C + 1) + s] * Bt[s] * Gk[s * dkp + j];
      else
        for (int s = 0; s <= r; ++s)
          acc += Ts[r * (C + 1) + s] * (Bt[s] * Ga[s]) * Ks[s * dkp + j];
      Ws[r * dkp + j] = acc;
    }
    for (int e = tid; e < C * kDvt; e += kThr) {
      const int r = e / kDvt, ii = e % kDvt;
      float acc = 0.f;
      for (int s = 0; s <= r; ++s) acc += Ts[r * (C + 1) + s] * Bt[s] * Vs[s * kDvt + ii];
      Us[e] = acc;
    }
    __syncthreads();
    // 6. V_new = U - W S^T
    for (int e = tid; e < C * kDvt; e += kThr) {
      const int r = e / kDvt, ii = e % kDvt;
      float acc = 0.f;
      for (int j = 0; j < dk; ++j) acc += Ws[r * dkp + j] * Ss[j * kDvt + ii];
      Vn[e] = Us[e] - acc;
    }
    __syncthreads();
    // 7. O = diag(gamma) Q S^T + P V_new   (old S)
    for (int e = tid; e < C * kDvt; e += kThr) {
      const int r = e / kDvt, ii = e % kDvt;
      if (r < L && i0 + ii < dv) {
        float acc = 0.f;
        for (int j = 0; j < dk; ++j) acc += Qs[r * dkp + j] * Ss[j * kDvt + ii];
        float acc2 = 0.f;
        for (int s = 0; s <= r; ++s) acc2 += Ps[r * (C + 1) + s] * Vn[s * kDvt + ii];
        st_from_f32(o + (size_t(ci.row0 + r) * H + h) * dv + i0 + ii,
                    (KDA ? acc : Ga[r] * acc) + acc2);
      }
    }
    __syncthreads();
    // 8. S <- gamma_last S + V_new^T diag(D) K
    for (int e = tid; e < dk * kDvt; e += kThr) {
      const int j = e / kDvt, ii = e % kDvt;
      float acc = 0.f;
      if (KDA) {
        for (int s = 0; s < C; ++s) acc += Ks[s * dkp + j] * Vn[s * kDvt + ii];
        Ss[e] = ex2_fast(Gl[j]) * Ss[e] + acc;
      } else {
        for (int s = 0; s < C; ++s) acc += Dd[s] * Ks[s * dkp + j] * Vn[s * kDvt + ii];
        Ss[e] = Ga[C - 1] * Ss[e] + acc;
      }
    }
  }
  __syncthreads();
  if (sN) {
    for (int e = tid; e < dk * kDvt; e += kThr) {
      const int j = e / kDvt, ii = e % kDvt;
      if (i0 + ii < dv) sN[((size_t(n) * H + h) * dk + j) * dv + i0 + ii] = Ss[e];
    }
  }
}

template <int C, typename T, bool KDA>
cudaError_t launch_simt_t(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *s0, int H, int dk, int dv, int N,
                          void *o, float *sN, uint32_t *ctrl, const ChunkInfo *table,
                          const int32_t *seq_first, cudaStream_t s) {
  const size_t floats = size_t(3) * C * (dk + 1) + size_t(3) * C * kDvt + size_t(dk) * kDvt +
                        size_t(3) * C * (C + 1) + 4 * C +
                        (KDA ? size_t(C) * (dk + 1) + dk : 0);
  const size_t bytes = floats * sizeof(float);
  auto kern = gdn_chunk_simt_kernel<C, T, KDA>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(bytes));
  if (e != cudaSuccess) return e;
  dim3 grid(N, H, (dv + kDvt - 1) / kDvt);
  kern<<<grid, simt_threads<KDA>(), bytes, s>>>(
      static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), g, beta,
      s0, H, dk, dv, static_cast<T *>(o), sN, ctrl, table, seq_first);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_simt(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *s0, const int32_t *cu, int B,
                              int T, int H, int dk, int dv, int N, int chunk, int dtype, void *o,
                              float *sN, uint32_t *ws_ctrl, cudaStream_t s, bool channel_gate) {
  (void)cu; (void)B; (void)T;
  char *base = reinterpret_cast<char *>(ws_ctrl);
  // The layout of the chunk table is the same for both paths.
  const WsLayout L = ws_layout(B, T, H, cu ? N : 0, chunk, false);
  const ChunkInfo *table = reinterpret_cast<const ChunkInfo *>(base + L.chunk_table);
  const int32_t *seq_first = reinterpret_cast<const int32_t *>(base + L.seq_first);
#define GDN_SIMT_CASE(CC, KK)                                                                   \
  if (chunk == CC && channel_gate == KK)                                                         \
    return dtype == GDN_BF16                                                                     \
               ? launch_simt_t<CC, __nv_bfloat16, KK>(q, k, v, g, beta, s0, H, dk, dv, N, o, \
                                                      sN, ws_ctrl, table, seq_first, s)         \
               : launch_simt_t<CC, float, KK>(q, k, v, g, beta, s0, H, dk, dv, N, o, sN,       \
                                              ws_ctrl, table, seq_first, s);
  GDN_SIMT_CASE(16, false)
  GDN_SIMT_CASE(32, false)
  GDN_SIMT_CASE(64, false)
  GDN_SIMT_CASE(16, true)
  GDN_SIMT_CASE(32, true)
  GDN_SIMT_CASE(64, true)
#undef GDN_SIMT_CASE
  return cudaErrorInvalidValue;
}

}  // namespace gdn
