// Chunkwise backward pass on the tensor cores (bf16 inputs, d_k = d_v = 128,
// 64-token chunks): the gradients of gdn_chunk_fwd for the loss
// L = sum(d_o * o) + sum(d_final_state * final_state).
//
// The pages present the chunkwise WY / UT-transform algorithm as a training
// algorithm ("Gated Delta Networks", phantomic12 page, mechanism paragraph)
// but give no gradients. These follow by reverse-mode differentiation of the
// chunk equations of the forward pass. Per chunk, with S = S_c the state
// entering it, G' = dL/dS_{c+1}, Gamma = cumsum(g), gamma = e^Gamma,
// D_s = e^(Gamma_last - Gamma_s), E_rs = e^(Gamma_r - Gamma_s), T diag(beta)
// = TB, W = T diag(beta gamma) K, P = (Q K^T) .* E (s <= r):
//   X   = TB V - W S^T                      (V_new, recomputed)
//   dX  = P^T dO + (D K) G'^T
//   dS  = gamma_last G' - dX^T W + (gamma dO)^T Q            (the chain)
//   dV  = TB^T dX
//   L   = (K K^T) .* E (s < r)   [A = diag(beta) L]
//   dY  = dX - L^T dV            (= (I + A)^-T dX without dividing by beta)
//   e   = V - gamma (K S^T) - L X (the residual v_r - alpha_r S_{r-1} k_r)
//   dbeta_r = dY_r . e_r
//   dP  = dO X^T;  R = -(dV X^T) .* E (s < r)
//   dQ  = gamma (dO S) + (dP .* E, s <= r) K
//   dK  = (dP .* E)^T Q + D (X G') - gamma (dV S) + R K + R^T K
//   dGamma_r = gamma_r q_r.(dO S)_r - gamma_r k_r.(dV S)_r
//            + rowsum_r(dP .* P) - colsum_r(dP .* P)
//            + rowsum_r(-(dV X^T) .* L) - colsum_r(-(dV X^T) .* L)
//            - delta_r,   delta_s = D_s X_s . (G' k_s)
//     and on the chunk's last token also + sum(delta) + gamma_last <G', S>;
//   dg  = reverse cumsum of dGamma over the chunk.
// The kernels of one call:
//   1. the forward's chunk map, prep and state scan, the scan also writing
//      every chunk's entering state S_c (bf16) and no output;
//   2. gdn_bwd_chain_kernel, one CTA per (sequence, head): the reverse chain
//      dS_c = gamma_last dS_{c+1} - dX^T W + (gamma dO)^T Q over the chunks,
//      writing each chunk's G' = dS_{c+1} (bf16) and d_initial_state;
//   3. gdn_bwd_unit_kernel, persistent over (chunk, head) units: everything
//      else above, from the chunk's tiles, S_c and G'.
// Products run on the warp-level tensor-core path (mma.sync m16n8k16, bf16
// operands, fp32 accumulation) from padded shared-memory tiles.
#include <cuda_bf16.h>

#include "bwd_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using bf16 = __nv_bfloat16;
constexpr int kC = 64, kD = 128;
// Row strides (bf16 elements) of the shared tiles: 272- and 144-byte rows put
// the 8 rows an ldmatrix reads in 8 distinct 16-byte bank groups.
constexpr int kLd128 = 136, kLd64 = 72;
constexpr uint32_t kT64x128 = 64 * kLd128 * 2;    // [64][128] tile, 17,408 B
constexpr uint32_t kT128x128 = 128 * kLd128 * 2;  // [128][128] tile, 34,816 B
constexpr uint32_t kT64x64 = 64 * kLd64 * 2;      // [64][64] tile, 9,216 B
constexpr uint32_t kT128x64 = 128 * kLd64 * 2;    // [128][64] tile, 18,432 B
constexpr int kThreads = 256, kWarps = kThreads / 32;   // the unit kernel's block
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One warp: acc[MT][NT] (16 x 8 tiles, rows m0 + 16 mt, columns n0 + 8 nt)
// += op(A) op(B) over k in [0, K) (fully unrolled). A is stored [m][k] (AT = false) or [k][m]
// (AT = true) at shared address A with row stride lda elements; B is stored
// [n][k] (BT = false) or [k][n] (BT = true). Fragment layout of acc[mt][nt]:
// with g = lane / 4, t = lane % 4, elements (g, 2t), (g, 2t+1), (g+8, 2t),
// (g+8, 2t+1) of the tile. NT is even (B is read two n-tiles at a time).
template <int MT, int NT, bool AT, bool BT, int K>
__device__ __forceinline__ void warp_mma(float (&acc)[MT][NT][4], uint32_t A, int lda, int m0,
                                         uint32_t B, int ldb, int n0, int lane) {
#pragma unroll
  for (int k0 = 0; k0 < K; k0 += 16) {
    uint32_t a[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      if (!AT) {
        const int r = m0 + 16 * mt + (lane & 15), c = k0 + 8 * (lane >> 4);
        ldsm_x4(A + 2u * uint32_t(r * lda + c), a[mt]);
      } else {
        const int r = k0 + (lane & 7) + 8 * (lane >> 4), c = m0 + 16 * mt + 8 * ((lane >> 3) & 1);
        ldsm_x4_trans(A + 2u * uint32_t(r * lda + c), a[mt]);
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; nt += 2) {
      uint32_t b[4];
      if (!BT) {
        const int r = n0 + 8 * nt + 8 * (lane >> 4) + (lane & 7), c = k0 + 8 * ((lane >> 3) & 1);
        ldsm_x4(B + 2u * uint32_t(r * ldb + c), b);
      } else {
        const int r = k0 + (lane & 7) + 8 * ((lane >> 3) & 1), c = n0 + 8 * nt + 8 * (lane >> 4);
        ldsm_x4_trans(B + 2u * uint32_t(r * ldb + c), b);
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        mma16816(acc[mt][nt], a[mt], b[0], b[1]);
        mma16816(acc[mt][nt + 1], a[mt], b[2], b[3]);
      }
    }
  }
}

// Two independent products of the same shape and depth in one loop (twice
// the independent accumulators per step): acc1 += op(A1) op(B1), acc2 +=
// op(A2) op(B2), operands as for warp_mma.
template <int MT, int NT, bool AT1, bool BT1, bool AT2, bool BT2, int K>
__device__ __forceinline__ void warp_mma2(float (&acc1)[MT][NT][4], uint32_t A1, int lda1,
                                          uint32_t B1, int ldb1, float (&acc2)[MT][NT][4],
                                          uint32_t A2, int lda2, uint32_t B2, int ldb2, int m0,
                                          int n0, int lane) {
#pragma unroll
  for (int k0 = 0; k0 < K; k0 += 16) {
    uint32_t a1[MT][4], a2[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      if (!AT1)
        ldsm_x4(A1 + 2u * uint32_t((m0 + 16 * mt + (lane & 15)) * lda1 + k0 + 8 * (lane >> 4)), a1[mt]);
      else
        ldsm_x4_trans(A1 + 2u * uint32_t((k0 + (lane & 7) + 8 * (lane >> 4)) * lda1 + m0 + 16 * mt +
                                         8 * ((lane >> 3) & 1)), a1[mt]);
      if (!AT2)
        ldsm_x4(A2 + 2u * uint32_t((m0 + 16 * mt + (lane & 15)) * lda2 + k0 + 8 * (lane >> 4)), a2[mt]);
      else
        ldsm_x4_trans(A2 + 2u * uint32_t((k0 + (lane & 7) + 8 * (lane >> 4)) * lda2 + m0 + 16 * mt +
                                         8 * ((lane >> 3) & 1)), a2[mt]);
    }
#pragma unroll
    for (int nt = 0; nt < NT; nt += 2) {
      uint32_t b1[4], b2[4];
      if (!BT1)
        ldsm_x4(B1 + 2u * uint32_t((n0 + 8 * nt + 8 * (lane >> 4) + (lane & 7)) * ldb1 + k0 +
                                   8 * ((lane >> 3) & 1)), b1);
      else
        ldsm_x4_trans(B1 + 2u * uint32_t((k0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * ldb1 + n0 +
                                         8 * nt + 8 * (lane >> 4)), b1);
      if (!BT2)
        ldsm_x4(B2 + 2u * uint32_t((n0 + 8 * nt + 8 * (lane >> 4) + (lane & 7)) * ldb2 + k0 +
                                   8 * ((lane >> 3) & 1)), b2);
      else
        ldsm_x4_trans(B2 + 2u * uint32_t((k0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * ldb2 + n0 +
                                         8 * nt + 8 * (lane >> 4)), b2);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        mma16816(acc1[mt][nt], a1[mt], b1[0], b1[1]);
        mma16816(acc2[mt][nt], a2[mt], b2[0], b2[1]);
        mma16816(acc1[mt][nt + 1], a1[mt], b1[2], b1[3]);
        mma16816(acc2[mt][nt + 1], a2[mt], b2[2], b2[3]);
      }
    }
  }
}

template <int MT, int NT>
__device__ __forceinline__ void zero_acc(float (&acc)[MT][NT][4]) {
#pragma unroll
  for (int i = 0; i < MT; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
}

// Fragment pair (row, 2 columns) of a [rows][ld] bf16 tile as two floats.
__device__ __forceinline__ float2 ld_pair(const bf16 *t, int ld, int r, int c) {
  const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(t + r * ld + c);
  return __bfloat1622float2(v);
}
__device__ __forceinline__ void st_pair(bf16 *t, int ld, int r, int c, float x, float y) {
  *reinterpret_cast<uint32_t *>(t + r * ld + c) = pack_bf16x2(x, y);
}

// Copies rows [0, 64) of a token tile (128 bf16 per row, row r at
// base + (row0 + r) * stride elements) into a [64][kLd128] shared tile; rows
// r >= len read as zero.
__device__ __forceinline__ void load_tokens(uint32_t dst, const bf16 *base, long long row0,
                                            long long stride, int len, int tid) {
  for (int e = tid; e < 64 * 16; e += kThreads) {
    const int r = e >> 4, c = e & 15;
    const bool ok = r < len;
    const bf16 *src = ok ? base + (row0 + r) * stride + 8 * c : base;
    cp_async16(dst + uint32_t(r * kLd128 + 8 * c) * 2u, src, ok ? 16u : 0u);
  }
}
// Copies a dense [rows][cols] bf16 tile (cols = 64 or 128) into a padded one.
template <int COLS>
__device__ __forceinline__ void load_dense(uint32_t dst, const bf16 *src, int rows, int tid) {
  constexpr int kPer = COLS / 8, kLd = COLS == 128 ? kLd128 : kLd64;
  for (int e = tid; e < rows * kPer; e += kThreads) {
    const int r = e / kPer, c = e - r * kPer;
    cp_async16(dst + uint32_t(r * kLd + 8 * c) * 2u, src + r * COLS + 8 * c, 16u);
  }
}

// ------------------------------------------------------------------ chain
// Row i of dS_c depends only on row i of dS_{c+1} (dX column i only on row i
// of G'), so each (sequence, head) chain runs as kSlices CTAs of kSlice d_v
// rows, two CTAs per SM. Shared memory: the G slice (bf16 [kSlice][d_k]), the
// dX slice (bf16 [tokens][kSlice]), one chunk's (D K)^T, P, -W and Q, and two
// stages of the dO slice and the decay factors. (D K)^T and P of the next
// chunk load while the G update runs, -W and Q while the next dX runs.
constexpr int kSlices = 4, kSlice = kD / kSlices, kLdS = kSlice + 8;
constexpr int kChainThreads = 256, kChainWarps = kChainThreads / 32;
constexpr uint32_t kTDoS = 64 * kLdS * 2;             // [64][kSlice] tile
constexpr uint32_t kCh_G = 0;                          // [kSlice][kLd128]
constexpr uint32_t kCh_DX = kCh_G + kSlice * kLd128 * 2;
constexpr uint32_t kCh_KT = kCh_DX + kTDoS;            // (D K)^T [d_k][tokens]
constexpr uint32_t kCh_PM = kCh_KT + kT128x64;         // P [r][s]
constexpr uint32_t kCh_WN = kCh_PM + kT64x64;          // -W [tokens][d_k]
constexpr uint32_t kCh_Q = kCh_WN + kT64x128;          // Q [tokens][d_k]
constexpr uint32_t kCh_DO = kCh_Q + kT64x128;          // 2 x dO slice, then gamma dO
constexpr uint32_t kCh_GAM = kCh_DO + 2 * kTDoS;       // 2 x (gamma [64], D [64])
constexpr uint32_t kChainSmem = kCh_GAM + 2 * 128 * 4;
static_assert(2 * (kChainSmem + 1024) <= 233472, "chain kernel: two CTAs per SM");

__global__ void __launch_bounds__(kChainThreads, 2) gdn_bwd_chain_kernel(
    const bf16 *__restrict__ q, const bf16 *__restrict__ d_o, const float *__restrict__ d_sN,
    float *__restrict__ ds0, const uint8_t *__restrict__ ws_w, const uint8_t *__restrict__ ws_kt,
    const uint8_t *__restrict__ ws_pm, const float *__restrict__ ws_gam,
    bf16 *__restrict__ gprime, int H, uint32_t *__restrict__ ctrl,
    const ChunkInfo *__restrict__ table, const int32_t *__restrict__ seq_first, int N,
    long long rows, int max_chunks) {
  (void)rows;
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n = blockIdx.x, h = blockIdx.y, i0 = kSlice * int(blockIdx.z);
  const uint32_t sb = smem_u32(smem);
  bf16 *Gs = reinterpret_cast<bf16 *>(smem + kCh_G);
  bf16 *DXs = reinterpret_cast<bf16 *>(smem + kCh_DX);
  int c0 = 0, nch = 0;
  if (!(ctrl[0] & kErrBadSeqlens) && GDN_IN_BOUNDS(ctrl, n + 1, N + 1)) {
    c0 = seq_first[n];
    nch = seq_first[n + 1] - c0;
  }
  // G = dL/dS rows [i0, i0 + kSlice) (formula orientation [d_v i][d_k j]);
  // warp w: local rows [gm0, gm0 + 16), columns [gn0, gn0 + 32).
  constexpr int kGT = 4;
  const int gm0 = 16 * (warp & 1), gn0 = 32 * (warp >> 1);
  float G[1][kGT][4];
  {
    const float *src = d_sN ? d_sN + (size_t(n) * H + h) * kD * kD : nullptr;
#pragma unroll
    for (int nt = 0; nt < kGT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = i0 + gm0 + g + 8 * (e >> 1), j = gn0 + 8 * nt + 2 * t + (e & 1);
        G[0][nt][e] = src ? src[j * kD + i] : 0.f;   // stored [d_k][d_v]
      }
  }
  auto unit_of = [&](int c) { return (long long)(c0 + c) * H + h; };
  auto info_of = [&](int c) {
    const long long chunk = c0 + c;
    return GDN_IN_BOUNDS(ctrl, chunk, max_chunks) ? table[chunk] : ChunkInfo{0, 0, 0, 0};
  };
  // group A: (D K)^T, P, the dO slice and the decay factors of chunk c
  auto load_a = [&](int c, int st) {
    if (c >= 0) {
      const long long unit = unit_of(c);
      const ChunkInfo ci = info_of(c);
      for (int e = tid; e < 128 * 8; e += kChainThreads) {
        const int r = e >> 3, cc = e & 7;
        cp_async16(sb + kCh_KT + uint32_t(r * kLd64 + 8 * cc) * 2u,
                   reinterpret_cast<const bf16 *>(ws_kt) + unit * (kD * kC) + r * kC + 8 * cc, 16u);
      }
      for (int e = tid; e < 64 * 8; e += kChainThreads) {
        const int r = e >> 3, cc = e & 7;
        cp_async16(sb + kCh_PM + uint32_t(r * kLd64 + 8 * cc) * 2u,
                   reinterpret_cast<const bf16 *>(ws_pm) + unit * (kC * kC) + r * kC + 8 * cc, 16u);
      }
      for (int e = tid; e < 64 * (kSlice / 8); e += kChainThreads) {
        const int r = e / (kSlice / 8), cc = e - r * (kSlice / 8);
        const bool ok = r < ci.len;
        const bf16 *src = ok ? d_o + ((long long)ci.row0 + r) * H * kD + size_t(h) * kD + i0 + 8 * cc
                             : d_o;
        cp_async16(sb + kCh_DO + st * kTDoS + uint32_t(r * kLdS + 8 * cc) * 2u, src, ok ? 16u : 0u);
      }
      if (tid < 32)
        cp_async16(sb + kCh_GAM + st * 512 + 16 * tid, ws_gam + unit * 128 + 4 * tid, 16u);
    }
    cp_async_commit();
  };
  // group B: -W and Q of chunk c
  auto load_b = [&](int c) {
    if (c >= 0) {
      const long long unit = unit_of(c);
      const ChunkInfo ci = info_of(c);
      for (int e = tid; e < 64 * 16; e += kChainThreads) {
        const int r = e >> 4, cc = e & 15;
        cp_async16(sb + kCh_WN + uint32_t(r * kLd128 + 8 * cc) * 2u,
                   reinterpret_cast<const bf16 *>(ws_w) + unit * (kC * kD) + r * kD + 8 * cc, 16u);
        const bool ok = r < ci.len;
        const bf16 *src = ok ? q + ((long long)ci.row0 + r) * H * kD + size_t(h) * kD + 8 * cc : q;
        cp_async16(sb + kCh_Q + uint32_t(r * kLd128 + 8 * cc) * 2u, src, ok ? 16u : 0u);
      }
    }
    cp_async_commit();
  };
  load_a(nch - 1, 0);
  load_b(nch - 1);
  for (int it = 0; it < nch; ++it) {
    const int c = nch - 1 - it, st = it & 1;
    const long long unit = unit_of(c);
    // G' slice of this chunk: bf16 into shared memory (operand) and the workspace
#pragma unroll
    for (int nt = 0; nt < kGT; ++nt) {
      const int i = gm0 + g, j = gn0 + 8 * nt + 2 * t;
      st_pair(Gs, kLd128, i, j, G[0][nt][0], G[0][nt][1]);
      st_pair(Gs, kLd128, i + 8, j, G[0][nt][2], G[0][nt][3]);
    }
    cp_async_wait<1>();   // group A of this chunk (B may still be in flight)
    __syncthreads();
    if (GDN_IN_BOUNDS(ctrl, unit, (long long)max_chunks * H)) {
      uint4 *dst = reinterpret_cast<uint4 *>(gprime + unit * (kD * kD) + size_t(i0) * kD);
      for (int e = tid; e < kSlice * 16; e += kChainThreads) {
        const int r = e >> 4, cc = e & 15;
        dst[r * 16 + cc] = *reinterpret_cast<const uint4 *>(Gs + r * kLd128 + 8 * cc);
      }
    }
    const float *gam = reinterpret_cast<const float *>(smem + kCh_GAM + st * 512);
    bf16 *DO = reinterpret_cast<bf16 *>(smem + kCh_DO + st * kTDoS);
    {
      // dX slice = P^T dO + (D K) G^T: warp w -> tokens [16 (w % 4), +16),
      // local d_v [16 (w / 4), +16)
      const int m0 = 16 * (warp & 3), n0 = 16 * (warp >> 2);
      float acc[1][2][4];
      zero_acc(acc);
      warp_mma<1, 2, true, true, 64>(acc, sb + kCh_PM, kLd64, m0, sb + kCh_DO + st * kTDoS, kLdS, n0, lane);
      warp_mma<1, 2, true, false, 128>(acc, sb + kCh_KT, kLd64, m0, sb + kCh_G, kLd128, n0, lane);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int r = m0 + g, cc = n0 + 8 * nt + 2 * t;
        st_pair(DXs, kLdS, r, cc, acc[0][nt][0], acc[0][nt][1]);
        st_pair(DXs, kLdS, r + 8, cc, acc[0][nt][2], acc[0][nt][3]);
      }
    }
    __syncthreads();   // dX complete; (D K)^T, P and the unscaled dO no longer read
    load_a(c - 1, st ^ 1);
    // gamma dO in place (bf16, rounded once)
    for (int e = tid; e < 64 * (kSlice / 2); e += kChainThreads) {
      const int r = e / (kSlice / 2), cc = 2 * (e - r * (kSlice / 2));
      const float2 x = ld_pair(DO, kLdS, r, cc);
      st_pair(DO, kLdS, r, cc, gam[r] * x.x, gam[r] * x.y);
    }
    cp_async_wait<1>();   // group B of this chunk
    __syncthreads();
    {
      // G <- gamma_last G - dX^T W + (gamma dO)^T Q
      const float gl = gam[kC - 1];
#pragma unroll
      for (int nt = 0; nt < kGT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) G[0][nt][e] *= gl;
      warp_mma<1, kGT, true, true, 64>(G, sb + kCh_DX, kLdS, gm0, sb + kCh_WN, kLd128, gn0, lane);
      warp_mma<1, kGT, true, true, 64>(G, sb + kCh_DO + st * kTDoS, kLdS, gm0, sb + kCh_Q, kLd128, gn0, lane);
    }
    __syncthreads();   // G slice, dX, -W and Q free
    load_b(c - 1);
  }
  cp_async_wait<0>();
  if (!(ctrl[0] & kErrBadSeqlens) && GDN_IN_BOUNDS(ctrl, (long long)n * H + h, (long long)N * H)) {
    float *dst = ds0 + (size_t(n) * H + h) * kD * kD;
#pragma unroll
    for (int nt = 0; nt < kGT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = i0 + gm0 + g + 8 * (e >> 1), j = gn0 + 8 * nt + 2 * t + (e & 1);
        dst[j * kD + i] = G[0][nt][e];
      }
  }
}

// ------------------------------------------------------------------ units
constexpr uint32_t kU_Q = 0;
constexpr uint32_t kU_K = kU_Q + kT64x128;
constexpr uint32_t kU_V = kU_K + kT64x128;
constexpr uint32_t kU_DO = kU_V + kT64x128;
constexpr uint32_t kU_S = kU_DO + kT64x128;       // S_c [d_v][d_k]
constexpr uint32_t kU_GP = kU_S + kT128x128;      // G' [d_v][d_k]
constexpr uint32_t kU_TB = kU_GP + kT128x128;     // T diag(beta); then -L; then R
constexpr uint32_t kU_P = kU_TB + kT64x64;        // P; then dP .* E
constexpr uint32_t kU_W = kU_P + kT64x64;         // -W; then dX
constexpr uint32_t kU_KT = kU_W + kT64x128;       // (D K)^T [d_k][tokens]; then dV
constexpr uint32_t kU_X = kU_KT + kT128x64;       // X
constexpr uint32_t kU_VEC = kU_X + kT64x128;      // Gamma, gamma, D, dGamma, dbeta, delta [64] each
constexpr uint32_t kU_RED = kU_VEC + 6 * 64 * 4;  // block reduction scratch [kWarps]
constexpr uint32_t kUnitSmem = kU_RED + 4 * kWarps;
static_assert(kT128x64 >= kT64x128 && kUnitSmem <= 232448, "unit kernel shared memory");

// Calls f(mt, nt, hf, row, col) for every fragment pair (row, col..col+1)
// of a warp's acc[MT][NT] tile with origin (m0, n0); the pair is
// acc[mt][nt][2 hf], acc[mt][nt][2 hf + 1].
template <int MT, int NT, typename F>
__device__ __forceinline__ void each_pair(int m0, int n0, int lane, F &&f) {
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
        f(mt, nt, hf, m0 + 16 * mt + (lane >> 2) + 8 * hf, n0 + 8 * nt + 2 * (lane & 3));
}

// Adds the per-row partial sums part[mt][hf] of a warp tile (rows m0 + 16 mt
// + lane / 4 + 8 hf) over the four lanes of a row, then into dst[row].
template <int MT>
__device__ __forceinline__ void add_rows(float *dst, float (&part)[MT][2], int m0, int lane) {
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float x = part[mt][hf];
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      if ((lane & 3) == 0) atomicAdd(dst + m0 + 16 * mt + (lane >> 2) + 8 * hf, x);
    }
}

// Subtracts the per-column partial sums part[nt][2] (columns n0 + 8 nt + 2 t,
// +1) over the eight lanes of a column, then from dst[col].
template <int NT>
__device__ __forceinline__ void sub_cols(float *dst, float (&part)[NT][2], int n0, int lane) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      float x = part[nt][b];
      x += __shfl_xor_sync(0xffffffffu, x, 4);
      x += __shfl_xor_sync(0xffffffffu, x, 8);
      x += __shfl_xor_sync(0xffffffffu, x, 16);
      if ((lane >> 2) == 0) atomicAdd(dst + n0 + 8 * nt + 2 * (lane & 3) + b, -x);
    }
}

__global__ void __launch_bounds__(kThreads, 1) gdn_bwd_unit_kernel(
    const bf16 *__restrict__ q, const bf16 *__restrict__ k, const bf16 *__restrict__ v,
    const float *__restrict__ g, const bf16 *__restrict__ d_o,
    const uint8_t *__restrict__ ws_w, const uint8_t *__restrict__ ws_kt,
    const uint8_t *__restrict__ ws_tb, const uint8_t *__restrict__ ws_pm,
    const bf16 *__restrict__ s_chunks, const bf16 *__restrict__ gprime, float *__restrict__ dq,
    float *__restrict__ dk, float *__restrict__ dv, float *__restrict__ dg,
    float *__restrict__ dbeta, int H, uint32_t *__restrict__ ctrl,
    const ChunkInfo *__restrict__ table, long long rows, int max_chunks) {
  (void)rows;
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sb = smem_u32(smem);
  bf16 *Qs = reinterpret_cast<bf16 *>(smem + kU_Q);
  bf16 *Ks = reinterpret_cast<bf16 *>(smem + kU_K);
  bf16 *Vs = reinterpret_cast<bf16 *>(smem + kU_V);
  bf16 *Ss = reinterpret_cast<bf16 *>(smem + kU_S);
  bf16 *Gp = reinterpret_cast<bf16 *>(smem + kU_GP);
  bf16 *Ls = reinterpret_cast<bf16 *>(smem + kU_TB);
  bf16 *Ps = reinterpret_cast<bf16 *>(smem + kU_P);
  bf16 *DXs = reinterpret_cast<bf16 *>(smem + kU_W);
  bf16 *DVs = reinterpret_cast<bf16 *>(smem + kU_KT);
  bf16 *Xs = reinterpret_cast<bf16 *>(smem + kU_X);
  float *Gam = reinterpret_cast<float *>(smem + kU_VEC);   // log2(e) Gamma
  float *gam = Gam + 64, *Dv = Gam + 128, *dGam = Gam + 192, *dBet = Gam + 256,
        *delta = Gam + 320;
  float *red = reinterpret_cast<float *>(smem + kU_RED);
  const int nunits = (ctrl[0] & kErrBadSeqlens) ? 0 : int(ctrl[1]) * H;
  // Warp tiles: 64 x 128 outputs as 2 x 4 tiles of 32 x 32 (rows m0, columns
  // n0); 64 x 64 outputs as 2 x 4 tiles of 32 x 16 (columns p0).
  constexpr int kMT = 2, kNT = 4, kNP = 2;
  const int m0 = 32 * (warp & 1), n0 = 32 * (warp >> 1), p0 = 16 * (warp >> 1);
  using Acc = float[kMT][kNT][4];
  using AccP = float[kMT][kNP][4];
  // stores a 64 x 128 fp32 result tile (rows < len) to out [B*T][H][128]
  auto store_out = [&](float *out, Acc &a, const ChunkInfo &ci, int h) {
    each_pair<kMT, kNT>(m0, n0, lane, [&](int mt, int nt, int hf, int r, int c) {
      const long long o = (((long long)ci.row0 + r) * H + h) * kD + c;
      if (r < ci.len && GDN_IN_BOUNDS(ctrl, o + 1, rows * H * kD))
        *reinterpret_cast<float2 *>(out + o) = make_float2(a[mt][nt][2 * hf], a[mt][nt][2 * hf + 1]);
    });
  };
  auto store_tile = [&](bf16 *t, Acc &a) {
    each_pair<kMT, kNT>(m0, n0, lane, [&](int mt, int nt, int hf, int r, int c) {
      st_pair(t, kLd128, r, c, a[mt][nt][2 * hf], a[mt][nt][2 * hf + 1]);
    });
  };
  for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x) {
    const int chunk = unit / H, h = unit - chunk * H;
    const ChunkInfo ci =
        GDN_IN_BOUNDS(ctrl, chunk, max_chunks) ? table[chunk] : ChunkInfo{0, 0, 0, 0};
    const int len = ci.len;
    const long long ustride = (long long)H * kD;
    load_tokens(sb + kU_Q, q + size_t(h) * kD, ci.row0, ustride, len, tid);
    load_tokens(sb + kU_K, k + size_t(h) * kD, ci.row0, ustride, len, tid);
    load_tokens(sb + kU_V, v + size_t(h) * kD, ci.row0, ustride, len, tid);
    load_tokens(sb + kU_DO, d_o + size_t(h) * kD, ci.row0, ustride, len, tid);
    {
      // S_c: piece p (columns 8 p .. 8 p + 7) of row i at piece index p * 128 + i
      const bf16 *src = s_chunks + (long long)unit * (kD * kD);
      for (int e = tid; e < 128 * 16; e += kThreads) {
        const int p = e >> 7, i = e & 127;
        cp_async16(sb + kU_S + uint32_t(i * kLd128 + 8 * p) * 2u, src + (p * 128 + i) * 8, 16u);
      }
    }
    load_dense<128>(sb + kU_GP, gprime + (long long)unit * (kD * kD), 128, tid);
    load_dense<64>(sb + kU_TB, reinterpret_cast<const bf16 *>(ws_tb) + (long long)unit * (kC * kC), 64, tid);
    load_dense<64>(sb + kU_P, reinterpret_cast<const bf16 *>(ws_pm) + (long long)unit * (kC * kC), 64, tid);
    load_dense<128>(sb + kU_W, reinterpret_cast<const bf16 *>(ws_w) + (long long)unit * (kC * kD), 64, tid);
    load_dense<64>(sb + kU_KT, reinterpret_cast<const bf16 *>(ws_kt) + (long long)unit * (kD * kC), 128, tid);
    cp_async_commit();
    if (warp == 0) {
      // log2(e) Gamma by a warp scan over the 64 tokens (g = 0 past the end)
      float x0 = 0.f, x1 = 0.f;
      const long long i0 = ((long long)ci.row0 + lane) * H + h, i1 = i0 + 32LL * H;
      if (lane < len && GDN_IN_BOUNDS(ctrl, i0, rows * H)) x0 = g[i0] * kLog2e;
      if (lane + 32 < len && GDN_IN_BOUNDS(ctrl, i1, rows * H)) x1 = g[i1] * kLog2e;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y0 = __shfl_up_sync(0xffffffffu, x0, off);
        const float y1 = __shfl_up_sync(0xffffffffu, x1, off);
        if (lane >= off) {
          x0 += y0;
          x1 += y1;
        }
      }
      x1 += __shfl_sync(0xffffffffu, x0, 31);
      const float last = __shfl_sync(0xffffffffu, x1, 31);
      Gam[lane] = x0;
      Gam[lane + 32] = x1;
      gam[lane] = ex2(x0);
      gam[lane + 32] = ex2(x1);
      Dv[lane] = ex2(last - x0);
      Dv[lane + 32] = ex2(last - x1);
    } else if (warp == 1) {
      dGam[lane] = dGam[lane + 32] = 0.f;
      dBet[lane] = dBet[lane + 32] = 0.f;
      delta[lane] = delta[lane + 32] = 0.f;
    }
    cp_async_wait<0>();
    __syncthreads();
    // <G', S> (for the last token's dGamma)
    {
      float gs_dot = 0.f;
      for (int e = tid; e < 128 * 64; e += kThreads) {
        const int r = e >> 6, c = 2 * (e & 63);
        const float2 a = ld_pair(Gp, kLd128, r, c), b = ld_pair(Ss, kLd128, r, c);
        gs_dot += a.x * b.x + a.y * b.y;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) gs_dot += __shfl_xor_sync(0xffffffffu, gs_dot, off);
      if (lane == 0) red[warp] = gs_dot;
    }

    // X = TB V + (-W) S^T; kept in fp32 for delta
    Acc xr;
    zero_acc(xr);
    warp_mma<kMT, kNT, false, true, 64>(xr, sb + kU_TB, kLd64, m0, sb + kU_V, kLd128, n0, lane);
    warp_mma<kMT, kNT, false, false, 128>(xr, sb + kU_W, kLd128, m0, sb + kU_S, kLd128, n0, lane);
    store_tile(Xs, xr);
    __syncthreads();   // X complete; -W no longer read
    // dX = P^T dO + (D K) G'^T;  delta_s = X_s . ((D K) G'^T)_s
    Acc dx;
    zero_acc(dx);
    warp_mma<kMT, kNT, true, false, 128>(dx, sb + kU_KT, kLd64, m0, sb + kU_GP, kLd128, n0, lane);
    {
      float part[kMT][2] = {};
      each_pair<kMT, kNT>(m0, n0, lane, [&](int mt, int nt, int hf, int, int) {
        part[mt][hf] += xr[mt][nt][2 * hf] * dx[mt][nt][2 * hf] +
                        xr[mt][nt][2 * hf + 1] * dx[mt][nt][2 * hf + 1];
      });
      add_rows<kMT>(delta, part, m0, lane);
    }
    warp_mma<kMT, kNT, true, true, 64>(dx, sb + kU_P, kLd64, m0, sb + kU_DO, kLd128, n0, lane);
    store_tile(DXs, dx);
    __syncthreads();   // dX complete; (D K)^T no longer read
    // dV = TB^T dX -> output and bf16 operand
    {
      Acc acc;
      zero_acc(acc);
      warp_mma<kMT, kNT, true, true, 64>(acc, sb + kU_TB, kLd64, m0, sb + kU_W, kLd128, n0, lane);
      store_tile(DVs, acc);
      store_out(dv, acc, ci, h);
    }
    __syncthreads();   // dV complete; TB no longer read
    // -L = -(K K^T) .* E, s < r (bf16, in place of TB)
    {
      AccP acc;
      zero_acc(acc);
      warp_mma<kMT, kNP, false, false, 128>(acc, sb + kU_K, kLd128, m0, sb + kU_K, kLd128, p0, lane);
      each_pair<kMT, kNP>(m0, p0, lane, [&](int mt, int nt, int hf, int r, int s) {
        const float e0 = s < r ? -ex2(Gam[r] - Gam[s]) : 0.f;
        const float e1 = s + 1 < r ? -ex2(Gam[r] - Gam[s + 1]) : 0.f;
        st_pair(Ls, kLd64, r, s, e0 * acc[mt][nt][2 * hf], e1 * acc[mt][nt][2 * hf + 1]);
      });
    }
    __syncthreads();
    // dY = dX - L^T dV (in dx);  e = V - gamma (K S^T) - L X;  dbeta = rowsum(dY .* e)
    warp_mma<kMT, kNT, true, true, 64>(dx, sb + kU_TB, kLd64, m0, sb + kU_KT, kLd128, n0, lane);
    {
      Acc ee;
      zero_acc(ee);
      warp_mma<kMT, kNT, false, false, 128>(ee, sb + kU_K, kLd128, m0, sb + kU_S, kLd128, n0, lane);
      each_pair<kMT, kNT>(m0, n0, lane, [&](int mt, int nt, int hf, int r, int c) {
        const float2 vv = ld_pair(Vs, kLd128, r, c);
        ee[mt][nt][2 * hf] = vv.x - gam[r] * ee[mt][nt][2 * hf];
        ee[mt][nt][2 * hf + 1] = vv.y - gam[r] * ee[mt][nt][2 * hf + 1];
      });
      warp_mma<kMT, kNT, false, true, 64>(ee, sb + kU_TB, kLd64, m0, sb + kU_X, kLd128, n0, lane);
      float part[kMT][2] = {};
      each_pair<kMT, kNT>(m0, n0, lane, [&](int mt, int nt, int hf, int, int) {
        part[mt][hf] += dx[mt][nt][2 * hf] * ee[mt][nt][2 * hf] +
                        dx[mt][nt][2 * hf + 1] * ee[mt][nt][2 * hf + 1];
      });
      add_rows<kMT>(dBet, part, m0, lane);
    }
    __syncthreads();   // every read of -L as an operand done
    // dP = dO X^T -> dGamma (dP .* P), then dP .* E (s <= r) over P;
    // R' = dV X^T -> dGamma (-R' .* L), then R = -R' .* E (s < r) over -L
    {
      AccP dp, rp;
      zero_acc(dp);
      zero_acc(rp);
      warp_mma2<kMT, kNP, false, false, false, false, 128>(dp, sb + kU_DO, kLd128, sb + kU_X,
                                                           kLd128, rp, sb + kU_KT, kLd128,
                                                           sb + kU_X, kLd128, m0, p0, lane);
      float rows_[kMT][2] = {}, cols_[kNP][2] = {};
      each_pair<kMT, kNP>(m0, p0, lane, [&](int mt, int nt, int hf, int r, int s) {
        const float2 pp = ld_pair(Ps, kLd64, r, s);
        const float2 nl = ld_pair(Ls, kLd64, r, s);   // -L
        const float* a = &dp[mt][nt][2 * hf];
        const float* b = &rp[mt][nt][2 * hf];
        const float f0 = a[0] * pp.x + b[0] * nl.x, f1 = a[1] * pp.y + b[1] * nl.y;
        rows_[mt][hf] += f0 + f1;
        cols_[nt][0] += f0;
        cols_[nt][1] += f1;
        const float e0 = s <= r ? ex2(Gam[r] - Gam[s]) : 0.f;
        const float e1 = s + 1 <= r ? ex2(Gam[r] - Gam[s + 1]) : 0.f;
        st_pair(Ps, kLd64, r, s, e0 * a[0], e1 * a[1]);
        // R = -R' .* E, strictly below the diagonal
        st_pair(Ls, kLd64, r, s, s < r ? -e0 * b[0] : 0.f, s + 1 < r ? -e1 * b[1] : 0.f);
      });
      add_rows<kMT>(dGam, rows_, m0, lane);
      sub_cols<kNP>(dGam, cols_, p0, lane);
    }
    __syncthreads();   // dP .* E and R complete
    // dQ = gamma (dO S) + (dP .* E) K;  dGamma_r += gamma_r q_r . (dO S)_r
    {
      Acc acc;
      zero_acc(acc);
      warp_mma<kMT, kNT, false, true, 128>(acc, sb + kU_DO, kLd128, m0, sb + kU_S, kLd128, n0, lane);
      float part[kMT][2] = {};
      each_pair<kMT, kNT>(m0, n0, lane, [&](int mt, int nt, int hf, int r, int c) {
        const float2 qq = ld_pair(Qs, kLd128, r, c);
        part[mt][hf] += gam[r] * (qq.x * acc[mt][nt][2 * hf] + qq.y * acc[mt][nt][2 * hf + 1]);
        acc[mt][nt][2 * hf] *= gam[r];
        acc[mt][nt][2 * hf + 1] *= gam[r];
      });
      add_rows<kMT>(dGam, part, m0, lane);
      warp_mma<kMT, kNT, false, true, 64>(acc, sb + kU_P, kLd64, m0, sb + kU_K, kLd128, n0, lane);
      store_out(dq, acc, ci, h);
    }
    // dK = (dP .* E)^T Q + D (X G') - gamma (dV S) + R K + R^T K;
    // dGamma_r -= gamma_r k_r . (dV S)_r
    {
      Acc acc, vs;
      zero_acc(acc);
      zero_acc(vs);
      warp_mma2<kMT, kNT, false, true, false, true, 128>(acc, sb + kU_X, kLd128, sb + kU_GP,
                                                         kLd128, vs, sb + kU_KT, kLd128,
                                                         sb + kU_S, kLd128, m0, n0, lane);
      float part[kMT][2] = {};
      each_pair<kMT, kNT>(m0, n0, lane, [&](int mt, int nt, int hf, int r, int c) {
        const float2 kk = ld_pair(Ks, kLd128, r, c);
        float *a = &acc[mt][nt][2 * hf];
        const float *b = &vs[mt][nt][2 * hf];
        part[mt][hf] -= gam[r] * (kk.x * b[0] + kk.y * b[1]);
        a[0] = Dv[r] * a[0] - gam[r] * b[0];
        a[1] = Dv[r] * a[1] - gam[r] * b[1];
      });
      add_rows<kMT>(dGam, part, m0, lane);
      warp_mma<kMT, kNT, true, true, 64>(acc, sb + kU_P, kLd64, m0, sb + kU_Q, kLd128, n0, lane);
      warp_mma<kMT, kNT, false, true, 64>(acc, sb + kU_TB, kLd64, m0, sb + kU_K, kLd128, n0, lane);
      warp_mma<kMT, kNT, true, true, 64>(acc, sb + kU_TB, kLd64, m0, sb + kU_K, kLd128, n0, lane);
      store_out(dk, acc, ci, h);
    }
    __syncthreads();   // dGamma, dbeta, delta and the <G', S> partials complete
    if (warp == 0) {
      // dGamma_s -= delta_s; the last token adds sum(delta) + gamma_last <G', S>;
      // dg = reverse cumsum of dGamma over the valid tokens (Gam holds
      // log2(e) Gamma, but dGamma is the derivative with respect to Gamma).
      float gsd = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) gsd += red[w];
      const float dl0 = delta[lane], dl1 = delta[lane + 32];
      float tot = dl0 + dl1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
      const int last = len - 1;
      float x0 = dGam[lane] - dl0, x1 = dGam[lane + 32] - dl1;
      const float extra = tot + gam[kC - 1] * gsd;
      if (lane == last) x0 += extra;
      if (lane + 32 == last) x1 += extra;
      if (lane > last) x0 = 0.f;
      if (lane + 32 > last) x1 = 0.f;
      // reverse inclusive scan over the 64 tokens: each half, then x0 += sum(x1)
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y0 = __shfl_down_sync(0xffffffffu, x0, off);
        const float y1 = __shfl_down_sync(0xffffffffu, x1, off);
        if (lane + off < 32) {
          x0 += y0;
          x1 += y1;
        }
      }
      x0 += __shfl_sync(0xffffffffu, x1, 0);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = lane + 32 * hf;
        const long long o = ((long long)ci.row0 + r) * H + h;
        if (r < len && GDN_IN_BOUNDS(ctrl, o, rows * H)) {
          dg[o] = hf ? x1 : x0;
          dbeta[o] = dBet[r];
        }
      }
    }
    __syncthreads();   // shared memory free for the next unit
  }
}

}  // namespace

cudaError_t launch_bwd_tc(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *s0, const int32_t *cu,
                          const void *d_o, const float *d_sN, int N, int B, int T, int H,
                          int num_seqs, float *dq, float *dkk, float *dvv, float *dg,
                          float *dbeta, float *ds0, void *ws, const BwdTcLayout &L,
                          cudaStream_t s) {
  char *base = static_cast<char *>(ws);
  cudaError_t e = launch_chunk_map(cu, B, T, num_seqs, kC, ws, L.fwd, s);
  if (e != cudaSuccess) return e;
  bf16 *sc = reinterpret_cast<bf16 *>(base + L.s_chunks);
  bf16 *gp = reinterpret_cast<bf16 *>(base + L.gprime);
  e = launch_chunk_tc(q, k, v, g, beta, s0, B, T, H, N, nullptr, nullptr, ws, L.fwd, s, sc);
  if (e != cudaSuccess) return e;
  uint32_t *ctrl = reinterpret_cast<uint32_t *>(base);
  const ChunkInfo *table = reinterpret_cast<const ChunkInfo *>(base + L.fwd.chunk_table);
  const int32_t *seq_first = reinterpret_cast<const int32_t *>(base + L.fwd.seq_first);
  const long long rows = (long long)B * T;
  e = cudaFuncSetAttribute(gdn_bwd_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kChainSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gdn_bwd_unit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kUnitSmem);
  if (e != cudaSuccess) return e;
  gdn_bwd_chain_kernel<<<dim3(N, H, kSlices), kChainThreads, kChainSmem, s>>>(
      static_cast<const bf16 *>(q), static_cast<const bf16 *>(d_o), d_sN, ds0,
      reinterpret_cast<const uint8_t *>(base + L.fwd.w),
      reinterpret_cast<const uint8_t *>(base + L.fwd.kt),
      reinterpret_cast<const uint8_t *>(base + L.fwd.pm),
      reinterpret_cast<const float *>(base + L.fwd.gam), gp, H, ctrl, table, seq_first, N, rows,
      L.fwd.max_chunks);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int sms = device_sms();
  const long long units = (long long)L.fwd.max_chunks * H;
  const int grid = int(std::min<long long>(units, sms > 0 ? sms : 148));
  gdn_bwd_unit_kernel<<<grid, kThreads, kUnitSmem, s>>>(
      static_cast<const bf16 *>(q), static_cast<const bf16 *>(k), static_cast<const bf16 *>(v),
      g, static_cast<const bf16 *>(d_o), reinterpret_cast<const uint8_t *>(base + L.fwd.w),
      reinterpret_cast<const uint8_t *>(base + L.fwd.kt),
      reinterpret_cast<const uint8_t *>(base + L.fwd.tb),
      reinterpret_cast<const uint8_t *>(base + L.fwd.pm), sc, gp, dq, dkk, dvv, dg, dbeta, H,
      ctrl, table, rows, L.fwd.max_chunks);
  (void)beta;
  return cudaGetLastError();
}

}  // namespace gdn
