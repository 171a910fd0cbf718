// Tensor-core (tcgen05 + TMEM + TMA) implementation of the chunkwise forward
// pass for bf16 inputs with d_k = d_v = 128 and chunks of 64 tokens.
//
// The method ("Gated Delta Networks: Improving Mamba2 with Delta Rule"): the
// gated delta rule computed chunkwise with the WY representation / UT
// transform, extended to carry the decay gate (phantomic12 page, mechanism
// paragraph; dmarx anthology LIT-137, "Standing in the anthology"; SOTA-135,
// "Source"). Per chunk (rows r, s in [0, 64), Gamma = inclusive cumsum of
// log alpha, gamma = exp(Gamma)):
//   A = strictly-lower diag(beta) (K K^T .* exp(Gamma_r - Gamma_s)),  T = (I + A)^-1
//   W = T diag(beta gamma) K,   U = T diag(beta) V
//   V_new = U - W S^T
//   O = diag(gamma) Q S^T + (Q K^T .* M) V_new,   M_rs = exp(Gamma_r - Gamma_s), s <= r
//   S <- gamma_last S + V_new^T diag(exp(Gamma_last - Gamma)) K
//
// Two kernels:
//   gdn_prep_kernel  one CTA per (chunk, head), fully parallel. Everything that
//                    does not depend on the state: Gamma, A, P = (QK^T).*M,
//                    T by blocked forward substitution, W^T and U^T on tcgen05.
//                    Writes W^T, U^T, P (bf16) and Gamma (fp32) to the workspace.
//   gdn_scan_kernel  one CTA per (sequence, head), sequential over chunks:
//                    the state-dependent products on tcgen05 with the fp32
//                    master state in registers of the epilogue warps, and O.
//
// All matrices below are worked in the "transposed frame" where the 128-wide
// head dimension is the MMA M dimension, so every tcgen05.mma is M = 128 and
// each thread of the epilogue warpgroup owns one TMEM lane = one row of d_v
// (or d_k). Shared-memory operand tiles use the 128-byte swizzle with 64
// bf16 (128 bytes) per row; TMA loads have no cluster broadcast.
#include <cstdio>
#include <cstring>

#include "gdn_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

constexpr int kC = 64;    // chunk
constexpr int kD = 128;   // d_k = d_v
constexpr uint32_t kTile64x64 = 64 * 128;     // 64 rows x 128 B   = 8 KB
constexpr uint32_t kTile128x64 = 128 * 128;   // 128 rows x 128 B = 16 KB

// ===================================================================== prep
// Shared memory of the prep kernel (offsets from a 1024-aligned base).
constexpr uint32_t kP_KQ = 0;                       // 2 blocks x [K rows 0-63 | Q rows 64-127] = 32 KB
constexpr uint32_t kP_V = kP_KQ + 2 * kTile128x64;  // 2 blocks x 64 rows = 16 KB
constexpr uint32_t kP_TB = kP_V + 2 * kTile64x64;   // T diag(beta), bf16, K-major 64x64
constexpr uint32_t kP_TBG = kP_TB + kTile64x64;     // T diag(beta gamma)
constexpr uint32_t kP_PST = kP_TBG + kTile64x64;    // P staging for the TMA store
constexpr uint32_t kP_AS = kP_PST + kTile64x64;     // A, fp32 [64][65]
constexpr uint32_t kP_TS = kP_AS + 64 * 65 * 4;     // T, fp32 [64][65]
constexpr uint32_t kP_XS = kP_TS + 64 * 65 * 4;     // scratch, fp32 3 x 16 x 16
constexpr uint32_t kP_VEC = kP_XS + 3 * 256 * 4;    // Gamma, beta, gamma: 3 x 64 fp32
constexpr uint32_t kP_BAR = kP_VEC + 3 * 64 * 4;    // 2 mbarriers + tmem address
constexpr uint32_t kP_END = kP_BAR + 64;
constexpr uint32_t kPrepSmem = kP_END + 1024;       // + alignment slack
constexpr int kPrepThreads = 128;

// T = (I + A)^-1 for the strictly lower-triangular 64 x 64 A, in fp32 shared
// memory, with 16 x 16 blocks: the four diagonal blocks are inverted by
// column-wise forward substitution in registers, then each off-diagonal block
// follows from T_ij = -T_ii (sum_{m=j}^{i-1} A_im T_mj), one block diagonal
// at a time (every T_mj it needs lies on an earlier block diagonal).
__device__ void solve_unit_lower_64(const float *__restrict__ As, float *__restrict__ Ts,
                                    float *__restrict__ Xs, int tid) {
  constexpr int P = 65;
  if (tid < 64) {
    const int bb = tid >> 4, jj = tid & 15, base = bb * 16;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) x[r] = (r == jj) ? 1.f : 0.f;
#pragma unroll
    for (int r = 1; r < 16; ++r) {
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < r; ++m) acc += As[(base + r) * P + base + m] * x[m];
      if (r > jj) x[r] = -acc;
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) Ts[(base + r) * P + base + jj] = x[r];
  } else {
    // zero the blocks above the diagonal
    for (int e = tid - 64; e < 64 * 64; e += 64) {
      const int r = e >> 6, c = e & 63;
      if ((c >> 4) > (r >> 4)) Ts[r * P + c] = 0.f;
    }
  }
  __syncthreads();
  for (int d = 1; d < 4; ++d) {
    const int nblk = 4 - d;
    // X_ij = sum_{m=16j}^{16i-1} A[16i+r][m] T[m][16j+c]
    for (int o = tid; o < nblk * 256; o += kPrepThreads) {
      const int b = o >> 8, r = (o >> 4) & 15, c = o & 15;
      const int i = b + d, j = b;
      float acc = 0.f;
      for (int m = 16 * j; m < 16 * i; ++m) acc += As[(16 * i + r) * P + m] * Ts[m * P + 16 * j + c];
      Xs[o] = acc;
    }
    __syncthreads();
    // T_ij = -T_ii X_ij
    for (int o = tid; o < nblk * 256; o += kPrepThreads) {
      const int b = o >> 8, r = (o >> 4) & 15, c = o & 15;
      const int i = b + d, j = b;
      float acc = 0.f;
      for (int m = 0; m <= r; ++m) acc += Ts[(16 * i + r) * P + 16 * i + m] * Xs[(b << 8) + (m << 4) + c];
      Ts[(16 * i + r) * P + 16 * j + c] = -acc;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kPrepThreads, 2) gdn_prep_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_wt,
    const __grid_constant__ CUtensorMap tm_ut, const __grid_constant__ CUtensorMap tm_pm,
    const float *__restrict__ g, const float *__restrict__ beta, float *__restrict__ gam_out,
    int H, uint32_t *__restrict__ ctrl, const ChunkInfo *__restrict__ table) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~uintptr_t(1023));
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x, h = blockIdx.y;
  if (ctrl[0] & kErrBadSeqlens) return;
  if (chunk >= int(ctrl[1])) return;
  const ChunkInfo ci = table[chunk];
  const int L = ci.len;
  const int unit = chunk * H + h;

  float *As = reinterpret_cast<float *>(sm + kP_AS);
  float *Ts = reinterpret_cast<float *>(sm + kP_TS);
  float *Xs = reinterpret_cast<float *>(sm + kP_XS);
  float *Gm = reinterpret_cast<float *>(sm + kP_VEC);
  float *Bt = Gm + 64;
  float *Ga = Bt + 64;
  uint64_t *bar_load = reinterpret_cast<uint64_t *>(sm + kP_BAR);
  uint64_t *bar_mma = bar_load + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_load + 2);

  if (tid == 0) {
    abort_flag = 0;
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    mbar_arrive_expect_tx(bar_load, 2 * kTile128x64 + 2 * kTile64x64);
    tma_load_3d(sm + kP_KQ, &tm_k, bar_load, 0, h, ci.row0);
    tma_load_3d(sm + kP_KQ + kTile64x64, &tm_q, bar_load, 0, h, ci.row0);
    tma_load_3d(sm + kP_KQ + kTile128x64, &tm_k, bar_load, 64, h, ci.row0);
    tma_load_3d(sm + kP_KQ + kTile128x64 + kTile64x64, &tm_q, bar_load, 64, h, ci.row0);
    tma_load_3d(sm + kP_V, &tm_v, bar_load, 0, h, ci.row0);
    tma_load_3d(sm + kP_V + kTile64x64, &tm_v, bar_load, 64, h, ci.row0);
  }
  if (tid < kC) {
    const bool ok = tid < L;
    Gm[tid] = ok ? g[size_t(ci.row0 + tid) * H + h] : 0.f;
    Bt[tid] = ok ? beta[size_t(ci.row0 + tid) * H + h] : 0.f;
  }
  __syncthreads();
  if (warp == 0) {  // inclusive cumsum of the 64 log-gates
    float a0 = Gm[2 * lane], a1 = Gm[2 * lane + 1];
    float s = a0 + a1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float t = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += t;
    }
    const float excl = s - (a0 + a1);
    Gm[2 * lane] = excl + a0;
    Gm[2 * lane + 1] = s;
  }
  const bool loaded = mbar_wait(bar_load, 0, ctrl, &abort_flag);
  if (loaded && L < kC) {
    // Rows past the sequence end act as k = q = v = 0.
    for (int e = tid; e < (kC - L) * 8; e += kPrepThreads) {
      const int r = L + e / 8, ch = e % 8;
      const uint4 z = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4 *>(sm + kP_KQ + r * 128 + ch * 16) = z;
      *reinterpret_cast<uint4 *>(sm + kP_KQ + kTile64x64 + r * 128 + ch * 16) = z;
      *reinterpret_cast<uint4 *>(sm + kP_KQ + kTile128x64 + r * 128 + ch * 16) = z;
      *reinterpret_cast<uint4 *>(sm + kP_KQ + kTile128x64 + kTile64x64 + r * 128 + ch * 16) = z;
      *reinterpret_cast<uint4 *>(sm + kP_V + r * 128 + ch * 16) = z;
      *reinterpret_cast<uint4 *>(sm + kP_V + kTile64x64 + r * 128 + ch * 16) = z;
    }
    fence_proxy_async_smem();
  }
  __syncthreads();
  if (!abort_flag && tid == 0) {
    // G = [K; Q] K^T : M = 128 (K rows then Q rows), N = 64, K = 128 (d_k)
    tc_fence_after();
    const uint32_t idesc = make_idesc_bf16(128, 64, 0, 0);
    const uint32_t kq = smem_u32(sm + kP_KQ);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t off = (kk >> 2) * kTile128x64 + (kk & 3) * 32;
      tc_mma_bf16(tmem, make_sdesc(kq + off, 16, 1024), make_sdesc(kq + off, 16, 1024), idesc,
                  kk > 0);
    }
    tc_commit(bar_mma);
  }
  if (tid < kC) Ga[tid] = expf(Gm[tid]);
  mbar_wait(bar_mma, 0, ctrl, &abort_flag);
  tc_fence_after();
  const int m = warp * 32 + lane;  // TMEM lane = row of G
  if (!abort_flag) {
    uint32_t r0[32], r1[32];
    const uint32_t taddr = tmem + (uint32_t(warp * 32) << 16);
    tmem_ld32(taddr, r0);
    tmem_ld32(taddr + 32, r1);
    tmem_ld_wait();
    if (m < kC) {
      const int r = m;
      const float br = Bt[r], gr = Gm[r];
#pragma unroll
      for (int s = 0; s < 32; ++s)
        As[r * 65 + s] = (s < r) ? br * expf(gr - Gm[s]) * __uint_as_float(r0[s]) : 0.f;
#pragma unroll
      for (int s = 0; s < 32; ++s)
        As[r * 65 + 32 + s] = (32 + s < r) ? br * expf(gr - Gm[32 + s]) * __uint_as_float(r1[s]) : 0.f;
    } else {
      const int c = m - kC;
      const float gc = Gm[c];
      uint8_t *prow = sm + kP_PST;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int s = ch * 8 + e;
          const float gv = __uint_as_float(ch < 4 ? r0[s & 31] : r1[s & 31]);
          f[e] = (s <= c) ? expf(gc - Gm[s]) * gv : 0.f;
        }
        uint4 pk = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                              pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
        *reinterpret_cast<uint4 *>(prow + sw128_offset(c, ch)) = pk;
      }
    }
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (!abort_flag && tid == 0) {
    tma_store_2d(&tm_pm, sm + kP_PST, 0, unit * kC);
    tma_store_commit();
  }
  if (!abort_flag) solve_unit_lower_64(As, Ts, Xs, tid);
  // T diag(beta) and T diag(beta gamma) as bf16 K-major operand tiles
  {
    const int r = tid >> 1, half = tid & 1;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int ch = half * 4 + cc;
      float fb[8], fg[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int s = ch * 8 + e;
        const float t = Ts[r * 65 + s] * Bt[s];
        fb[e] = t;
        fg[e] = t * Ga[s];
      }
      *reinterpret_cast<uint4 *>(sm + kP_TB + sw128_offset(r, ch)) =
          make_uint4(pack_bf16x2(fb[0], fb[1]), pack_bf16x2(fb[2], fb[3]),
                     pack_bf16x2(fb[4], fb[5]), pack_bf16x2(fb[6], fb[7]));
      *reinterpret_cast<uint4 *>(sm + kP_TBG + sw128_offset(r, ch)) =
          make_uint4(pack_bf16x2(fg[0], fg[1]), pack_bf16x2(fg[2], fg[3]),
                     pack_bf16x2(fg[4], fg[5]), pack_bf16x2(fg[6], fg[7]));
    }
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (!abort_flag && tid == 0) {
    tc_fence_after();
    // W^T = K^T (T diag(beta gamma))^T : M = 128 (d_k), N = 64, K = 64 (tokens)
    // U^T = V^T (T diag(beta))^T       : M = 128 (d_v), N = 64, K = 64
    const uint32_t idesc = make_idesc_bf16(128, 64, 1, 0);
    const uint32_t kq = smem_u32(sm + kP_KQ), vv = smem_u32(sm + kP_V);
    const uint32_t tbg = smem_u32(sm + kP_TBG), tb = smem_u32(sm + kP_TB);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      tc_mma_bf16(tmem + 64, make_sdesc(kq + kk * 2048, kTile128x64, 1024),
                  make_sdesc(tbg + kk * 32, 16, 1024), idesc, kk > 0);
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      tc_mma_bf16(tmem + 128, make_sdesc(vv + kk * 2048, kTile64x64, 1024),
                  make_sdesc(tb + kk * 32, 16, 1024), idesc, kk > 0);
    }
    tc_commit(bar_mma);
  }
  if (tid < kC) gam_out[size_t(unit) * kC + tid] = Gm[tid];
  mbar_wait(bar_mma, 1, ctrl, &abort_flag);
  tc_fence_after();
  if (!abort_flag) {
    // Row m of W^T / U^T -> bf16 staging tiles (reusing the K/Q and V areas).
    const uint32_t taddr = tmem + (uint32_t(warp * 32) << 16);
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      uint32_t r0[32], r1[32];
      tmem_ld32(taddr + 64 + which * 64, r0);
      tmem_ld32(taddr + 96 + which * 64, r1);
      tmem_ld_wait();
      uint8_t *dst = sm + (which == 0 ? kP_KQ : kP_V);
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const uint32_t *src = ch < 4 ? r0 : r1;
        const int b = (ch & 3) * 8;
        *reinterpret_cast<uint4 *>(dst + sw128_offset(m, ch)) = make_uint4(
            pack_bf16x2(__uint_as_float(src[b + 0]), __uint_as_float(src[b + 1])),
            pack_bf16x2(__uint_as_float(src[b + 2]), __uint_as_float(src[b + 3])),
            pack_bf16x2(__uint_as_float(src[b + 4]), __uint_as_float(src[b + 5])),
            pack_bf16x2(__uint_as_float(src[b + 6]), __uint_as_float(src[b + 7])));
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    if (!abort_flag) {
      tma_store_2d(&tm_wt, sm + kP_KQ, 0, unit * kD);
      tma_store_2d(&tm_ut, sm + kP_V, 0, unit * kD);
      tma_store_commit();
    }
    tma_store_wait_all();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ===================================================================== scan
// Per stage (one chunk of one head): W^T, U^T, Q, K, P, Gamma.
constexpr uint32_t kS_WT = 0;                       // [128 d_k][64 c]   MN-major B of S W^T
constexpr uint32_t kS_UT = kS_WT + kTile128x64;     // [128 d_v][64 s]
constexpr uint32_t kS_Q = kS_UT + kTile128x64;      // 2 x [64 c][64 d]  K-major B of S Q^T
constexpr uint32_t kS_K = kS_Q + 2 * kTile64x64;    // 2 x [64 s][64 d]  MN-major B of dS
constexpr uint32_t kS_P = kS_K + 2 * kTile64x64;    // [64 c][64 s]      K-major B of Y
constexpr uint32_t kS_G = kS_P + kTile64x64;        // 64 fp32
constexpr uint32_t kStageBytes = kS_G + 1024;       // keep stages 1024-aligned
constexpr uint32_t kStageTx = 4 * kTile128x64 + kTile64x64 + 256;
constexpr int kStages = 2;
constexpr uint32_t kS_STATE = kStages * kStageBytes;          // S, bf16 [128 d_v][128 d_k]: 2 blocks
constexpr uint32_t kS_A1 = kS_STATE + 2 * kTile128x64;        // V_new^T           [128][64]
constexpr uint32_t kS_A2 = kS_A1 + kTile128x64;               // V_new^T diag(D)   [128][64]
constexpr uint32_t kS_BAR = kS_A2 + kTile128x64;
constexpr uint32_t kS_END = kS_BAR + 128;
constexpr uint32_t kScanSmem = kS_END + 1024;
constexpr int kScanThreads = 256;
// TMEM columns
constexpr uint32_t kT_X = 0, kT_Z = 64, kT_Y = 192, kT_DS = 320;

__global__ void __launch_bounds__(kScanThreads, 1) gdn_scan_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_wt, const __grid_constant__ CUtensorMap tm_ut,
    const __grid_constant__ CUtensorMap tm_pm, const __grid_constant__ CUtensorMap tm_gam,
    const float *__restrict__ s0, float *__restrict__ sN, __nv_bfloat16 *__restrict__ o, int H,
    uint32_t *__restrict__ ctrl, const ChunkInfo *__restrict__ table,
    const int32_t *__restrict__ seq_first) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~uintptr_t(1023));
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x, h = blockIdx.y;
  if (ctrl[0] & kErrBadSeqlens) return;
  const int c0 = seq_first[n], nch = seq_first[n + 1] - c0;

  uint64_t *full = reinterpret_cast<uint64_t *>(sm + kS_BAR);  // [2]
  uint64_t *empty = full + 2;                                   // [2]
  uint64_t *s_ready = full + 4;
  uint64_t *x_full = full + 5;
  uint64_t *vnew_ready = full + 6;
  uint64_t *s_full = full + 7;
  uint64_t *y_full = full + 8;
  uint64_t *drain = full + 9;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(full + 10);

  if (tid == 0) {
    abort_flag = 0;
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_wt);
    tma_prefetch_desc(&tm_ut);
    tma_prefetch_desc(&tm_pm);
    tma_prefetch_desc(&tm_gam);
    for (int i = 0; i < 10; ++i) mbar_init(full + i, 1);
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    for (int c = 0; c < nch; ++c) {
      const int st = c & 1;
      if (c >= 2 && !mbar_wait(empty + st, ((c >> 1) - 1) & 1, ctrl, &abort_flag)) break;
      const ChunkInfo ci = table[c0 + c];
      const int unit = (c0 + c) * H + h;
      uint8_t *sb = sm + st * kStageBytes;
      mbar_arrive_expect_tx(full + st, kStageTx);
      tma_load_2d(sb + kS_WT, &tm_wt, full + st, 0, unit * kD);
      tma_load_2d(sb + kS_UT, &tm_ut, full + st, 0, unit * kD);
      tma_load_3d(sb + kS_Q, &tm_q, full + st, 0, h, ci.row0);
      tma_load_3d(sb + kS_Q + kTile64x64, &tm_q, full + st, 64, h, ci.row0);
      tma_load_3d(sb + kS_K, &tm_k, full + st, 0, h, ci.row0);
      tma_load_3d(sb + kS_K + kTile64x64, &tm_k, full + st, 64, h, ci.row0);
      tma_load_2d(sb + kS_P, &tm_pm, full + st, 0, unit * kC);
      tma_load_2d(sb + kS_G, &tm_gam, full + st, 0, unit);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t id_x = make_idesc_bf16(128, 64, 0, 1);    // S W^T : B MN-major
    const uint32_t id_z = make_idesc_bf16(128, 64, 0, 0);    // S Q^T : B K-major
    const uint32_t id_s = make_idesc_bf16(128, 128, 0, 1);   // A2 K  : B MN-major
    const uint32_t id_y = make_idesc_bf16(128, 64, 0, 0);    // A1 P^T: B K-major
    const uint32_t sS = smem_u32(sm + kS_STATE);
    const uint32_t sA1 = smem_u32(sm + kS_A1), sA2 = smem_u32(sm + kS_A2);
    for (int c = 0; c < nch; ++c) {
      const int st = c & 1;
      const uint32_t sb = smem_u32(sm + st * kStageBytes);
      if (!mbar_wait(full + st, (c >> 1) & 1, ctrl, &abort_flag)) break;
      if (!mbar_wait(s_ready, c & 1, ctrl, &abort_flag)) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t a = make_sdesc(sS + (kk >> 2) * kTile128x64 + (kk & 3) * 32, 16, 1024);
        tc_mma_bf16(tmem + kT_X, a, make_sdesc(sb + kS_WT + kk * 2048, kTile64x64, 1024), id_x,
                    kk > 0);
      }
      tc_commit(x_full);
      const uint32_t zcol = kT_Z + (c & 1) * 64;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t a = make_sdesc(sS + (kk >> 2) * kTile128x64 + (kk & 3) * 32, 16, 1024);
        const uint64_t b =
            make_sdesc(sb + kS_Q + (kk >> 2) * kTile64x64 + (kk & 3) * 32, 16, 1024);
        tc_mma_bf16(tmem + zcol, a, b, id_z, kk > 0);
      }
      if (!mbar_wait(vnew_ready, c & 1, ctrl, &abort_flag)) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        tc_mma_bf16(tmem + kT_DS, make_sdesc(sA2 + kk * 32, 16, 1024),
                    make_sdesc(sb + kS_K + kk * 2048, kTile64x64, 1024), id_s, kk > 0);
      }
      tc_commit(s_full);
      const uint32_t ycol = kT_Y + (c & 1) * 64;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        tc_mma_bf16(tmem + ycol, make_sdesc(sA1 + kk * 32, 16, 1024),
                    make_sdesc(sb + kS_P + kk * 32, 16, 1024), id_y, kk > 0);
      }
      tc_commit(y_full);
    }
    // Every MMA issued above has completed once this fires.
    tc_commit(drain);
    mbar_wait(drain, 0, ctrl, &abort_flag);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int i = tid - 128;                      // TMEM lane = row of d_v
    const uint32_t lane_base = tmem + (uint32_t((warp - 4) * 32) << 16);
    float S[kD];                                  // S[i][j], fp32 master
    {
      const float *src = s0 ? s0 + (size_t(n) * H + h) * kD * kD : nullptr;
#pragma unroll
      for (int j = 0; j < kD; ++j) S[j] = src ? src[size_t(j) * kD + i] : 0.f;
    }
    auto store_state_bf16 = [&]() {
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const int j = ch * 8;
        *reinterpret_cast<uint4 *>(sm + kS_STATE + (ch >> 3) * kTile128x64 +
                                   sw128_offset(i, ch & 7)) =
            make_uint4(pack_bf16x2(S[j], S[j + 1]), pack_bf16x2(S[j + 2], S[j + 3]),
                       pack_bf16x2(S[j + 4], S[j + 5]), pack_bf16x2(S[j + 6], S[j + 7]));
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (i == 0) mbar_arrive(s_ready);
    };
    store_state_bf16();
    // Every epilogue thread runs every iteration and every named barrier, even
    // after an abort (waits then return at once), so no thread is stranded.
    auto wait = [&](uint64_t *bar, uint32_t parity) {
      if (!abort_flag) mbar_wait(bar, parity, ctrl, &abort_flag);
    };
    for (int c = 0; c < nch; ++c) {
      const int st = c & 1;
      uint8_t *sb = sm + st * kStageBytes;
      wait(full + st, (c >> 1) & 1);
      const ChunkInfo ci = table[c0 + c];
      const float *G = reinterpret_cast<const float *>(sb + kS_G);
      const float glast = G[kC - 1];
      wait(x_full, c & 1);
      tc_fence_after();
      // V_new^T row i = U^T row i - (S W^T) row i
      {
        uint32_t x0[32], x1[32];
        tmem_ld32(lane_base + kT_X, x0);
        tmem_ld32(lane_base + kT_X + 32, x1);
        tmem_ld_wait();
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 u4 = *reinterpret_cast<const uint4 *>(sb + kS_UT + sw128_offset(i, ch));
          const __nv_bfloat162 *u2 = reinterpret_cast<const __nv_bfloat162 *>(&u4);
          float vn[8], vd[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int s = ch * 8 + e;
            const float u = (e & 1) ? __high2float(u2[e >> 1]) : __low2float(u2[e >> 1]);
            const float xv = __uint_as_float(ch < 4 ? x0[s & 31] : x1[s & 31]);
            vn[e] = u - xv;
            vd[e] = vn[e] * expf(glast - G[s]);
          }
          *reinterpret_cast<uint4 *>(sm + kS_A1 + sw128_offset(i, ch)) =
              make_uint4(pack_bf16x2(vn[0], vn[1]), pack_bf16x2(vn[2], vn[3]),
                         pack_bf16x2(vn[4], vn[5]), pack_bf16x2(vn[6], vn[7]));
          *reinterpret_cast<uint4 *>(sm + kS_A2 + sw128_offset(i, ch)) =
              make_uint4(pack_bf16x2(vd[0], vd[1]), pack_bf16x2(vd[2], vd[3]),
                         pack_bf16x2(vd[4], vd[5]), pack_bf16x2(vd[6], vd[7]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(1, 128);
      if (i == 0) mbar_arrive(vnew_ready);
      // S <- gamma_last S + dS
      wait(s_full, c & 1);
      tc_fence_after();
      {
        const float gl = expf(glast);
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
          uint32_t d[32];
          tmem_ld32(lane_base + kT_DS + jb * 32, d);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < 32; ++t) S[jb * 32 + t] = gl * S[jb * 32 + t] + __uint_as_float(d[t]);
        }
      }
      tc_fence_before();
      store_state_bf16();
      // O rows of this chunk: o[c'][i] = gamma_c' (S Q^T)[i][c'] + Y[i][c']
      wait(y_full, c & 1);
      tc_fence_after();
      {
        uint32_t z[32], y[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          tmem_ld32(lane_base + kT_Z + (c & 1) * 64 + half * 32, z);
          tmem_ld32(lane_base + kT_Y + (c & 1) * 64 + half * 32, y);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const int cc = half * 32 + t;
            if (cc < ci.len) {
              const float val = expf(G[cc]) * __uint_as_float(z[t]) + __uint_as_float(y[t]);
              o[(size_t(ci.row0 + cc) * H + h) * kD + i] = __float2bfloat16_rn(val);
            }
          }
        }
      }
      tc_fence_before();
      named_bar_sync(1, 128);
      if (i == 0) mbar_arrive(empty + st);
    }
    if (sN && !abort_flag) {
      float *dst = sN + (size_t(n) * H + h) * kD * kD;
#pragma unroll
      for (int j = 0; j < kD; ++j) dst[size_t(j) * kD + i] = S[j];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [rows, H, d] bf16 tokens (d innermost), box 64 x 1 x 64, 128-byte swizzle.
bool map_tokens(CUtensorMap *m, const void *base, long long rows, int H) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(kD), cuuint64_t(H), cuuint64_t(rows)};
  cuuint64_t strides[2] = {cuuint64_t(kD) * 2, cuuint64_t(H) * kD * 2};
  cuuint32_t box[3] = {64, 1, 64};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
             box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// [rows, inner] 2-D map with box (inner, box_rows).
bool map_2d(CUtensorMap *m, const void *base, CUtensorMapDataType t, int esize, long long rows,
            int inner, int box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cuuint64_t(inner), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(inner) * esize};
  cuuint32_t box[2] = {cuuint32_t(inner), cuuint32_t(box_rows)};
  cuuint32_t es[2] = {1, 1};
  return enc(m, t, 2, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *s0, int B, int T, int H, int N,
                            void *o, float *sN, void *ws, const WsLayout &L, cudaStream_t s) {
  char *base = static_cast<char *>(ws);
  uint32_t *ctrl = reinterpret_cast<uint32_t *>(base);
  const ChunkInfo *table = reinterpret_cast<const ChunkInfo *>(base + L.chunk_table);
  const int32_t *seq_first = reinterpret_cast<const int32_t *>(base + L.seq_first);
  const long long rows = (long long)B * T;
  const long long units = (long long)L.max_chunks * H;
  if (T > 0 && L.max_chunks > 0) {
    CUtensorMap mq, mk, mv, mwt, mut, mpm, mgm;
    if (!map_tokens(&mq, q, rows, H) || !map_tokens(&mk, k, rows, H) ||
        !map_tokens(&mv, v, rows, H) ||
        !map_2d(&mwt, base + L.wt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kD, 64, kD,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mut, base + L.ut, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kD, 64, kD,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mpm, base + L.pm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kC, 64, kC,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mgm, base + L.gam, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, units, 64, 1,
                CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(gdn_prep_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kPrepSmem);
    if (e != cudaSuccess) return e;
    prof_record(g_profile.prep, s);
    gdn_prep_kernel<<<dim3(L.max_chunks, H), kPrepThreads, kPrepSmem, s>>>(
        mq, mk, mv, mwt, mut, mpm, g, beta, reinterpret_cast<float *>(base + L.gam), H, ctrl,
        table);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gdn_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kScanSmem);
    if (e != cudaSuccess) return e;
    prof_record(g_profile.scan, s);
    gdn_scan_kernel<<<dim3(N, H), kScanThreads, kScanSmem, s>>>(
        mq, mk, mwt, mut, mpm, mgm, s0, sN, static_cast<__nv_bfloat16 *>(o), H, ctrl, table,
        seq_first);
    return cudaGetLastError();
  }
  // No tokens: the final state is the initial state.
  prof_record(g_profile.prep, s);
  prof_record(g_profile.scan, s);
  if (sN) {
    const size_t bytes = size_t(N) * H * kD * kD * sizeof(float);
    return s0 ? cudaMemcpyAsync(sN, s0, bytes, cudaMemcpyDeviceToDevice, s)
              : cudaMemsetAsync(sN, 0, bytes, s);
  }
  return cudaSuccess;
}

}  // namespace gdn
