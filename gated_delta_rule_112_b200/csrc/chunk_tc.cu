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
//   gdn_prep_kernel  one CTA per (chunk, head), fully parallel: everything that
//                    depends only on the chunk's own K, Q, g, beta -- Gamma, A,
//                    P = (Q K^T) .* M, T by blocked forward substitution, and on
//                    tcgen05 W = T diag(beta gamma) K and (D K)^T with
//                    D = diag(exp(Gamma_last - Gamma)). Writes -W, (D K)^T,
//                    T diag(beta), P (bf16) and the decay factors (fp32).
//   gdn_scan_kernel  one CTA per (sequence, head), sequential over chunks:
//                    U^T = V^T (T diag(beta))^T and the state-dependent
//                    products on tcgen05, the fp32 state in registers of the
//                    epilogue warps, and O. Products that share an A operand
//                    are issued as one wide MMA (N = 128 or 192): a tcgen05.mma
//                    costs about the same whatever its N, so fewer, wider
//                    instructions shorten the sequential chain.
//
// All products are worked in the "transposed frame" where the 128-wide head
// dimension is the MMA M dimension, so every tcgen05.mma is M = 128 and each
// epilogue thread owns one TMEM lane = one row of d_v (or d_k). Shared-memory
// operand tiles use the 128-byte swizzle with 64 bf16 (128 bytes) per row;
// TMA loads have no cluster broadcast.
#include <algorithm>
#include <cstdio>
#include <cstring>

#include "gdn_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdn {

#ifdef GDN_TRACE
__device__ unsigned long long g_gdn_trace[2][kTraceSlots][kTraceEvents];
#endif

namespace {

constexpr int kC = 64;    // chunk
constexpr int kD = 128;   // d_k = d_v
constexpr uint32_t kTile64x64 = 64 * 128;     // 64 rows x 128 B   = 8 KB
constexpr uint32_t kTile128x64 = 128 * 128;   // 128 rows x 128 B = 16 KB

// ===================================================================== prep
// Shared memory of the prep kernel (offsets from a 1024-aligned base).
constexpr int kLd = 68;                              // fp32 row stride of A and T (16-byte rows)
constexpr uint32_t kP_KQ = 0;                        // 2 blocks x [K rows 0-63 | Q rows 64-127] = 32 KB
constexpr uint32_t kP_PST = kP_KQ + kTile64x64;      // P staging, over Q of block 0 (dead after G)
constexpr uint32_t kP_WST = kP_KQ;                   // -W staging [64 c][128 d] (2 blocks), over K/Q
constexpr uint32_t kP_KST = kP_KQ + kTile128x64;     // (D K)^T staging [128 d][64 s], over K/Q
constexpr uint32_t kP_TT = kP_KST + kTile64x64;      // solve: T transposed, fp32 [48][36], over Q of block 1
constexpr uint32_t kP_AS = kP_KQ + 2 * kTile128x64;  // A, fp32 [64][68]; after the solve it
constexpr uint32_t kP_TB = kP_AS;                    //   holds T diag(beta)       (bf16 64x64)
constexpr uint32_t kP_TBG = kP_AS + kTile64x64;      //   and   T diag(beta gamma) (bf16 64x64)
constexpr uint32_t kP_TS = kP_AS + 64 * kLd * 4;     // T, fp32 [64][68]; then diag(D) (bf16 64x64)
constexpr uint32_t kP_DIAG = kP_TS;
constexpr int kLy = 36;                              // fp32 row stride of the solve scratch
constexpr uint32_t kP_XS = kP_TS + 64 * kLd * 4;     // solve scratch, fp32 [32][36]
static_assert(kLy % 32 == 4 && kLd % 32 == 4 && 48 * kLy * 4 <= kTile64x64,
              "solve strides and the transposed-T area");
constexpr uint32_t kP_VEC = kP_XS + 32 * kLy * 4;    // Gamma, beta, gamma, Gamma log2(e): 4 x 64 fp32
constexpr uint32_t kP_BAR = kP_VEC + 4 * 64 * 4;     // 2 mbarriers + tmem address
constexpr uint32_t kP_END = kP_BAR + 64;
constexpr uint32_t kPrepSmem = kP_END + 1024;        // + alignment slack
constexpr int kPrepThreads = 256;
static_assert(2 * kTile64x64 <= 64 * kLd * 4, "T tiles must fit in the A area");
static_assert(kP_AS % 1024 == 0 && kP_PST % 1024 == 0 && kP_KST % 1024 == 0 &&
                  kP_DIAG % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");

// 2^x on the special-function unit (PTX ex2.approx, flush-to-zero).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float4 lds4(const float *p) {
  return *reinterpret_cast<const float4 *>(p);
}

// Shared address of this lane's row for an ldmatrix.x4 A fragment (16 x 8,
// rows r0.., columns c0..) of a row-major fp32 matrix with row stride ld.
__device__ __forceinline__ uint32_t frag_a(const float *m, int ld, int r0, int c0, int lane) {
  return smem_u32(m + (r0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * ld + c0 + 4 * (lane >> 4));
}
// ... and for a B fragment (8 x 8, k x n) read from the transposed copy
// (row n, word k): x2 gives k0.. k0 + 7, x4 also k0 + 8 .. k0 + 15.
__device__ __forceinline__ uint32_t frag_bt(const float *mt, int ld, int n0, int k0, int lane) {
  return smem_u32(mt + (n0 + (lane & 7)) * ld + k0 + 4 * (lane >> 3));
}

// d += a b for fp32 fragments on the tf32 tensor-core path, each operand split
// into tf32 parts x = hi + lo (|lo| <= 2^-11 |x|, the rest <= 2^-22 |x|) and
// the three products that matter: lo hi + hi lo + hi hi. The dropped lo lo
// term and the tails keep each product term within about 2^-21 of fp32.
__device__ __forceinline__ void mma_3xtf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                           uint32_t b1) {
  uint32_t ah[4], al[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    ah[i] = cvt_tf32(__uint_as_float(a[i]));
    al[i] = cvt_tf32(__uint_as_float(a[i]) - __uint_as_float(ah[i]));
  }
  const uint32_t bh0 = cvt_tf32(__uint_as_float(b0)), bh1 = cvt_tf32(__uint_as_float(b1));
  const uint32_t bl0 = cvt_tf32(__uint_as_float(b0) - __uint_as_float(bh0));
  const uint32_t bl1 = cvt_tf32(__uint_as_float(b1) - __uint_as_float(bh1));
  mma_tf32_m16n8k8(d, al, bh0, bh1);
  mma_tf32_m16n8k8(d, ah, bl0, bl1);
  mma_tf32_m16n8k8(d, ah, bh0, bh1);
}

// T = (I + A)^-1 for the strictly lower-triangular 64 x 64 A (fp32 shared
// memory, row stride kLd), by recursive 2 x 2 blocking: for a lower block
// triangular [[L11, 0], [L21, L22]], the inverse is [[T11, 0], [-T22 L21 T11, T22]].
//   step 0  the four 16 x 16 diagonal blocks, by column-wise forward
//           substitution in registers (thread = one column of one block);
//           their upper triangles are written as zeros. Blocks 0-2 are also
//           written transposed into Tt (row stride kLy): T(0,0), T(1,1) at
//           [0, 32) x [0, 32), T(2,2) at rows [32, 48)
//   step 1  T(1,0) and T(3,2): Y_b = A(i,j) T(j,j), then T(i,j) = -T(i,i) Y_b
//           (i = 2b + 1, j = 2b); warp (b, column half) computes both
//           products for its 8 columns, so only a warp sync lies between them
//   step 2  T([2,3],[0,1]): Y = A(..) T([0,1],[0,1]), then -T([2,3],[2,3]) Y;
//           warp = one 16 x 8 tile of each product, the two warps that share
//           a column tile meet on a named barrier
// The products are warp-level tensor-core tiles (m16n8k8, split tf32, fp32
// accumulation) whose operands are read with ldmatrix: A operands from the
// row-major A and T, B operands from transposed copies (Tt, and Y stored
// transposed in Xs), all with row strides = 4 (mod 32) words, so that an
// 8-row ldmatrix and the transposed fragment stores are free of bank
// conflicts. Loop bounds skip the blocks of T above the diagonal, which are
// never written, and are uniform within a warp.
__device__ void solve_unit_lower_64(const float *__restrict__ As, float *__restrict__ Ts,
                                    float *__restrict__ Tt, float *__restrict__ Xs, int tid) {
  const int warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  if (tid < 64) {
    const int base = (tid >> 4) * 16, jj = tid & 15;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) x[r] = (r == jj) ? 1.f : 0.f;
#pragma unroll
    for (int r = 1; r < 16; ++r) {
      const float *arow = As + (base + r) * kLd + base;
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
      for (int m4 = 0; m4 < r; m4 += 4) {
        const float4 a = lds4(arow + m4);
        acc0 = fmaf(a.x, x[m4], acc0);
        if (m4 + 1 < r) acc1 = fmaf(a.y, x[m4 + 1], acc1);
        if (m4 + 2 < r) acc0 = fmaf(a.z, x[m4 + 2], acc0);
        if (m4 + 3 < r) acc1 = fmaf(a.w, x[m4 + 3], acc1);
      }
      if (r > jj) x[r] = -(acc0 + acc1);
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) Ts[(base + r) * kLd + base + jj] = x[r];
    if (base < 48) {   // transposed: row = column of T, word = row of T
      float *dst = Tt + (base + jj) * kLy + (base < 32 ? base : 0);
#pragma unroll
      for (int r = 0; r < 16; r += 4)
        *reinterpret_cast<float4 *>(dst + r) = make_float4(x[r], x[r + 1], x[r + 2], x[r + 3]);
    }
  }
  __syncthreads();
  if (warp < 4) {  // step 1
    const int b = warp >> 1, n0 = 8 * (warp & 1);
    const int i = 16 * (2 * b + 1), j = i - 16;
    const float *tjt = Tt + (b ? 32 * kLy : 0);   // T(j,j) transposed, block-local indices
    float *yt = Xs + b * 16 * kLy;                // Y_b transposed
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    // columns n >= 8 of T(j,j) are zero in rows k < 8
    for (int k0 = n0; k0 < 16; k0 += 8) {
      uint32_t a[4], bb[2];
      ldsm_x4(frag_a(As, kLd, i, j + k0, lane), a);
      ldsm_x2(frag_bt(tjt, kLy, n0, k0, lane), bb);
      mma_3xtf32(c, a, bb[0], bb[1]);
    }
    const int n = n0 + 2 * t;
    yt[n * kLy + g] = c[0];
    yt[(n + 1) * kLy + g] = c[1];
    yt[n * kLy + g + 8] = c[2];
    yt[(n + 1) * kLy + g + 8] = c[3];
    __syncwarp();
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t bb[4];
    ldsm_x4(frag_bt(yt, kLy, n0, 0, lane), bb);
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      uint32_t a[4];
      ldsm_x4(frag_a(Ts, kLd, i, i + 8 * kk, lane), a);
      mma_3xtf32(d, a, bb[2 * kk], bb[2 * kk + 1]);
    }
    *reinterpret_cast<float2 *>(Ts + (i + g) * kLd + j + n) = make_float2(-d[0], -d[1]);
    *reinterpret_cast<float2 *>(Ts + (i + g + 8) * kLd + j + n) = make_float2(-d[2], -d[3]);
    if (b == 0) {   // T(1,0) is also a B operand of step 2
      Tt[n * kLy + i + g] = -d[0];
      Tt[(n + 1) * kLy + i + g] = -d[1];
      Tt[n * kLy + i + g + 8] = -d[2];
      Tt[(n + 1) * kLy + i + g + 8] = -d[3];
    }
  }
  __syncthreads();
  {  // step 2: output tile rows 32 + m0 .. + 15, columns n0 .. n0 + 7
    const int mi = warp >> 2, m0 = 16 * mi, n0 = 8 * (warp & 3);
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    // columns n of T([0,1],[0,1]) are zero in rows k < n: start at k = n0
    for (int k0 = n0; k0 < 32; k0 += 8) {
      uint32_t a[4], bb[2];
      ldsm_x4(frag_a(As, kLd, 32 + m0, k0, lane), a);
      ldsm_x2(frag_bt(Tt, kLy, n0, k0, lane), bb);
      mma_3xtf32(c, a, bb[0], bb[1]);
    }
    const int n = n0 + 2 * t;
    Xs[n * kLy + m0 + g] = c[0];
    Xs[(n + 1) * kLy + m0 + g] = c[1];
    Xs[n * kLy + m0 + g + 8] = c[2];
    Xs[(n + 1) * kLy + m0 + g + 8] = c[3];
    named_bar_sync(1 + (warp & 3), 64);   // Y rows [0, 32) of columns n0.. are in Xs
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    // rows [32, 48) of T([2,3],[2,3]) have columns [32, 48) only
    for (int k0 = 0; k0 < m0 + 16; k0 += 16) {
      uint32_t bb[4];
      ldsm_x4(frag_bt(Xs, kLy, n0, k0, lane), bb);
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        uint32_t a[4];
        ldsm_x4(frag_a(Ts, kLd, 32 + m0, 32 + k0 + 8 * kk, lane), a);
        mma_3xtf32(d, a, bb[2 * kk], bb[2 * kk + 1]);
      }
    }
    *reinterpret_cast<float2 *>(Ts + (32 + m0 + g) * kLd + n) = make_float2(-d[0], -d[1]);
    *reinterpret_cast<float2 *>(Ts + (32 + m0 + g + 8) * kLd + n) = make_float2(-d[2], -d[3]);
  }
  __syncthreads();
}

// Persistent: each CTA loops over (chunk, head) units u = blockIdx.x + i *
// gridDim.x (u = chunk * H + h). The tensor memory, barriers and tensor-map
// prefetches are set up once; while a unit runs, the next unit's K and Q
// tiles are prefetched into L2 and its g and beta into registers, and the
// unit's TMA stores drain while the next unit starts (a store only has to
// finish reading shared memory before that memory is written again).
// Warp roles: all 8 warps share the epilogues. TMEM lane quarter = warp % 4,
// column half = warp / 4.
__global__ void __launch_bounds__(kPrepThreads, 3) gdn_prep_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_kt,
    const __grid_constant__ CUtensorMap tm_tb, const __grid_constant__ CUtensorMap tm_pm,
    const float *__restrict__ g,
    const float *__restrict__ beta, float *__restrict__ gam_out, int H,
    uint32_t *__restrict__ ctrl, const ChunkInfo *__restrict__ table) {
  extern __shared__ uint8_t smem_raw[];
  // Pointer arithmetic (not integer casts) keeps the shared address space.
  uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  grid_launch_dependents();   // the scan may start its prologue on freed SMs

  float *As = reinterpret_cast<float *>(sm + kP_AS);
  float *Ts = reinterpret_cast<float *>(sm + kP_TS);
  float *Xs = reinterpret_cast<float *>(sm + kP_XS);
  float *Tt = reinterpret_cast<float *>(sm + kP_TT);
  float *Gm = reinterpret_cast<float *>(sm + kP_VEC);
  float *Bt = Gm + 64;
  float *Ga = Bt + 64;
  float *Gl = Ga + 64;                     // Gamma log2(e)
  uint64_t *bar_load = reinterpret_cast<uint64_t *>(sm + kP_BAR);
  uint64_t *bar_mma = bar_load + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_load + 2);

  if (tid == 0) {
    abort_flag = 0;
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Everything above overlaps the chunk-map kernel; the chunk table, the
  // chunk count and the error word are read only after it completes.
  grid_dependency_wait();
  const int nunits = (ctrl[0] & kErrBadSeqlens) ? 0 : int(ctrl[1]) * H;
  const int m = (warp & 3) * 32 + lane;   // TMEM lane = row of G
  const int hc = warp >> 2;               // column half
  const uint32_t lane_base = tmem + (uint32_t((warp & 3) * 32) << 16);

  // g and beta of unit u (rows past the sequence end read as 0), one row per
  // thread of the first two warps.
  float g_reg = 0.f, b_reg = 0.f;
  auto fetch_gb = [&](int u) {
    if (tid < kC && u < nunits) {
      const int cu = u / H, hu = u - cu * H;
      const ChunkInfo cf = table[cu];
      const bool ok = tid < cf.len;
      g_reg = ok ? g[size_t(cf.row0 + tid) * H + hu] : 0.f;
      b_reg = ok ? beta[size_t(cf.row0 + tid) * H + hu] : 0.f;
    }
  };
  fetch_gb(blockIdx.x);
  int it = 0;
  for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x, ++it) {
  const int chunk = unit / H, h = unit - chunk * H;
  const ChunkInfo ci = table[chunk];
  const int L = ci.len;
  const bool tr = (h == 0 && tid == 0);   // traced thread (GDN_TRACE builds only)
  (void)tr;
  GDN_TRACE_POINT(tr && chunk < 64, 1, chunk, 0);
  if (tid == 0) {
    // The previous unit's TMA stores read the K/Q and A areas: wait until
    // they have (they need not have reached global memory).
    tma_store_wait_read();
    if (!abort_flag) {
      mbar_arrive_expect_tx(bar_load, 2 * kTile128x64);
      tma_load_3d(sm + kP_KQ, &tm_k, bar_load, 0, h, ci.row0);
      tma_load_3d(sm + kP_KQ + kTile64x64, &tm_q, bar_load, 0, h, ci.row0);
      tma_load_3d(sm + kP_KQ + kTile128x64, &tm_k, bar_load, 64, h, ci.row0);
      tma_load_3d(sm + kP_KQ + kTile128x64 + kTile64x64, &tm_q, bar_load, 64, h, ci.row0);
    }
    const int nu = unit + int(gridDim.x);
    if (nu < nunits) {
      const int cn = nu / H, hn = nu - cn * H;
      const int rn = table[cn].row0;
      tma_prefetch_l2_3d(&tm_k, 0, hn, rn);
      tma_prefetch_l2_3d(&tm_k, 64, hn, rn);
      tma_prefetch_l2_3d(&tm_q, 0, hn, rn);
      tma_prefetch_l2_3d(&tm_q, 64, hn, rn);
    }
  }
  if (tid < kC) {
    Gm[tid] = g_reg;
    Bt[tid] = b_reg;
  }
  fetch_gb(unit + int(gridDim.x));
  __syncthreads();
  if (warp == 0) {  // inclusive cumsum of the 64 log-gates
    const float a0 = Gm[2 * lane], a1 = Gm[2 * lane + 1];
    float s = a0 + a1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float t = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += t;
    }
    const float excl = s - (a0 + a1);
    Gm[2 * lane] = excl + a0;
    Gm[2 * lane + 1] = s;
    constexpr float kLog2e = 1.4426950408889634f;
    Gl[2 * lane] = (excl + a0) * kLog2e;
    Gl[2 * lane + 1] = s * kLog2e;
  }
  const bool loaded = mbar_wait(bar_load, it & 1, ctrl, &abort_flag);
  GDN_TRACE_POINT(tr && chunk < 64, 1, chunk, 1);
  if (loaded && L < kC) {
    // Rows past the sequence end act as k = q = 0 (beta = g = 0 above).
    for (int e = tid; e < (kC - L) * 8; e += kPrepThreads) {
      const int r = L + e / 8, ch = e % 8;
      const uint4 z = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4 *>(sm + kP_KQ + r * 128 + ch * 16) = z;
      *reinterpret_cast<uint4 *>(sm + kP_KQ + kTile64x64 + r * 128 + ch * 16) = z;
      *reinterpret_cast<uint4 *>(sm + kP_KQ + kTile128x64 + r * 128 + ch * 16) = z;
      *reinterpret_cast<uint4 *>(sm + kP_KQ + kTile128x64 + kTile64x64 + r * 128 + ch * 16) = z;
    }
    fence_proxy_async_smem();
  }
  __syncthreads();
  if (!abort_flag && tid == 0) {
    // G = [K; Q] K^T : M = 128 (K rows then Q rows), N = 64, K = 128 (d_k)
    tc_fence_after();
    const uint32_t idesc = make_idesc_bf16(128, 64, 0, 0);
    // One descriptor, k steps added to its start-address field (see the scan's
    // MMA warp): no dependent integer chain between the MMAs.
    const uint64_t dkq = make_sdesc(smem_u32(sm + kP_KQ), 16, 1024);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t d = dkq + uint64_t(((kk >> 2) * kTile128x64 + (kk & 3) * 32) >> 4);
      tc_mma_bf16(tmem, d, d, idesc, kk > 0);
    }
    tc_commit(bar_mma);
  }
  if (tid < kC) {
    Ga[tid] = __expf(Gm[tid]);
    gam_out[size_t(unit) * 128 + tid] = expf(Gm[tid]);                   // gamma_c
    gam_out[size_t(unit) * 128 + 64 + tid] = expf(Gm[kC - 1] - Gm[tid]);  // D_s
  }
  mbar_wait(bar_mma, 0, ctrl, &abort_flag);
  GDN_TRACE_POINT(tr && chunk < 64, 1, chunk, 2);
  tc_fence_after();

  // A[r][s] = beta_r 2^(Gl_r - Gl_s) G[r][s] for s < r (fp32, for the solve);
  // P[c][s] = 2^(Gl_c - Gl_s) G[c][s] for s <= c (bf16 operand tile). Warps 4
  // (A rows 0-31) and 6 (P rows 0-31) hold columns 32-63, all above the
  // diagonal: they write zeros without touching tensor memory.
  const bool zero_warp = (hc == 1) && ((warp & 1) == 0);
  if (!abort_flag) {
    uint32_t r0[32];
    if (!zero_warp) {
      tmem_ld32(lane_base + 32 * hc, r0);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int t = 0; t < 32; ++t) r0[t] = 0u;
    }
    if (m < kC) {
      const int r = m;
      const float br = Bt[r], glr = Gl[r];
#pragma unroll
      for (int t = 0; t < 32; t += 4) {
        const int s = 32 * hc + t;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if (!zero_warp) {
          const float4 gs = lds4(Gl + s);
          a.x = (s + 0 < r) ? br * ex2_approx(glr - gs.x) * __uint_as_float(r0[t + 0]) : 0.f;
          a.y = (s + 1 < r) ? br * ex2_approx(glr - gs.y) * __uint_as_float(r0[t + 1]) : 0.f;
          a.z = (s + 2 < r) ? br * ex2_approx(glr - gs.z) * __uint_as_float(r0[t + 2]) : 0.f;
          a.w = (s + 3 < r) ? br * ex2_approx(glr - gs.w) * __uint_as_float(r0[t + 3]) : 0.f;
        }
        *reinterpret_cast<float4 *>(As + r * kLd + s) = a;
      }
    } else {
      const int c = m - kC;
      const float glc = Gl[c];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int ch = 4 * hc + cc;
        float f[8];
        if (!zero_warp) {
          const float4 g0 = lds4(Gl + ch * 8), g1 = lds4(Gl + ch * 8 + 4);
          const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int s = ch * 8 + e;
            f[e] = (s <= c) ? ex2_approx(glc - gv[e]) * __uint_as_float(r0[8 * cc + e]) : 0.f;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = 0.f;
        }
        *reinterpret_cast<uint4 *>(sm + kP_PST + sw128_offset(c, ch)) =
            make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                       pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (!abort_flag && tid == 0) {
    tma_store_2d(&tm_pm, sm + kP_PST, 0, unit * kC);
    tma_store_commit();
  }
  GDN_TRACE_POINT(tr && chunk < 64, 1, chunk, 3);
  if (!abort_flag) solve_unit_lower_64(As, Ts, Tt, Xs, tid);
  GDN_TRACE_POINT(tr && chunk < 64, 1, chunk, 4);
  // T diag(beta) and T diag(beta gamma) as bf16 K-major operand tiles (A is
  // dead now). Thread: row r, columns [16 q4, 16 q4 + 16); T is lower
  // triangular and its upper blocks are unwritten, so s > r reads as zero.
  {
    const int r = tid >> 2, q4 = tid & 3;
    float fb[16], fg[16];
    if (16 * q4 <= r) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int s0 = 16 * q4 + 4 * i;
        const float4 t = lds4(Ts + r * kLd + s0);
        const float4 bt = lds4(Bt + s0), ga = lds4(Ga + s0);
        const float tv[4] = {t.x, t.y, t.z, t.w}, bv[4] = {bt.x, bt.y, bt.z, bt.w},
                    gv[4] = {ga.x, ga.y, ga.z, ga.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float v = (s0 + e <= r) ? tv[e] * bv[e] : 0.f;
          fb[4 * i + e] = v;
          fg[4 * i + e] = v * gv[e];
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) fb[e] = fg[e] = 0.f;
    }
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int ch = q4 * 2 + cc;
      const float *xb = fb + 8 * cc, *xg = fg + 8 * cc;
      *reinterpret_cast<uint4 *>(sm + kP_TB + sw128_offset(r, ch)) =
          make_uint4(pack_bf16x2(xb[0], xb[1]), pack_bf16x2(xb[2], xb[3]),
                     pack_bf16x2(xb[4], xb[5]), pack_bf16x2(xb[6], xb[7]));
      *reinterpret_cast<uint4 *>(sm + kP_TBG + sw128_offset(r, ch)) =
          make_uint4(pack_bf16x2(xg[0], xg[1]), pack_bf16x2(xg[2], xg[3]),
                     pack_bf16x2(xg[4], xg[5]), pack_bf16x2(xg[6], xg[7]));
    }
  }
  __syncthreads();
  // T is dead: its area now holds diag(D), D_s = exp(Gamma_last - Gamma_s), as a
  // bf16 K-major tile, the B operand that turns K^T into (D K)^T.
  {
    const int r = tid >> 2, q4 = tid & 3;
    const float dr = expf(Gm[kC - 1] - Gm[r]);
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int ch = q4 * 2 + cc;
      float f[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = (ch * 8 + e == r) ? dr : 0.f;
      *reinterpret_cast<uint4 *>(sm + kP_DIAG + sw128_offset(r, ch)) =
          make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                     pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
    }
  }
  fence_proxy_async_smem();
  __syncthreads();
  GDN_TRACE_POINT(tr && chunk < 64, 1, chunk, 5);
  if (!abort_flag && tid == 0) {
    tma_store_2d(&tm_tb, sm + kP_TB, 0, unit * kC);
    tma_store_commit();
    tc_fence_after();
    // W^T    = K^T (T diag(beta gamma))^T : M = 128 (d_k), N = 64, K = 64 -> cols [64, 128)
    // (DK)^T = K^T diag(D)                : M = 128 (d_k), N = 64, K = 64 -> cols [0, 64)
    const uint32_t idesc = make_idesc_bf16(128, 64, 1, 0);
    const uint64_t dkt = make_sdesc(smem_u32(sm + kP_KQ), kTile128x64, 1024);
    const uint64_t dtbg = make_sdesc(smem_u32(sm + kP_TBG), 16, 1024);
    const uint64_t ddg = make_sdesc(smem_u32(sm + kP_DIAG), 16, 1024);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      tc_mma_bf16(tmem + 64, dkt + uint64_t(kk * 2048 >> 4), dtbg + uint64_t(kk * 32 >> 4), idesc,
                  kk > 0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      tc_mma_bf16(tmem, dkt + uint64_t(kk * 2048 >> 4), ddg + uint64_t(kk * 32 >> 4), idesc,
                  kk > 0);
    tc_commit(bar_mma);
  }
  mbar_wait(bar_mma, 1, ctrl, &abort_flag);
  GDN_TRACE_POINT(tr && chunk < 64, 1, chunk, 6);
  if (tid == 0) tma_store_wait_read();   // the P staging lies under the W staging
  tc_fence_after();
  __syncthreads();
  if (!abort_flag) {
    if (hc == 0) {
      // -W, K-major [64 c][128 d]: read W^T (lanes = d, columns = c) as
      // mma-accumulator fragments and store them transposed with stmatrix.
      const int q = warp & 3, mj = lane & 7, mm = lane >> 3;
      const uint32_t wst = smem_u32(sm + kP_WST);
#pragma unroll
      for (int lb = 0; lb < 32; lb += 16) {
#pragma unroll
        for (int cb = 0; cb < 64; cb += 16) {
          uint32_t w8[8];
          tmem_ld16x256_x2(lane_base + (uint32_t(lb) << 16) + 64 + cb, w8);
          tmem_ld_wait();
          uint32_t w[4];
#pragma unroll
          for (int mq = 0; mq < 4; ++mq)
            w[mq] = pack_bf16x2(-__uint_as_float(w8[2 * mq]), -__uint_as_float(w8[2 * mq + 1]));
          const int d0 = q * 32 + lb + 8 * (mm & 1);   // first d index of my matrix
          const int crow = cb + 8 * (mm >> 1) + mj;     // chunk row this thread addresses
          stmatrix_x4_trans(wst + (d0 >> 6) * kTile64x64 + sw128_offset(crow, (d0 & 63) >> 3),
                            w[0], w[1], w[2], w[3]);
        }
      }
    } else {
      // (D K)^T row m (= d) -> [128 d][64 s] staging.
      uint32_t r0[32], r1[32];
      tmem_ld32(lane_base, r0);
      tmem_ld32(lane_base + 32, r1);
      tmem_ld_wait();
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const uint32_t *src = ch < 4 ? r0 : r1;
        const int b = (ch & 3) * 8;
        *reinterpret_cast<uint4 *>(sm + kP_KST + sw128_offset(m, ch)) = make_uint4(
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
      tma_store_2d(&tm_w, sm + kP_WST, 0, unit * kC);
      tma_store_2d(&tm_w, sm + kP_WST + kTile64x64, 64, unit * kC);
      tma_store_2d(&tm_kt, sm + kP_KST, 0, unit * kD);
      tma_store_commit();
    }
    GDN_TRACE_POINT(tr && chunk < 64, 1, chunk, 7);
  }
  __syncthreads();   // shared memory and tensor memory free for the next unit
  }
  if (tid == 0) tma_store_wait_all();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ===================================================================== scan
// One stage (one chunk of one head), as the B operands of three wide MMAs:
//   BXZ  2 x [ -W rows 0-63 | Q rows 64-127 ]  (128 rows, K = d_k in two blocks)
//   BU   [ T diag(beta) rows 0-63 | zeros ]    (128 rows, K = 64 tokens)
//   BSY  stage 0: [ (D K)^T rows 0-127 | P rows 128-191 ]  (192 rows, K = 64 tokens)
//        stage 1: [ P rows 0-63 | (D K)^T rows 64-191 ]
// plus V (the MN-major A operand of U^T). The zero half of BU is written
// once; TMA never touches it. The two BSY orders put dS in the same tensor
// memory columns for every chunk and Y in one of two buffers (Y0 after dS,
// Y1 before it), so SY(c+1) never waits for the output warps to finish Y(c).
// The per-chunk decay factors (gamma[64], D[64]) travel in a separate 4-slot
// ring so the output warps never hold a stage.
constexpr uint32_t kS_BXZ = 0;                        // 32 KB
constexpr uint32_t kS_V = kS_BXZ + 2 * kTile128x64;   // 16 KB, 2 x [64 s][64 d]
constexpr uint32_t kS_BU = kS_V + 2 * kTile64x64;     // 16 KB
constexpr uint32_t kS_BSY = kS_BU + kTile128x64;      // 24 KB
constexpr uint32_t kStageBytes = kS_BSY + kTile128x64 + kTile64x64;   // 88 KB
constexpr int kStages = 2, kGamSlots = 4;
constexpr int kPrefetchAhead = 2;     // chunks prefetched into L2 ahead of the stage loads
constexpr uint32_t kS_OST = kStages * kStageBytes;            // O staging, 2 x [64 c][64 d]
constexpr uint32_t kS_GAM = kS_OST + 2 * kTile64x64;          // kGamSlots x 128 fp32
constexpr uint32_t kS_BAR = kS_GAM + kGamSlots * 512;         // mbarriers, tmem slot, flags
constexpr uint32_t kS_END = kS_BAR + 256;
constexpr uint32_t kScanSmem = kS_END;   // the dynamic window starts 1024-aligned (checked)
constexpr uint32_t kStageTxA = kS_BSY - kTile64x64;   // BXZ, V and Tb (not the zero tile)
constexpr uint32_t kStageTxB = kTile128x64 + kTile64x64;   // (D K)^T and P
constexpr int kScanThreads = 512;
// TMEM columns (fp32 accumulators, then the bf16 A operands held in TMEM)
constexpr uint32_t kT_XZ = 0;     // [X | Z] = [U^T - S W^T | S Q^T]      fp32 [128][128]
constexpr uint32_t kT_Y1 = 128;   // Y of odd chunks  = V_new^T P^T       fp32 [128][64]
constexpr uint32_t kT_DS = 192;   // dS = V_new^T (D K)                    fp32 [128][128]
constexpr uint32_t kT_Y0 = 320;   // Y of even chunks                      fp32 [128][64]
constexpr uint32_t kT_S = 384;    // S        bf16 [128][128] (64 columns)
constexpr uint32_t kT_A1 = 448;   // V_new^T  bf16 [128][64]  (32 columns)
// Named barriers (0 is __syncthreads)
constexpr uint32_t kBarOut = 2;
// The chain warps hand each finished epilogue to the MMA warp through a
// hardware named barrier (chain warps bar.arrive, the MMA warp bar.sync):
// kBarA1 after V_new^T is in tensor memory, kBarS after S_{c+1} is. A chain
// warp cannot arrive twice before the MMA warp syncs once: its next arrival
// needs an MMA result that the MMA warp only issues after that sync.
constexpr uint32_t kBarA1 = 3, kBarS = 4;
constexpr uint32_t kChainHandoff = 8 * 32 + 32;   // 8 chain warps + the MMA warp
// Barrier slots in the kS_BAR area
// y_full[b] completes when Y buffer b holds a new chunk; the output warps wait
// on it, the chain on s_full. (One barrier for both would let a slow output
// warp miss a phase: it reports Z consumed before it waits for Y.)
// Each stage has two parts with their own full/empty pairs: part A (BXZ, V,
// BU) is last read by XZ(c) and part B (BSY) by SY(c), so the next loads of
// part A start while SY(c) and the S epilogue still run.
constexpr int kB_FULLA = 0, kB_EMPTYA = 2, kB_FULLB = 4, kB_EMPTYB = 6, kB_GFULL = 8,
              kB_GEMPTY = 12, kB_XFULL = 16, kB_SFULL = 17, kB_YFULL = 18, kB_ZFREE = 20,
              kB_DRAIN = 21, kB_COUNT = 22;

// Warp roles (16 warps). Every role runs its loop with all 32 lanes, so the
// lanes of a warp wait on barriers together; one lane issues TMA copies,
// MMAs and arrivals.
//   warp 0        TMA producer
//   warp 1        TMEM allocation and every tcgen05.mma
//   warps 4-11    state chain: two warpgroups, warpgroup h owns columns
//                 [32h, 32h+32) of V_new and [64h, 64h+64) of S; thread =
//                 TMEM lane = row i of d_v; the fp32 S lives in its registers,
//                 its bf16 copy (an MMA operand) in tensor memory. Each finished
//                 epilogue is handed to the MMA warp through a named barrier.
//   warps 12-15   output: O = diag(gamma) Z + Y, staged for TMA stores
// Per chunk c the tensor core runs three wide products:
//   U(c)   [X|Z]  = V^T [Tb | 0]^T            (4 MMAs, N = 128)  -- before S_c is known
//   XZ(c)  [X|Z] += S [-W | Q]^T              (8 MMAs, N = 128)  -> X = V_new^T, Z = S Q^T
//   SY(c)  [dS|Y] = V_new^T [(DK)^T | P]^T    (4 MMAs, N = 192)
// and the chain is XZ -> V_new epilogue -> SY -> S epilogue -> XZ(c+1), with
// U(c+1) running during the S epilogue. The MMA warp does its other waits
// (output done with Z, next stage loaded) while the V_new epilogue runs, so
// only the two epilogue handshakes sit on the chain.
__global__ void __launch_bounds__(kScanThreads, 1) gdn_scan_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_v,
    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_kt,
    const __grid_constant__ CUtensorMap tm_tb, const __grid_constant__ CUtensorMap tm_pm,
    const __grid_constant__ CUtensorMap tm_gam, const __grid_constant__ CUtensorMap tm_o,
    const float *__restrict__ s0, float *__restrict__ sN, __nv_bfloat16 *__restrict__ o, int H,
    uint32_t *__restrict__ ctrl, const ChunkInfo *__restrict__ table,
    const int32_t *__restrict__ seq_first, int split, float *__restrict__ sN_trans,
    int sN_group) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = smem_raw;                 // pointer arithmetic keeps the shared space
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Sequences (or segments of sequences) n = blockIdx.x. With split > 0, the
  // CTAs from `split` on run segment n = blockIdx.x - split as a transition:
  // V = 0 (no U product) from S = I, writing the resulting state to sN_trans.
  // o == nullptr: no output is written. The final state of n goes to
  // sN[n / sN_group] when n % sN_group == sN_group - 1 (sN_group = 1: every n).
  const bool trans = split > 0 && int(blockIdx.x) >= split;
  const int n = trans ? int(blockIdx.x) - split : int(blockIdx.x), h = blockIdx.y;
  const bool write_o = o != nullptr;
  if (smem_u32(sm) & 1023) {              // swizzled tiles need a 1024-aligned base
    grid_dependency_wait();               // the error word is the map kernel's until then
    if (tid == 0) atomicOr(ctrl, kErrLayout);
    return;
  }
  const bool tr = (n == 0 && h == 0);     // traced CTA (GDN_TRACE builds only)
  (void)tr;

  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kS_BAR);
  uint64_t *full_a = bars + kB_FULLA, *empty_a = bars + kB_EMPTYA;
  uint64_t *full_b = bars + kB_FULLB, *empty_b = bars + kB_EMPTYB;
  uint64_t *gfull = bars + kB_GFULL, *gempty = bars + kB_GEMPTY;
  uint64_t *x_full = bars + kB_XFULL, *s_full = bars + kB_SFULL, *y_full = bars + kB_YFULL;
  uint64_t *z_free = bars + kB_ZFREE, *drain = bars + kB_DRAIN;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kB_COUNT);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  if (tid == 0) {
    *abort_flag = 0;
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_kt);
    tma_prefetch_desc(&tm_tb);
    tma_prefetch_desc(&tm_pm);
    tma_prefetch_desc(&tm_gam);
    tma_prefetch_desc(&tm_o);
    for (int b = 0; b < kB_COUNT; ++b) {
      uint32_t count = 1;
      if (b >= kB_GEMPTY && b < kB_GEMPTY + 4) count = 2;        // MMA warp + output
      mbar_init(bars + b, count);
    }
    fence_mbar_init();
  }
  // The zero half of BU in both stages.
  for (int e = tid; e < kStages * (kTile64x64 / 16); e += kScanThreads) {
    const int st = e / (kTile64x64 / 16), off = e % (kTile64x64 / 16);
    *reinterpret_cast<uint4 *>(sm + st * kStageBytes + kS_BU + kTile64x64 + off * 16) =
        make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Waits inside the role loops: after an abort they return at once, so every
  // loop runs to its end and named barriers stay in step.
  auto wait = [&](uint64_t *bar, uint32_t parity) { mbar_wait(bar, parity, ctrl, abort_flag); };
  // The chunk table and the prep kernel's outputs are read only after the
  // kernels that write them have completed (the chain warps first load the
  // initial state, which no earlier kernel of this call writes).
  int c0 = 0, nch = 0;
  auto read_chunks = [&]() {
    grid_dependency_wait();
    if (!(ctrl[0] & kErrBadSeqlens)) {
      c0 = seq_first[n];
      nch = seq_first[n + 1] - c0;
    }
  };
  if (warp < 4 || warp >= 12) read_chunks();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    for (int c = 0; c < nch && !*abort_flag; ++c) {
      const int st = c & 1, gs = c & 3;
      const ChunkInfo ci = table[c0 + c];
      const int unit = (c0 + c) * H + h;
      uint8_t *sb = sm + st * kStageBytes;
      if (c >= 2) wait(empty_a + st, ((c >> 1) - 1) & 1);
      if (lane == 0) {
        GDN_TRACE_POINT(tr, 0, c, 0);
        // Only what this CTA's products read: a run without output needs
        // neither Q nor P, a transition run neither V nor T diag(beta).
        mbar_arrive_expect_tx(full_a + st, (write_o ? kStageTxA : kStageTxA - kTile128x64) -
                                               (trans ? 2 * kTile64x64 + kTile64x64 : 0u));
        tma_load_2d(sb + kS_BXZ, &tm_w, full_a + st, 0, unit * kC);
        tma_load_2d(sb + kS_BXZ + kTile128x64, &tm_w, full_a + st, 64, unit * kC);
        if (write_o) {
          tma_load_3d(sb + kS_BXZ + kTile64x64, &tm_q, full_a + st, 0, h, ci.row0);
          tma_load_3d(sb + kS_BXZ + kTile128x64 + kTile64x64, &tm_q, full_a + st, 64, h,
                      ci.row0);
        }
        if (!trans) {
          tma_load_3d(sb + kS_V, &tm_v, full_a + st, 0, h, ci.row0);
          tma_load_3d(sb + kS_V + kTile64x64, &tm_v, full_a + st, 64, h, ci.row0);
          tma_load_2d(sb + kS_BU, &tm_tb, full_a + st, 0, unit * kC);
        }
      }
      __syncwarp();
      if (c >= 2) wait(empty_b + st, ((c >> 1) - 1) & 1);
      if (lane == 0) {
        // Without output, (D K)^T goes first in both stages and P is not loaded.
        const bool swap = st && write_o;
        mbar_arrive_expect_tx(full_b + st, write_o ? kStageTxB : kTile128x64);
        tma_load_2d(sb + kS_BSY + (swap ? kTile64x64 : 0u), &tm_kt, full_b + st, 0, unit * kD);
        if (write_o)
          tma_load_2d(sb + kS_BSY + (st ? 0u : kTile128x64), &tm_pm, full_b + st, 0, unit * kC);
        // The loads above take about one chunk period to land from HBM; the
        // chunk after next goes to L2 now, so its own loads come from L2.
        if (c + kPrefetchAhead < nch) {
          const ChunkInfo cp = table[c0 + c + kPrefetchAhead];
          const int up = (c0 + c + kPrefetchAhead) * H + h;
          tma_prefetch_l2_2d(&tm_w, 0, up * kC);
          tma_prefetch_l2_2d(&tm_w, 64, up * kC);
          tma_prefetch_l2_2d(&tm_kt, 0, up * kD);
          if (write_o) {
            tma_prefetch_l2_3d(&tm_q, 0, h, cp.row0);
            tma_prefetch_l2_3d(&tm_q, 64, h, cp.row0);
            tma_prefetch_l2_2d(&tm_pm, 0, up * kC);
          }
          if (!trans) {
            tma_prefetch_l2_3d(&tm_v, 0, h, cp.row0);
            tma_prefetch_l2_3d(&tm_v, 64, h, cp.row0);
            tma_prefetch_l2_2d(&tm_tb, 0, up * kC);
          }
        }
      }
      __syncwarp();
      if (c >= 4) wait(gempty + gs, ((c >> 2) - 1) & 1);
      if (lane == 0) {
        mbar_arrive_expect_tx(gfull + gs, 512);
        tma_load_2d(sm + kS_GAM + gs * 512, &tm_gam, gfull + gs, 0, unit);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Without output, Z and Y are not needed: U and XZ shrink to X (N = 64),
    // SY to dS (N = 128, (D K)^T then first in both stages).
    const uint32_t id_u = make_idesc_bf16(128, write_o ? 128 : 64, 1, 0);   // V^T [Tb|0]^T
    const uint32_t id_xz = make_idesc_bf16(128, write_o ? 128 : 64, 0, 0);  // S [-W|Q]^T
    const uint32_t id_sy = make_idesc_bf16(128, write_o ? 192 : 128, 0, 0); // A1 [(DK)^T|P]^T
    const bool issuer = lane == 0;
    // Shared-memory descriptors of the operand tiles of both stages, built
    // once: a single issuing thread pays the latency of every dependent
    // integer op, so rebuilding descriptors between MMAs doubles the issue
    // time. A k step is added to the start-address field (smem offsets >> 4
    // stay below 2^14, so the field never carries into the next one).
    uint64_t dV[kStages], dBU[kStages], dBXZ[kStages], dBSY[kStages];
#pragma unroll
    for (int st = 0; st < kStages; ++st) {
      const uint32_t sb = smem_u32(sm + st * kStageBytes);
      dV[st] = make_sdesc(sb + kS_V, kTile64x64, 1024);
      dBU[st] = make_sdesc(sb + kS_BU, 16, 1024);
      dBXZ[st] = make_sdesc(sb + kS_BXZ, 16, 1024);
      dBSY[st] = make_sdesc(sb + kS_BSY, 16, 1024);
    }
    // U(c) into [X|Z]. The caller has seen chunk c loaded and the output
    // warps done reading Z of chunk c - 1.
    auto issue_u = [&](int c) {
      if (issuer) {
        const uint64_t da = (c & 1) ? dV[1] : dV[0], db = (c & 1) ? dBU[1] : dBU[0];
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_bf16(tmem + kT_XZ, da + uint64_t(kk * 2048 >> 4), db + uint64_t(kk * 32 >> 4),
                      id_u, kk > 0);
      }
      __syncwarp();
    };
    // XZ(c) += S_c [-W|Q]^T, reading the bf16 copy of S_c.
    auto issue_xz = [&](int c) {
      if (issuer) {
        GDN_TRACE_POINT(tr, 0, c, 1);
        const uint64_t db = (c & 1) ? dBXZ[1] : dBXZ[0];
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // a transition run has no U: XZ starts the sum
          tc_mma_bf16_ts(tmem + kT_XZ, tmem + kT_S + 8 * kk,
                         db + uint64_t(((kk >> 2) * kTile128x64 + (kk & 3) * 32) >> 4), id_xz,
                         (kk > 0) || !trans);
        tc_commit(x_full);
        tc_commit(empty_a + (c & 1));     // U(c) and XZ(c) were the last readers of part A
      }
      __syncwarp();
    };
    if (nch > 0) {
      wait(full_a, 0);
      if (!trans) issue_u(0);
    }
    named_bar_sync(kBarS, kChainHandoff);     // S_0 stored (the chain hands it over even if nch = 0)
    if (nch > 0) issue_xz(0);
    for (int c = 0; c < nch; ++c) {
      const int st = c & 1, gs = c & 3;
      const bool more = c + 1 < nch;
      wait(full_b + st, (c >> 1) & 1);    // (D K)^T and P of chunk c (while XZ(c) runs)
      named_bar_sync(kBarA1, kChainHandoff);  // V_new^T of chunk c in tensor memory
      GDN_TRACE_POINT(tr && issuer, 0, c, 6);
      if (issuer) {
        const uint64_t db = st ? dBSY[1] : dBSY[0];
        tc_fence_after();
        // even chunks: D = [dS | Y0] at kT_DS; odd: D = [Y1 | dS] at kT_Y1
        // (without output: D = dS at kT_DS for every chunk)
        const uint32_t d = tmem + ((st && write_o) ? kT_Y1 : kT_DS);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_bf16_ts(d, tmem + kT_A1 + 8 * kk, db + uint64_t(kk * 32 >> 4), id_sy, kk > 0);
        tc_commit(s_full);
        tc_commit(y_full + st);
        tc_commit(empty_b + st);          // SY(c) was the last reader of part B
        GDN_TRACE_POINT(tr, 0, c, 12);
      }
      __syncwarp();
      // Off the chain (SY(c) and the S epilogue are running): U(c+1) needs the
      // output warps done with Z(c) and part A of chunk c + 1.
      if (more) {
        wait(z_free, c & 1);
        GDN_TRACE_POINT(tr && issuer, 0, c, 13);
        wait(full_a + (st ^ 1), ((c + 1) >> 1) & 1);
        GDN_TRACE_POINT(tr && issuer, 0, c, 14);
        if (!trans) issue_u(c + 1);
      }
      named_bar_sync(kBarS, kChainHandoff);   // S_{c+1} stored, decay factors of c read
      GDN_TRACE_POINT(tr && issuer, 0, c, 8);
      if (more) issue_xz(c + 1);
      if (issuer) mbar_arrive(gempty + gs);
      __syncwarp();
    }
    if (issuer) tc_commit(drain);         // fires once every MMA above has completed
    __syncwarp();
    // Waited for even after an abort (bounded): tensor memory is freed below.
    volatile int keep_waiting = 0;
    mbar_wait(drain, 0, ctrl, &keep_waiting);
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ state chain
    const int hh = (warp - 4) >> 2;                     // column half
    const int i = ((warp & 3) << 5) + lane;             // TMEM lane = row of d_v
    const uint32_t lane_base = tmem + (uint32_t((warp & 3) * 32) << 16);
    const bool tl = tr && warp == 4 && lane == 0;       // traced lane
    (void)tl;
    float S[64];                                        // S[i][64 hh + t], fp32 master
    {
      const float *src = (s0 && !trans) ? s0 + (size_t(n) * H + h) * kD * kD : nullptr;
#pragma unroll
      for (int t = 0; t < 64; ++t)
        S[t] = trans ? (64 * hh + t == i ? 1.f : 0.f) : (src ? src[size_t(64 * hh + t) * kD + i] : 0.f);
    }
    read_chunks();
    // bf16 copy of S (row i, columns [64 hh, 64 hh + 64)) into tensor memory,
    // then hand it to the MMA warp.
    auto store_state = [&]() {
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) pk[t] = pack_bf16x2(S[32 * q + 2 * t], S[32 * q + 2 * t + 1]);
        tmem_st16(lane_base + kT_S + 32 * hh + 16 * q, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      named_bar_arrive(kBarS, kChainHandoff);
    };
    store_state();
    for (int c = 0; c < nch; ++c) {
      const int gs = c & 3;
      wait(x_full, c & 1);
      GDN_TRACE_POINT(tl, 0, c, 5);
      tc_fence_after();
      // V_new^T[i][s] = X[i][s] for s in [32 hh, 32 hh + 32): bf16 back to TMEM
      // as the A operand of SY.
      {
        uint32_t x[32], a1[16];
        tmem_ld32(lane_base + kT_XZ + 32 * hh, x);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e)
          a1[e] = pack_bf16x2(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1]));
        tmem_st16(lane_base + kT_A1 + 16 * hh, a1);
      }
      tmem_st_wait();
      tc_fence_before();
      named_bar_arrive(kBarA1, kChainHandoff);
      // S <- gamma_last S + dS on columns [64 hh, 64 hh + 64)
      wait(gfull + gs, (c >> 2) & 1);
      const float gl = reinterpret_cast<const float *>(sm + kS_GAM + gs * 512)[kC - 1];
      wait(s_full, c & 1);
      GDN_TRACE_POINT(tl, 0, c, 7);
      tc_fence_after();
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        uint32_t d[32];
        tmem_ld32(lane_base + kT_DS + 64 * hh + 32 * b, d);
        tmem_ld_wait();
        GDN_TRACE_POINT(tl && b == 0, 0, c, 3);
#pragma unroll
        for (int t = 0; t < 32; t += 2) {
          const float2 r = ffma2(make_float2(gl, gl), make_float2(S[32 * b + t], S[32 * b + t + 1]),
                                 make_float2(__uint_as_float(d[t]), __uint_as_float(d[t + 1])));
          S[32 * b + t] = r.x;
          S[32 * b + t + 1] = r.y;
        }
      }
      store_state();
      GDN_TRACE_POINT(tl, 0, c, 4);
      GDN_TRACE_POINT(tr && warp == 11 && lane == 0, 0, c, 15);
    }
    float *sNp = trans ? sN_trans : sN;
    const int sN_idx = trans ? n : n / sN_group;
    if (sNp && (trans || n % sN_group == sN_group - 1) && !*abort_flag) {
      float *dst = sNp + (size_t(sN_idx) * H + h) * kD * kD;
#pragma unroll
      for (int t = 0; t < 64; ++t) dst[size_t(64 * hh + t) * kD + i] = S[t];
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ output
    // O[c'][i] = gamma_c' Z[i][c'] + Y[i][c'] (Z, Y are O^T in TMEM). Each warp
    // reads its 32 lanes as mma-accumulator fragments (16 lanes x 8 columns),
    // Z as soon as XZ is done (so U of the next chunk may overwrite it), Y
    // after SY, and writes O transposed into the swizzled staging tile with
    // stmatrix, 16 bytes per row; a TMA store (whole chunks) or a 16-byte copy
    // loop (a sequence's last, partial chunk) moves the tile to o.
    const int q = warp & 3, ot = tid - 384;           // output thread 0..127
    const uint32_t lane_q = tmem + (uint32_t(q * 32) << 16);
    const bool leader = (warp == 12 && lane == 0);
    const uint32_t ost = smem_u32(sm + kS_OST);
    const int fc = 2 * (lane & 3);                     // fragment column pair
    const int mj = lane & 7, mm = lane >> 3;           // stmatrix: row j of matrix m
    for (int c = 0; c < nch && !write_o; ++c) {
      // No output: keep only this role's side of the barrier protocol.
      const int gs = c & 3;
      wait(x_full, c & 1);
      if (leader) mbar_arrive(z_free);
      wait(gfull + gs, (c >> 2) & 1);
      if (leader) mbar_arrive(gempty + gs);
      __syncwarp();
    }
    for (int c = 0; c < nch && write_o; ++c) {
      const int gs = c & 3;
      const float *gam = reinterpret_cast<const float *>(sm + kS_GAM + gs * 512);
      const ChunkInfo ci = table[c0 + c];
      const bool whole = ci.len == kC;
      uint32_t z[2][32], ynext[8];
      wait(x_full, c & 1);
      tc_fence_after();
      tmem_ld16x256_x8(lane_q + kT_XZ + 64, z[0]);
      tmem_ld16x256_x8(lane_q + (16u << 16) + kT_XZ + 64, z[1]);
      tmem_ld_wait();
      tc_fence_before();
      named_bar_sync(kBarOut, 128);
      if (leader) mbar_arrive(z_free);
      wait(gfull + gs, (c >> 2) & 1);
      if (leader) tma_store_wait_read();     // staging free again
      named_bar_sync(kBarOut, 128);
      wait(y_full + (c & 1), (c >> 1) & 1);
      GDN_TRACE_POINT(tr && leader, 0, c, 9);
      const uint32_t ycol = (c & 1) ? kT_Y1 : kT_Y0;
      tc_fence_after();
#pragma unroll
      for (int lb = 0; lb < 2; ++lb) {
#pragma unroll
        for (int cbi = 0; cbi < 4; ++cbi) {
          const int cb = 16 * cbi;
          uint32_t y[8];
          if ((cbi & 1) == 0) {              // two loads in flight per wait
            tmem_ld16x256_x2(lane_q + (uint32_t(16 * lb) << 16) + ycol + cb, y);
            tmem_ld16x256_x2(lane_q + (uint32_t(16 * lb) << 16) + ycol + cb + 16, ynext);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = ynext[e];
          }
          const float2 g0 = *reinterpret_cast<const float2 *>(gam + cb + fc);
          const float2 g1 = *reinterpret_cast<const float2 *>(gam + cb + 8 + fc);
          uint32_t w[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const float2 gg = (m < 2) ? g0 : g1;
            const int k = 2 * m;
            w[m] = pack_bf16x2(
                fmaf(gg.x, __uint_as_float(z[lb][8 * cbi + k]), __uint_as_float(y[k])),
                fmaf(gg.y, __uint_as_float(z[lb][8 * cbi + k + 1]), __uint_as_float(y[k + 1])));
          }
          // matrices: 0 = (lanes +0..7, cols +0..7), 1 = (lanes +8..15, cols +0..7),
          //           2 = (lanes +0..7, cols +8..15), 3 = (lanes +8..15, cols +8..15)
          const int i0 = q * 32 + 16 * lb + 8 * (mm & 1);  // first d_v index of my matrix
          const int crow = cb + 8 * (mm >> 1) + mj;        // token row this thread addresses
          const uint32_t addr =
              ost + (i0 >> 6) * kTile64x64 + sw128_offset(crow, (i0 & 63) >> 3);
          stmatrix_x4_trans(addr, w[0], w[1], w[2], w[3]);
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      named_bar_sync(kBarOut, 128);
      GDN_TRACE_POINT(tr && leader, 0, c, 11);
      if (leader) {
        mbar_arrive(gempty + gs);
        if (whole && !*abort_flag) {
          tma_store_3d(&tm_o, sm + kS_OST, 0, h, ci.row0);
          tma_store_3d(&tm_o, sm + kS_OST + kTile64x64, 64, h, ci.row0);
          tma_store_commit();
        }
        GDN_TRACE_POINT(tr, 0, c, 10);
      }
      __syncwarp();
      if (!whole && !*abort_flag) {
        // rows [0, len) of the tile, 16 bytes at a time
        for (int e = ot; e < ci.len * 16; e += 128) {
          const int row = e >> 4, k = e & 15;
          const uint4 v = *reinterpret_cast<const uint4 *>(
              sm + kS_OST + (k >> 3) * kTile64x64 + sw128_offset(row, k & 7));
          *reinterpret_cast<uint4 *>(o + (size_t(ci.row0 + row) * H + h) * kD + 8 * k) = v;
        }
      }
    }
    if (leader) tma_store_wait_all();
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================ segment composition
// For a sequence whose state scan was split into `segs` segments: the first
// pass gave each segment's state from S = 0 (H_g, in hbuf) and its transition
// (the state from S = I with V = 0, P_g, in pbuf), so S_{g+1} = S_g P_g + H_g
// (the chunk map S -> S (gamma_last I - W^T D K) + U^T D K is affine in S).
// In the stored orientation X = S^T ([d_k][d_v]) that is X_{g+1} = P~_g X_g +
// H~_g, where P~_g is pbuf's stored matrix. Every column of X evolves alone,
// so one CTA owns 16 columns of one (sequence, head); fp32 throughout.
// Writes X_g, the start state of segment g, to sstart.
__global__ void __launch_bounds__(256) gdn_segment_combine_kernel(
    const float *__restrict__ s0, const float *__restrict__ hbuf,
    const float *__restrict__ pbuf, float *__restrict__ sstart, int H, int segs,
    const uint32_t *__restrict__ ctrl) {
  __shared__ __align__(16) float X[kD][16];
  const int b = blockIdx.x / H, h = blockIdx.x - b * H, col0 = 16 * blockIdx.y;
  const int tid = threadIdx.x;
  if (ctrl[0] & kErrBadSeqlens) return;
  for (int e = tid; e < kD * 16; e += blockDim.x) {
    const int j = e >> 4, c = e & 15;
    X[j][c] = s0 ? s0[((size_t(b) * H + h) * kD + j) * kD + col0 + c] : 0.f;
  }
  __syncthreads();
  const int j = tid >> 1, c0 = (tid & 1) * 8;   // this thread's row and 8 columns
  for (int gi = 0; gi < segs; ++gi) {
    const size_t base = ((size_t(b) * segs + gi) * H + h) * kD * kD;
    float4 *dst = reinterpret_cast<float4 *>(sstart + base + size_t(j) * kD + col0 + c0);
    dst[0] = *reinterpret_cast<const float4 *>(&X[j][c0]);
    dst[1] = *reinterpret_cast<const float4 *>(&X[j][c0 + 4]);
    if (gi == segs - 1) break;
    const float4 h0 = *reinterpret_cast<const float4 *>(hbuf + base + size_t(j) * kD + col0 + c0);
    const float4 h1 =
        *reinterpret_cast<const float4 *>(hbuf + base + size_t(j) * kD + col0 + c0 + 4);
    float acc[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
    const float4 *prow = reinterpret_cast<const float4 *>(pbuf + base + size_t(j) * kD);
#pragma unroll 4
    for (int m4 = 0; m4 < kD / 4; ++m4) {
      const float4 p = prow[m4];
      const float pv[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 xa = *reinterpret_cast<const float4 *>(&X[4 * m4 + e][c0]);
        const float4 xb = *reinterpret_cast<const float4 *>(&X[4 * m4 + e][c0 + 4]);
        acc[0] = fmaf(pv[e], xa.x, acc[0]); acc[1] = fmaf(pv[e], xa.y, acc[1]);
        acc[2] = fmaf(pv[e], xa.z, acc[2]); acc[3] = fmaf(pv[e], xa.w, acc[3]);
        acc[4] = fmaf(pv[e], xb.x, acc[4]); acc[5] = fmaf(pv[e], xb.y, acc[5]);
        acc[6] = fmaf(pv[e], xb.z, acc[6]); acc[7] = fmaf(pv[e], xb.w, acc[7]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 8; ++e) X[j][c0 + e] = acc[e];
    __syncthreads();
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

// [rows, inner] 2-D map with box (box_inner, box_rows).
bool map_2d(CUtensorMap *m, const void *base, CUtensorMapDataType t, int esize, long long rows,
            int inner, int box_inner, int box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cuuint64_t(inner), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(inner) * esize};
  cuuint32_t box[2] = {cuuint32_t(box_inner), cuuint32_t(box_rows)};
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
    CUtensorMap mq, mk, mv, mo, mw, mkt, mtb, mpm, mgm;
    if (!map_tokens(&mq, q, rows, H) || !map_tokens(&mk, k, rows, H) ||
        !map_tokens(&mv, v, rows, H) || !map_tokens(&mo, o, rows, H) ||
        !map_2d(&mw, base + L.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kC, kD, 64, kC,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mkt, base + L.kt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kD, 64, 64, kD,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mtb, base + L.tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kC, 64, 64, kC,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mpm, base + L.pm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kC, 64, 64, kC,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mgm, base + L.gam, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, units, 128, 128, 1,
                CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(gdn_prep_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kPrepSmem);
    if (e != cudaSuccess) return e;
    prof_record(g_profile.prep, s);
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long prep_ctas = std::min<long long>(units, 3LL * sms);
    // Both kernels start with programmatic dependent launch: their prologues
    // overlap the tail of the kernel before them.
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(prep_ctas));
    cfg.blockDim = dim3(kPrepThreads);
    cfg.dynamicSmemBytes = kPrepSmem;
    cfg.stream = s;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, gdn_prep_kernel, mq, mk, mw, mkt, mtb, mpm, g, beta,
                           reinterpret_cast<float *>(base + L.gam), H, ctrl, table);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gdn_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kScanSmem);
    if (e != cudaSuccess) return e;
    prof_record(g_profile.scan, s);
    cfg.blockDim = dim3(kScanThreads);
    cfg.dynamicSmemBytes = kScanSmem;
    if (L.segs <= 1) {
      cfg.gridDim = dim3(N, H);
      return cudaLaunchKernelEx(&cfg, gdn_scan_kernel, mq, mv, mw, mkt, mtb, mpm, mgm, mo, s0,
                                sN, static_cast<__nv_bfloat16 *>(o), H, ctrl,
                                static_cast<const ChunkInfo *>(table), seq_first, 0,
                                static_cast<float *>(nullptr), 1);
    }
    // Segmented state scan (few long sequences): three passes over B * segs
    // segments. (1) every segment from S = 0 and as a transition, no output;
    // (2) the segments' start states; (3) every segment from its start state,
    // writing o and, for each sequence's last segment, the final state.
    const int nseg = B * L.segs;
    const int32_t *seg_first = reinterpret_cast<const int32_t *>(base + L.seg_first);
    float *hbuf = reinterpret_cast<float *>(base + L.hbuf);
    float *pbuf = reinterpret_cast<float *>(base + L.pbuf);
    float *sstart = reinterpret_cast<float *>(base + L.sstart);
    cfg.gridDim = dim3(2 * nseg, H);
    e = cudaLaunchKernelEx(&cfg, gdn_scan_kernel, mq, mv, mw, mkt, mtb, mpm, mgm, mo,
                           static_cast<const float *>(nullptr), hbuf,
                           static_cast<__nv_bfloat16 *>(nullptr), H, ctrl,
                           static_cast<const ChunkInfo *>(table), seg_first, nseg, pbuf, 1);
    if (e != cudaSuccess) return e;
    gdn_segment_combine_kernel<<<dim3(B * H, kD / 16), 256, 0, s>>>(s0, hbuf, pbuf, sstart, H,
                                                                   L.segs, ctrl);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // A plain launch: the start states come from the kernel just before it.
    cfg.gridDim = dim3(nseg, H);
    cfg.numAttrs = 0;
    return cudaLaunchKernelEx(&cfg, gdn_scan_kernel, mq, mv, mw, mkt, mtb, mpm, mgm, mo,
                              static_cast<const float *>(sstart), sN,
                              static_cast<__nv_bfloat16 *>(o), H, ctrl,
                              static_cast<const ChunkInfo *>(table), seg_first, 0,
                              static_cast<float *>(nullptr), L.segs);
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

#ifdef GDN_TRACE
// Trace builds only: copy the phase timestamps to `host` (2*64*16 u64).
extern "C" int gdn_trace_fetch(unsigned long long *host) {
  return cudaMemcpyFromSymbol(host, gdn::g_gdn_trace, sizeof(gdn::g_gdn_trace)) == cudaSuccess
             ? 0
             : -1;
}
#endif
