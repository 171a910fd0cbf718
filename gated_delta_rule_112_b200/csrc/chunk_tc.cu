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
__device__ unsigned long long g_gdn_cta_ns[1024][4];   // per scan CTA: start, XZ(0), last XZ, end
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

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
constexpr uint32_t kP_TT = kP_KQ + kTile128x64 + kTile64x64;   // solve: T transposed, fp32 [48][36], over Q of block 1
constexpr uint32_t kP_AS = kP_KQ + 2 * kTile128x64;  // A, fp32 [64][68]; after the solve it
constexpr uint32_t kP_TB = kP_AS;                    //   holds T diag(beta)       (bf16 64x64)
constexpr uint32_t kP_TBG = kP_AS + kTile64x64;      //   and   T diag(beta gamma) (bf16 64x64)
constexpr uint32_t kP_TS = kP_AS + 64 * kLd * 4;     // T, fp32 [64][68]; then the (D K)^T
constexpr uint32_t kP_KST = kP_TS;                   //   staging [128 d][64 s] (bf16, 16 KB)
constexpr int kLy = 36;                              // fp32 row stride of the solve scratch
constexpr uint32_t kP_XS = kP_TS + 64 * kLd * 4;     // solve scratch, fp32 [32][36]
static_assert(kLy % 32 == 4 && kLd % 32 == 4 && 48 * kLy * 4 <= kTile64x64,
              "solve strides and the transposed-T area");
constexpr uint32_t kP_VEC = kP_XS + 32 * kLy * 4;    // Gamma, beta, gamma, Gamma log2(e), D: 5 x 64 fp32
constexpr uint32_t kP_BAR = kP_VEC + 5 * 64 * 4;     // 2 mbarriers + tmem address
constexpr uint32_t kP_END = kP_BAR + 64;
constexpr uint32_t kPrepSmem = kP_END + 1024;        // + alignment slack
constexpr int kPrepThreads = 256;
static_assert(2 * kTile64x64 <= 64 * kLd * 4, "T tiles must fit in the A area");
static_assert(kTile128x64 <= 64 * kLd * 4, "the (D K)^T staging must fit in the T area");
static_assert(kP_AS % 1024 == 0 && kP_PST % 1024 == 0 && kP_KST % 1024 == 0,
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

// d += a b for fp32 fragments on the warp-level tf32 tensor-core path, each
// operand rounded once to tf32 (10-bit mantissa, round to nearest). T is
// rounded to bf16 (8-bit mantissa) before any product uses it, and the block
// products' tf32 error stays about ten times below that rounding.
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  uint32_t ar[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) ar[i] = cvt_tf32(__uint_as_float(a[i]));
  mma_tf32_m16n8k8(d, ar, cvt_tf32(__uint_as_float(b0)), cvt_tf32(__uint_as_float(b1)));
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
// The products are warp-level tensor-core tiles (m16n8k8, tf32, fp32
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
      mma_tf32(c, a, bb[0], bb[1]);
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
      mma_tf32(d, a, bb[2 * kk], bb[2 * kk + 1]);
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
      mma_tf32(c, a, bb[0], bb[1]);
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
        mma_tf32(d, a, bb[2 * kk], bb[2 * kk + 1]);
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
    uint32_t *__restrict__ ctrl, const ChunkInfo *__restrict__ table, long long rows,
    int max_chunks) {
  (void)rows;
  (void)max_chunks;   // extents of the bounds checks (GDN_CHECKS builds)
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
  float *Dv = Gl + 64;                     // D_s = exp(Gamma_last - Gamma_s)
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
      const ChunkInfo cf = GDN_IN_BOUNDS(ctrl, cu, max_chunks) ? table[cu] : ChunkInfo{0, 0, 0, 0};
      const long long idx = (long long)(cf.row0 + tid) * H + hu;
      const bool ok = tid < cf.len && GDN_IN_BOUNDS(ctrl, idx, rows * H);
      g_reg = ok ? g[idx] : 0.f;
      b_reg = ok ? beta[idx] : 0.f;
    }
  };
  fetch_gb(blockIdx.x);
  int it = 0;
  for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x, ++it) {
  const int chunk = unit / H, h = unit - chunk * H;
  const ChunkInfo ci =
      GDN_IN_BOUNDS(ctrl, chunk, max_chunks) ? table[chunk] : ChunkInfo{0, 0, 0, 0};
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
      const int rn = GDN_IN_BOUNDS(ctrl, cn, max_chunks) ? table[cn].row0 : 0;
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
    const float ga = expf(Gm[tid]), dv = expf(Gm[kC - 1] - Gm[tid]);
    Ga[tid] = ga;
    Dv[tid] = dv;
    if (GDN_IN_BOUNDS(ctrl, (long long)unit * 128 + 64 + tid, (long long)max_chunks * H * 128)) {
      gam_out[size_t(unit) * 128 + tid] = ga;        // gamma_c
      gam_out[size_t(unit) * 128 + 64 + tid] = dv;   // D_s
    }
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
  fence_proxy_async_smem();
  __syncthreads();
  GDN_TRACE_POINT(tr && chunk < 64, 1, chunk, 5);
  if (!abort_flag && tid == 0) {
    tma_store_2d(&tm_tb, sm + kP_TB, 0, unit * kC);
    tma_store_commit();
    tc_fence_after();
    // W^T = K^T (T diag(beta gamma))^T : M = 128 (d_k), N = 64, K = 64 -> cols [64, 128)
    const uint32_t idesc = make_idesc_bf16(128, 64, 1, 0);
    const uint64_t dkt = make_sdesc(smem_u32(sm + kP_KQ), kTile128x64, 1024);
    const uint64_t dtbg = make_sdesc(smem_u32(sm + kP_TBG), 16, 1024);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      tc_mma_bf16(tmem + 64, dkt + uint64_t(kk * 2048 >> 4), dtbg + uint64_t(kk * 32 >> 4), idesc,
                  kk > 0);
    tc_commit(bar_mma);
  }
  // While the tensor core computes W^T (both read K), (D K)^T goes straight
  // from the K tile into its staging tile (the dead T area): 8 x 8 blocks are
  // read transposed with ldmatrix (thread t gets tokens 2(t%4), 2(t%4)+1 of
  // d_k row t/4), scaled by (D_s, D_s+1) in bf16 with one rounding -- the
  // bits the MMA against a bf16 diag(D) tile gave -- and stored with
  // stmatrix. Warp w owns d_k rows [16 w, 16 w + 16).
  if (!abort_flag) {
    const int mj = lane & 7, mm = lane >> 3;
    const int sp = 2 * (lane & 3);                  // first token of this thread's pair
    const uint32_t kq = smem_u32(sm + kP_KQ), kst = smem_u32(sm + kP_KST);
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      // matrix mm: d_k block jb = 2 warp + (mm & 1), token block sb = 2 it + (mm >> 1)
      const int jb = 2 * warp + (mm & 1), sb = 2 * it + (mm >> 1);
      const int srow = 8 * sb + mj;                 // K row (token) this thread addresses
      uint32_t x[4];
      ldsm_x4_trans(kq + (jb >> 3) * kTile128x64 + sw128_offset(srow, jb & 7), x);
      uint32_t y[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int s0 = 16 * it + 8 * (m >> 1) + sp;
        y[m] = mul_bf16x2(x[m], pack_bf16x2(Dv[s0], Dv[s0 + 1]));
      }
      const int jrow = 8 * jb + mj;                 // (D K)^T row this thread addresses
      stmatrix_x4(kst + sw128_offset(jrow, sb), y[0], y[1], y[2], y[3]);
    }
  }
  mbar_wait(bar_mma, 1, ctrl, &abort_flag);
  GDN_TRACE_POINT(tr && chunk < 64, 1, chunk, 6);
  if (tid == 0) tma_store_wait_read();   // the P staging lies under the W staging
  tc_fence_after();
  __syncthreads();
  if (!abort_flag) {
    // -W, K-major [64 c][128 d]: read W^T (lanes = d, columns = c) as
    // mma-accumulator fragments and store them transposed with stmatrix.
    // Warp w: lane quarter w % 4, token columns [32 (w / 4), 32 (w / 4) + 32).
    const int q = warp & 3, mj = lane & 7, mm = lane >> 3;
    const uint32_t wst = smem_u32(sm + kP_WST);
#pragma unroll
    for (int lb = 0; lb < 32; lb += 16) {
#pragma unroll
      for (int cb = 32 * hc; cb < 32 * hc + 32; cb += 16) {
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

// ============================================================ channel-wise gate: prep
// The channel-wise (Kimi Delta Attention) gate of dmarx anthology LIT-137,
// "Standing in the anthology", and SOTA-135, "Sequence": alpha_t has one value
// per d_k channel, S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t
// v_t k_t^T. Per chunk, with Gamma_rj = sum_{s <= r} log alpha_sj:
//   A_rs = beta_r sum_j k_rj k_sj e^(Gamma_rj - Gamma_sj)   (s < r)
//   P_rs = sum_j q_rj k_sj e^(Gamma_rj - Gamma_sj)          (s <= r)
//   W = T diag(beta) (K .* e^Gamma),  U = T diag(beta) V,  T = (I + A)^-1
//   O = (Q .* e^Gamma) S^T + P V_new
//   S <- S diag(e^Gamma_last) + V_new^T (K .* e^(Gamma_last - Gamma))
// The decay sits inside the dot products. For the 16-row block R of A and P
// the factor splits through the block's first row b = 16 R:
//   e^(Gamma_r - Gamma_s) = e^(Gamma_r - Gamma_b) e^(Gamma_b - Gamma_s),
// so block row R is one product of a left operand (K or Q rows of the block
// scaled by e^(Gamma_r - Gamma_b) <= 1) with a right operand (K rows 0 ..
// 16 R + 15 scaled by e^(Gamma_b - Gamma_s): <= 1 below the block, within
// e^(15 max |log alpha|) inside it), on the warp-level tensor-core path
// (mma.sync m16n8k16, bf16 operands, fp32 accumulation). Everything after A
// is the scalar gate's prep: the same blocked solve, T diag(beta) and W on
// tcgen05. The state scan then consumes the same operand tiles, with
// Q .* e^Gamma in place of Q (gamma = 1 in the decay record) and the
// per-channel state decay e^Gamma_last.
// Shared memory holds one unit at a time, laid out for two CTAs per SM
// (each CTA: this window, 1 KB of static shared memory and the 1 KB the
// hardware reserves); areas are reused once their last reader is done. P
// goes to global memory straight from the mma fragments.
constexpr uint32_t kK_KQ = 0;                          // K, Q (bf16, 128-byte swizzle) as in prep;
                                                       // later Q .* e^Gamma, K .* e^Gamma, -W
constexpr uint32_t kK_GM = kK_KQ + 2 * kTile128x64;    // log2(e) Gamma fp32 [64][128]; then the
                                                       // solve's T, T^T blocks and scratch
constexpr uint32_t kK_AS = kK_GM + 64 * 128 * 4;       // A fp32 [64][68]
constexpr uint32_t kK_RR = (kK_AS + 64 * kLd * 4 + 1023) / 1024 * 1024;   // right operand of
                                                       // block row R [64][128] (256-B rows);
                                                       // later the (D K)^T staging [128][64]
constexpr uint32_t kK_LK = kK_RR + 64 * 256;           // left operands of block row R [16][128]
constexpr uint32_t kK_LQ = kK_LK + 16 * 256;           // (LK, LQ: later T diag(beta) bf16)
constexpr uint32_t kK_VEC = kK_LQ + 16 * 256;          // beta[64], e^Gamma_last[128]
constexpr uint32_t kK_BAR = kK_VEC + 192 * 4;
constexpr uint32_t kKdaPrepSmem = kK_BAR + 64;         // the dynamic window starts 1024-aligned (checked)
constexpr uint32_t kK_TS = kK_GM;                      // solve: T fp32 [64][68]
constexpr uint32_t kK_TT = kK_TS + 64 * kLd * 4;       // solve: T transposed fp32 [48][36]
constexpr uint32_t kK_XS = kK_TT + 48 * kLy * 4;       // solve scratch fp32 [32][36]
constexpr uint32_t kK_TB = kK_LK;
constexpr int kKdaPrepThreads = 256;
static_assert(kK_GM % 1024 == 0 && kK_RR % 1024 == 0 && kK_LK % 1024 == 0 &&
                  kK_XS + 32 * kLy * 4 <= kK_AS && 2 * 16 * 256 >= kTile64x64 &&
                  kTile128x64 <= 64 * 256 && 2 * (kKdaPrepSmem + 2048) <= 233472,
              "channel-wise prep layout: two CTAs per SM");

// Byte offset of 16-byte chunk c (0..15) of row r in a [rows][128 bf16] tile
// with 256-byte rows, XOR-swizzled so that 8 consecutive rows at the same
// chunk hit distinct banks (ldmatrix reads 8 rows x 16 bytes).
__device__ __forceinline__ uint32_t sw256(uint32_t r, uint32_t c) {
  return r * 256u + ((c ^ (r & 7u)) << 4);
}

// d += a b, m16n8k16, bf16 operands, fp32 accumulators (fragment layouts as
// for m16n8k8 with each register holding two consecutive k).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Eight bf16 (one 16-byte chunk) times eight fp32 factors, rounded once.
__device__ __forceinline__ uint4 scale8(uint4 x, const float (&f)[8]) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xffff0000u);
    o[i] = pack_bf16x2(lo * f[2 * i], hi * f[2 * i + 1]);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// 2^(a_x - b_x) for the eight channels of two float4 pairs.
__device__ __forceinline__ void ex2_diff8(float (&f)[8], float4 a0, float4 a1, float4 b0,
                                          float4 b1) {
  f[0] = ex2_approx(a0.x - b0.x);
  f[1] = ex2_approx(a0.y - b0.y);
  f[2] = ex2_approx(a0.z - b0.z);
  f[3] = ex2_approx(a0.w - b0.w);
  f[4] = ex2_approx(a1.x - b1.x);
  f[5] = ex2_approx(a1.y - b1.y);
  f[6] = ex2_approx(a1.z - b1.z);
  f[7] = ex2_approx(a1.w - b1.w);
}

__global__ void __launch_bounds__(kKdaPrepThreads, 2) gdn_kda_prep_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_kt,
    const __grid_constant__ CUtensorMap tm_tb, const __grid_constant__ CUtensorMap tm_qt,
    const float *__restrict__ g, const float *__restrict__ beta, float *__restrict__ gam_out,
    uint32_t *__restrict__ pm_out, int H, uint32_t *__restrict__ ctrl,
    const ChunkInfo *__restrict__ table, long long rows, int max_chunks) {
  (void)rows;
  (void)max_chunks;   // extents of the bounds checks (GDN_CHECKS builds)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = smem_raw;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  grid_launch_dependents();
  if (smem_u32(sm) & 1023) {
    grid_dependency_wait();
    if (tid == 0) atomicOr(ctrl, kErrLayout);
    return;
  }
  float *Gm = reinterpret_cast<float *>(sm + kK_GM);   // log2(e) Gamma
  float *As = reinterpret_cast<float *>(sm + kK_AS);
  float *Ts = reinterpret_cast<float *>(sm + kK_TS);
  float *Xs = reinterpret_cast<float *>(sm + kK_XS);
  float *Tt = reinterpret_cast<float *>(sm + kK_TT);
  float *Bt = reinterpret_cast<float *>(sm + kK_VEC);   // beta [64]
  float *El = Bt + 64;                                  // e^Gamma_last [128]
  uint64_t *bar_load = reinterpret_cast<uint64_t *>(sm + kK_BAR);
  uint64_t *bar_mma = bar_load + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_load + 2);
  constexpr float kLog2e = 1.4426950408889634f;
  if (tid == 0) {
    abort_flag = 0;
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();
  const int nunits = (ctrl[0] & kErrBadSeqlens) ? 0 : int(ctrl[1]) * H;
  const long long pm_words = (long long)max_chunks * H * (64 * 64 / 2);
  (void)pm_words;
  int it = 0;
  for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x, ++it) {
    const int chunk = unit / H, h = unit - chunk * H;
    const ChunkInfo ci =
        GDN_IN_BOUNDS(ctrl, chunk, max_chunks) ? table[chunk] : ChunkInfo{0, 0, 0, 0};
    const int L = ci.len;
    uint32_t *pm = pm_out + (long long)unit * (64 * 64 / 2);   // P of this unit, [64][64] bf16
    if (tid == 0) {
      // The previous unit's stores must have read the areas reused below.
      tma_store_wait_read();
      if (!abort_flag) {
        mbar_arrive_expect_tx(bar_load, 2 * kTile128x64);
        tma_load_3d(sm + kK_KQ, &tm_k, bar_load, 0, h, ci.row0);
        tma_load_3d(sm + kK_KQ + kTile64x64, &tm_q, bar_load, 0, h, ci.row0);
        tma_load_3d(sm + kK_KQ + kTile128x64, &tm_k, bar_load, 64, h, ci.row0);
        tma_load_3d(sm + kK_KQ + kTile128x64 + kTile64x64, &tm_q, bar_load, 64, h, ci.row0);
      }
    }
    __syncthreads();   // every thread is past the previous unit's reads of Gm, RR, LK, LQ
    // log2(e) Gamma: inclusive cumsum of g over the tokens (rows past the
    // sequence end read as 0) as a blocked scan. Thread t owns channels
    // 4 (t % 32) .. +3 of rows 8 (t / 32) .. +7: a scan over its 8 rows, the
    // 8 blocks' totals through shared memory (the right-operand area, free
    // here), then each block adds the totals of the blocks before it.
    float4 *Tot = reinterpret_cast<float4 *>(sm + kK_RR);   // [8 blocks][32 channel groups]
    {
      const int c4 = tid & 31, rb = tid >> 5;
      float4 run = make_float4(0.f, 0.f, 0.f, 0.f), part[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 8 * rb + i;
        const long long idx = ((long long)(ci.row0 + r) * H + h) * 128 + 4 * c4;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < L && GDN_IN_BOUNDS(ctrl, idx + 3, rows * H * 128))
          x = *reinterpret_cast<const float4 *>(g + idx);
        run.x = fmaf(x.x, kLog2e, run.x);
        run.y = fmaf(x.y, kLog2e, run.y);
        run.z = fmaf(x.z, kLog2e, run.z);
        run.w = fmaf(x.w, kLog2e, run.w);
        part[i] = run;
      }
      Tot[rb * 32 + c4] = run;
      __syncthreads();
      float4 off = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int b = 0; b < rb; ++b) {
        const float4 t4 = Tot[b * 32 + c4];
        off.x += t4.x;
        off.y += t4.y;
        off.z += t4.z;
        off.w += t4.w;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
        *reinterpret_cast<float4 *>(Gm + (8 * rb + i) * 128 + 4 * c4) =
            make_float4(part[i].x + off.x, part[i].y + off.y, part[i].z + off.z,
                        part[i].w + off.w);
      if (rb == 7) {
        El[4 * c4] = ex2_approx(part[7].x + off.x);
        El[4 * c4 + 1] = ex2_approx(part[7].y + off.y);
        El[4 * c4 + 2] = ex2_approx(part[7].z + off.z);
        El[4 * c4 + 3] = ex2_approx(part[7].w + off.w);
      }
    }
    if (tid < 64) {
      const long long idx = (long long)(ci.row0 + tid) * H + h;
      Bt[tid] = (tid < L && GDN_IN_BOUNDS(ctrl, idx, rows * H)) ? beta[idx] : 0.f;
    }
    // P is zero above its diagonal 16 x 16 blocks: blocks (R, S), S > R, are
    // written here, the others by the block-row products below.
    if (tid < 192) {
      const int bi = tid >> 5, rr = (tid >> 1) & 15, half = tid & 1;
      const int R = bi < 3 ? 0 : (bi < 5 ? 1 : 2), S = bi < 3 ? bi + 1 : (bi < 5 ? bi - 1 : 3);
      const long long wi = (long long)(16 * R + rr) * 32 + 8 * S + 4 * half;
      if (GDN_IN_BOUNDS(ctrl, (long long)unit * 2048 + wi + 3, pm_words))
        *reinterpret_cast<uint4 *>(pm + wi) = make_uint4(0, 0, 0, 0);
    }
    const bool loaded = mbar_wait(bar_load, it & 1, ctrl, &abort_flag);
    if (loaded && L < kC) {
      // Rows past the sequence end act as k = q = 0.
      for (int e = tid; e < (kC - L) * 8; e += kKdaPrepThreads) {
        const int r = L + e / 8, ch = e % 8;
        const uint4 z = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>(sm + kK_KQ + r * 128 + ch * 16) = z;
        *reinterpret_cast<uint4 *>(sm + kK_KQ + kTile64x64 + r * 128 + ch * 16) = z;
        *reinterpret_cast<uint4 *>(sm + kK_KQ + kTile128x64 + r * 128 + ch * 16) = z;
        *reinterpret_cast<uint4 *>(sm + kK_KQ + kTile128x64 + kTile64x64 + r * 128 + ch * 16) = z;
      }
    }
    __syncthreads();
    // A and P, one 16-row block row R at a time, b = 16 R.
    for (int R = 0; R < 4; ++R) {
      const int b = 16 * R, nrow = b + 16;
      {  // left operands: rows of block R, K and Q .* e^(Gamma_r - Gamma_b); one pair per thread
        const int r = b + (tid >> 4), c = tid & 15;
        const uint32_t kq = kK_KQ + (c >> 3) * kTile128x64 + sw128_offset(r, c & 7);
        const float *gr = Gm + r * 128 + 8 * c, *gb = Gm + b * 128 + 8 * c;
        float f[8];
        ex2_diff8(f, lds4(gr), lds4(gr + 4), lds4(gb), lds4(gb + 4));
        *reinterpret_cast<uint4 *>(sm + kK_LK + sw256(r - b, c)) =
            scale8(*reinterpret_cast<const uint4 *>(sm + kq), f);
        *reinterpret_cast<uint4 *>(sm + kK_LQ + sw256(r - b, c)) =
            scale8(*reinterpret_cast<const uint4 *>(sm + kq + kTile64x64), f);
      }
      // right operand: K rows s < b + 16 scaled by e^(Gamma_b - Gamma_s)
      for (int e = tid; e < nrow * 16; e += kKdaPrepThreads) {
        const int s = e >> 4, c = e & 15;
        const uint32_t kq = kK_KQ + (c >> 3) * kTile128x64 + sw128_offset(s, c & 7);
        const float *gs = Gm + s * 128 + 8 * c, *gb = Gm + b * 128 + 8 * c;
        float f[8];
        ex2_diff8(f, lds4(gb), lds4(gb + 4), lds4(gs), lds4(gs + 4));
        *reinterpret_cast<uint4 *>(sm + kK_RR + sw256(s, c)) =
            scale8(*reinterpret_cast<const uint4 *>(sm + kq), f);
      }
      __syncthreads();
      // jobs: (n-tile of 8 columns, A or P); warp w takes jobs w and w + 8
      const int njobs = 4 * (R + 1);
      for (int job = warp; job < njobs; job += 8) {
        const int nt = job >> 1, isP = job & 1;
        const uint32_t left = smem_u32(sm + (isP ? kK_LQ : kK_LK));
        const uint32_t right = smem_u32(sm + kK_RR);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const int ar = (lane & 7) + 8 * ((lane >> 3) & 1);   // A fragment row within the block
        const int brow = 8 * nt + (lane & 7);                // B fragment row (= column s)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          uint32_t a[4], bb[2];
          ldsm_x4(left + sw256(ar, 2 * kk + (lane >> 4)), a);
          ldsm_x2(right + sw256(brow, 2 * kk + ((lane >> 3) & 1)), bb);
          mma_bf16_16816(acc, a, bb[0], bb[1]);
        }
        const int gq = lane >> 2, tq = lane & 3;
        const int r0 = b + gq, s0 = 8 * nt + 2 * tq;
        if (!isP) {
          const float b0 = Bt[r0], b1 = Bt[r0 + 8];
          *reinterpret_cast<float2 *>(As + r0 * kLd + s0) = make_float2(b0 * acc[0], b0 * acc[1]);
          *reinterpret_cast<float2 *>(As + (r0 + 8) * kLd + s0) =
              make_float2(b1 * acc[2], b1 * acc[3]);
        } else {
          const uint32_t p0 = pack_bf16x2(s0 <= r0 ? acc[0] : 0.f, s0 + 1 <= r0 ? acc[1] : 0.f);
          const uint32_t p1 =
              pack_bf16x2(s0 <= r0 + 8 ? acc[2] : 0.f, s0 + 1 <= r0 + 8 ? acc[3] : 0.f);
          const long long w0 = (long long)r0 * 32 + (s0 >> 1);
          if (GDN_IN_BOUNDS(ctrl, (long long)unit * 2048 + w0 + 8 * 32, pm_words)) {
            pm[w0] = p0;
            pm[w0 + 8 * 32] = p1;
          }
        }
      }
      __syncthreads();   // LK, LQ and RR are rewritten by the next block row
    }
    // (D K)^T with D_sj = e^(Gamma_last,j - Gamma_sj), straight from the K tile
    // (ldmatrix.trans gives thread t tokens s, s + 1 of d_k row t / 4), staged
    // in the right-operand area; warp w owns d_k rows [16 w, 16 w + 16).
    {
      const int mj = lane & 7, mm = lane >> 3, sp = 2 * (lane & 3), jq = lane >> 2;
      const uint32_t kq = smem_u32(sm + kK_KQ), kst = smem_u32(sm + kK_RR);
#pragma unroll
      for (int it2 = 0; it2 < 4; ++it2) {
        const int jb = 2 * warp + (mm & 1), sb = 2 * it2 + (mm >> 1);
        uint32_t x[4];
        ldsm_x4_trans(kq + (jb >> 3) * kTile128x64 + sw128_offset(8 * sb + mj, jb & 7), x);
        uint32_t y[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int j = 8 * (2 * warp + (m & 1)) + jq, s0 = 8 * (2 * it2 + (m >> 1)) + sp;
          const float gl = Gm[63 * 128 + j];
          const float d0 = ex2_approx(gl - Gm[s0 * 128 + j]);
          const float d1 = ex2_approx(gl - Gm[(s0 + 1) * 128 + j]);
          y[m] = pack_bf16x2(__uint_as_float(x[m] << 16) * d0,
                             __uint_as_float(x[m] & 0xffff0000u) * d1);
        }
        stmatrix_x4(kst + sw128_offset(8 * jb + mj, sb), y[0], y[1], y[2], y[3]);
      }
    }
    __syncthreads();   // every read of the plain K tile is done
    // Q .* e^Gamma (the scan's Q) and K .* e^Gamma (the W operand), in place.
    for (int e = tid; e < 64 * 16; e += kKdaPrepThreads) {
      const int r = e >> 4, c = e & 15;
      const uint32_t kq = kK_KQ + (c >> 3) * kTile128x64 + sw128_offset(r, c & 7);
      const float *gr = Gm + r * 128 + 8 * c;
      const float4 r0 = lds4(gr), r1 = lds4(gr + 4);
      const float f[8] = {ex2_approx(r0.x), ex2_approx(r0.y), ex2_approx(r0.z),
                          ex2_approx(r0.w), ex2_approx(r1.x), ex2_approx(r1.y),
                          ex2_approx(r1.z), ex2_approx(r1.w)};
      *reinterpret_cast<uint4 *>(sm + kq) = scale8(*reinterpret_cast<const uint4 *>(sm + kq), f);
      *reinterpret_cast<uint4 *>(sm + kq + kTile64x64) =
          scale8(*reinterpret_cast<const uint4 *>(sm + kq + kTile64x64), f);
    }
    fence_proxy_async_smem();
    __syncthreads();   // Gamma is dead: the solve's scratch takes its place
    if (tid == 0 && !abort_flag) {
      tma_store_2d(&tm_qt, sm + kK_KQ + kTile64x64, 0, unit * kC);
      tma_store_2d(&tm_qt, sm + kK_KQ + kTile128x64 + kTile64x64, 64, unit * kC);
      tma_store_2d(&tm_kt, sm + kK_RR, 0, unit * kD);
      tma_store_commit();
    }
    solve_unit_lower_64(As, Ts, Tt, Xs, tid);   // ends with __syncthreads
    // T diag(beta), bf16 K-major (T is lower triangular; its upper blocks are
    // unwritten, so s > r reads as zero).
    {
      const int r = tid >> 2, q4 = tid & 3;
      float fb[16];
      if (16 * q4 <= r) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int s0 = 16 * q4 + 4 * i;
          const float4 t4 = lds4(Ts + r * kLd + s0);
          const float4 bt = lds4(Bt + s0);
          const float tv[4] = {t4.x, t4.y, t4.z, t4.w}, bv[4] = {bt.x, bt.y, bt.z, bt.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) fb[4 * i + e] = (s0 + e <= r) ? tv[e] * bv[e] : 0.f;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) fb[e] = 0.f;
      }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int ch = q4 * 2 + cc;
        const float *xb = fb + 8 * cc;
        *reinterpret_cast<uint4 *>(sm + kK_TB + sw128_offset(r, ch)) =
            make_uint4(pack_bf16x2(xb[0], xb[1]), pack_bf16x2(xb[2], xb[3]),
                       pack_bf16x2(xb[4], xb[5]), pack_bf16x2(xb[6], xb[7]));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (!abort_flag && tid == 0) {
      tma_store_2d(&tm_tb, sm + kK_TB, 0, unit * kC);
      tma_store_commit();
      tc_fence_after();
      // W^T = (K .* e^Gamma)^T (T diag(beta))^T : M = 128 (d_k), N = 64, K = 64
      const uint32_t idesc = make_idesc_bf16(128, 64, 1, 0);
      const uint64_t dkt = make_sdesc(smem_u32(sm + kK_KQ), kTile128x64, 1024);
      const uint64_t dtb = make_sdesc(smem_u32(sm + kK_TB), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc_mma_bf16(tmem, dkt + uint64_t(kk * 2048 >> 4), dtb + uint64_t(kk * 32 >> 4), idesc,
                    kk > 0);
      tc_commit(bar_mma);
    }
    // The decay record: gamma = 1 (the output uses Q .* e^Gamma directly),
    // then the per-channel state decay e^Gamma_last.
    {
      const long long base = (long long)unit * 256;
      if (GDN_IN_BOUNDS(ctrl, base + 255, (long long)max_chunks * H * 256)) {
        // [0, 64): gamma = 1, [64, 128): unused, [128, 256): e^Gamma_last
        gam_out[base + tid] = tid < 64 ? 1.f : (tid < 128 ? 0.f : El[tid - 128]);
      }
    }
    mbar_wait(bar_mma, it & 1, ctrl, &abort_flag);
    if (tid == 0) tma_store_wait_read();   // Q .* e^Gamma is staged where -W goes
    tc_fence_after();
    __syncthreads();
    if (!abort_flag) {
      // -W, K-major [64 c][128 d], from W^T (lanes = d, columns = c); warp w:
      // lane quarter w % 4, token columns [32 (w / 4), 32 (w / 4) + 32).
      const int q = warp & 3, hc = warp >> 2, mj = lane & 7, mm = lane >> 3;
      const uint32_t lane_base = tmem + (uint32_t(32 * q) << 16);
      const uint32_t wst = smem_u32(sm + kK_KQ);
#pragma unroll
      for (int lb = 0; lb < 32; lb += 16) {
#pragma unroll
        for (int cb = 32 * hc; cb < 32 * hc + 32; cb += 16) {
          uint32_t w8[8];
          tmem_ld16x256_x2(lane_base + (uint32_t(lb) << 16) + cb, w8);
          tmem_ld_wait();
          uint32_t w[4];
#pragma unroll
          for (int mq = 0; mq < 4; ++mq)
            w[mq] = pack_bf16x2(-__uint_as_float(w8[2 * mq]), -__uint_as_float(w8[2 * mq + 1]));
          const int d0 = q * 32 + lb + 8 * (mm & 1);
          const int crow = cb + 8 * (mm >> 1) + mj;
          stmatrix_x4_trans(wst + (d0 >> 6) * kTile64x64 + sw128_offset(crow, (d0 & 63) >> 3),
                            w[0], w[1], w[2], w[3]);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && !abort_flag) {
      tma_store_2d(&tm_w, sm + kK_KQ, 0, unit * kC);
      tma_store_2d(&tm_w, sm + kK_KQ + kTile64x64, 64, unit * kC);
      tma_store_commit();
    }
  }
  if (tid == 0) tma_store_wait_all();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

// ===================================================================== scan
// One chunk of one head is loaded in three parts, each with its own ring so
// that it can come in as soon as its last reader is done:
//   X part  BXZ  2 x [ -W rows 0-63 | Q rows 64-127 ]  (128 rows, K = d_k in two
//                blocks), the B operand of XZ; 3 stages, freed by XZ(c): a
//                load from HBM takes about a chunk period here, so it is
//                issued two chunks ahead
//   U part  V (MN-major A operand of U^T, 2 x [64 s][64 d]) and
//           BU = T diag(beta) (64 rows, K = 64 tokens); 2 slots, freed by U(c),
//           which runs early in the previous chunk
//   B part  BSY  stage 0: [ (D K)^T rows 0-127 | P rows 128-191 ]  (192 rows,
//                K = 64 tokens), stage 1: [ P rows 0-63 | (D K)^T rows 64-191 ];
//                2 stages, freed by SY(c)
// The two BSY orders put dS in the same tensor
// memory columns for every chunk and Y in one of two buffers (Y0 after dS,
// Y1 before it), so SY(c+1) never waits for the output warps to finish Y(c).
// The per-chunk decay factors (gamma[64], D[64]) travel in a separate 4-slot
// ring so the output warps never hold a stage.
constexpr int kStages = 2, kXStages = 3, kUSlots = 2, kGamSlots = 4;
constexpr uint32_t kXStage = 2 * kTile128x64;                  // 32 KB
constexpr uint32_t kUSlot = 2 * kTile64x64 + kTile64x64;       // 24 KB: V, then BU
constexpr uint32_t kBStage = kTile128x64 + kTile64x64;         // 24 KB
constexpr uint32_t kS_X = 0;
constexpr uint32_t kS_U = kS_X + kXStages * kXStage;
constexpr uint32_t kS_B = kS_U + kUSlots * kUSlot;
constexpr int kPrefetchAhead = 0;     // chunks prefetched into L2 ahead of the stage loads (0: none)
constexpr uint32_t kS_OST = kS_B + kStages * kBStage;          // O staging, 2 x [64 c][64 d]
constexpr uint32_t kS_GAM = kS_OST + 2 * kTile64x64;          // kGamSlots x 128 fp32
constexpr uint32_t kGamRec = 1024;   // decay record slot: 128 fp32 (scalar) or 256 (channel-wise)
constexpr uint32_t kS_BAR = kS_GAM + kGamSlots * kGamRec;      // mbarriers, tmem slot, flags
constexpr uint32_t kS_END = kS_BAR + 512;
constexpr uint32_t kScanSmem = kS_END;   // the dynamic window starts 1024-aligned (checked)
static_assert(kS_U % 1024 == 0 && kUSlot % 1024 == 0 && kS_B % 1024 == 0 &&
                  kS_OST % 1024 == 0 && kScanSmem <= 232448,
              "scan shared-memory layout");
constexpr int kScanThreads = 512;
// TMEM columns (fp32 accumulators, then the bf16 A operands held in TMEM)
constexpr uint32_t kT_XZ = 0;     // [X | Z] = [U^T - S W^T | S Q^T]      fp32 [128][128]
constexpr uint32_t kT_Z = 64;     //   (Z: zeroed by the output warps once they have read it)
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
// Barrier slots in the kS_BAR area (full_a / empty_a: the X part; full_u /
// empty_u: the U part)
// y_full[b] completes when Y buffer b holds a new chunk; the output warps wait
// on it, the chain on s_full. (One barrier for both would let a slow output
// warp miss a phase: it reports Z consumed before it waits for Y.)
// Each stage has two parts with their own full/empty pairs: part A (BXZ, V,
// BU) is last read by XZ(c) and part B (BSY) by SY(c), so the next loads of
// part A start while SY(c) and the S epilogue still run.
// x_free / u_done hand U(c+1) to its own issuing warp and back: x_free(c)
// completes once the V_new epilogue has read X(c), u_done(c+1) once U(c+1)
// has run (XZ(c+1) accumulates on it).
constexpr int kB_FULLA = 0, kB_EMPTYA = 3, kB_FULLB = 6, kB_EMPTYB = 8, kB_GFULL = 10,
              kB_GEMPTY = 14, kB_XFULL = 18, kB_SFULL = 19, kB_YFULL = 20, kB_ZFREE = 22,
              kB_DRAIN = 23, kB_XFREE = 24, kB_UDONE = 25, kB_DRAINU = 26, kB_FULLU = 27,
              kB_EMPTYU = 29, kB_COUNT = 31;
static_assert(kB_COUNT * 8 + 8 <= 512, "barrier area");

// Warp roles (16 warps). Every role runs its loop with all 32 lanes, so the
// lanes of a warp wait on barriers together; one lane issues TMA copies,
// MMAs and arrivals.
//   warp 0        TMA producer
//   warp 1        TMEM allocation and the chain's tcgen05.mma (XZ, SY)
//   warp 2        U = V^T Tb^T (tcgen05.mma): a thread issues MMAs only about
//                 as fast as the tensor core runs them, so U has an issuer of
//                 its own and the chain's issuer is free when S is ready
//   warps 4-11    state chain: two warpgroups, warpgroup h owns columns
//                 [32h, 32h+32) of V_new and [64h, 64h+64) of S; thread =
//                 TMEM lane = row i of d_v; the fp32 S lives in its registers,
//                 its bf16 copy (an MMA operand) in tensor memory. Each finished
//                 epilogue is handed to the MMA warp through a named barrier.
//   warps 12-15   output: O = diag(gamma) Z + Y, staged for TMA stores
// Per chunk c the tensor core runs three wide products:
//   U(c)   X      = V^T Tb^T                  (4 MMAs, N = 64)   -- before S_c is known
//   XZ(c)  [X|Z] += S [-W | Q]^T              (8 MMAs, N = 128)  -> X = V_new^T, Z = S Q^T
//   SY(c)  [dS|Y] = V_new^T [(DK)^T | P]^T    (4 MMAs, N = 192)
// and the chain is XZ -> V_new epilogue -> SY -> S epilogue -> XZ(c+1), with
// U(c+1) running during the S epilogue. XZ
// accumulates Z on zeros: the output warps read Z(c), store zeros in its
// place and then free it (z_free), which only XZ(c+1) waits for -- by then
// the output warps are long done. So only the two epilogue handshakes sit on
// the chain.
__global__ void __launch_bounds__(kScanThreads, 1) gdn_scan_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_v,
    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_kt,
    const __grid_constant__ CUtensorMap tm_tb, const __grid_constant__ CUtensorMap tm_pm,
    const __grid_constant__ CUtensorMap tm_gam, const __grid_constant__ CUtensorMap tm_o,
    const float *__restrict__ s0, float *__restrict__ sN, __nv_bfloat16 *__restrict__ o, int H,
    uint32_t *__restrict__ ctrl, const ChunkInfo *__restrict__ table,
    const int32_t *__restrict__ seq_first, int split, float *__restrict__ sN_trans,
    int sN_group, long long rows, int max_chunks, int n_first, int n_s0, int n_sN, int kda,
    __nv_bfloat16 *__restrict__ s_chunks) {
  // s_chunks (may be null): the state entering every chunk in bf16, for the
  // backward pass: per unit (chunk * H + head) 128 x 128 values of S
  // (formula orientation, row i = d_v, column j = d_k), the 16-byte piece
  // holding columns 8 p .. 8 p + 7 of row i at piece index p * 128 + i.
  // kda: the channel-wise gate. Q comes per unit from the prep (Q .* e^Gamma,
  // 2-D map tm_q over [units * 64][128]), the decay records are 256 wide and
  // S decays per d_k channel.
  // rows, max_chunks: token rows of q/k/v/o and chunk-table entries; n_first:
  // entries of seq_first; n_s0 / n_sN: states in s0 and in the array the final
  // states go to (the extents of the bounds checks of GDN_CHECKS builds).
  (void)rows;
  (void)max_chunks;
  (void)n_first;
  (void)n_s0;
  (void)n_sN;
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
#ifdef GDN_TRACE
  const int cta_id = int(blockIdx.y * gridDim.x + blockIdx.x);
  if (tid == 0 && cta_id < 1024) g_gdn_cta_ns[cta_id][0] = global_ns();
#endif

  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kS_BAR);
  uint64_t *full_a = bars + kB_FULLA, *empty_a = bars + kB_EMPTYA;
  uint64_t *full_b = bars + kB_FULLB, *empty_b = bars + kB_EMPTYB;
  uint64_t *gfull = bars + kB_GFULL, *gempty = bars + kB_GEMPTY;
  uint64_t *x_full = bars + kB_XFULL, *s_full = bars + kB_SFULL, *y_full = bars + kB_YFULL;
  uint64_t *z_free = bars + kB_ZFREE, *drain = bars + kB_DRAIN;
  uint64_t *x_free = bars + kB_XFREE, *u_done = bars + kB_UDONE;
  uint64_t *full_u = bars + kB_FULLU, *empty_u = bars + kB_EMPTYU;
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
  // A sequence's (or segment's) chunks are consecutive 64-token blocks from
  // its first row, only the last one possibly partial: chunk c starts at row
  // row_first + 64 c and is last_len long if c == nch - 1, else 64. Read once
  // here rather than a table entry per chunk (a dependent global load on the
  // producer's path).
  int c0 = 0, nch = 0, row_first = 0, last_len = kC;
  auto read_chunks = [&]() {
    grid_dependency_wait();
    if (!(ctrl[0] & kErrBadSeqlens)) {
      if (GDN_IN_BOUNDS(ctrl, n + 1, n_first)) {
        c0 = seq_first[n];
        nch = seq_first[n + 1] - c0;
      }
      if (nch > 0 && GDN_IN_BOUNDS(ctrl, c0, max_chunks) &&
          GDN_IN_BOUNDS(ctrl, c0 + nch - 1, max_chunks)) {
        row_first = table[c0].row0;
        last_len = table[c0 + nch - 1].len;
      } else {
        nch = 0;
      }
    }
  };
  auto chunk_row0 = [&](int c) { return row_first + kC * c; };
  auto chunk_len = [&](int c) { return c == nch - 1 ? last_len : kC; };
  if (warp < 4 || warp >= 12) read_chunks();   // warps 0-2 issue, 3 idles

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    for (int c = 0; c < nch && !*abort_flag; ++c) {
      const int st = c & 1, gs = c & 3, us = c % kUSlots;
      const int row0 = chunk_row0(c);
      const int unit = (c0 + c) * H + h;
      GDN_TRACE_POINT(tr && lane == 0, 0, c, 0);
      // Only what this CTA's products read: a run without output needs
      // neither Q nor P, a transition run neither V nor T diag(beta).
      if (!trans) {
        if (c >= kUSlots) wait(empty_u + us, ((c / kUSlots) - 1) & 1);
        if (lane == 0) {
          uint8_t *ub = sm + kS_U + us * kUSlot;
          mbar_arrive_expect_tx(full_u + us, kUSlot);
          tma_load_3d(ub, &tm_v, full_u + us, 0, h, row0);
          tma_load_3d(ub + kTile64x64, &tm_v, full_u + us, 64, h, row0);
          tma_load_2d(ub + 2 * kTile64x64, &tm_tb, full_u + us, 0, unit * kC);
        }
        __syncwarp();
      }
      const int xs = c % kXStages;
      uint8_t *xb = sm + kS_X + xs * kXStage;
      if (c >= kXStages) wait(empty_a + xs, ((c / kXStages) - 1) & 1);
      if (lane == 0) {
        mbar_arrive_expect_tx(full_a + xs, write_o ? kXStage : kTile128x64);
        tma_load_2d(xb, &tm_w, full_a + xs, 0, unit * kC);
        tma_load_2d(xb + kTile128x64, &tm_w, full_a + xs, 64, unit * kC);
        if (write_o && kda) {
          tma_load_2d(xb + kTile64x64, &tm_q, full_a + xs, 0, unit * kC);
          tma_load_2d(xb + kTile128x64 + kTile64x64, &tm_q, full_a + xs, 64, unit * kC);
        } else if (write_o) {
          tma_load_3d(xb + kTile64x64, &tm_q, full_a + xs, 0, h, row0);
          tma_load_3d(xb + kTile128x64 + kTile64x64, &tm_q, full_a + xs, 64, h, row0);
        }
      }
      __syncwarp();
      uint8_t *bb = sm + kS_B + st * kBStage;
      if (c >= 2) wait(empty_b + st, ((c >> 1) - 1) & 1);
      if (lane == 0) {
        // Without output, (D K)^T goes first in both stages and P is not loaded.
        const bool swap = st && write_o;
        mbar_arrive_expect_tx(full_b + st, write_o ? kBStage : kTile128x64);
        tma_load_2d(bb + (swap ? kTile64x64 : 0u), &tm_kt, full_b + st, 0, unit * kD);
        if (write_o) tma_load_2d(bb + (st ? 0u : kTile128x64), &tm_pm, full_b + st, 0, unit * kC);
        // Stage loads wait for their ring slot; the chunks ahead go to L2 now,
        // so those loads come from L2.
        if (kPrefetchAhead > 0 && c + kPrefetchAhead < nch) {
          const int rp = chunk_row0(c + kPrefetchAhead);
          const int up = (c0 + c + kPrefetchAhead) * H + h;
          tma_prefetch_l2_2d(&tm_w, 0, up * kC);
          tma_prefetch_l2_2d(&tm_w, 64, up * kC);
          tma_prefetch_l2_2d(&tm_kt, 0, up * kD);
          if (write_o) {
            tma_prefetch_l2_3d(&tm_q, 0, h, rp);
            tma_prefetch_l2_3d(&tm_q, 64, h, rp);
            tma_prefetch_l2_2d(&tm_pm, 0, up * kC);
          }
          if (!trans) {
            tma_prefetch_l2_3d(&tm_v, 0, h, rp);
            tma_prefetch_l2_3d(&tm_v, 64, h, rp);
            tma_prefetch_l2_2d(&tm_tb, 0, up * kC);
          }
        }
      }
      __syncwarp();
      if (c >= 4) wait(gempty + gs, ((c >> 2) - 1) & 1);
      if (lane == 0) {
        mbar_arrive_expect_tx(gfull + gs, kda ? 1024 : 512);
        tma_load_2d(sm + kS_GAM + gs * kGamRec, &tm_gam, gfull + gs, 0, unit);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Without output, Z and Y are not needed: U and XZ shrink to X (N = 64),
    // SY to dS (N = 128, (D K)^T then first in both stages).
    const uint32_t id_xz = make_idesc_bf16(128, write_o ? 128 : 64, 0, 0);  // S [-W|Q]^T
    const uint32_t id_sy = make_idesc_bf16(128, write_o ? 192 : 128, 0, 0); // A1 [(DK)^T|P]^T
    const bool issuer = lane == 0;
    // Shared-memory descriptors of the operand tiles of both stages, built
    // once: a single issuing thread pays the latency of every dependent
    // integer op, so rebuilding descriptors between MMAs doubles the issue
    // time. A k step is added to the start-address field (smem offsets >> 4
    // stay below 2^14, so the field never carries into the next one).
    uint64_t dBSY[kStages];
#pragma unroll
    for (int st = 0; st < kStages; ++st)
      dBSY[st] = make_sdesc(smem_u32(sm + kS_B + st * kBStage), 16, 1024);
    // XZ(c) += S_c [-W|Q]^T, reading the bf16 copy of S_c.
    auto issue_xz = [&](int c) {
      if (issuer) {
        GDN_TRACE_POINT(tr, 0, c, 1);
#ifdef GDN_TRACE
        if (cta_id < 1024) g_gdn_cta_ns[cta_id][c == 0 ? 1 : 2] = global_ns();
#endif
        const uint64_t db = make_sdesc(smem_u32(sm + kS_X + (c % kXStages) * kXStage), 16, 1024);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // a transition run has no U: XZ starts the sum
          tc_mma_bf16_ts(tmem + kT_XZ, tmem + kT_S + 8 * kk,
                         db + uint64_t(((kk >> 2) * kTile128x64 + (kk & 3) * 32) >> 4), id_xz,
                         (kk > 0) || !trans);
        tc_commit(x_full);
        tc_commit(empty_a + (c % kXStages));   // XZ(c) was the last reader of the X part
      }
      __syncwarp();
    };
    if (nch > 0) {
      wait(full_a, 0);                        // -W and Q of chunk 0 (stage 0)
      if (!trans) wait(u_done, 0);            // X = U(0)
      wait(z_free, 0);                        // Z zeroed at the start
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
        mbar_arrive(x_free);              // X(c) read: U(c + 1) may overwrite it
        const uint64_t db = st ? dBSY[1] : dBSY[0];
        tc_fence_after();
        // even chunks: D = [dS | Y0] at kT_DS; odd: D = [Y1 | dS] at kT_Y1
        // (without output: D = dS at kT_DS for every chunk). One N = 192
        // group: a separate Y group would hold this issuer up as well.
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
      // While SY(c) and the S epilogue run: XZ(c + 1) needs U(c + 1) done,
      // -W and Q of chunk c + 1, and Z(c) read and zeroed by the output warps.
      if (more) {
        if (!trans) wait(u_done, (c + 1) & 1);
        wait(full_a + (c + 1) % kXStages, ((c + 1) / kXStages) & 1);
        GDN_TRACE_POINT(tr && issuer, 0, c, 14);
        wait(z_free, (c + 1) & 1);
        GDN_TRACE_POINT(tr && issuer, 0, c, 13);
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
  } else if (warp == 2) {
    // ------------------------------------------------------------ U issuer
    // U(c) = V^T Tb^T into X (accumulate = 0). U(c) needs chunk c loaded and,
    // for c > 0, X(c - 1) read by the V_new epilogue.
    const bool issuer = lane == 0;
    const uint32_t id_u = make_idesc_bf16(128, 64, 1, 0);
    for (int c = 0; c < nch && !trans; ++c) {
      const int us = c % kUSlots;
      if (c > 0) wait(x_free, (c - 1) & 1);
      wait(full_u + us, (c / kUSlots) & 1);
      if (issuer) {
        const uint32_t ub = smem_u32(sm + kS_U + us * kUSlot);
        const uint64_t da = make_sdesc(ub, kTile64x64, 1024);
        const uint64_t db = make_sdesc(ub + 2 * kTile64x64, 16, 1024);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_bf16(tmem + kT_XZ, da + uint64_t(kk * 2048 >> 4), db + uint64_t(kk * 32 >> 4),
                      id_u, kk > 0);
        tc_commit(u_done);
        tc_commit(empty_u + us);
      }
      __syncwarp();
    }
    if (issuer) tc_commit(bars + kB_DRAINU);  // fires once every U above has completed
    __syncwarp();
    volatile int keep_waiting = 0;
    mbar_wait(bars + kB_DRAINU, 0, ctrl, &keep_waiting);
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ state chain
    const int hh = (warp - 4) >> 2;                     // column half
    const int i = ((warp & 3) << 5) + lane;             // TMEM lane = row of d_v
    const uint32_t lane_base = tmem + (uint32_t((warp & 3) * 32) << 16);
    const bool tl = tr && warp == 4 && lane == 0;       // traced lane
    (void)tl;
    float S[64];                                        // S[i][64 hh + t], fp32 master
    {
      const float *src = (s0 && !trans && GDN_IN_BOUNDS(ctrl, (long long)n * H + h, (long long)n_s0 * H))
                             ? s0 + (size_t(n) * H + h) * kD * kD
                             : nullptr;
#pragma unroll
      for (int t = 0; t < 64; ++t)
        S[t] = trans ? (64 * hh + t == i ? 1.f : 0.f) : (src ? src[size_t(64 * hh + t) * kD + i] : 0.f);
    }
    read_chunks();
    // bf16 copy of S (row i, columns [64 hh, 64 hh + 64)) into tensor memory,
    // then hand it to the MMA warp.
    // cs: the chunk the state enters (its bf16 copy also goes to s_chunks).
    auto store_state = [&](int cs) {
      uint32_t pk[2][16];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
#pragma unroll
        for (int t = 0; t < 16; ++t) pk[q][t] = pack_bf16x2(S[32 * q + 2 * t], S[32 * q + 2 * t + 1]);
        tmem_st16(lane_base + kT_S + 32 * hh + 16 * q, pk[q]);
      }
      tmem_st_wait();
      tc_fence_before();
      named_bar_arrive(kBarS, kChainHandoff);
      // off the chain's path: the MMA warp already has the state. Layout per
      // unit: 16-byte piece p (= columns 8 p .. 8 p + 7) of row i at piece
      // index p * 128 + i, so each store instruction of a warp writes 32
      // consecutive pieces (512 contiguous bytes).
      if (s_chunks && cs < nch) {
        const long long u = (long long)(c0 + cs) * H + h;
        if (GDN_IN_BOUNDS(ctrl, u, (long long)max_chunks * H)) {
          uint4 *dst = reinterpret_cast<uint4 *>(s_chunks + u * kD * kD) + i;
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int t = 0; t < 16; t += 4)
              dst[(8 * hh + 4 * q + t / 4) * kD] =
                  make_uint4(pk[q][t], pk[q][t + 1], pk[q][t + 2], pk[q][t + 3]);
        }
      }
    };
    store_state(0);
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
      const float *rec = reinterpret_cast<const float *>(sm + kS_GAM + gs * kGamRec);
      const float gl = rec[kC - 1];
      wait(s_full, c & 1);
      GDN_TRACE_POINT(tl, 0, c, 7);
      tc_fence_after();
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        uint32_t d[32];
        tmem_ld32(lane_base + kT_DS + 64 * hh + 32 * b, d);
        tmem_ld_wait();
        GDN_TRACE_POINT(tl && b == 0, 0, c, 3);
        if (!kda) {
#pragma unroll
          for (int t = 0; t < 32; t += 2) {
            const float2 r = ffma2(make_float2(gl, gl), make_float2(S[32 * b + t], S[32 * b + t + 1]),
                                   make_float2(__uint_as_float(d[t]), __uint_as_float(d[t + 1])));
            S[32 * b + t] = r.x;
            S[32 * b + t + 1] = r.y;
          }
        } else {
          // channel-wise gate: column j of S (d_k channel) decays by e^Gamma_last,j
          const float *dec = rec + 128 + 64 * hh + 32 * b;
#pragma unroll
          for (int t = 0; t < 32; t += 2) {
            const float2 r = ffma2(*reinterpret_cast<const float2 *>(dec + t),
                                   make_float2(S[32 * b + t], S[32 * b + t + 1]),
                                   make_float2(__uint_as_float(d[t]), __uint_as_float(d[t + 1])));
            S[32 * b + t] = r.x;
            S[32 * b + t + 1] = r.y;
          }
        }
      }
      store_state(c + 1);
      GDN_TRACE_POINT(tl, 0, c, 4);
      GDN_TRACE_POINT(tr && warp == 11 && lane == 0, 0, c, 15);
    }
    float *sNp = trans ? sN_trans : sN;
    const int sN_idx = trans ? n : n / sN_group;
    if (sNp && (trans || n % sN_group == sN_group - 1) && !*abort_flag &&
        GDN_IN_BOUNDS(ctrl, (long long)sN_idx * H + h, (long long)n_sN * H)) {
      float *dst = sNp + (size_t(sN_idx) * H + h) * kD * kD;
#pragma unroll
      for (int t = 0; t < 64; ++t) dst[size_t(64 * hh + t) * kD + i] = S[t];
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ output
    // O[c'][i] = gamma_c' Z[i][c'] + Y[i][c'] (Z, Y are O^T in TMEM). Each warp
    // reads its 32 lanes as mma-accumulator fragments (16 lanes x 8 columns),
    // Z as soon as XZ is done (then zeroes it for XZ of the next chunk), Y
    // after SY, and writes O transposed into the swizzled staging tile with
    // stmatrix, 16 bytes per row; a TMA store (whole chunks) or a 16-byte copy
    // loop (a sequence's last, partial chunk) moves the tile to o.
    const int q = warp & 3, ot = tid - 384;           // output thread 0..127
    const uint32_t lane_q = tmem + (uint32_t(q * 32) << 16);
    const bool leader = (warp == 12 && lane == 0);
    const uint32_t ost = smem_u32(sm + kS_OST);
    const int fc = 2 * (lane & 3);                     // fragment column pair
    const int mj = lane & 7, mm = lane >> 3;           // stmatrix: row j of matrix m
    // Zeros into this warp's 32 lanes of the Z columns (waited for here).
    auto zero_z = [&]() {
      uint32_t zr[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) zr[t] = 0u;
      tmem_st32(lane_q + kT_Z, zr);
      tmem_st32(lane_q + kT_Z + 32, zr);
      tmem_st_wait();
    };
    // z_free phase 0: Z starts at zero (XZ accumulates it on top).
    if (write_o) zero_z();
    tc_fence_before();
    named_bar_sync(kBarOut, 128);
    if (leader) mbar_arrive(z_free);
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
      const float *gam = reinterpret_cast<const float *>(sm + kS_GAM + gs * kGamRec);
      const int row0 = chunk_row0(c), len = chunk_len(c);
      const bool whole = len == kC;
      uint32_t z[2][32], ynext[8];
      wait(x_full, c & 1);
      tc_fence_after();
      tmem_ld16x256_x8(lane_q + kT_XZ + 64, z[0]);
      tmem_ld16x256_x8(lane_q + (16u << 16) + kT_XZ + 64, z[1]);
      tmem_ld_wait();
      zero_z();                                  // for XZ(c + 1)
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
          tma_store_3d(&tm_o, sm + kS_OST, 0, h, row0);
          tma_store_3d(&tm_o, sm + kS_OST + kTile64x64, 64, h, row0);
          tma_store_commit();
        }
        GDN_TRACE_POINT(tr, 0, c, 10);
      }
      __syncwarp();
      if (!whole && !*abort_flag) {
        // rows [0, len) of the tile, 16 bytes at a time
        for (int e = ot; e < len * 16; e += 128) {
          const int row = e >> 4, k = e & 15;
          const uint4 v = *reinterpret_cast<const uint4 *>(
              sm + kS_OST + (k >> 3) * kTile64x64 + sw128_offset(row, k & 7));
          const long long oi = ((long long)(row0 + row) * H + h) * kD + 8 * k;
          if (GDN_IN_BOUNDS(ctrl, oi + 7, rows * H * kD))
            *reinterpret_cast<uint4 *>(o + oi) = v;
        }
      }
    }
    if (leader) tma_store_wait_all();
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
#ifdef GDN_TRACE
  if (tid == 0 && cta_id < 1024) g_gdn_cta_ns[cta_id][3] = global_ns();
#endif
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
    uint32_t *__restrict__ ctrl) {
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
    // (uniform across the CTA, so the barriers below stay matched)
    if (!GDN_IN_BOUNDS(ctrl, (long long)(b * segs + gi) * H + h,
                       (long long)(gridDim.x / H) * segs * H))
      break;
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

}  // namespace

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encoder() {
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

cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *s0, int B, int T, int H, int N,
                            void *o, float *sN, void *ws, const WsLayout &L, cudaStream_t s,
                            __nv_bfloat16 *s_chunks) {
  // s_chunks != null (the backward pass): the scan also stores every chunk's
  // entering state; o may then be null (no output written; its tensor map
  // is built over q and never stored through).
  char *base = static_cast<char *>(ws);
  uint32_t *ctrl = reinterpret_cast<uint32_t *>(base);
  const ChunkInfo *table = reinterpret_cast<const ChunkInfo *>(base + L.chunk_table);
  const int32_t *seq_first = reinterpret_cast<const int32_t *>(base + L.seq_first);
  const long long rows = (long long)B * T;
  const long long units = (long long)L.max_chunks * H;
  if (T > 0 && L.max_chunks > 0) {
    CUtensorMap mq, mk, mv, mo, mw, mkt, mtb, mpm, mgm, mqt;
    const int rec = L.kda ? 256 : 128;   // decay record width
    if (!map_tokens(&mq, q, rows, H) || !map_tokens(&mk, k, rows, H) ||
        !map_tokens(&mv, v, rows, H) || !map_tokens(&mo, o ? o : q, rows, H) ||
        !map_2d(&mw, base + L.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kC, kD, 64, kC,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mkt, base + L.kt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kD, 64, 64, kD,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mtb, base + L.tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kC, 64, 64, kC,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mpm, base + L.pm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kC, 64, 64, kC,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mgm, base + L.gam, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, units, rec, rec, 1,
                CU_TENSOR_MAP_SWIZZLE_NONE) ||
        (L.kda && !map_2d(&mqt, base + L.qt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kC, kD,
                          64, kC, CU_TENSOR_MAP_SWIZZLE_128B)))
      return cudaErrorInvalidValue;
    cudaError_t e = L.kda ? cudaFuncSetAttribute(gdn_kda_prep_kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kKdaPrepSmem)
                          : cudaFuncSetAttribute(gdn_prep_kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kPrepSmem);
    if (e != cudaSuccess) return e;
    prof_record(g_profile.prep, s);
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long prep_ctas = std::min<long long>(units, (L.kda ? 2LL : 3LL) * sms);
    // Both kernels start with programmatic dependent launch: their prologues
    // overlap the tail of the kernel before them.
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(prep_ctas));
    cfg.blockDim = dim3(L.kda ? kKdaPrepThreads : kPrepThreads);
    cfg.dynamicSmemBytes = L.kda ? kKdaPrepSmem : kPrepSmem;
    cfg.stream = s;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    if (L.kda)
      e = cudaLaunchKernelEx(&cfg, gdn_kda_prep_kernel, mq, mk, mw, mkt, mtb, mqt, g, beta,
                             reinterpret_cast<float *>(base + L.gam),
                             reinterpret_cast<uint32_t *>(base + L.pm), H, ctrl, table, rows,
                             L.max_chunks);
    else
      e = cudaLaunchKernelEx(&cfg, gdn_prep_kernel, mq, mk, mw, mkt, mtb, mpm, g, beta,
                             reinterpret_cast<float *>(base + L.gam), H, ctrl, table, rows,
                             L.max_chunks);
    if (e != cudaSuccess) return e;
    // the scan reads Q from the prep's Q .* e^Gamma with the channel-wise gate
    const CUtensorMap mqs = L.kda ? mqt : mq;
    e = cudaFuncSetAttribute(gdn_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kScanSmem);
    if (e != cudaSuccess) return e;
    prof_record(g_profile.scan, s);
    cfg.blockDim = dim3(kScanThreads);
    cfg.dynamicSmemBytes = kScanSmem;
    if (L.segs <= 1) {
      cfg.gridDim = dim3(N, H);
      return cudaLaunchKernelEx(&cfg, gdn_scan_kernel, mqs, mv, mw, mkt, mtb, mpm, mgm, mo, s0,
                                sN, static_cast<__nv_bfloat16 *>(o), H, ctrl,
                                static_cast<const ChunkInfo *>(table), seq_first, 0,
                                static_cast<float *>(nullptr), 1, rows, L.max_chunks, N + 1, N,
                                N, int(L.kda), s_chunks);
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
    e = cudaLaunchKernelEx(&cfg, gdn_scan_kernel, mqs, mv, mw, mkt, mtb, mpm, mgm, mo,
                           static_cast<const float *>(nullptr), hbuf,
                           static_cast<__nv_bfloat16 *>(nullptr), H, ctrl,
                           static_cast<const ChunkInfo *>(table), seg_first, nseg, pbuf, 1, rows,
                           L.max_chunks, nseg + 1, 0, nseg, int(L.kda),
                           static_cast<__nv_bfloat16 *>(nullptr));
    if (e != cudaSuccess) return e;
    gdn_segment_combine_kernel<<<dim3(B * H, kD / 16), 256, 0, s>>>(s0, hbuf, pbuf, sstart, H,
                                                                   L.segs, ctrl);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // A plain launch: the start states come from the kernel just before it.
    cfg.gridDim = dim3(nseg, H);
    cfg.numAttrs = 0;
    return cudaLaunchKernelEx(&cfg, gdn_scan_kernel, mqs, mv, mw, mkt, mtb, mpm, mgm, mo,
                              static_cast<const float *>(sstart), sN,
                              static_cast<__nv_bfloat16 *>(o), H, ctrl,
                              static_cast<const ChunkInfo *>(table), seg_first, 0,
                              static_cast<float *>(nullptr), L.segs, rows, L.max_chunks, nseg + 1,
                              nseg, B, int(L.kda), static_cast<__nv_bfloat16 *>(nullptr));
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
extern "C" int gdn_trace_fetch_cta(unsigned long long *host) {
  return cudaMemcpyFromSymbol(host, gdn::g_gdn_cta_ns, sizeof(gdn::g_gdn_cta_ns)) == cudaSuccess
             ? 0
             : -1;
}
extern "C" int gdn_trace_fetch(unsigned long long *host) {
  return cudaMemcpyFromSymbol(host, gdn::g_gdn_trace, sizeof(gdn::g_gdn_trace)) == cudaSuccess
             ? 0
             : -1;
}
#endif
