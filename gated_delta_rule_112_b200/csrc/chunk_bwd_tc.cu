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
//   2. gdn_bwd_chain_kernel, two CTAs per (sequence, head): the reverse chain
//      dS_c = gamma_last dS_{c+1} - dX^T W + (gamma dO)^T Q over the chunks,
//      writing each chunk's G' = dS_{c+1} (bf16) and d_initial_state;
//   3. gdn_bwd_unit_kernel, persistent over (chunk, head) units: everything
//      else above, from the chunk's tiles, S_c and G'.
// Every product of kernels 2 and 3 is a tcgen05.mma (bf16 operands from
// 128-byte-swizzled shared tiles, fp32 accumulators in tensor memory).
#include <cuda_bf16.h>

#include "bwd_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using bf16 = __nv_bfloat16;
constexpr int kC = 64, kD = 128;
// the unit kernel's block: 16 epilogue warps (four per TMEM lane quadrant,
// each with a quarter of an accumulator's columns) and one issuer warp (TMA
// and MMAs)
constexpr int kThreads = 512, kWarps = kThreads / 32, kUnitThreads = kThreads + 32;
constexpr float kLog2e = 1.4426950408889634f;

// One contiguous copy global -> shared (16-byte aligned, size a multiple of
// 16) that completes `bytes` of the mbarrier's transaction count; no cluster
// broadcast.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------------ units
// Per (chunk, head) unit on tcgen05: every product is an M = 64 (tokens)
// tcgen05.mma issued by one thread of the issuer warp, operands read by the
// tensor core straight from shared memory, fp32 accumulators in tensor memory
// (512 columns, one CTA per SM). M = 64 accumulator row r sits in TMEM lane
// 32 (r / 16) + r % 16, so epilogue warp w reads rows 16 (w % 4) .. +15 with
// tcgen05.ld.16x256b in the mma-fragment layout (rows g, g + 8; columns 2 t,
// 2 t + 1), a quarter (w / 4) of the columns. All tiles are bf16 in
// 128-byte-swizzled panels of 64 columns; a stored tile serves as a K-major
// operand (rows = M or N) or as an MN-major one (rows = K) per product.
// Six phases, each one or two MMA groups (a commit per group) and an epilogue
// by the 16 epilogue warps:
//   1  X = TB V + (-W) S^T [X];  DKG = (D K) G'^T [D];  K K^T [KK]
//      -> X bf16, delta = rowsum(X .* DKG), L = K K^T .* E (s < r) bf16
//   2  D += P^T dO (= dX);  K S^T [KS]          -> dX bf16
//   3  dV = TB^T dX [X]                         -> dv, dV bf16
//   4  D -= L^T dV (= dY);  L X [LX];  dO X^T [dP];  dV X^T [R']
//      -> e = V - gamma KS - LX, dbeta = rowsum(dY .* e); dGamma from dP .* P
//         and -R' .* L; dP .* E (s <= r) and R = -R' .* E (s < r) bf16
//   5  dO S [A];  (dP .* E) K [B];  X G' [C];  dV S [E]
//      -> dq = gamma A + B; dGamma terms; the first part of dk in registers
//   6  (dP .* E)^T Q + R K + R^T K [A]          -> dk
constexpr uint32_t kV_Q = 0;                  // [64][128]: two 8 KB panels
constexpr uint32_t kV_K = kV_Q + 16384;
constexpr uint32_t kV_V = kV_K + 16384;
constexpr uint32_t kV_DO = kV_V + 16384;
constexpr uint32_t kV_S = kV_DO + 16384;      // S_c [128 d_v][128 d_k] in the scan's piece order, unswizzled
constexpr uint32_t kV_GP = kV_S + 32768;      // G' [d_v][d_k]
constexpr uint32_t kV_TB = kV_GP + 32768;     // [64][64]: one 8 KB panel
constexpr uint32_t kV_P = kV_TB + 8192;       // P; then dP .* E
constexpr uint32_t kV_W = kV_P + 8192;        // -W [64][128]; then dX
constexpr uint32_t kV_KT = kV_W + 16384;      // (D K)^T [128][64] (one 16 KB panel); then dV [64][128]
constexpr uint32_t kV_X = kV_KT + 16384;      // X [64][128]
constexpr uint32_t kV_L = kV_X + 16384;       // L [64][64]; then R
constexpr uint32_t kV_VEC = kV_L + 8192;      // Gamma, gamma, D, dGamma, dbeta, delta [64] fp32
constexpr uint32_t kV_RED = kV_VEC + 6 * 64 * 4;
constexpr uint32_t kV_BAR = kV_RED + 4 * kWarps;   // 4 mbarriers, TMEM slot, abort flag
constexpr uint32_t kUnitSmem = kV_BAR + 64 + 1024;  // + 1024: the window is aligned up to 1 KB
static_assert(kV_Q % 1024 == 0 && kV_S % 1024 == 0 && kV_TB % 1024 == 0 && kV_KT % 1024 == 0 &&
                  kV_X % 1024 == 0 && kV_L % 1024 == 0 && kUnitSmem <= 232448,
              "unit kernel shared memory");
// tensor-memory columns of the accumulators
constexpr uint32_t kC0 = 0, kC1 = 128, kC2 = 256, kC3 = 384;

// Byte offset of element (r, c) of a [rows][*] bf16 tile stored as 64-column
// panels with the 128-byte swizzle (8-row atoms; tile base 1024-aligned).
__device__ __forceinline__ uint32_t swz(int rows, int r, int c) {
  return uint32_t((c >> 6) * rows * 128 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) +
                  (c & 7) * 2);
}

// One operand of a product: tile base, its rows and whether it is read
// MN-major (stored [K rows][M or N]) or K-major (stored [M or N rows][K]).
// piece: a 128 x 128 tile stored unswizzled in 16-byte pieces, element (i, j)
// at byte (j / 8) * 2048 + i * 16 + (j % 8) * 2 (the state scan's store order);
// its rows i are then N (K-major) or K (MN-major).
struct Opnd {
  uint32_t base;
  int rows;
  bool mn;
  bool piece = false;
};
// Descriptor of an unswizzled operand (layout type 0): 8 x 16-byte core
// matrices, lbo / sbo their strides along K / along M or N for K-major
// operands and along K / along M or N, swapped, for MN-major ones.
__device__ __forceinline__ uint64_t make_sdesc_plain(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFFu);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;              // descriptor version (sm_100); layout 0: no swizzle
  return d;
}
// Shared-memory descriptor of k-step kk (16 elements of K).
__device__ __forceinline__ uint64_t opnd_desc(const Opnd &o, int kk) {
  if (o.piece) {
    // K-major (rows i = N, K = j): the two core matrices of a k-step are two
    // pieces (2048 B apart), 8-row groups 128 B apart. MN-major (K = i, N = j):
    // a k-step is 16 rows (256 B); 8-column groups (pieces) 2048 B apart,
    // 8-row groups of K 128 B apart.
    if (o.mn) return make_sdesc_plain(o.base + uint32_t(kk) * 256u, 128, 2048);
    return make_sdesc_plain(o.base + uint32_t(kk) * 4096u, 2048, 128);
  }
  if (o.mn) return make_sdesc(o.base + uint32_t(kk) * 2048u, uint32_t(o.rows) * 128u, 1024);
  return make_sdesc(o.base + uint32_t(kk >> 2) * uint32_t(o.rows) * 128u + uint32_t(kk & 3) * 32u,
                    16, 1024);
}
// acc[tmem col] (+)= A B over K = 16 ksteps; M = 64; N = n.
__device__ __forceinline__ void mma_product(uint32_t tmem, uint32_t col, const Opnd &a,
                                            const Opnd &b, int n, int ksteps, bool accumulate,
                                            bool negate = false) {
  const uint32_t idesc = make_idesc_bf16(64, n, a.mn ? 1 : 0, b.mn ? 1 : 0, negate ? 1 : 0);
  for (int kk = 0; kk < ksteps; ++kk)
    tc_mma_bf16(tmem + col, opnd_desc(a, kk), opnd_desc(b, kk), idesc,
                (accumulate || kk > 0) ? 1u : 0u);
}

// 32 (x4: 16) columns of an M = 64 accumulator: r[4 j + 0..3] = rows
// lane/4 and lane/4 + 8 of the warp's 16-row block, columns 8 j + 2 (lane % 4), +1.
__device__ __forceinline__ void tmem_ld16x256_x4(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// After tcgen05.wait::ld: ties later uses of the loaded registers to the wait.
template <int N>
__device__ __forceinline__ void reg_dep(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}
template <int NJ>
__device__ __forceinline__ void to_acc(float (&acc)[NJ][4], const uint32_t (&r)[4 * NJ]) {
#pragma unroll
  for (int j = 0; j < NJ; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[j][e] = __uint_as_float(r[4 * j + e]);
}

// A warp's share of an M = 64 accumulator: rows 16 (w % 4) + g (+ 8), columns
// col0 + 8 j + 2 t (+1) for j < NJ, as acc[j][0..3] (NJ = 8: 64 columns per
// warp, N = 128 split over the two warps of each row block; NJ = 4: 32 of 64).
template <int NJ>
__device__ __forceinline__ void load_acc(float (&acc)[NJ][4], uint32_t taddr) {
  if constexpr (NJ == 2) {
    uint32_t r[8];
    tmem_ld16x256_x2(taddr, r);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][e] = __uint_as_float(r[4 * j + e]);
  } else if constexpr (NJ == 8) {
    uint32_t r[32];
    tmem_ld16x256_x8(taddr, r);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][e] = __uint_as_float(r[4 * j + e]);
  } else {
    uint32_t r[16];
    tmem_ld16x256_x4(taddr, r);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][e] = __uint_as_float(r[4 * j + e]);
  }
}

// Calls f(j, hf, row, col) for the fragment pairs (row, col..col+1) of a
// warp's tile with origin (m0, n0); the pair is acc[j][2 hf], acc[j][2 hf + 1].
template <int NJ, typename F>
__device__ __forceinline__ void each_pair(int m0, int n0, int lane, F &&f) {
#pragma unroll
  for (int j = 0; j < NJ; ++j)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf)
      f(j, hf, m0 + (lane >> 2) + 8 * hf, n0 + 8 * j + 2 * (lane & 3));
}

// Adds the per-row partial sums part[hf] (rows m0 + lane/4 + 8 hf) over the
// four lanes of a row, then into dst[row].
__device__ __forceinline__ void add_rows(float *dst, const float (&part)[2], int m0, int lane) {
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    float x = part[hf];
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    if ((lane & 3) == 0) atomicAdd(dst + m0 + (lane >> 2) + 8 * hf, x);
  }
}
// Subtracts the per-column partial sums part[j][b] (columns n0 + 8 j + 2 t + b)
// over the eight lanes of a column from dst[col].
template <int NJ>
__device__ __forceinline__ void sub_cols(float *dst, const float (&part)[NJ][2], int n0, int lane) {
#pragma unroll
  for (int j = 0; j < NJ; ++j)
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      float x = part[j][b];
      x += __shfl_xor_sync(0xffffffffu, x, 4);
      x += __shfl_xor_sync(0xffffffffu, x, 8);
      x += __shfl_xor_sync(0xffffffffu, x, 16);
      if ((lane >> 2) == 0) atomicAdd(dst + n0 + 8 * j + 2 * (lane & 3) + b, -x);
    }
}

__device__ __forceinline__ float2 swz_ld(const uint8_t *t, int rows, int r, int c) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(t + swz(rows, r, c)));
}
__device__ __forceinline__ void swz_st(uint8_t *t, int rows, int r, int c, float x, float y) {
  *reinterpret_cast<uint32_t *>(t + swz(rows, r, c)) = pack_bf16x2(x, y);
}

// Loads by TMA (one thread; coordinates past the tensors read as zero):
// tokens q, k, v, dO [rows, H, 128] (box 64 x 1 x 64, two per tile); -W, T
// diag(beta), P [units * 64][*] and (D K)^T [units * 128][64] (box 64 x rows);
// G' [units * 128][128] (box 64 x 128). S_c, stored by the scan in 16-byte
// pieces (piece p of row i at p * 128 + i), arrives by one 32 KB bulk copy in
// that order and is read by the MMAs through unswizzled descriptors.
__global__ void __launch_bounds__(kUnitThreads, 1) gdn_bwd_unit_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_kt,
    const __grid_constant__ CUtensorMap tm_tb, const __grid_constant__ CUtensorMap tm_pm,
    const __grid_constant__ CUtensorMap tm_gp, const bf16 *__restrict__ s_chunks,
    const float *__restrict__ g, float *__restrict__ dq, float *__restrict__ dk,
    float *__restrict__ dv, float *__restrict__ dg, float *__restrict__ dbeta, int H,
    uint32_t *__restrict__ ctrl, const ChunkInfo *__restrict__ table, long long rows,
    int max_chunks) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool epi = warp < kWarps, issuer = warp == kWarps && lane == 0;
  const uint32_t sb = smem_u32(sm);
  float *Gam = reinterpret_cast<float *>(sm + kV_VEC);   // log2(e) Gamma
  float *gam = Gam + 64, *Dv = Gam + 128, *dGam = Gam + 192, *dBet = Gam + 256,
        *delta = Gam + 320;
  float *red = reinterpret_cast<float *>(sm + kV_RED);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kV_BAR);   // MMA groups (2), loads A, B
  uint64_t *ld_a = bars + 2, *ld_b = bars + 3;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kV_BAR + 32);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kV_BAR + 36);
  if (tid == 0) {
    *abort_flag = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) mbar_init(bars + b, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // epilogue ownership: rows [m0, m0 + 16) (TMEM lanes 32 (w % 4) ..), columns
  // [n0, n0 + 32) of N = 128 accumulators, [p0, p0 + 16) of N = 64 ones
  const int m0 = 16 * (warp & 3), n0 = 32 * (warp >> 2), p0 = 16 * (warp >> 2);
  const uint32_t lanes = tmem + (uint32_t(32 * (warp & 3)) << 16);
  // operands
  const Opnd Qm{sb + kV_Q, 64, true};
  const Opnd Kk{sb + kV_K, 64, false}, Km{sb + kV_K, 64, true};
  const Opnd Vm{sb + kV_V, 64, true};
  const Opnd DOk{sb + kV_DO, 64, false}, DOm{sb + kV_DO, 64, true};
  const Opnd Sk{sb + kV_S, 128, false, true}, Sm{sb + kV_S, 128, true, true};
  const Opnd GPk{sb + kV_GP, 128, false}, GPm{sb + kV_GP, 128, true};
  const Opnd TBk{sb + kV_TB, 64, false}, TBm{sb + kV_TB, 64, true};
  const Opnd Pk{sb + kV_P, 64, false}, Pm{sb + kV_P, 64, true};
  const Opnd Wk{sb + kV_W, 64, false}, DXm{sb + kV_W, 64, true};
  const Opnd KTm{sb + kV_KT, 128, true}, DVk{sb + kV_KT, 64, false}, DVm{sb + kV_KT, 64, true};
  const Opnd Xk{sb + kV_X, 64, false}, Xm{sb + kV_X, 64, true};
  const Opnd Lk{sb + kV_L, 64, false}, Lm{sb + kV_L, 64, true};
  // Each phase is one or two MMA groups, committed to the two mbarriers in
  // turn (at most one phase of a barrier is ever outstanding): `issue` hands
  // the shared-memory writes to the tensor core and one thread issues the
  // groups; `wait_group` waits for the oldest outstanding group.
  uint32_t parity[2] = {0u, 0u};
  int next_commit = 0, next_wait = 0;
  auto issue = [&](auto &&a, auto &&b, bool two) {
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (issuer) {
      tc_fence_after();
      if (!*abort_flag) a();
      tc_commit(bars + (next_commit & 1));
      if (two) {
        if (!*abort_flag) b();
        tc_commit(bars + ((next_commit + 1) & 1));
      }
    }
    next_commit += two ? 2 : 1;
  };
  auto wait_group = [&]() {   // epilogue warps: the oldest outstanding group
    const int b = next_wait & 1;
    mbar_wait(bars + b, parity[b], ctrl, abort_flag);
    parity[b] ^= 1u;
    ++next_wait;
    tc_fence_after();
  };
  auto none = [] {};
  const int nunits = (ctrl[0] & kErrBadSeqlens) ? 0 : int(ctrl[1]) * H;
  auto info = [&](int u) {
    const int c = u / H;
    return GDN_IN_BOUNDS(ctrl, c, max_chunks) ? table[c] : ChunkInfo{0, 0, 0, 0};
  };
  // group A (Q, K, P) and group B (V, dO, S_c, G', T diag(beta), -W, (D K)^T)
  // of unit u, issued by the issuer thread; each load completes one phase of
  // its barrier.
  int na = 0, nb = 0;
  auto load_a = [&](int u) {
    const ChunkInfo c = info(u);
    const int hu = u % H;
    mbar_arrive_expect_tx(ld_a, 2 * 16384 + 8192);
    tma_load_3d(sm + kV_Q, &tm_q, ld_a, 0, hu, c.row0);
    tma_load_3d(sm + kV_Q + 8192, &tm_q, ld_a, 64, hu, c.row0);
    tma_load_3d(sm + kV_K, &tm_k, ld_a, 0, hu, c.row0);
    tma_load_3d(sm + kV_K + 8192, &tm_k, ld_a, 64, hu, c.row0);
    tma_load_2d(sm + kV_P, &tm_pm, ld_a, 0, u * kC);
    ++na;
  };
  auto load_b = [&](int u) {
    const ChunkInfo c = info(u);
    const int hu = u % H;
    mbar_arrive_expect_tx(ld_b, 4 * 16384 + 2 * 32768 + 8192);
    bulk_load(sm + kV_S, s_chunks + (long long)u * (kD * kD), 32768, ld_b);
    tma_load_3d(sm + kV_V, &tm_v, ld_b, 0, hu, c.row0);
    tma_load_3d(sm + kV_V + 8192, &tm_v, ld_b, 64, hu, c.row0);
    tma_load_3d(sm + kV_DO, &tm_do, ld_b, 0, hu, c.row0);
    tma_load_3d(sm + kV_DO + 8192, &tm_do, ld_b, 64, hu, c.row0);
    tma_load_2d(sm + kV_GP, &tm_gp, ld_b, 0, u * kD);
    tma_load_2d(sm + kV_GP + 16384, &tm_gp, ld_b, 64, u * kD);
    tma_load_2d(sm + kV_TB, &tm_tb, ld_b, 0, u * kC);
    tma_load_2d(sm + kV_W, &tm_w, ld_b, 0, u * kC);
    tma_load_2d(sm + kV_W + 8192, &tm_w, ld_b, 64, u * kC);
    tma_load_2d(sm + kV_KT, &tm_kt, ld_b, 0, u * kD);
    ++nb;
  };
  bool first = true;
  int it_count = 0;
  for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x) {
    const int chunk = unit / H, h = unit - chunk * H;
    const ChunkInfo ci =
        GDN_IN_BOUNDS(ctrl, chunk, max_chunks) ? table[chunk] : ChunkInfo{0, 0, 0, 0};
    const int len = ci.len;
    // ---- loads. Both groups of this unit were issued during the previous
    // one, each as soon as its last reader there was done (group B after phase
    // 5's products, group A (Q, K, P) after phase 6's); the first unit's here.
    if (issuer && first) {
      load_b(unit);
      load_a(unit);
    }
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
    {
      // this unit's tiles landed (group B was issued during the previous unit);
      // rows of q, k, v, dO past the chunk's end (the next sequence's) to zero
      const uint32_t ph = uint32_t(it_count) & 1u;
      mbar_wait(ld_a, ph, ctrl, abort_flag);
      mbar_wait(ld_b, ph, ctrl, abort_flag);
      for (int e = tid; epi && e < (kC - len) * 16; e += kThreads) {
        const int r = len + (e >> 4), c8 = 8 * (e & 15);
        const uint32_t o = swz(64, r, c8);
        const uint4 z = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>(sm + kV_Q + o) = z;
        *reinterpret_cast<uint4 *>(sm + kV_K + o) = z;
        *reinterpret_cast<uint4 *>(sm + kV_V + o) = z;
        *reinterpret_cast<uint4 *>(sm + kV_DO + o) = z;
      }
    }
    // ---- phase 1
    issue([&] {
      mma_product(tmem, kC0, TBk, Vm, 128, 4, false);       // X = TB V
      mma_product(tmem, kC0, Wk, Sk, 128, 8, true);         //   + (-W) S^T
      mma_product(tmem, kC1, KTm, GPk, 128, 8, false);      // DKG = (D K) G'^T
    }, [&] {
      mma_product(tmem, kC3, Kk, Kk, 64, 8, false);         // K K^T
    }, true);
    if (epi) {
      // <G', S> for the last token's dGamma: S_c's piece e = (p, i) holds
      // row i, columns 8 p .. 8 p + 7, found in G' (swizzled rows) by swz
      float gs_dot = 0.f;
      for (int e = tid; e < 128 * 16; e += kThreads) {
        const int p = e >> 7, i = e & 127;
        const uint4 a = *reinterpret_cast<const uint4 *>(sm + kV_GP + swz(128, i, 8 * p));
        const uint4 b = *reinterpret_cast<const uint4 *>(sm + kV_S + 16 * e);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          gs_dot = fmaf(__uint_as_float(aw[i] << 16), __uint_as_float(bw[i] << 16), gs_dot);
          gs_dot = fmaf(__uint_as_float(aw[i] & 0xffff0000u), __uint_as_float(bw[i] & 0xffff0000u),
                        gs_dot);
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) gs_dot += __shfl_xor_sync(0xffffffffu, gs_dot, off);
      if (lane == 0) red[warp] = gs_dot;
      wait_group();
      float xr[4][4], dkg[4][4];
      {
        uint32_t r1[16], r2[16];
        tmem_ld16x256_x4(lanes + kC0 + n0, r1);
        tmem_ld16x256_x4(lanes + kC1 + n0, r2);
        tmem_ld_wait();
        reg_dep(r1);
        reg_dep(r2);
        to_acc<4>(xr, r1);
        to_acc<4>(dkg, r2);
      }
      float part[2] = {0.f, 0.f};
      each_pair<4>(m0, n0, lane, [&](int j, int hf, int r, int c) {
        swz_st(sm + kV_X, 64, r, c, xr[j][2 * hf], xr[j][2 * hf + 1]);
        part[hf] += xr[j][2 * hf] * dkg[j][2 * hf] + xr[j][2 * hf + 1] * dkg[j][2 * hf + 1];
      });
      add_rows(delta, part, m0, lane);
      wait_group();
      float kk[2][4];
      load_acc<2>(kk, lanes + kC3 + p0);
      each_pair<2>(m0, p0, lane, [&](int j, int hf, int r, int s) {
        const float e0 = s < r ? ex2(Gam[r] - Gam[s]) : 0.f;
        const float e1 = s + 1 < r ? ex2(Gam[r] - Gam[s + 1]) : 0.f;
        swz_st(sm + kV_L, 64, r, s, e0 * kk[j][2 * hf], e1 * kk[j][2 * hf + 1]);
      });
    }
    // ---- phase 2
    issue([&] {
      mma_product(tmem, kC1, Pm, DOm, 128, 4, true);        // dX = DKG + P^T dO
    }, [&] {
      mma_product(tmem, kC2, Kk, Sk, 128, 8, false);        // K S^T (read in phase 4)
    }, true);
    if (epi) {
      wait_group();
      float dx[4][4];
      load_acc<4>(dx, lanes + kC1 + n0);
      each_pair<4>(m0, n0, lane, [&](int j, int hf, int r, int c) {
        swz_st(sm + kV_W, 64, r, c, dx[j][2 * hf], dx[j][2 * hf + 1]);
      });
    }
    // ---- phase 3
    issue([&] { mma_product(tmem, kC0, TBm, DXm, 128, 4, false); }, none, false);   // dV = TB^T dX
    if (epi) {
      wait_group();   // K S^T
      wait_group();   // dV
      float a[4][4];
      load_acc<4>(a, lanes + kC0 + n0);
      each_pair<4>(m0, n0, lane, [&](int j, int hf, int r, int c) {
        swz_st(sm + kV_KT, 64, r, c, a[j][2 * hf], a[j][2 * hf + 1]);
        const long long o = (((long long)ci.row0 + r) * H + h) * kD + c;
        if (r < len && GDN_IN_BOUNDS(ctrl, o + 1, rows * H * kD))
          *reinterpret_cast<float2 *>(dv + o) = make_float2(a[j][2 * hf], a[j][2 * hf + 1]);
      });
    }
    // ---- phase 4
    // L is read by the second group's products and rewritten (as R) after
    // it: the first group's epilogue handles dP, then waits for the second
    issue([&] {
      mma_product(tmem, kC0, DOk, Xk, 64, 8, false);        // dP = dO X^T  (cols 0..63)
      mma_product(tmem, kC0 + 64, DVk, Xk, 64, 8, false);   // R' = dV X^T (cols 64..127)
    }, [&] {
      mma_product(tmem, kC1, Lm, DVm, 128, 4, true, true);  // dY = dX - L^T dV
      mma_product(tmem, kC3, Lk, Xm, 128, 4, false);        // L X
    }, true);
    if (epi) {
      wait_group();
      float dp[2][4], rp[2][4];
      {
        uint32_t r1[8], r2[8];
        tmem_ld16x256_x2(lanes + kC0 + p0, r1);
        tmem_ld16x256_x2(lanes + kC0 + 64 + p0, r2);
        tmem_ld_wait();
        reg_dep(r1);
        reg_dep(r2);
        to_acc<2>(dp, r1);
        to_acc<2>(rp, r2);
      }
      // dP .* P -> dGamma and dP .* E (s <= r) over P, while the second group runs
      float rows_[2] = {0.f, 0.f}, cols_[2][2] = {};
      each_pair<2>(m0, p0, lane, [&](int j, int hf, int r, int s) {
        const float2 pp = swz_ld(sm + kV_P, 64, r, s);
        const float *a = &dp[j][2 * hf];
        const float f0 = a[0] * pp.x, f1 = a[1] * pp.y;
        rows_[hf] += f0 + f1;
        cols_[j][0] += f0;
        cols_[j][1] += f1;
        const float e0 = s <= r ? ex2(Gam[r] - Gam[s]) : 0.f;
        const float e1 = s + 1 <= r ? ex2(Gam[r] - Gam[s + 1]) : 0.f;
        swz_st(sm + kV_P, 64, r, s, e0 * a[0], e1 * a[1]);
      });
      wait_group();   // L is free once L^T dV and L X are done
      // -R' .* L -> dGamma, and R = -R' .* E (s < r) over L
      each_pair<2>(m0, p0, lane, [&](int j, int hf, int r, int s) {
        const float2 ll = swz_ld(sm + kV_L, 64, r, s);
        const float *b = &rp[j][2 * hf];
        const float f0 = -b[0] * ll.x, f1 = -b[1] * ll.y;
        rows_[hf] += f0 + f1;
        cols_[j][0] += f0;
        cols_[j][1] += f1;
        const float e0 = s < r ? ex2(Gam[r] - Gam[s]) : 0.f;
        const float e1 = s + 1 < r ? ex2(Gam[r] - Gam[s + 1]) : 0.f;
        swz_st(sm + kV_L, 64, r, s, -e0 * b[0], -e1 * b[1]);
      });
      add_rows(dGam, rows_, m0, lane);
      sub_cols<2>(dGam, cols_, p0, lane);
      // e = V - gamma (K S^T) - L X;  dbeta = rowsum(dY .* e)
      {
        float dy[4][4], ks[4][4], lx[4][4];
        load_acc<4>(dy, lanes + kC1 + n0);
        load_acc<4>(ks, lanes + kC2 + n0);
        load_acc<4>(lx, lanes + kC3 + n0);
        float part[2] = {0.f, 0.f};
        each_pair<4>(m0, n0, lane, [&](int j, int hf, int r, int c) {
          const float2 vv = swz_ld(sm + kV_V, 64, r, c);
          const float e0 = vv.x - gam[r] * ks[j][2 * hf] - lx[j][2 * hf];
          const float e1 = vv.y - gam[r] * ks[j][2 * hf + 1] - lx[j][2 * hf + 1];
          part[hf] += dy[j][2 * hf] * e0 + dy[j][2 * hf + 1] * e1;
        });
        add_rows(dBet, part, m0, lane);
      }
    }
    // ---- phase 5
    issue([&] {
      mma_product(tmem, kC0, DOk, Sm, 128, 8, false);       // dO S
      mma_product(tmem, kC1, Pk, Km, 128, 4, false);        // (dP .* E) K
    }, [&] {
      mma_product(tmem, kC2, Xk, GPm, 128, 8, false);       // X G'
      mma_product(tmem, kC3, DVk, Sm, 128, 8, false);       // dV S
    }, true);
    float dkp[4][4];   // D (X G') - gamma (dV S): the first part of dk
    if (epi) {
      wait_group();
      float a[4][4], b[4][4];
      {
        uint32_t r1[16], r2[16];
        tmem_ld16x256_x4(lanes + kC0 + n0, r1);
        tmem_ld16x256_x4(lanes + kC1 + n0, r2);
        tmem_ld_wait();
        reg_dep(r1);
        reg_dep(r2);
        to_acc<4>(a, r1);
        to_acc<4>(b, r2);
      }
      float part[2] = {0.f, 0.f};
      each_pair<4>(m0, n0, lane, [&](int j, int hf, int r, int c) {
        const float2 qq = swz_ld(sm + kV_Q, 64, r, c);
        part[hf] += gam[r] * (qq.x * a[j][2 * hf] + qq.y * a[j][2 * hf + 1]);
        const long long o = (((long long)ci.row0 + r) * H + h) * kD + c;
        if (r < len && GDN_IN_BOUNDS(ctrl, o + 1, rows * H * kD))
          *reinterpret_cast<float2 *>(dq + o) =
              make_float2(gam[r] * a[j][2 * hf] + b[j][2 * hf],
                          gam[r] * a[j][2 * hf + 1] + b[j][2 * hf + 1]);
      });
      add_rows(dGam, part, m0, lane);
      wait_group();
      {
        uint32_t r1[16], r2[16];
        tmem_ld16x256_x4(lanes + kC2 + n0, r1);
        tmem_ld16x256_x4(lanes + kC3 + n0, r2);
        tmem_ld_wait();
        reg_dep(r1);
        reg_dep(r2);
        to_acc<4>(a, r1);
        to_acc<4>(b, r2);
      }
      float part2[2] = {0.f, 0.f};
      each_pair<4>(m0, n0, lane, [&](int j, int hf, int r, int c) {
        const float2 kk2 = swz_ld(sm + kV_K, 64, r, c);
        part2[hf] -= gam[r] * (kk2.x * b[j][2 * hf] + kk2.y * b[j][2 * hf + 1]);
        dkp[j][2 * hf] = Dv[r] * a[j][2 * hf] - gam[r] * b[j][2 * hf];
        dkp[j][2 * hf + 1] = Dv[r] * a[j][2 * hf + 1] - gam[r] * b[j][2 * hf + 1];
      });
      add_rows(dGam, part2, m0, lane);
    }
    if (issuer && unit + int(gridDim.x) < nunits) {
      // phase 5's second group (the last reader of the group-B tiles) done:
      // the next unit's group B loads during the rest of this one
      const int gidx = next_commit - 1;
      mbar_wait(bars + (gidx & 1), uint32_t(gidx >> 1) & 1u, ctrl, abort_flag);
      load_b(unit + int(gridDim.x));
    }
    // ---- phase 6
    issue([&] {
      mma_product(tmem, kC0, Pm, Qm, 128, 4, false);        // (dP .* E)^T Q
      mma_product(tmem, kC0, Lk, Km, 128, 4, true);         //   + R K
      mma_product(tmem, kC0, Lm, Km, 128, 4, true);         //   + R^T K
    }, none, false);
    if (issuer && unit + int(gridDim.x) < nunits) {
      // phase 6's group (the last reader of Q, K and P; the epilogues read
      // them before its issue) done: the next unit's group A loads now
      const int gidx = next_commit - 1;
      mbar_wait(bars + (gidx & 1), uint32_t(gidx >> 1) & 1u, ctrl, abort_flag);
      load_a(unit + int(gridDim.x));
    }
    if (epi) {
      wait_group();
      float a[4][4];
      load_acc<4>(a, lanes + kC0 + n0);
      each_pair<4>(m0, n0, lane, [&](int j, int hf, int r, int c) {
        const long long o = (((long long)ci.row0 + r) * H + h) * kD + c;
        if (r < len && GDN_IN_BOUNDS(ctrl, o + 1, rows * H * kD))
          *reinterpret_cast<float2 *>(dk + o) =
              make_float2(dkp[j][2 * hf] + a[j][2 * hf], dkp[j][2 * hf + 1] + a[j][2 * hf + 1]);
      });
    }
    tc_fence_before();
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
    first = false;
    ++it_count;
  }
  if (issuer) {
    // after an abort: copies still in flight land before the CTA exits (bounded)
    volatile int keep_waiting = 0;
    if (na > 0) mbar_wait(ld_a, uint32_t(na - 1) & 1u, ctrl, &keep_waiting);
    if (nb > 0) mbar_wait(ld_b, uint32_t(nb - 1) & 1u, ctrl, &keep_waiting);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ chain
// The reverse chain over a sequence's chunks on tcgen05. Row i of dS_c depends
// only on row i of dS_{c+1}, so each (sequence, head) runs as two CTAs of 64
// d_v rows. The slice of G = dL/dS (64 d_v x 128 d_k, fp32) lives in tensor
// memory as an M = 64 accumulator; per chunk c, with G = dS_{c+1}:
//   E0  G -> bf16 G' (operand, and dS_{c+1} for the unit kernel)
//   M1  dX = P^T dO + (D K) G'^T                    [64 tokens x 64 d_v]
//       then, behind it in the tensor pipe: G *= gamma_last (tcgen05.st) and
//       G += dO^T (gamma Q)
//   E1  dX -> bf16
//   M2  G += dX^T (-W)                              [64 d_v x 128 d_k]
// Only E0 -> M1 -> E1 -> M2 is sequential. Warp 8 is the issuer: one thread
// loads the chunks' tiles by TMA (three stages, two chunks ahead, 128-byte
// swizzle: the layouts the MMAs read) and issues every MMA, each group when
// the mbarrier of its operands completes. Warps 0-7 run the epilogues E0 and
// E1 and the gamma_last scaling of G; warps 9-12 copy each G' tile to global
// memory and prepare each landed stage (the dO tail zeroed, Q scaled by
// gamma), all handing over on mbarriers.
constexpr int kChainEpi = 256, kChainLoad = 128, kChainThreads = kChainEpi + 32 + kChainLoad;
constexpr int kChainSlices = 2, kChainRows = kD / kChainSlices;
constexpr uint32_t kH_G = 0;                  // G' bf16 [64 d_v][128 d_k]: two 8 KB panels
constexpr uint32_t kH_DX = kH_G + 16384;      // dX bf16 [64 tokens][64 d_v]: one panel
constexpr uint32_t kH_STAGE = kH_DX + 8192;
constexpr uint32_t kHs_KT = 0;                // (D K)^T [128 d_k][64 tokens]: one 16 KB panel
constexpr uint32_t kHs_P = kHs_KT + 16384;    // P [64][64]
constexpr uint32_t kHs_DO = kHs_P + 8192;     // dO slice [64 tokens][64 d_v]
constexpr uint32_t kHs_W = kHs_DO + 8192;     // -W [64][128]
constexpr uint32_t kHs_Q = kHs_W + 16384;     // Q [64][128], then gamma Q
constexpr uint32_t kHs_GAM = kHs_Q + 16384;   // gamma [64], D [64]
constexpr uint32_t kHStage = kHs_GAM + 1024;  // (1 KB keeps the stages 1024-aligned)
constexpr uint32_t kStageBytes = 16384 + 8192 + 8192 + 16384 + 16384 + 512;   // one stage's TMA bytes
constexpr int kChainStages = 3;
constexpr uint32_t kH_BAR = kH_STAGE + kChainStages * kHStage;   // 13 mbarriers, TMEM slot, abort flag
constexpr uint32_t kChainSmem = kH_BAR + 128 + 1024;
static_assert(kHStage % 1024 == 0 && kH_STAGE % 1024 == 0 && kChainSmem <= 232448,
              "chain kernel shared memory");

__device__ __forceinline__ void tmem_st16x256_x8(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Tensor maps: q and dO as [rows, H, 128] tokens (box 64 x 1 x 64); -W
// [units * 64][128], (D K)^T [units * 128][64] and P [units * 64][64] (box
// 64 x rows); the decay factors [units][128] fp32 (one row).
__global__ void __launch_bounds__(kChainThreads, 1) gdn_bwd_chain_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_kt,
    const __grid_constant__ CUtensorMap tm_pm, const __grid_constant__ CUtensorMap tm_gm,
    const float *__restrict__ d_sN, float *__restrict__ ds0, bf16 *__restrict__ gprime, int H,
    uint32_t *__restrict__ ctrl, const ChunkInfo *__restrict__ table,
    const int32_t *__restrict__ seq_first, int N, int max_chunks) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x, h = blockIdx.y, i0 = kChainRows * int(blockIdx.z);
  const uint32_t sb = smem_u32(sm);
  // mbarriers. One phase per chunk unless noted; "x8": one arrival per epilogue warp.
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kH_BAR);
  uint64_t *full = bar;           // [3] stage's TMA bytes landed (one phase per use of the stage)
  uint64_t *ready = bar + 3;      // [3] x4: stage's dO tail zeroed and Q scaled (per use)
  uint64_t *gb_full = bar + 6;    // x8: G' (bf16) written
  uint64_t *g_scaled = bar + 7;   // x8: G *= gamma_last stored to tensor memory
  uint64_t *dx_full = bar + 8;    // commit: dX accumulated
  uint64_t *dxs_full = bar + 9;   // x8: dX (bf16) written, dX columns read
  uint64_t *g_full = bar + 10;    // commit: every product of the chunk done
  uint64_t *drain = bar + 11;     // commit: the issuer's last MMAs done (teardown)
  uint64_t *gb_free = bar + 12;   // x4: G' copied to global memory (the tile may be rewritten)
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kH_BAR + 104);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kH_BAR + 108);
  if (tid == 0) {
    *abort_flag = 0;
    for (int st = 0; st < kChainStages; ++st) {
      mbar_init(full + st, 1);
      mbar_init(ready + st, kChainLoad / 32);
    }
    mbar_init(gb_free, kChainLoad / 32);
    mbar_init(gb_full, kChainEpi / 32);
    mbar_init(g_scaled, kChainEpi / 32);
    mbar_init(dx_full, 1);
    mbar_init(dxs_full, kChainEpi / 32);
    mbar_init(g_full, 1);
    mbar_init(drain, 1);
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
  constexpr uint32_t kCG = 0, kCX = 128;      // TMEM columns: G (128), dX (64)
  int c0 = 0, nch = 0;
  if (!(ctrl[0] & kErrBadSeqlens) && GDN_IN_BOUNDS(ctrl, n + 1, N + 1)) {
    c0 = seq_first[n];
    nch = seq_first[n + 1] - c0;
  }
  auto info_of = [&](int c) {
    const long long chunk = c0 + c;
    return GDN_IN_BOUNDS(ctrl, chunk, max_chunks) ? table[chunk] : ChunkInfo{0, 0, 0, 0};
  };
  // Iteration k runs chunk nch - 1 - k from stage k % 3 (the stage's (k / 3)-th use).
  if (warp == kChainEpi / 32) {
    // ------------------------------------------------------------ issuer
    if (lane == 0) {
      int issued = 0;
      auto load = [&](int k) {   // TMA of iteration k's tiles (coordinates past the tensors read as zero)
        const int c = nch - 1 - k;
        const int unit = (c0 + c) * H + h;
        const ChunkInfo ci = info_of(c);
        uint8_t *stage = sm + kH_STAGE + (k % kChainStages) * kHStage;
        uint64_t *fb = full + k % kChainStages;
        mbar_arrive_expect_tx(fb, kStageBytes);
        tma_load_2d(stage + kHs_KT, &tm_kt, fb, 0, unit * kD);
        tma_load_2d(stage + kHs_P, &tm_pm, fb, 0, unit * kC);
        tma_load_3d(stage + kHs_DO, &tm_do, fb, i0, h, ci.row0);
        tma_load_2d(stage + kHs_W, &tm_w, fb, 0, unit * kC);
        tma_load_2d(stage + kHs_W + 8192, &tm_w, fb, 64, unit * kC);
        tma_load_3d(stage + kHs_Q, &tm_q, fb, 0, h, ci.row0);
        tma_load_3d(stage + kHs_Q + 8192, &tm_q, fb, 64, h, ci.row0);
        tma_load_2d(stage + kHs_GAM, &tm_gm, fb, 0, unit);
        issued = k + 1;
      };
      auto wait_on = [&](uint64_t *b, uint32_t ph) {
        mbar_wait(b, ph, ctrl, abort_flag);
        tc_fence_after();
        return !*abort_flag;
      };
      for (int k = 0; k < kChainStages && k < nch; ++k) load(k);
      for (int it = 0; it < nch; ++it) {
        const int st = it % kChainStages;
        const uint32_t ph = uint32_t(it) & 1u, sa = sb + kH_STAGE + uint32_t(st) * kHStage;
        const Opnd Pm{sa + kHs_P, 64, true}, DOm{sa + kHs_DO, 64, true};
        const Opnd KTm{sa + kHs_KT, 128, true}, Gk{sb + kH_G, 64, false};
        const Opnd Wm{sa + kHs_W, 64, true}, Qm{sa + kHs_Q, 64, true};
        const Opnd DXm{sb + kH_DX, 64, true};
        // the previous chunk's stage is free once its products are done
        if (it >= 1 && wait_on(g_full, ph ^ 1u) && it + 2 < nch) load(it + 2);
        if (wait_on(ready + st, uint32_t(it / kChainStages) & 1u))
          mma_product(tmem, kCX, Pm, DOm, 64, 4, false);       // dX = P^T dO
        if (wait_on(gb_full, ph)) mma_product(tmem, kCX, KTm, Gk, 64, 8, true);   // + (D K) G'^T
        tc_commit(dx_full);
        if (wait_on(g_scaled, ph)) mma_product(tmem, kCG, DOm, Qm, 128, 4, true);   // G += dO^T (gamma Q)
        if (wait_on(dxs_full, ph)) mma_product(tmem, kCG, DXm, Wm, 128, 4, true);   // G += dX^T (-W)
        tc_commit(g_full);
      }
      // teardown: every MMA complete and (after an abort) every copy landed
      tc_commit(drain);
      volatile int keep_waiting = 0;
      mbar_wait(drain, 0, ctrl, &keep_waiting);
      for (int k = issued - kChainStages < 0 ? 0 : issued - kChainStages; k < issued; ++k)
        mbar_wait(full + k % kChainStages, uint32_t(k / kChainStages) & 1u, ctrl, &keep_waiting);
    }
    __syncwarp();
  } else if (warp > kChainEpi / 32) {
    // ------------------------------------------------------------ loader warps
    const int lt = tid - (kChainEpi + 32);
    auto arrive = [&](uint64_t *b) {
      __syncwarp();
      if (lane == 0) mbar_arrive(b);
    };
    // Wait for iteration k's stage, zero the rows of dO past the chunk's end
    // (they belong to the next sequence) and scale Q rows by gamma (rows past
    // the end to zero).
    auto land = [&](int k) {
      const int st = k % kChainStages;
      mbar_wait(full + st, uint32_t(k / kChainStages) & 1u, ctrl, abort_flag);
      const int len = info_of(nch - 1 - k).len;
      uint8_t *stage = sm + kH_STAGE + st * kHStage;
      const float *gam = reinterpret_cast<const float *>(stage + kHs_GAM);
      for (int e = lt; e < (kC - len) * 8; e += kChainLoad) {
        const int rr = len + (e >> 3), c8 = 8 * (e & 7);
        *reinterpret_cast<uint4 *>(stage + kHs_DO + swz(64, rr, c8)) = make_uint4(0, 0, 0, 0);
      }
      for (int e = lt; e < 64 * 16; e += kChainLoad) {
        const int rr = e >> 4, c8 = 8 * (e & 15);
        uint4 *p = reinterpret_cast<uint4 *>(stage + kHs_Q + swz(64, rr, c8));
        uint4 x = make_uint4(0, 0, 0, 0);
        if (rr < len) {
          x = *p;
          const float gr = gam[rr];
          uint32_t *w = reinterpret_cast<uint32_t *>(&x);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(w + u));
            w[u] = pack_bf16x2(gr * f.x, gr * f.y);
          }
        }
        *p = x;
      }
      fence_proxy_async_smem();
      arrive(ready + st);
    };
    if (nch > 0) land(0);
    for (int it = 0; it < nch; ++it) {
      const long long unit = (long long)(c0 + nch - 1 - it) * H + h;
      // dS_{c+1} (bf16, row-major [d_v][d_k]) for the unit kernel, from the G' tile
      mbar_wait(gb_full, uint32_t(it) & 1u, ctrl, abort_flag);
      if (GDN_IN_BOUNDS(ctrl, unit, (long long)max_chunks * H)) {
        uint4 *dst = reinterpret_cast<uint4 *>(gprime + unit * (kD * kD) + size_t(i0) * kD);
        for (int e = lt; e < kChainRows * 16; e += kChainLoad) {
          const int rr = e >> 4, c16 = e & 15;
          dst[rr * 16 + c16] = *reinterpret_cast<const uint4 *>(sm + kH_G + swz(64, rr, 8 * c16));
        }
      }
      arrive(gb_free);
      if (it + 1 < nch) land(it + 1);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t lanes = tmem + (uint32_t(32 * (warp & 3)) << 16);
    const int m0 = 16 * (warp & 3);           // rows of this warp (d_v for G, tokens for dX)
    const int gn0 = 64 * (warp >> 2), xn0 = 32 * (warp >> 2);
    auto arrive = [&](uint64_t *b) {
      __syncwarp();
      if (lane == 0) mbar_arrive(b);
    };
    // G slice = d_final_state rows [i0, i0 + 64) (stored [d_k][d_v]) into tensor memory
    {
      const float *src = d_sN ? d_sN + (size_t(n) * H + h) * kD * kD : nullptr;
      uint32_t r[32];
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = i0 + m0 + (lane >> 2) + 8 * (e >> 1);
          const int jj = gn0 + 8 * j + 2 * (lane & 3) + (e & 1);
          r[4 * j + e] = __float_as_uint(src ? src[jj * kD + i] : 0.f);
        }
      tmem_st16x256_x8(lanes + kCG + gn0, r);
      tmem_st_wait();
    }
    for (int it = 0; it < nch; ++it) {
      const uint32_t ph = uint32_t(it) & 1u;
      const float *gam =
          reinterpret_cast<const float *>(sm + kH_STAGE + (it % kChainStages) * kHStage + kHs_GAM);
      if (it >= 1) {
        mbar_wait(g_full, ph ^ 1u, ctrl, abort_flag);
        tc_fence_after();
      }
      // the stage landed (gamma_last is read below)
      mbar_wait(ready + it % kChainStages, uint32_t(it / kChainStages) & 1u, ctrl, abort_flag);
      // E0: G' -> bf16 (operand of the dX product)
      uint32_t r[32];
      tmem_ld16x256_x8(lanes + kCG + gn0, r);
      tmem_ld_wait();
      reg_dep(r);
      if (it >= 1) mbar_wait(gb_free, ph ^ 1u, ctrl, abort_flag);   // previous G' copied out
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
          swz_st(sm + kH_G, 64, m0 + (lane >> 2) + 8 * hf, gn0 + 8 * j + 2 * (lane & 3),
                 __uint_as_float(r[4 * j + 2 * hf]), __uint_as_float(r[4 * j + 2 * hf + 1]));
      fence_proxy_async_smem();
      arrive(gb_full);
      // G *= gamma_last in tensor memory (the chunk's products then accumulate on it)
      const float gl = gam[kC - 1];
#pragma unroll
      for (int u = 0; u < 32; ++u) r[u] = __float_as_uint(gl * __uint_as_float(r[u]));
      tmem_st16x256_x8(lanes + kCG + gn0, r);
      tmem_st_wait();
      tc_fence_before();
      arrive(g_scaled);
      // E1: dX -> bf16 [tokens][d_v]
      mbar_wait(dx_full, ph, ctrl, abort_flag);
      tc_fence_after();
      {
        float a[4][4];
        load_acc<4>(a, lanes + kCX + xn0);
        each_pair<4>(m0, xn0, lane, [&](int j, int hf, int rr, int cc) {
          swz_st(sm + kH_DX, 64, rr, cc, a[j][2 * hf], a[j][2 * hf + 1]);
        });
      }
      fence_proxy_async_smem();
      tc_fence_before();
      arrive(dxs_full);
    }
    if (nch > 0) {
      mbar_wait(g_full, uint32_t(nch - 1) & 1u, ctrl, abort_flag);
      tc_fence_after();
    }
    if (!(ctrl[0] & kErrBadSeqlens) &&
        GDN_IN_BOUNDS(ctrl, (long long)n * H + h, (long long)N * H)) {
      uint32_t r[32];
      tmem_ld16x256_x8(lanes + kCG + gn0, r);
      tmem_ld_wait();
      reg_dep(r);
      float *dst = ds0 + (size_t(n) * H + h) * kD * kD;
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = i0 + m0 + (lane >> 2) + 8 * (e >> 1);
          const int jj = gn0 + 8 * j + 2 * (lane & 3) + (e & 1);
          dst[jj * kD + i] = __uint_as_float(r[4 * j + e]);
        }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

cudaError_t launch_bwd_tc(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *s0, const int32_t *cu,
                          const void *d_o, const float *d_sN, int N, int B, int T, int H,
                          int num_seqs, float *dq, float *dkk, float *dvv, float *dg,
                          float *dbeta, float *ds0, void *ws, const BwdTcLayout &L,
                          cudaStream_t s, bool replay) {
  char *base = static_cast<char *>(ws);
  bf16 *sc = reinterpret_cast<bf16 *>(base + L.s_chunks);
  bf16 *gp = reinterpret_cast<bf16 *>(base + L.gprime);
  cudaError_t e = cudaSuccess;
  if (replay) {
    e = launch_chunk_map(cu, B, T, num_seqs, kC, ws, L.fwd, s);
    if (e != cudaSuccess) return e;
    e = launch_chunk_tc(q, k, v, g, beta, s0, B, T, H, N, nullptr, nullptr, ws, L.fwd, s, sc);
    if (e != cudaSuccess) return e;
  }
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
  // tensor maps (all zero when there are no chunks: no kernel then loads)
  CUtensorMap mq{}, mk{}, mv{}, mdo{}, mw{}, mkt{}, mtb{}, mpm{}, mgm{}, mgp{};
  const long long units = (long long)L.fwd.max_chunks * H;
  if (T > 0 && L.fwd.max_chunks > 0) {
    if (!map_tokens(&mq, q, rows, H) || !map_tokens(&mk, k, rows, H) ||
        !map_tokens(&mv, v, rows, H) || !map_tokens(&mdo, d_o, rows, H) ||
        !map_2d(&mw, base + L.fwd.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kC, kD, 64, kC,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mkt, base + L.fwd.kt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kD, kC, 64,
                kD, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mtb, base + L.fwd.tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kC, kC, 64,
                kC, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mpm, base + L.fwd.pm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kC, kC, 64,
                kC, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map_2d(&mgm, base + L.fwd.gam, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, units, 128, 128, 1,
                CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !map_2d(&mgp, gp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, units * kD, kD, 64, kD,
                CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  gdn_bwd_chain_kernel<<<dim3(N, H, kChainSlices), kChainThreads, kChainSmem, s>>>(
      mq, mdo, mw, mkt, mpm, mgm, d_sN, ds0, gp, H, ctrl, table, seq_first, N, L.fwd.max_chunks);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int sms = device_sms();
  const int grid = int(std::min<long long>(units > 0 ? units : 1, sms > 0 ? sms : 148));
  gdn_bwd_unit_kernel<<<grid, kUnitThreads, kUnitSmem, s>>>(
      mq, mk, mv, mdo, mw, mkt, mtb, mpm, mgp, sc, g, dq, dkk, dvv, dg, dbeta, H, ctrl, table,
      rows, L.fwd.max_chunks);
  (void)beta;
  return cudaGetLastError();
}

}  // namespace gdn
