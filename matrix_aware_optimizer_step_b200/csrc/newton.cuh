// newton.cuh -- Newton-Muon right-preconditioning ("The Newton-Muon
// Optimizer", section "What Is Newton-Muon?"): each layer gradient G is
// right-multiplied by the inverse of the activation second moment
// S = X^T X / N before the standard Muon step; the MLP contraction uses a
// four-block diagonal S, one d x d inverse per block of d gradient columns.
//
//   act_transpose_kernel  a d-wide activation block, transposed to bf16
//                         d x tokens: the K-major operand of S = Xt Xt^T / N,
//                         which the tensor-core engine computes (GRAM32).
//   act_split_kernel      the same for fp32 activations, split into bf16
//                         high and low parts laid out so that one GRAM32
//                         product over three times the tokens sums the
//                         three significant cross products.
//   chol_panel_kernel, chol_update_kernel  S = L L^T in place (fp32),
//                         panels of 32, two batched launches per panel
//                         (d <= 1536).
//   linv_init_kernel, linv_level_kernel  L^-1 from the diagonal blocks'
//                         inverses by recursive doubling, two batched tile
//                         products per level.
//   spd_inverse_product_kernel  S^-1 = L^-T L^-1 in 64x64 tiles of the lower
//                         triangle (mirrored), then copy_inverse_kernel.
//   cholesky_kernel, chol_solve_kernel  unblocked versions for larger d.
//   precond_prep_kernel   S^-1 split into bf16 hi + lo, once per distinct
//                         S^-1: the B operand of G' = G [S_hi; S_lo] on the
//                         tensor-core engine (PRECOND), which reads G in
//                         place.
//   precond_kernel        G' = G blockdiag(S_b^-1) with fp32 FMAs, for block
//                         widths that are not a multiple of 64.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "elementwise.cuh"   // tsw: the swizzled transposing tile

namespace muon {

template <typename D>
__device__ __forceinline__ int find_tile_desc(const D* __restrict__ d, int n, int64_t tile) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (d[mid].tile_start <= tile) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ---------------------------------------------------------------------------
// Cholesky factorisation and inverse
// ---------------------------------------------------------------------------
constexpr int CHOL_THREADS = 1024;
constexpr int CHOL_MAX_D = 4096;
constexpr int SOLVE_ROWS_PER_BLOCK = 64;    // rows of S^-1 per solve block
constexpr int SOLVE_THREADS = 512;
constexpr int kDevErrNotSPD = 2;

struct CholDesc {
  float* a;          // d x d scratch: S in, L (lower) out; strict upper: L^T
                     // (unblocked path); blocked path: the 32x32 diagonal
                     // blocks keep their input values (see t)
  float* inv;        // d x d output S^-1
  float* t;          // d x d scratch (blocked path): each 32x32 diagonal
                     // block holds that block's factor D (lower) and D^-1
                     // transposed (strict upper); elsewhere the recursive
                     // L^-1's products
  int32_t d;
  int32_t pad;
};

__global__ void __launch_bounds__(CHOL_THREADS)
    cholesky_kernel(const CholDesc* __restrict__ descs, float damping, int* err) {
  const CholDesc& c = descs[blockIdx.x];
  float* a = c.a;
  const int d = c.d;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = CHOL_THREADS / 32;
  __shared__ float s_lkk;
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  if (damping != 0.f)
    for (int i = threadIdx.x; i < d; i += CHOL_THREADS) a[int64_t(i) * d + i] += damping;
  __syncthreads();
  for (int k = 0; k < d; ++k) {
    if (threadIdx.x == 0) {
      const float akk = a[int64_t(k) * d + k];
      float l = akk > 0.f ? sqrtf(akk) : 0.f;
      if (!(akk > 0.f)) { s_bad = 1; l = 1.f; }
      a[int64_t(k) * d + k] = l;
      s_lkk = l;
    }
    __syncthreads();
    const float inv = 1.0f / s_lkk;
    for (int i = k + 1 + threadIdx.x; i < d; i += CHOL_THREADS) {
      const float l = a[int64_t(i) * d + k] * inv;
      a[int64_t(i) * d + k] = l;
      a[int64_t(k) * d + i] = l;     // L^T row k, read along rows below
    }
    __syncthreads();
    // trailing update of the lower triangle: A[i][j] -= L[i][k] L[j][k], k < j <= i
    for (int i = k + 1 + warp; i < d; i += nwarps) {
      const float lik = a[int64_t(k) * d + i];
      float* row = a + int64_t(i) * d;
      const float* lk = a + int64_t(k) * d;
      for (int j = k + 1 + lane; j <= i; j += 32) row[j] -= lik * lk[j];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0 && s_bad) atomicOr(err, kDevErrNotSPD);
}

// ---------------------------------------------------------------------------
// Blocked versions (panel width 32), used when d <= CHOL_BLOCKED_MAX_D.
// ---------------------------------------------------------------------------
constexpr int CB = 32;                      // panel width
constexpr int CBP = CB + 1;                 // padded row of a panel in smem
constexpr int CHOL_BLOCKED_MAX_D = 1536;    // widest block the blocked path takes (larger: unblocked kernels)
constexpr int CP_THREADS = 256;
constexpr int CPR = 64;                     // panel rows per chol_panel_kernel block

// Right-looking blocked Cholesky S = L L^T in place (lower triangle), batched
// over matrices, two launches per 32-wide panel at p0:
//
//   chol_panel_kernel   every block factors the panel's 32x32 diagonal block
//                       D (one warp, in shared memory) and inverts it (lane j
//                       solves for column j of D^-1); block 0 writes D to the
//                       lower triangle and D^-1 transposed to the strict
//                       upper triangle of the same block of the t scratch
//                       (read back by linv_init_kernel), never over the
//                       input that the launch's other blocks are still
//                       reading; each block then forms CPR rows of the panel
//                       below D, P = A_panel D^-T, as a product over all
//                       threads.
//   chol_update_kernel  the trailing lower triangle minus P P^T, in 64x64
//                       tiles with 4x4 register tiles (grid.x: tile).
//
// Damping (added to the diagonal) is applied to each diagonal block as it is
// loaded for factoring: every trailing update only subtracts, so the order
// does not matter.  A non-positive pivot raises kDevErrNotSPD and continues
// with pivot 1 so the launch sequence stays well defined.
__global__ void __launch_bounds__(CP_THREADS)
    chol_panel_kernel(const CholDesc* __restrict__ descs, int p0, float damping, int* err) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  const CholDesc& c = descs[blockIdx.y];
  const int d = c.d;
  if (p0 >= d) return;
  float* a = c.a;
  const int nb = min(CB, d - p0);
  const int r0 = p0 + nb + blockIdx.x * CPR;           // first panel row of this block
  if (blockIdx.x > 0 && r0 >= d) return;
  __shared__ float dg[CB][CBP];
  __shared__ float dinv[CB][CBP];
  __shared__ float ap[CPR][CBP];
  __shared__ float rdiag[CB];                          // 1 / L_ii of D
  __shared__ int bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) bad = 0;
  for (int e = tid; e < CB * CB; e += CP_THREADS) {
    const int i = e / CB, j = e % CB;
    float v = (i < nb && j <= i) ? a[int64_t(p0 + i) * d + p0 + j] : 0.f;
    if (i == j && i < nb) v += damping;
    dg[i][j] = v;
  }
  for (int e = tid; e < CPR * CB; e += CP_THREADS) {
    const int rr = e / CB, j = e % CB;
    ap[rr][j] = (r0 + rr < d && j < nb) ? a[int64_t(r0 + rr) * d + p0 + j] : 0.f;
  }
  __syncthreads();
  if (warp == 0) {
    // unblocked Cholesky of D in registers: lane i holds row i (zero above
    // the diagonal and past nb); column k travels by shuffle.  This warp's
    // serial chain is the panel launch's critical path, so the pivot's
    // reciprocal square root q (rsqrtf, within 2 ulp) gives both L_kk =
    // a_kk q and the column scaling by one multiply each, and the
    // inverse below multiplies by the stored q instead of dividing.
    float a[CB];
#pragma unroll
    for (int j = 0; j < CB; ++j) a[j] = dg[lane][j];
    bool neg = false;
#pragma unroll
    for (int k = 0; k < CB; ++k) {
      if (k < nb) {
        float akk = __shfl_sync(0xffffffffu, a[k], k);
        if (!(akk > 0.f)) { neg = true; akk = 1.f; }
        const float q = rsqrtf(akk);
        if (lane == k) { a[k] = akk * q; rdiag[k] = q; }
        else if (lane > k) a[k] *= q;
        const float lik = a[k];
#pragma unroll
        for (int j = k + 1; j < CB; ++j) {
          const float ljk = __shfl_sync(0xffffffffu, a[k], j);
          if (lane >= j) a[j] -= lik * ljk;
        }
      }
    }
    if (lane == 0 && neg) bad = 1;
#pragma unroll
    for (int j = 0; j < CB; ++j) dg[lane][j] = a[j];
    __syncwarp();
    // D x = e_lane: x = column `lane` of D^-1, forward substitution with
    // four independent partial sums per row (the chain of dependent adds is
    // a quarter as long)
    float x[CB];
#pragma unroll
    for (int i = 0; i < CB; ++i) {
      float s0 = (i == lane) ? 1.f : 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
      for (int k = 0; k + 3 < i; k += 4) {
        s0 -= dg[i][k] * x[k];
        s1 -= dg[i][k + 1] * x[k + 1];
        s2 -= dg[i][k + 2] * x[k + 2];
        s3 -= dg[i][k + 3] * x[k + 3];
      }
#pragma unroll
      for (int k = i & ~3; k < i; ++k) s0 -= dg[i][k] * x[k];
      x[i] = (i < nb) ? ((s0 + s1) + (s2 + s3)) * rdiag[i] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < CB; ++i) dinv[i][lane] = x[i];
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    // into t, not a: the other blocks of this launch read D's input from a
    float* t = c.t;
    for (int e = tid; e < nb * nb; e += CP_THREADS) {
      const int i = e / nb, j = e % nb;
      if (j <= i) t[int64_t(p0 + i) * d + p0 + j] = dg[i][j];
      else t[int64_t(p0 + i) * d + p0 + j] = dinv[j][i];     // D^-1[j][i], j > i, at (p0 + i, p0 + j)
    }
    if (tid == 0 && bad) atomicOr(err, kDevErrNotSPD);
  }
  // P[rr][j] = sum over k <= j of A[rr][k] D^-1[j][k]; 8 outputs per thread
  const int rr = tid >> 2, jb = (tid & 3) * 8;
  float out[8] = {};
#pragma unroll 4
  for (int k = 0; k < CB; ++k) {
    const float av = ap[rr][k];
#pragma unroll
    for (int v = 0; v < 8; ++v) out[v] += av * dinv[jb + v][k];   // zero for k > jb + v
  }
  if (r0 + rr < d) {
#pragma unroll
    for (int v = 0; v < 8; ++v)
      if (jb + v < nb) a[int64_t(r0 + rr) * d + p0 + jb + v] = out[v];
  }
}

// Trailing update after the panel at p0: A[i][j] -= sum over k < 32 of
// P[i][k] P[j][k] for p0 + 32 <= j <= i < d, one 64x64 lower tile per block.
constexpr int CU_T = 64;
constexpr int CU_P = CU_T + 4;              // padded row of the transposed panel slices (16-byte rows)
__global__ void __launch_bounds__(CP_THREADS) chol_update_kernel(const CholDesc* __restrict__ descs, int p0) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  const CholDesc& c = descs[blockIdx.y];
  const int d = c.d;
  const int q0 = p0 + CB;
  if (q0 >= d) return;
  const int nt = (d - q0 + CU_T - 1) / CU_T;
  const int t = blockIdx.x;
  if (t >= nt * (nt + 1) / 2) return;
  int ti = int((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
  while (ti * (ti + 1) / 2 > t) --ti;
  while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
  const int tj = t - ti * (ti + 1) / 2;
  const int i0 = q0 + ti * CU_T, j0 = q0 + tj * CU_T;
  float* a = c.a;
  __shared__ __align__(16) float pi_s[CB][CU_P];   // pi_s[k][r] = P[i0 + r][k]
  __shared__ __align__(16) float pj_s[CB][CU_P];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  for (int e = tid; e < CU_T * CB; e += CP_THREADS) {
    const int r = e / CB, k = e % CB;
    pi_s[k][r] = (i0 + r < d) ? a[int64_t(i0 + r) * d + p0 + k] : 0.f;
    pj_s[k][r] = (j0 + r < d) ? a[int64_t(j0 + r) * d + p0 + k] : 0.f;
  }
  __syncthreads();
  float acc[4][4] = {};
#pragma unroll 8
  for (int k = 0; k < CB; ++k) {
    const float4 x = *reinterpret_cast<const float4*>(&pi_s[k][ty * 4]);
    const float4 y = *reinterpret_cast<const float4*>(&pj_s[k][tx * 4]);
    const float xv[4] = {x.x, x.y, x.z, x.w}, yv[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] += xv[u] * yv[v];
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ty * 4 + u;
    if (i >= d) continue;
    const int j = j0 + tx * 4;
    float* row = a + int64_t(i) * d;
    if (j + 3 <= i && j + 3 < d && (d % 4) == 0) {
      float4 w = *reinterpret_cast<float4*>(row + j);
      w.x -= acc[u][0]; w.y -= acc[u][1]; w.z -= acc[u][2]; w.w -= acc[u][3];
      *reinterpret_cast<float4*>(row + j) = w;
    } else {
#pragma unroll
      for (int v = 0; v < 4; ++v)
        if (j + v <= i && j + v < d) row[j + v] -= acc[u][v];
    }
  }
}

// L^-1 by recursive doubling of the 32x32 diagonal blocks: for a lower
// triangular [[A, 0], [C, B]], the inverse is [[A^-1, 0], [-B^-1 C A^-1,
// B^-1]].  Level l pairs consecutive blocks of s = 32 * 2^l rows: block p
// of the level spans rows r0 = 2 s p .. r0 + s + s2 (s2 = min(s, d - r0 - s),
// the second block may be short), and once A^-1 and B^-1 are in X its
// off-diagonal block is two products,
//   T   = C A^-1         (rows r0+s.., columns r0..; A^-1 lower: k >= j)
//   X21 = -B^-1 T        (B^-1 lower: k <= i)
// so the chain of dependent launches is 2 log2(d / 32) long instead of d /
// 32 row blocks.  X is written to c.inv, T to c.t; C is read from L's lower
// triangle in c.a.  Every output is an fp32 sum of products of fp32 values,
// as in forward substitution, in a different order.
//
// linv_init_kernel: X's 64x64 diagonal tiles (grid.x: tile, grid.y: matrix)
// hold the two 32x32 diagonal-block inverses and zeros above the diagonal
// (the upper triangle of these tiles is read as zeros by the tile products
// below and by spd_inverse_product_kernel); the lower-left 32x32 block is
// left to level 0.
__global__ void __launch_bounds__(256) linv_init_kernel(const CholDesc* __restrict__ descs) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  const CholDesc& c = descs[blockIdx.y];
  const int d = c.d;
  const int t0 = blockIdx.x * 64;
  if (t0 >= d) return;
  for (int e = threadIdx.x; e < 64 * 64; e += 256) {
    const int r = t0 + (e >> 6), col = t0 + (e & 63);
    if (r >= d || col >= d) continue;
    const int br = r / CB, bc = col / CB;
    float v;
    if (bc > br || col > r) {
      v = 0.f;
    } else if (bc == br) {
      // D^-1 of the 32-block starting at p0: strict lower part stored
      // transposed above the diagonal of the factor's block in t, diagonal
      // 1/L_ii
      const int p0 = br * CB;
      v = col == r ? 1.f / c.t[int64_t(r) * d + r] : c.t[int64_t(col) * d + p0 + (r - p0)];
    } else {
      continue;      // lower-left 32x32 block: level 0
    }
    c.inv[int64_t(r) * d + col] = v;
  }
}

// 8x8 register tile of a 64x64 output tile over 64 threads: thread (ty, tx)
// owns rows {4ty .. 4ty+3, 32+4ty .. 32+4ty+3} and the same columns with tx,
// so each 16-byte shared-memory load of a warp reads contiguous bytes, and a
// thread issues 64 FMAs per four loads (a 4x4 tile over 256 threads issues
// 16 per two, which leaves the FMA pipes waiting on shared memory).
__device__ __forceinline__ int rc8(int t, int u) { return (u < 4) ? t * 4 + u : 32 + t * 4 + (u - 4); }

template <int LD>
__device__ __forceinline__ void fma_tile8(const float (*xs)[LD], const float (*ys)[LD], int kk, int ty, int tx,
                                          float (&acc)[8][8]) {
  const float4 x0 = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
  const float4 x1 = *reinterpret_cast<const float4*>(&xs[kk][32 + ty * 4]);
  const float4 y0 = *reinterpret_cast<const float4*>(&ys[kk][tx * 4]);
  const float4 y1 = *reinterpret_cast<const float4*>(&ys[kk][32 + tx * 4]);
  const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
  const float yv[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int v = 0; v < 8; ++v) acc[u][v] += xv[u] * yv[v];
}

// One product of a doubling level (grid.x: pair x output tile, grid.y:
// matrix), 64x64 output tiles, 8x8 per thread, K staged 32 at a time.
// mode 0: T = C A^-1, mode 1: X21 = -B^-1 T.  Each output is summed over k
// in increasing order, one FMA per k, whatever the register tiling.
constexpr int LV_T = 64, LV_K = 32, LV_THREADS = 64;
constexpr int LV_LOADS = LV_T * LV_K / 4 / LV_THREADS;   // 16-byte loads per thread per panel
__global__ void __launch_bounds__(LV_THREADS) linv_level_kernel(const CholDesc* __restrict__ descs, int s, int mode) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  const CholDesc& c = descs[blockIdx.y];
  const int d = c.d;
  if (d <= s) return;
  const int tiles = (s + LV_T - 1) / LV_T;                // per side of a pair's output
  const int pair = blockIdx.x / (tiles * tiles);
  const int rem = blockIdx.x % (tiles * tiles);
  const int r0 = 2 * s * pair;
  if (r0 + s >= d) return;                                // no second block
  const int s2 = min(s, d - r0 - s);
  const int it = rem / tiles, jt = rem % tiles;
  const int i0 = it * LV_T, j0 = jt * LV_T;               // output tile, relative to (r0 + s, r0)
  if (i0 >= s2) return;
  // K range: mode 0, k in [j0, s) (A^-1 lower); mode 1, k in [0, min(i0 + 64, s2)) (B^-1 lower)
  const int klo = mode == 0 ? j0 : 0;
  const int khi = mode == 0 ? s : min(i0 + LV_T, s2);
  // P[i][k], Q[k][j] (relative indices) and the output, as row-major views
  const float* P = mode == 0 ? c.a + int64_t(r0 + s) * d + r0 : c.inv + int64_t(r0 + s) * d + (r0 + s);
  const float* Q = mode == 0 ? c.inv + int64_t(r0) * d + r0 : c.t + int64_t(r0 + s) * d + r0;
  float* O = mode == 0 ? c.t + int64_t(r0 + s) * d + r0 : c.inv + int64_t(r0 + s) * d + r0;
  const int kdim = mode == 0 ? s : s2;                    // valid k of the operands
  __shared__ __align__(16) float ps[LV_K][LV_T + 4];     // P transposed: ps[k][i]
  __shared__ __align__(16) float qs[LV_K][LV_T + 4];
  const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
  float acc[8][8] = {};
  // 16-byte loads need rows that start 16-byte aligned; every operand view
  // starts at a column that is a multiple of 32
  const bool vec = (d % 4) == 0;
  const int klim = min(khi, kdim);
  // The next panel pair is loaded into registers while this one is
  // multiplied: each thread issues its 16 loads (16 bytes each) together,
  // one latency per panel, hidden behind 2048 FMAs.  Loaded one element at a
  // time into shared memory, with 64 accumulators per thread, the compiler
  // spaced the loads out and exposed each one's latency (measured 2.5x
  // slower at the same instruction count).
  float4 pv[LV_LOADS], qv[LV_LOADS];
  auto load = [&](int k0) {
#pragma unroll
    for (int n = 0; n < LV_LOADS; ++n) {
      const int e = tid + n * LV_THREADS;
      const int i = e >> 3, k4 = (e & 7) * 4;             // P: row i, k4 .. k4 + 3 of the panel
      const int gi = i0 + i, gk = k0 + k4;
      if (vec && gi < s2 && gk + 3 < klim) {
        pv[n] = *reinterpret_cast<const float4*>(P + int64_t(gi) * d + gk);
      } else {
        float* pp = reinterpret_cast<float*>(&pv[n]);
#pragma unroll
        for (int c = 0; c < 4; ++c) pp[c] = (gi < s2 && gk + c < klim) ? P[int64_t(gi) * d + gk + c] : 0.f;
      }
      const int qk = e >> 4, qj4 = (e & 15) * 4;          // Q: row qk, columns qj4 .. qj4 + 3
      const int hk = k0 + qk, hj = j0 + qj4;
      if (vec && hk < klim && hj + 3 < s) {
        qv[n] = *reinterpret_cast<const float4*>(Q + int64_t(hk) * d + hj);
      } else {
        float* qq = reinterpret_cast<float*>(&qv[n]);
#pragma unroll
        for (int c = 0; c < 4; ++c) qq[c] = (hk < klim && hj + c < s) ? Q[int64_t(hk) * d + hj + c] : 0.f;
      }
    }
  };
  if (klo < khi) load(klo);
  for (int k0 = klo; k0 < khi; k0 += LV_K) {
#pragma unroll
    for (int n = 0; n < LV_LOADS; ++n) {
      const int e = tid + n * LV_THREADS;
      const int i = e >> 3, k4 = (e & 7) * 4;
      ps[k4][i] = pv[n].x; ps[k4 + 1][i] = pv[n].y; ps[k4 + 2][i] = pv[n].z; ps[k4 + 3][i] = pv[n].w;
      *reinterpret_cast<float4*>(&qs[e >> 4][(e & 15) * 4]) = qv[n];
    }
    __syncthreads();
    if (k0 + LV_K < khi) load(k0 + LV_K);
#pragma unroll 4
    for (int kk = 0; kk < LV_K; ++kk) fma_tile8<LV_T + 4>(ps, qs, kk, ty, tx, acc);
    __syncthreads();
  }
  const float sign = mode == 0 ? 1.f : -1.f;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int i = i0 + rc8(ty, u);
    if (i >= s2) continue;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int j = j0 + rc8(tx, v);
      if (j < s) O[int64_t(i) * d + j] = sign * acc[u][v];
    }
  }
}

// S^-1 = L^-T L^-1: S^-1[i][j] = sum over k >= max(i, j) of L^-1[k][i] L^-1[k][j].
// One 64x64 tile of the lower triangle per block (grid.x: tile, grid.y:
// matrix), K in chunks of 32 rows of L^-1 staged in shared memory, 4x4
// register tiles; the tile and its mirror are written to c.a.
constexpr int SIP_T = 64, SIP_K = 32, SIP_THREADS = 256;
__global__ void __launch_bounds__(SIP_THREADS) spd_inverse_product_kernel(const CholDesc* __restrict__ descs) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  const CholDesc& c = descs[blockIdx.y];
  const int d = c.d;
  const int nt = (d + SIP_T - 1) / SIP_T;
  const int t = blockIdx.x;
  if (t >= nt * (nt + 1) / 2) return;
  int ti = int((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
  while (ti * (ti + 1) / 2 > t) --ti;
  while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
  const int tj = t - ti * (ti + 1) / 2;
  const int i0 = ti * SIP_T, j0 = tj * SIP_T;
  const float* li = c.inv;
  __shared__ __align__(16) float as[SIP_K][SIP_T];
  __shared__ __align__(16) float bs[SIP_K][SIP_T];
  __shared__ float cs[SIP_T][SIP_T + 1];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const bool vec = (d % 4) == 0;
  float acc[4][4] = {};
  for (int k0 = i0; k0 < d; k0 += SIP_K) {
    for (int e = tid; e < SIP_K * SIP_T / 4; e += SIP_THREADS) {
      const int kr = e >> 4, c4 = (e & 15) * 4;
      const int k = k0 + kr;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
      if (k < d) {
        const float* row = li + int64_t(k) * d;
        if (vec && i0 + c4 + 4 <= d) {
          a = *reinterpret_cast<const float4*>(row + i0 + c4);
        } else {
          float* pa = reinterpret_cast<float*>(&a);
          for (int u = 0; u < 4; ++u) pa[u] = i0 + c4 + u < d ? row[i0 + c4 + u] : 0.f;
        }
        if (vec && j0 + c4 + 4 <= d) {
          b = *reinterpret_cast<const float4*>(row + j0 + c4);
        } else {
          float* pb = reinterpret_cast<float*>(&b);
          for (int u = 0; u < 4; ++u) pb[u] = j0 + c4 + u < d ? row[j0 + c4 + u] : 0.f;
        }
      }
      *reinterpret_cast<float4*>(&as[kr][c4]) = a;
      *reinterpret_cast<float4*>(&bs[kr][c4]) = b;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < SIP_K; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&as[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&bs[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] += av[u] * bv[v];
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) cs[ty * 4 + u][tx * 4 + v] = acc[u][v];
  __syncthreads();
  float* out = c.a;
  for (int e = tid; e < SIP_T * SIP_T; e += SIP_THREADS) {
    const int r = e >> 6, q = e & 63;
    if (i0 + r < d && j0 + q < d) out[int64_t(i0 + r) * d + j0 + q] = cs[r][q];
  }
  if (ti != tj) {
    for (int e = tid; e < SIP_T * SIP_T; e += SIP_THREADS) {
      const int q = e >> 6, r = e & 63;      // output row j0 + q, column i0 + r
      if (i0 + r < d && j0 + q < d) out[int64_t(j0 + q) * d + i0 + r] = cs[r][q];
    }
  }
}

// c.inv = c.a (d x d), grid.y = matrix.
__global__ void __launch_bounds__(256) copy_inverse_kernel(const CholDesc* __restrict__ descs) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  const CholDesc& c = descs[blockIdx.y];
  const int64_t n = int64_t(c.d) * c.d;
  const int64_t stride = int64_t(gridDim.x) * 256;
  if (n % 4 == 0) {
    const float4* src = reinterpret_cast<const float4*>(c.a);
    float4* dst = reinterpret_cast<float4*>(c.inv);
    for (int64_t e = blockIdx.x * 256 + threadIdx.x; e < n / 4; e += stride) dst[e] = src[e];
  } else {
    for (int64_t e = blockIdx.x * 256 + threadIdx.x; e < n; e += stride) c.inv[e] = c.a[e];
  }
}

// Row j of S^-1 (= column j, S^-1 symmetric): forward L y = e_j, backward
// L^T x = y, y and x kept in the output row.
__global__ void __launch_bounds__(SOLVE_THREADS)
    chol_solve_kernel(const CholDesc* __restrict__ descs, int blocks_per_mat) {
  const CholDesc& c = descs[blockIdx.x / blocks_per_mat];
  const int part = blockIdx.x % blocks_per_mat;
  const int d = c.d;
  const float* a = c.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = SOLVE_THREADS / 32;
  for (int j = part * SOLVE_ROWS_PER_BLOCK + warp; j < min(d, (part + 1) * SOLVE_ROWS_PER_BLOCK); j += nwarps) {
    float* x = c.inv + int64_t(j) * d;
    for (int i = lane; i < j; i += 32) x[i] = 0.f;
    __syncwarp();
    // forward: y_i = (delta_ij - sum_{j<=k<i} L[i][k] y_k) / L[i][i]
    for (int i = j; i < d; ++i) {
      const float* li = a + int64_t(i) * d;
      float s = 0.f;
      for (int k = j + lane; k < i; k += 32) s += li[k] * x[k];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) x[i] = ((i == j ? 1.f : 0.f) - s) / li[i];
      __syncwarp();
    }
    // backward: x_i = (y_i - sum_{k>i} L[k][i] x_k) / L[i][i]; L[k][i] = upper row i
    for (int i = d - 1; i >= 0; --i) {
      const float* ui = a + int64_t(i) * d;
      float s = 0.f;
      for (int k = i + 1 + lane; k < d; k += 32) s += ui[k] * x[k];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) x[i] = (x[i] - s) / ui[i];
      __syncwarp();
    }
  }
}

// ---------------------------------------------------------------------------
// G' = G blockdiag(S^-1)
// ---------------------------------------------------------------------------
constexpr int PRE_BM = 64;
constexpr int PRE_BN = 64;
constexpr int PRE_BK = 32;
constexpr int PRE_THREADS = 256;

struct PrecondDesc {
  const __nv_bfloat16* grad;   // rows x cols
  const float* s_inv;          // blocks x d x d
  float* out;                  // rows x cols
  int64_t rows, cols, d;
  int64_t tile_start;
  int32_t tiles_r, tiles_c;    // per block: ceil(rows/64), ceil(d/64)
};

__global__ void __launch_bounds__(PRE_THREADS)
    precond_kernel(const PrecondDesc* __restrict__ descs, int n, const int* skip) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  if (halted(skip)) return;
  __shared__ float gs[PRE_BK][PRE_BM + 4];   // G tile, transposed (k, row)
  __shared__ float ss[PRE_BK][PRE_BN + 4];   // S^-1 tile (k, col)
  const int64_t gt = blockIdx.x;
  const PrecondDesc& p = descs[find_tile_desc(descs, n, gt)];
  int64_t lt = gt - p.tile_start;
  const int64_t per_block = int64_t(p.tiles_r) * p.tiles_c;
  const int64_t b = lt / per_block;
  lt -= b * per_block;
  const int64_t r0 = (lt / p.tiles_c) * PRE_BM, c0 = (lt % p.tiles_c) * PRE_BN;
  const int64_t gcol0 = b * p.d;                      // first gradient column of the block
  const float* s = p.s_inv + b * p.d * p.d;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < p.d; k0 += PRE_BK) {
    for (int e = threadIdx.x; e < PRE_BM * PRE_BK; e += PRE_THREADS) {
      const int rr = e / PRE_BK, kk = e % PRE_BK;
      const int64_t r = r0 + rr, k = k0 + kk;
      gs[kk][rr] = (r < p.rows && k < p.d) ? __bfloat162float(p.grad[r * p.cols + gcol0 + k]) : 0.f;
    }
    for (int e = threadIdx.x; e < PRE_BK * PRE_BN; e += PRE_THREADS) {
      const int kk = e / PRE_BN, cc = e % PRE_BN;
      const int64_t k = k0 + kk, cidx = c0 + cc;
      ss[kk][cc] = (k < p.d && cidx < p.d) ? s[k * p.d + cidx] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < PRE_BK; ++kk) {
      float a[4], bb[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) { a[u] = gs[kk][ty * 4 + u]; bb[u] = ss[kk][tx * 4 + u]; }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] += a[u] * bb[v];
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t r = r0 + ty * 4 + u;
    if (r >= p.rows) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int64_t cidx = c0 + tx * 4 + v;
      if (cidx < p.d) p.out[r * p.cols + gcol0 + cidx] = acc[u][v];
    }
  }
}

// ---------------------------------------------------------------------------
// Staging for the tensor-core Newton-Muon products
// ---------------------------------------------------------------------------
constexpr int TPOSE_T = 64;

// One d-wide column block of a tokens x width activation matrix, to be
// written transposed (d rows of `tokens`, leading dimension ldt) as the
// K-major operand of the second-moment product.
struct ActBlock {
  const __nv_bfloat16* acts;
  __nv_bfloat16* xt;
  int64_t tokens, width, col0, d, ldt;
};

// grid.y = block, grid.x = 64x64 tiles of (tokens x d).  16-byte loads and
// stores through a swizzled 64x64 tile (tsw, conflict-free in both
// directions) when the widths allow, elementwise at ragged edges.
__global__ void __launch_bounds__(256) act_transpose_kernel(const ActBlock* __restrict__ blocks) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  __shared__ __align__(16) __nv_bfloat16 t[TPOSE_T][TPOSE_T];   // t[j][tsw(j, tok)]
  const ActBlock& b = blocks[blockIdx.y];
  const int64_t tiles_j = (b.d + TPOSE_T - 1) / TPOSE_T;
  const int64_t t0 = (blockIdx.x / tiles_j) * TPOSE_T, j0 = (blockIdx.x % tiles_j) * TPOSE_T;
  if (t0 >= b.tokens) return;
  const bool vec = (b.width % 8 == 0) && (b.col0 % 8 == 0) && (b.ldt % 8 == 0);
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int v = threadIdx.x + it * 256;
    const int tt = v >> 3, jv = (v & 7) * 8;
    const int64_t tok = t0 + tt, j = j0 + jv;
    __nv_bfloat16 x[8];
    if (vec && tok < b.tokens && j + 8 <= b.d) {
      const uint4 w = *reinterpret_cast<const uint4*>(b.acts + tok * b.width + b.col0 + j);
      const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&w);
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = e[k];
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        x[k] = (tok < b.tokens && j + k < b.d) ? b.acts[tok * b.width + b.col0 + j + k] : __float2bfloat16_rn(0.f);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) t[jv + k][tsw(jv + k, tt)] = x[k];
  }
  __syncthreads();
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int v = threadIdx.x + it * 256;
    const int jj = v >> 3, tv = (v & 7) * 8;
    const int64_t j = j0 + jj, tok = t0 + tv;
    if (j >= b.d) continue;
    __nv_bfloat16* dst = b.xt + j * b.ldt + tok;
    if (vec && tok + 8 <= b.tokens) {
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(&t[jj][tsw(jj, tv)]);
    } else {
      for (int k = 0; k < 8 && tok + k < b.tokens; ++k) dst[k] = t[jj][tsw(jj, tv + k)];
    }
  }
}

// One d-wide column block of an fp32 tokens x width activation, written as
// the two K-major operands of its second moment on the tensor cores: with
// H = bf16(x) and L = bf16(x - H) (so x - H - L is below 2^-16 |x|),
//   xa (d rows of 3 tokens, leading dimension ld3) = [H^T | H^T | L^T],
//   xb (same shape)                                 = [H^T | L^T | H^T],
// and xa xb^T = H^T H + H^T L + L^T H = X^T X up to the dropped L^T L term
// and the rounding of L, both below 2^-16 relative per product.
struct ActSplitBlock {
  const float* acts;
  __nv_bfloat16* xa;
  __nv_bfloat16* xb;
  int64_t tokens, width, col0, d, ld3;
};

__global__ void __launch_bounds__(256) act_split_kernel(const ActSplitBlock* __restrict__ blocks) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  __shared__ __align__(16) __nv_bfloat16 th[TPOSE_T][TPOSE_T];   // th[j][tsw(j, tok)]: H
  __shared__ __align__(16) __nv_bfloat16 tl[TPOSE_T][TPOSE_T];   //                     L
  const ActSplitBlock& b = blocks[blockIdx.y];
  const int64_t tiles_j = (b.d + TPOSE_T - 1) / TPOSE_T;
  const int64_t t0 = (blockIdx.x / tiles_j) * TPOSE_T, j0 = (blockIdx.x % tiles_j) * TPOSE_T;
  if (t0 >= b.tokens) return;
  const bool vin = (b.width % 4 == 0) && (b.col0 % 4 == 0);
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int v = threadIdx.x + it * 256;
    const int tt = v >> 3, jv = (v & 7) * 8;
    const int64_t tok = t0 + tt, j = j0 + jv;
    float x[8];
    if (vin && tok < b.tokens && j + 8 <= b.d) {
      const float4* p = reinterpret_cast<const float4*>(b.acts + tok * b.width + b.col0 + j);
      const float4 u = p[0], w = p[1];
      x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w; x[4] = w.x; x[5] = w.y; x[6] = w.z; x[7] = w.w;
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = (tok < b.tokens && j + k < b.d) ? b.acts[tok * b.width + b.col0 + j + k] : 0.f;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const __nv_bfloat16 h = __float2bfloat16_rn(x[k]);
      th[jv + k][tsw(jv + k, tt)] = h;
      tl[jv + k][tsw(jv + k, tt)] = __float2bfloat16_rn(x[k] - __bfloat162float(h));
    }
  }
  __syncthreads();
  // segment offsets along K: xa = [H, H, L], xb = [H, L, H]
  const int64_t T = b.tokens;
  const bool vout = (T % 8 == 0) && (b.ld3 % 8 == 0);
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int v = threadIdx.x + it * 256;
    const int jj = v >> 3, tv = (v & 7) * 8;
    const int64_t j = j0 + jj, tok = t0 + tv;
    if (j >= b.d) continue;
    __nv_bfloat16* ra = b.xa + j * b.ld3 + tok;
    __nv_bfloat16* rb = b.xb + j * b.ld3 + tok;
    if (vout && tok + 8 <= T) {
      const uint4 h = *reinterpret_cast<const uint4*>(&th[jj][tsw(jj, tv)]);
      const uint4 l = *reinterpret_cast<const uint4*>(&tl[jj][tsw(jj, tv)]);
      *reinterpret_cast<uint4*>(ra) = h;
      *reinterpret_cast<uint4*>(ra + T) = h;
      *reinterpret_cast<uint4*>(ra + 2 * T) = l;
      *reinterpret_cast<uint4*>(rb) = h;
      *reinterpret_cast<uint4*>(rb + T) = l;
      *reinterpret_cast<uint4*>(rb + 2 * T) = h;
    } else {
      for (int k = 0; k < 8 && tok + k < T; ++k) {
        const __nv_bfloat16 h = th[jj][tsw(jj, tv + k)], l = tl[jj][tsw(jj, tv + k)];
        ra[k] = h; ra[T + k] = h; ra[2 * T + k] = l;
        rb[k] = h; rb[T + k] = l; rb[2 * T + k] = h;
      }
    }
  }
}

// One S^-1 of a preconditioning launch (nb fp32 d x d blocks) split into
// bf16 hi/lo stacks, 2d x d per block: rows 0..d-1 = hi, d..2d-1 = lo, with
// hi + lo ~ S^-1.  Matrices that share an S^-1 share its stacks.
struct PrepDesc {
  const float* s_inv;
  __nv_bfloat16* sst;
  int32_t nb, d;
};

// grid.y = stack, grid.x strides over its nb*d*d elements, 8 per thread and
// step (16-byte loads and stores) when d*d is a multiple of 8, one
// otherwise.  Pointers are 16-byte aligned.
__global__ void __launch_bounds__(256) precond_prep_kernel(const PrepDesc* __restrict__ descs) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  const PrepDesc& p = descs[blockIdx.y];
  const int64_t dd = static_cast<int64_t>(p.d) * p.d;
  const int64_t ns = p.nb * dd;
  const bool svec = (dd % 8) == 0;
  const int64_t nsu = svec ? ns / 8 : ns;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * 256;
  for (int64_t e = blockIdx.x * 256 + threadIdx.x; e < nsu; e += stride) {
    if (svec) {
      const int64_t e8 = e * 8;
      const int64_t b = e8 / dd, rem = e8 - b * dd;
      const float4* src = reinterpret_cast<const float4*>(p.s_inv + e8);
      const float4 v0 = src[0], v1 = src[1];
      const float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __nv_bfloat16 h0 = __float2bfloat16_rn(v[2 * k]), h1 = __float2bfloat16_rn(v[2 * k + 1]);
        const __nv_bfloat16 l0 = __float2bfloat16_rn(v[2 * k] - __bfloat162float(h0));
        const __nv_bfloat16 l1 = __float2bfloat16_rn(v[2 * k + 1] - __bfloat162float(h1));
        hw[k] = uint32_t(__bfloat16_as_ushort(h0)) | (uint32_t(__bfloat16_as_ushort(h1)) << 16);
        lw[k] = uint32_t(__bfloat16_as_ushort(l0)) | (uint32_t(__bfloat16_as_ushort(l1)) << 16);
      }
      __nv_bfloat16* st = p.sst + b * 2 * dd;
      *reinterpret_cast<uint4*>(st + rem) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(st + dd + rem) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    } else {
      const int64_t b = e / dd, rem = e - b * dd;
      const float v = p.s_inv[e];
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
      __nv_bfloat16* st = p.sst + b * 2 * dd;
      st[rem] = hi;
      st[dd + rem] = lo;
    }
  }
}

}  // namespace muon
