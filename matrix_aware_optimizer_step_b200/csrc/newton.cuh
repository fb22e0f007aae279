// newton.cuh -- Newton-Muon right-preconditioning ("The Newton-Muon
// Optimizer", section "What Is Newton-Muon?"): each layer gradient G is
// right-multiplied by the inverse of the activation second moment
// S = X^T X / N before the standard Muon step; the MLP contraction uses a
// four-block diagonal S, one d x d inverse per block of d gradient columns.
//
//   act_transpose_kernel  a d-wide activation block, transposed to bf16
//                         d x tokens: the K-major operand of S = Xt Xt^T / N,
//                         which the tensor-core engine computes (GRAM32).
//   cholesky_blocked_kernel  S = L L^T in place (fp32), panels of 32, one
//                         block per matrix (d <= 1536).
//   chol_linv_kernel      L^-1, 32 columns per block, blocked forward
//                         substitution with the diagonal blocks' inverses.
//   spd_inverse_product_kernel  S^-1 = L^-T L^-1 in 64x64 tiles of the lower
//                         triangle (mirrored), then copy_inverse_kernel.
//   cholesky_kernel, chol_solve_kernel  unblocked versions for larger d.
//   precond_prep_kernel   bf16 copies of the gradients and S^-1 split into
//                         bf16 hi + lo, the operands of G' = G [S_hi; S_lo]
//                         on the tensor-core engine (PRECOND).
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
                     // (unblocked path) or, in each 32x32 diagonal block,
                     // the transpose of that block's inverse (blocked path)
  float* inv;        // d x d output S^-1
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
constexpr int CHOLB_THREADS = 512;
constexpr int CHOL_BLOCKED_MAX_D = 1536;    // panel of d x 33 floats fits in smem

__host__ __device__ inline int cholb_smem_bytes(int d) { return d * CBP * 4; }

// Right-looking Cholesky S = L L^T in place (lower triangle), one block per
// matrix: factor the 32x32 diagonal block (one warp), solve the panel below it
// row by row, subtract the panel's rank-32 product from the trailing lower
// triangle in 4x4 register tiles.  The panel lives in shared memory.  Warp 0
// also inverts each factored diagonal block D (column j of D^-1 by lane j) and
// stores D^-1 transposed in the block's strict upper triangle, where the
// inverse kernel turns its in-block substitutions into products.
__global__ void __launch_bounds__(CHOLB_THREADS)
    cholesky_blocked_kernel(const CholDesc* __restrict__ descs, float damping, int* err) {
  extern __shared__ float pan[];            // [d][CBP]: rows below the diagonal block
  __shared__ float dg[CB][CBP];
  __shared__ int bad;
  const CholDesc& c = descs[blockIdx.x];
  float* a = c.a;
  const int d = c.d;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) bad = 0;
  if (damping != 0.f)
    for (int i = tid; i < d; i += CHOLB_THREADS) a[int64_t(i) * d + i] += damping;
  __syncthreads();
  for (int p0 = 0; p0 < d; p0 += CB) {
    const int nb = min(CB, d - p0);
    for (int e = tid; e < CB * CB; e += CHOLB_THREADS) {
      const int i = e / CB, j = e % CB;
      dg[i][j] = (i < nb && j <= i) ? a[int64_t(p0 + i) * d + p0 + j] : 0.f;
    }
    __syncthreads();
    if (warp == 0) {                        // unblocked Cholesky of the diagonal block
      for (int k = 0; k < nb; ++k) {
        if (lane == 0) {
          float dkk = dg[k][k];
          if (!(dkk > 0.f)) { bad = 1; dkk = 1.f; }
          dg[k][k] = sqrtf(dkk);
        }
        __syncwarp();
        const float lkk = dg[k][k];
        if (lane > k && lane < nb) dg[lane][k] /= lkk;
        __syncwarp();
        if (lane > k && lane < nb)
          for (int j = k + 1; j <= lane; ++j) dg[lane][j] -= dg[lane][k] * dg[j][k];
        __syncwarp();
      }
    }
    __syncthreads();
    for (int e = tid; e < nb * nb; e += CHOLB_THREADS) {
      const int i = e / nb, j = e % nb;
      if (j <= i) a[int64_t(p0 + i) * d + p0 + j] = dg[i][j];
    }
    if (warp == 0) {
      // D x = e_lane by forward substitution; x = column `lane` of D^-1
      float x[CB];
#pragma unroll
      for (int i = 0; i < CB; ++i) {
        float sum = (i == lane) ? 1.f : 0.f;
#pragma unroll
        for (int k = 0; k < i; ++k) sum -= dg[i][k] * x[k];
        x[i] = (i < nb) ? sum / dg[i][i] : 0.f;
      }
      // D^-1[i][lane] (i > lane) goes to row p0 + lane, column p0 + i
#pragma unroll
      for (int i = 0; i < CB; ++i)
        if (i > lane && i < nb) a[int64_t(p0 + lane) * d + p0 + i] = x[i];
    }
    // panel: row i below solves x L11^T = a_i (forward substitution)
    const int r0 = p0 + nb, nrows = d - r0;
    for (int ii = tid; ii < nrows; ii += CHOLB_THREADS) {
      float x[CB];
      float* arow = a + int64_t(r0 + ii) * d + p0;
#pragma unroll
      for (int j = 0; j < CB; ++j) x[j] = j < nb ? arow[j] : 0.f;
#pragma unroll
      for (int j = 0; j < CB; ++j) {
        if (j < nb) {
          float sum = x[j];
#pragma unroll
          for (int k = 0; k < j; ++k) sum -= x[k] * dg[j][k];
          x[j] = sum / dg[j][j];
        }
      }
#pragma unroll
      for (int j = 0; j < CB; ++j)
        if (j < nb) {
          arow[j] = x[j];
          pan[ii * CBP + j] = x[j];
        }
    }
    __syncthreads();
    // trailing lower triangle: A[i][j] -= sum_k P[i][k] P[j][k], 4x4 tiles
    const int t4 = (nrows + 3) / 4;
    const int ntiles = t4 * (t4 + 1) / 2;
    for (int t = tid; t < ntiles; t += CHOLB_THREADS) {
      int ti = int((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
      while (ti * (ti + 1) / 2 > t) --ti;
      while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
      const int tj = t - ti * (ti + 1) / 2;
      float acc[4][4] = {};
      for (int k = 0; k < nb; ++k) {
        float pi[4], pj[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int ri = 4 * ti + u, rj = 4 * tj + u;
          pi[u] = ri < nrows ? pan[ri * CBP + k] : 0.f;
          pj[u] = rj < nrows ? pan[rj * CBP + k] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] += pi[u] * pj[v];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = 4 * ti + u;
        if (i >= nrows) continue;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int j = 4 * tj + v;
          if (j <= i) a[int64_t(r0 + i) * d + r0 + j] -= acc[u][v];
        }
      }
    }
    __syncthreads();
  }
  if (tid == 0 && bad) atomicOr(err, kDevErrNotSPD);
}

constexpr int CINV_THREADS = 256;

// dv = D^-1 for the diagonal block at rbase (zero outside the matrix):
// D^-1[i][k] for k < i sits at (rbase + k, rbase + i) of the factor's
// storage, the diagonal is 1 / L[i][i].
__device__ __forceinline__ void load_diag_inverse(const float* L, int d, int rbase, float (*dv)[CBP], int tid) {
  for (int e = tid; e < CB * CB; e += CINV_THREADS) {
    const int i = e / CB, k = e % CB;
    const int gi = rbase + i, gk = rbase + k;
    float v = 0.f;
    if (gi < d && gk < d) {
      if (k < i) v = L[int64_t(gk) * d + gi];
      else if (k == i) v = 1.f / L[int64_t(gi) * d + gi];
    }
    dv[i][k] = v;
  }
}
__host__ __device__ inline int cinv_smem_bytes(int d) { return d * CBP * 4; }

// L^-1, 32 columns per block: forward L Y = E (E = columns c0 .. c0+31 of
// I; rows of Y above c0 are zero), row blocks of 32 at a time, Y resident in
// shared memory.  Within a row block the substitution is a product with the
// diagonal block's inverse D^-1, spread over all threads.  Y is written to
// c.inv (rows from c0 rounded down to 64, zeros above c0), the operand of
// spd_inverse_product_kernel.  L is read from the lower triangle of c.a.
__global__ void __launch_bounds__(CINV_THREADS)
    chol_linv_kernel(const CholDesc* __restrict__ descs, int blocks_per_mat) {
  extern __shared__ float y[];              // [d][CBP]
  __shared__ float acc_s[CB][CBP];
  __shared__ float dv[CB][CBP];             // inverse of the current diagonal block
  const CholDesc& c = descs[blockIdx.x / blocks_per_mat];
  const int d = c.d;
  const int c0 = (blockIdx.x % blocks_per_mat) * CB;
  if (c0 >= d) return;
  const float* L = c.a;
  const int tid = threadIdx.x;
  const int orow = tid >> 3, ocol = (tid & 7) * 4;     // this thread's 4 outputs in a 32x32 block
  const int nrb = (d + CB - 1) / CB;
  const int rb0 = c0 / CB;
  // ---- forward ----
  for (int rb = rb0; rb < nrb; ++rb) {
    const int rbase = rb * CB;
    float acc[4];
    const int r = rbase + orow;
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[v] = (r == c0 + ocol + v) ? 1.f : 0.f;
    if (r < d) {
      const float* lrow = L + int64_t(r) * d;
      for (int k = c0; k < rbase; ++k) {
        const float l = lrow[k];
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[v] -= l * y[k * CBP + ocol + v];
      }
    }
#pragma unroll
    for (int v = 0; v < 4; ++v) acc_s[orow][ocol + v] = acc[v];
    load_diag_inverse(L, d, rbase, dv, tid);
    __syncthreads();
    // Y_block = D^-1 * acc
    {
      float out[4] = {0.f, 0.f, 0.f, 0.f};
      for (int k = 0; k <= orow; ++k) {
        const float dk = dv[orow][k];
#pragma unroll
        for (int v = 0; v < 4; ++v) out[v] += dk * acc_s[k][ocol + v];
      }
      if (r < d) {
#pragma unroll
        for (int v = 0; v < 4; ++v) y[r * CBP + ocol + v] = out[v];
      }
    }
    __syncthreads();
  }
  // ---- columns c0 .. c0+31 of L^-1 ----
  const int rw = c0 & ~63;
  for (int e = tid; e < (d - rw) * CB; e += CINV_THREADS) {
    const int i = rw + e / CB, j = e % CB;
    if (c0 + j < d) c.inv[int64_t(i) * d + c0 + j] = i < c0 ? 0.f : y[i * CBP + j];
  }
}

// S^-1 = L^-T L^-1: S^-1[i][j] = sum over k >= max(i, j) of L^-1[k][i] L^-1[k][j].
// One 64x64 tile of the lower triangle per block (grid.x: tile, grid.y:
// matrix), K in chunks of 32 rows of L^-1 staged in shared memory, 4x4
// register tiles; the tile and its mirror are written to c.a.
constexpr int SIP_T = 64, SIP_K = 32, SIP_THREADS = 256;
__global__ void __launch_bounds__(SIP_THREADS) spd_inverse_product_kernel(const CholDesc* __restrict__ descs) {
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
  if (skip != nullptr && *skip) return;
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

// One preconditioned matrix: its bf16 gradient copied to a batched layout
// (rows x ldc) and its nb fp32 inverses split into bf16 hi/lo stacks
// (2d x d each: rows 0..d-1 = hi, d..2d-1 = lo, with hi + lo ~ S^-1).
struct PrepDesc {
  const __nv_bfloat16* g;
  __nv_bfloat16* gc;
  const float* s_inv;
  __nv_bfloat16* sst;
  int64_t rows, cols, ldc;
  int32_t nb, d;
};

// grid.y = matrix, grid.x strides over max(rows*cols, nb*d*d) elements, 8
// per thread and step (16-byte loads and stores) when the gradient width and
// d*d are multiples of 8, one otherwise.  Pointers are 16-byte aligned.
__global__ void __launch_bounds__(256) precond_prep_kernel(const PrepDesc* __restrict__ descs) {
  const PrepDesc& p = descs[blockIdx.y];
  const int64_t ng = p.rows * p.cols;
  const int64_t dd = static_cast<int64_t>(p.d) * p.d;
  const int64_t ns = p.nb * dd;
  const bool gvec = (p.cols % 8) == 0;       // then ldc == cols: a flat copy
  const bool svec = (dd % 8) == 0;
  const int64_t ngu = gvec ? ng / 8 : ng;
  const int64_t nsu = svec ? ns / 8 : ns;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * 256;
  for (int64_t e = blockIdx.x * 256 + threadIdx.x; e < ngu || e < nsu; e += stride) {
    if (e < ngu) {
      if (gvec) {
        reinterpret_cast<uint4*>(p.gc)[e] = reinterpret_cast<const uint4*>(p.g)[e];
      } else {
        const int64_t r = e / p.cols, c = e - r * p.cols;
        p.gc[r * p.ldc + c] = p.g[e];
      }
    }
    if (e < nsu) {
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
}

}  // namespace muon
