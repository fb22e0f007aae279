// newton.cuh -- Newton-Muon right-preconditioning ("The Newton-Muon
// Optimizer", section "What Is Newton-Muon?"): each layer gradient G is
// right-multiplied by the inverse of the activation second moment
// S = X^T X / N before the standard Muon step; the MLP contraction uses a
// four-block diagonal S, one d x d inverse per block of d gradient columns.
//
//   act_gram_kernel     S_b = X_b^T X_b / N, fp32 accumulation of bf16
//                       activations (products of bf16 values are exact in
//                       fp32), one 64x64 tile of S per block.
//   cholesky_kernel     S = L L^T in place (fp32), one block per matrix;
//                       L^T is mirrored into the upper triangle so every
//                       later read is along a row.
//   chol_solve_kernel   S^-1 row by row: L y = e_j, then L^T x = y; one warp
//                       per row, blocks split the rows of each matrix.
//   precond_kernel      G' = G blockdiag(S_b^-1), bf16 G, fp32 S^-1 and
//                       output, 64x64 tiles with 4x4 outputs per thread.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace muon {

// ---------------------------------------------------------------------------
// second moment
// ---------------------------------------------------------------------------
constexpr int GRAM_T = 64;
constexpr int GRAM_K = 32;
constexpr int GRAM_THREADS = 256;

struct GramDesc {
  const __nv_bfloat16* acts;   // tokens x width
  float* s_out;                // d x d
  int64_t tokens, width, col0, d;
  int64_t tile_start;
  int32_t tiles;               // ceil(d / 64)
  int32_t pad;
};

template <typename D>
__device__ __forceinline__ int find_tile_desc(const D* __restrict__ d, int n, int64_t tile) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (d[mid].tile_start <= tile) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(GRAM_THREADS)
    act_gram_kernel(const GramDesc* __restrict__ descs, int n) {
  __shared__ float xi[GRAM_K][GRAM_T + 4];
  __shared__ float xj[GRAM_K][GRAM_T + 4];
  const int64_t gt = blockIdx.x;
  const GramDesc& g = descs[find_tile_desc(descs, n, gt)];
  const int64_t lt = gt - g.tile_start;
  const int64_t i0 = (lt / g.tiles) * GRAM_T, j0 = (lt % g.tiles) * GRAM_T;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // 16 x 16 threads, 4x4 outputs each
  float acc[4][4] = {};
  for (int64_t t0 = 0; t0 < g.tokens; t0 += GRAM_K) {
    // stage 32 tokens x 64 columns of both column blocks
    for (int e = threadIdx.x; e < GRAM_K * GRAM_T; e += GRAM_THREADS) {
      const int tk = e / GRAM_T, c = e % GRAM_T;
      const int64_t t = t0 + tk;
      const bool tok = t < g.tokens;
      const int64_t ci = i0 + c, cj = j0 + c;
      xi[tk][c] = (tok && ci < g.d) ? __bfloat162float(g.acts[t * g.width + g.col0 + ci]) : 0.f;
      xj[tk][c] = (tok && cj < g.d) ? __bfloat162float(g.acts[t * g.width + g.col0 + cj]) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int tk = 0; tk < GRAM_K; ++tk) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) { a[u] = xi[tk][ty * 4 + u]; b[u] = xj[tk][tx * 4 + u]; }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] += a[u] * b[v];
    }
    __syncthreads();
  }
  const float inv_n = 1.0f / float(g.tokens);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t i = i0 + ty * 4 + u;
    if (i >= g.d) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int64_t j = j0 + tx * 4 + v;
      if (j < g.d) g.s_out[i * g.d + j] = acc[u][v] * inv_n;
    }
  }
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
  float* a;          // d x d scratch: S in, L (lower) + L^T (strict upper) out
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

}  // namespace muon
