// elementwise.cuh -- the HBM-bound kernels of the Muon step.
//
//   momentum_kernel   Nesterov momentum in place on the fp32 buffer, the
//                     look-ahead U cast to bf16 and written in the wide
//                     (rows <= cols) layout the Newton-Schulz engine reads,
//                     transposing through shared memory for tall matrices,
//                     and one partial sum of U^2 per tile (block reduction).
//                     12 B/element with bf16 gradients.
//   norm_reduce_kernel  ||U||^2 per matrix from its tiles' partials (or from
//                     the preconditioning product's, when that product
//                     applied the momentum itself).
//   apply_kernel      W <- W (1 - lr wd) - lr scale O, O read from the final
//                     wide bf16 X (transposed back through shared memory for
//                     tall matrices); optionally O to an fp32 output.
//                     10 B/element.  Used when the weight step cannot be
//                     fused into the last Newton-Schulz product (an update_out
//                     was requested, a width is not a multiple of 4, or no
//                     iteration runs) and for the Newton-Schulz-only export.
//   finite_kernel     read-only NaN/Inf scan of the gradients.
//   adamw_kernel      fused AdamW over a list of tensors, bias-corrected.
//
// Sources: momentum 0.95 with Nesterov (first page, "Hyperparameter
// tuning"); EMA convention of the blog's section 1; decoupled decay and the
// shape scale (blog, PyTorch set-up after section 4); AdamW (first page,
// "Usage"; blog section 1).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace muon {

constexpr int EW_TILE = 64;        // 64 x 64 element tiles
constexpr int EW_THREADS = 256;
// momentum_kernel: 128 threads, four 8-element vectors each per 64 x 64 tile.
// Each warp's fixed work per tile (tile lookup, descriptor loads, the block
// reduction) is then shared by twice the elements of a 256-thread block; in
// a long step the power cap holds the SM clock near 1 GHz, where the kernel
// is limited by instruction issue rather than HBM, and this measured 6 %
// faster there (no change at full clock).
constexpr int MOM_THREADS = 128;
constexpr int MOM_VECS = EW_TILE * EW_TILE / 8 / MOM_THREADS;

// Transposing tile: element (c, r) of a 64 x 64 bf16 tile sits in row c at
// 16-byte unit (r / 8) ^ (c / 8 % 8).  Writing one column (8 rows c apart,
// 4 consecutive r per warp) and reading 8-element row units are both free of
// bank conflicts.
__device__ __forceinline__ int tsw(int c, int r) { return ((((r >> 3) ^ (c >> 3)) & 7) << 3) | (r & 7); }

// One matrix as the elementwise kernels see it.  Lives in a device table.
struct MatDesc {
  const void* grad;          // rows x cols, grad_dtype (momentum) / input (export)
  float* weight;             // rows x cols
  float* momentum;           // rows x cols
  float* update_out;         // rows x cols fp32 or nullptr
  __nv_bfloat16* x_in;       // wide layout (m x ld), where U is written
  const __nv_bfloat16* x_out;  // wide layout, final Newton-Schulz output
  float* norm2;              // this matrix's ||U||^2 slot
  float* partials;           // one partial sum per tile of the launch (indexed by tile)
  int64_t rows, cols;
  int64_t ld;                // leading dimension of the wide layout
  int64_t tile_start;        // first 64x64 tile of this matrix in the launch
  int32_t tiles_c;           // ceil(cols / 64)
  int32_t transposed;        // rows > cols: wide layout is the transpose
  int32_t grad_dtype;        // 0 f32, 1 bf16
  float lr_scale;            // lr * shape scale
  float decay;               // 1 - lr * wd
  int32_t nparts;            // > 0: momentum, U and the partials of ||U||^2 come
                             // from the preconditioning product's epilogue, the
                             // partials at partials[0 .. nparts); momentum_kernel
                             // skips the matrix
};

// Segments of equal-shape matrices in one launch (kernel parameter space,
// no global memory round trip): tile -> matrix is a short scan plus one
// division instead of a search through the descriptor table.  Tiles are
// counted from the launch's first block, so the lookup is 32-bit integer
// arithmetic: every thread of a block repeats it, and a 64-bit division is
// a long instruction sequence that, repeated per thread, made up about half
// of the momentum kernel's issued instructions.
constexpr int MAX_SEGS = 32;
struct SegTable {
  int n;
  int first_mat[MAX_SEGS];         // descriptor index of the segment's first matrix
  uint32_t tile_start[MAX_SEGS];   // first tile of the segment, from the launch's first block
  uint32_t tiles_per_mat[MAX_SEGS];
};

struct TileLoc {
  int mat;        // descriptor index
  uint32_t lt;    // tile index within the matrix
};

__device__ __forceinline__ TileLoc seg_locate(const SegTable& t, uint32_t b) {
  int s = 0;
#pragma unroll 1
  while (s + 1 < t.n && t.tile_start[s + 1] <= b) ++s;
  const uint32_t rel = b - t.tile_start[s];
  const uint32_t k = rel / t.tiles_per_mat[s];
  return {t.first_mat[s] + static_cast<int>(k), rel - k * t.tiles_per_mat[s]};
}

// Origin (row, column) of tile lt of a matrix with tiles_c tile columns.
__device__ __forceinline__ void tile_origin(uint32_t lt, int32_t tiles_c, int64_t& r0, int64_t& c0) {
  const uint32_t tc = static_cast<uint32_t>(tiles_c);
  const uint32_t tr = lt / tc;
  r0 = static_cast<int64_t>(tr) * EW_TILE;
  c0 = static_cast<int64_t>(lt - tr * tc) * EW_TILE;
}

__device__ __forceinline__ void load8_grad(const void* g, int dtype, int64_t idx, float (&x)[8]) {
  if (dtype == 1) {
    const uint4 w = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(g) + idx);
    float2 f;
    f = unpack_bf16x2(w.x); x[0] = f.x; x[1] = f.y;
    f = unpack_bf16x2(w.y); x[2] = f.x; x[3] = f.y;
    f = unpack_bf16x2(w.z); x[4] = f.x; x[5] = f.y;
    f = unpack_bf16x2(w.w); x[6] = f.x; x[7] = f.y;
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(g) + idx);
    const float4 a = p[0], b = p[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
}

__device__ __forceinline__ float load1_grad(const void* g, int dtype, int64_t idx) {
  return dtype == 1 ? __bfloat162float(static_cast<const __nv_bfloat16*>(g)[idx])
                    : static_cast<const float*>(g)[idx];
}

template <int NT = EW_THREADS>
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
  if (w == 0) {
    s = (l < NT / 32) ? red[l] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  }
  return s;   // valid in thread 0
}

// mode 0: momentum (buf updated, U = Nesterov look-ahead or buf)
// mode 1: plain load (U = input), for Newton-Schulz only
template <int MODE>
__global__ void __launch_bounds__(MOM_THREADS)
    momentum_kernel(const MatDesc* __restrict__ descs, const __grid_constant__ SegTable segs, int64_t tile_base,
                    float beta, int nesterov, const int* skip) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  if (halted(skip)) return;
  __shared__ __align__(16) __nv_bfloat16 tile[EW_TILE][EW_TILE];
  __shared__ float red[MOM_THREADS / 32];
  const int64_t gt = tile_base + blockIdx.x;
  const TileLoc loc = seg_locate(segs, blockIdx.x);
  const MatDesc& d = descs[loc.mat];
  if (d.nparts > 0) return;   // done in the preconditioning product (uniform per block)
  const int64_t lt = loc.lt;
  float ss = 0.f;
  if (!d.transposed && d.ld == d.cols && (d.cols % 8) == 0) {
    // Rows are contiguous in both layouts: block lt takes elements
    // [4096 lt, 4096 lt + 4096) of the flattened matrix, so each warp moves
    // 256 consecutive elements (the matrix has at least as many 64x64 tiles
    // as 4096-element runs; the blocks past its end store a zero partial).
    const int64_t n = d.rows * d.cols;
#pragma unroll
    for (int it = 0; it < MOM_VECS; ++it) {
      const int64_t e = lt * (EW_TILE * EW_TILE) + (threadIdx.x + it * MOM_THREADS) * 8;
      if (e >= n) continue;
      float g[8], u[8];
      load8_grad(d.grad, d.grad_dtype, e, g);
      if (MODE == 0) {
        float4* bp = reinterpret_cast<float4*>(d.momentum + e);
        const float4 b0 = bp[0], b1 = bp[1];
        float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          b[k] = beta * b[k] + (1.f - beta) * g[k];
          u[k] = nesterov ? (1.f - beta) * g[k] + beta * b[k] : b[k];
        }
        bp[0] = make_float4(b[0], b[1], b[2], b[3]);
        bp[1] = make_float4(b[4], b[5], b[6], b[7]);
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) u[k] = g[k];
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) ss += u[k] * u[k];
      uint4 w;
      w.x = pack_bf16x2(u[0], u[1]); w.y = pack_bf16x2(u[2], u[3]);
      w.z = pack_bf16x2(u[4], u[5]); w.w = pack_bf16x2(u[6], u[7]);
      *reinterpret_cast<uint4*>(d.x_in + e) = w;
    }
    const float tot = block_sum<MOM_THREADS>(ss, red);
    if (threadIdx.x == 0) d.partials[gt] = tot;
    return;
  }
  int64_t r0, c0;
  tile_origin(loc.lt, d.tiles_c, r0, c0);
  const bool vec_ok = (d.cols % 8 == 0) && (d.ld % 8 == 0);
  // 64 rows x 8 vectors of 8 columns = 512 vectors, 4 per thread
#pragma unroll
  for (int it = 0; it < MOM_VECS; ++it) {
    const int v = threadIdx.x + it * MOM_THREADS;
    const int rl = v >> 3, cl = (v & 7) * 8;
    const int64_t r = r0 + rl, c = c0 + cl;
    if (r >= d.rows) continue;
    float u[8];
    if (vec_ok && c + 8 <= d.cols) {
      const int64_t idx = r * d.cols + c;
      float g[8];
      load8_grad(d.grad, d.grad_dtype, idx, g);
      if (MODE == 0) {
        float4* bp = reinterpret_cast<float4*>(d.momentum + idx);
        float4 b0 = bp[0], b1 = bp[1];
        float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          b[k] = beta * b[k] + (1.f - beta) * g[k];
          u[k] = nesterov ? (1.f - beta) * g[k] + beta * b[k] : b[k];
        }
        bp[0] = make_float4(b[0], b[1], b[2], b[3]);
        bp[1] = make_float4(b[4], b[5], b[6], b[7]);
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) u[k] = g[k];
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) ss += u[k] * u[k];
      if (!d.transposed) {
        uint4 w;
        w.x = pack_bf16x2(u[0], u[1]); w.y = pack_bf16x2(u[2], u[3]);
        w.z = pack_bf16x2(u[4], u[5]); w.w = pack_bf16x2(u[6], u[7]);
        *reinterpret_cast<uint4*>(d.x_in + r * d.ld + c) = w;
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) tile[cl + k][tsw(cl + k, rl)] = __float2bfloat16_rn(u[k]);
      }
    } else {
      for (int k = 0; k < 8; ++k) {
        const int64_t cc = c + k;
        if (cc >= d.cols) break;
        const int64_t idx = r * d.cols + cc;
        const float g = load1_grad(d.grad, d.grad_dtype, idx);
        float uk;
        if (MODE == 0) {
          const float b = beta * d.momentum[idx] + (1.f - beta) * g;
          d.momentum[idx] = b;
          uk = nesterov ? (1.f - beta) * g + beta * b : b;
        } else {
          uk = g;
        }
        ss += uk * uk;
        if (!d.transposed) d.x_in[r * d.ld + cc] = __float2bfloat16_rn(uk);
        else tile[cl + k][tsw(cl + k, rl)] = __float2bfloat16_rn(uk);
      }
    }
  }
  if (d.transposed) {
    __syncthreads();
    // wide row = original column c0 + cl, wide columns = original rows r0 .. r0+63
#pragma unroll
    for (int it = 0; it < MOM_VECS; ++it) {
      const int v = threadIdx.x + it * MOM_THREADS;
      const int cl = v >> 3, rl = (v & 7) * 8;
      const int64_t wr = c0 + cl, wc = r0 + rl;
      if (wr >= d.cols) continue;
      __nv_bfloat16* dst = d.x_in + wr * d.ld + wc;
      if (wc + 8 <= d.rows && (d.ld % 8 == 0)) {
        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(&tile[cl][tsw(cl, rl)]);
      } else {
        for (int k = 0; k < 8 && wc + k < d.rows; ++k) dst[k] = tile[cl][tsw(cl, rl + k)];
      }
    }
  }
  // this tile's share of sum(U^2); norm_reduce_kernel adds the partials of
  // each matrix in tile order (deterministic, no atomics or fences here)
  const float tot = block_sum<MOM_THREADS>(ss, red);
  if (threadIdx.x == 0) d.partials[gt] = tot;
}

// ||U||^2 of matrix descs[blockIdx.x]: its tiles' partials summed in a fixed
// order (thread t takes tiles t, t + 256, ...; then a fixed tree), so the
// result is the same run to run.
__global__ void __launch_bounds__(EW_THREADS) norm_reduce_kernel(const MatDesc* __restrict__ descs, const int* skip) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  if (halted(skip)) return;
  __shared__ float red[EW_THREADS / 32];
  const MatDesc& d = descs[blockIdx.x];
  const bool fused = d.nparts > 0;
  const int64_t ntiles = fused ? d.nparts : ((d.rows + EW_TILE - 1) / EW_TILE) * d.tiles_c;
  const float* part = fused ? d.partials : d.partials + d.tile_start;
  float acc = 0.f;
  for (int64_t t = threadIdx.x; t < ntiles; t += EW_THREADS) acc += part[t];
  const float all = block_sum(acc, red);
  if (threadIdx.x == 0) *d.norm2 = all;
}

// W[0..8) <- W (1 - lr wd) - lr scale O, W already loaded into w.
__device__ __forceinline__ void store_weight8(float* dst, const float4 (&w)[2], const float (&o)[8], float decay,
                                              float lr_scale) {
  float4 w0 = w[0], w1 = w[1];
  w0.x = w0.x * decay - lr_scale * o[0]; w0.y = w0.y * decay - lr_scale * o[1];
  w0.z = w0.z * decay - lr_scale * o[2]; w0.w = w0.w * decay - lr_scale * o[3];
  w1.x = w1.x * decay - lr_scale * o[4]; w1.y = w1.y * decay - lr_scale * o[5];
  w1.z = w1.z * decay - lr_scale * o[6]; w1.w = w1.w * decay - lr_scale * o[7];
  float4* wp = reinterpret_cast<float4*>(dst);
  wp[0] = w0;
  wp[1] = w1;
}

__device__ __forceinline__ void store_f32x8(float* dst, const float (&o)[8]) {
  float4* op = reinterpret_cast<float4*>(dst);
  op[0] = make_float4(o[0], o[1], o[2], o[3]);
  op[1] = make_float4(o[4], o[5], o[6], o[7]);
}

// mode 0: apply update to W (and optionally write O)
// mode 1: export O only (Newton-Schulz only path)
// norm_scale: when no iteration ran, O = U / (||U|| + eps) is formed here.
template <int MODE>
__global__ void __launch_bounds__(EW_THREADS)
    apply_kernel(const MatDesc* __restrict__ descs, const __grid_constant__ SegTable segs,
                 int normalise, float eps, const int* skip) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  if (halted(skip)) return;
  __shared__ __align__(16) __nv_bfloat16 tile[EW_TILE][EW_TILE];
  const TileLoc loc = seg_locate(segs, blockIdx.x);
  const MatDesc& d = descs[loc.mat];
  const int64_t lt = loc.lt;
  int64_t r0, c0;
  tile_origin(loc.lt, d.tiles_c, r0, c0);
  const float s = normalise ? 1.0f / (sqrtf(*d.norm2) + eps) : 1.0f;
  if (!d.transposed && d.ld == d.cols && (d.cols % 8) == 0) {
    // contiguous rows: the flat element run of momentum_kernel, loads of both
    // vectors issued before any store
    const int64_t n = d.rows * d.cols;
    float o[2][8];
    float4 w[2][2];
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int64_t e = lt * (EW_TILE * EW_TILE) + (threadIdx.x + it * EW_THREADS) * 8;
      if (e < n) {
        const uint4 x = *reinterpret_cast<const uint4*>(d.x_out + e);
        float2 f;
        f = unpack_bf16x2(x.x); o[it][0] = f.x; o[it][1] = f.y;
        f = unpack_bf16x2(x.y); o[it][2] = f.x; o[it][3] = f.y;
        f = unpack_bf16x2(x.z); o[it][4] = f.x; o[it][5] = f.y;
        f = unpack_bf16x2(x.w); o[it][6] = f.x; o[it][7] = f.y;
        if (MODE == 0) {
          const float4* wp = reinterpret_cast<const float4*>(d.weight + e);
          w[it][0] = wp[0];
          w[it][1] = wp[1];
        }
      }
    }
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int64_t e = lt * (EW_TILE * EW_TILE) + (threadIdx.x + it * EW_THREADS) * 8;
      if (e >= n) continue;
#pragma unroll
      for (int k = 0; k < 8; ++k) o[it][k] *= s;
      if (MODE == 0) store_weight8(d.weight + e, w[it], o[it], d.decay, d.lr_scale);
      if (d.update_out != nullptr) store_f32x8(d.update_out + e, o[it]);
    }
    return;
  }
  // 64x64 tile: W loads first (independent of O), then O (through shared
  // memory for tall matrices), then the stores
  const bool vec_ok = (d.cols % 8 == 0) && (d.ld % 8 == 0);
  float4 w[2][2];
  bool full[2];
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int v = threadIdx.x + it * EW_THREADS;
    const int64_t r = r0 + (v >> 3), c = c0 + (v & 7) * 8;
    full[it] = r < d.rows && vec_ok && c + 8 <= d.cols;
    if (full[it] && MODE == 0) {
      const float4* wp = reinterpret_cast<const float4*>(d.weight + r * d.cols + c);
      w[it][0] = wp[0];
      w[it][1] = wp[1];
    }
  }
  if (d.transposed) {
    // stage the 64x64 block of the wide X (rows c0.., cols r0..) in smem
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int v = threadIdx.x + it * EW_THREADS;
      const int cl = v >> 3, rl = (v & 7) * 8;
      const int64_t wr = c0 + cl, wc = r0 + rl;
      if (wr >= d.cols) continue;
      const __nv_bfloat16* src = d.x_out + wr * d.ld + wc;
      if (wc + 8 <= d.rows && (d.ld % 8 == 0)) {
        *reinterpret_cast<uint4*>(&tile[cl][tsw(cl, rl)]) = *reinterpret_cast<const uint4*>(src);
      } else {
        for (int k = 0; k < 8 && wc + k < d.rows; ++k) tile[cl][tsw(cl, rl + k)] = src[k];
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int v = threadIdx.x + it * EW_THREADS;
    const int rl = v >> 3, cl = (v & 7) * 8;
    const int64_t r = r0 + rl, c = c0 + cl;
    if (r >= d.rows) continue;
    if (full[it]) {
      float o[8];
      if (!d.transposed) {
        const uint4 x = *reinterpret_cast<const uint4*>(d.x_out + r * d.ld + c);
        float2 f;
        f = unpack_bf16x2(x.x); o[0] = f.x; o[1] = f.y;
        f = unpack_bf16x2(x.y); o[2] = f.x; o[3] = f.y;
        f = unpack_bf16x2(x.z); o[4] = f.x; o[5] = f.y;
        f = unpack_bf16x2(x.w); o[6] = f.x; o[7] = f.y;
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] = __bfloat162float(tile[cl + k][tsw(cl + k, rl)]);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] *= s;
      const int64_t idx = r * d.cols + c;
      if (MODE == 0) store_weight8(d.weight + idx, w[it], o, d.decay, d.lr_scale);
      if (d.update_out != nullptr) store_f32x8(d.update_out + idx, o);
    } else {
      for (int k = 0; k < 8; ++k) {
        const int64_t cc = c + k;
        if (cc >= d.cols) break;
        const float ok = s * (d.transposed ? __bfloat162float(tile[cl + k][tsw(cl + k, rl)])
                                           : __bfloat162float(d.x_out[r * d.ld + cc]));
        const int64_t idx = r * d.cols + cc;
        if (MODE == 0) d.weight[idx] = d.weight[idx] * d.decay - d.lr_scale * ok;
        if (d.update_out != nullptr) d.update_out[idx] = ok;
      }
    }
  }
}

// Sets *flag when any gradient element is NaN or Inf.  One 64x64 tile per
// block, same tiling as momentum_kernel.
__global__ void __launch_bounds__(EW_THREADS)
    finite_kernel(const MatDesc* __restrict__ descs, const __grid_constant__ SegTable segs,
                  int* flag) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  const TileLoc loc = seg_locate(segs, blockIdx.x);
  const MatDesc& d = descs[loc.mat];
  int64_t r0, c0;
  tile_origin(loc.lt, d.tiles_c, r0, c0);
  bool bad = false;
  for (int e = threadIdx.x; e < EW_TILE * EW_TILE; e += EW_THREADS) {
    const int64_t r = r0 + e / EW_TILE, c = c0 + e % EW_TILE;
    if (r < d.rows && c < d.cols) bad |= !isfinite(load1_grad(d.grad, d.grad_dtype, r * d.cols + c));
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(flag, 1);
}

// ----------------------------------------------------------------------------
// AdamW
// ----------------------------------------------------------------------------
constexpr int ADAM_CHUNK = 8192;   // elements per block

struct AdamDesc {
  float* param;
  const void* grad;
  float* m;
  float* v;
  int64_t numel;
  int64_t chunk_start;
  int32_t grad_dtype;
  int32_t pad;
};

struct AdamScalars {
  float lr, beta1, beta2, eps, decay;   // decay = 1 - lr * wd
  float bc1, bc2_sqrt;                  // 1 - beta1^t, sqrt(1 - beta2^t)
};

__device__ __forceinline__ int find_adam(const AdamDesc* __restrict__ d, int n, int64_t chunk) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (d[mid].chunk_start <= chunk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ void adam_one(float& p, float g, float& m, float& v, const AdamScalars& s) {
  m = s.beta1 * m + (1.f - s.beta1) * g;
  v = s.beta2 * v + (1.f - s.beta2) * g * g;
  const float denom = sqrtf(v) / s.bc2_sqrt + s.eps;
  p = p * s.decay - (s.lr / s.bc1) * (m / denom);
}

__global__ void __launch_bounds__(EW_THREADS)
    adamw_kernel(const AdamDesc* __restrict__ descs, int n, AdamScalars s, const int* skip) {
  pdl_wait();      // previous kernel's results visible (no-op without PDL)
  if (halted(skip)) return;
  const int64_t ch = blockIdx.x;
  const AdamDesc& d = descs[find_adam(descs, n, ch)];
  const int64_t base = (ch - d.chunk_start) * ADAM_CHUNK;
  const int64_t end = min(base + ADAM_CHUNK, d.numel);
  const bool vec_ok = ((reinterpret_cast<uintptr_t>(d.param) | reinterpret_cast<uintptr_t>(d.m) |
                        reinterpret_cast<uintptr_t>(d.v)) & 15) == 0 &&
                      (reinterpret_cast<uintptr_t>(d.grad) & (d.grad_dtype == 1 ? 7 : 15)) == 0;
  if (vec_ok) {
    const int64_t vend = base + ((end - base) / 4) * 4;
    for (int64_t i = base + threadIdx.x * 4; i < vend; i += EW_THREADS * 4) {
      float4 p = *reinterpret_cast<float4*>(d.param + i);
      float4 m = *reinterpret_cast<float4*>(d.m + i);
      float4 v = *reinterpret_cast<float4*>(d.v + i);
      float g[4];
      if (d.grad_dtype == 1) {
        const uint2 w = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(d.grad) + i);
        const float2 a = unpack_bf16x2(w.x), b = unpack_bf16x2(w.y);
        g[0] = a.x; g[1] = a.y; g[2] = b.x; g[3] = b.y;
      } else {
        const float4 q = *reinterpret_cast<const float4*>(static_cast<const float*>(d.grad) + i);
        g[0] = q.x; g[1] = q.y; g[2] = q.z; g[3] = q.w;
      }
      adam_one(p.x, g[0], m.x, v.x, s);
      adam_one(p.y, g[1], m.y, v.y, s);
      adam_one(p.z, g[2], m.z, v.z, s);
      adam_one(p.w, g[3], m.w, v.w, s);
      *reinterpret_cast<float4*>(d.param + i) = p;
      *reinterpret_cast<float4*>(d.m + i) = m;
      *reinterpret_cast<float4*>(d.v + i) = v;
    }
    const int64_t j = vend + threadIdx.x;   // at most 3 trailing elements
    if (j < end) {
      float p = d.param[j], m = d.m[j], v = d.v[j];
      adam_one(p, load1_grad(d.grad, d.grad_dtype, j), m, v, s);
      d.param[j] = p; d.m[j] = m; d.v[j] = v;
    }
  } else {
    for (int64_t j = base + threadIdx.x; j < end; j += EW_THREADS) {
      float p = d.param[j], m = d.m[j], v = d.v[j];
      adam_one(p, load1_grad(d.grad, d.grad_dtype, j), m, v, s);
      d.param[j] = p; d.m[j] = m; d.v[j] = v;
    }
  }
}

}  // namespace muon
