// small_ns.cuh -- the whole quintic Newton-Schulz iteration of a small matrix
// in ONE launch ("Muon: when the LLM optimizer treats weight matrices as
// matrices", section 3: X <- a X + b (X X^T) X + c (X X^T)^2 X, five times).
//
// For a wide X of m <= n <= 256 the batched engine (ns_gemm.cuh) needs 15
// dependent launches of one tile each, and each launch costs more than its
// tile's arithmetic.  Here one CTA pair owns the matrix for all iterations:
// the pair's shared memory holds X twice (as the K-major operand of the Gram
// product and as the MN-major operand of the update) and the Gram / B'
// matrix, TMEM holds two 128x256 fp32 accumulators per CTA, and the three
// products of an iteration follow each other with a cluster barrier between
// them instead of a kernel boundary.  Pairs take whole matrices; a batch of
// small matrices strides over the pairs.
//
// The data flow is the engine's, product for product: A = alpha X X^T
// rounded to bf16; B' = b A + c A A + a I from the bf16 A and the fp32 A A,
// rounded to bf16; X' = alpha B' X rounded to bf16 (alpha = s^2 and s in the
// first iteration, s = 1 / (||U||_F + eps)).  The last update either stores
// X' (bf16, wide layout) or applies the weight step
// W <- W (1 - lr wd) - lr scale * alpha B' X from the fp32 accumulator, like
// the engine's fused last update.
//
// Layout per CTA r of the pair (rows [128 r, 128 r + 128) of X, A, B'):
//   XR  X rows of this CTA, K-major (K = the n columns), 128-byte swizzle:
//       four 16 KB chunks of 64 columns, row i at i * 128 B, 16-byte unit u
//       of a row at u ^ (i % 8).  Operand A and B of the Gram product.
//   XC  X columns [128 r, 128 r + 128), MN-major (K = the m rows): four
//       16 KB blocks of 64 K-rows, each two 8 KB chunks of 64 columns,
//       K-row k at k * 128 B, unit u at u ^ (k % 8).  Operand B of the
//       update.  The update epilogue writes the other CTA's half of these
//       columns into the peer's XC through distributed shared memory.
//   AB  A, then B', rows of this CTA, K-major like XR (K = m).
// Rows and columns past m and n are zero in every operand.
#pragma once

#include "elementwise.cuh"
#include "sm100_ptx.cuh"

namespace muon {

namespace small_cfg {
constexpr int MAXD = 256;                  // m, n <= 256 (wide orientation)
constexpr int THREADS = 256;               // 8 warps, all epilogue; one thread issues the MMAs
constexpr int PANEL = 128 * MAXD * 2;      // 64 KB: 128 rows x 256 bf16, or 256 K-rows x 128 bf16
constexpr int CHUNK = 128 * 64 * 2;        // 16 KB: one 64-wide K chunk of a K-major panel
constexpr int SMEM = 3 * PANEL + 1024 + 128;
constexpr int ACC = 256;                   // TMEM columns of one accumulator
}  // namespace small_cfg

struct SmallNsArgs {
  const __nv_bfloat16* x_in;   // wide X0 of matrix z at x_in + z * bs (ld elements per row)
  __nv_bfloat16* x_out;        // wide final X (when apply == nullptr)
  int64_t ld, bs;
  const float* norm2;          // ||U||_F^2 of matrix z at norm2[z]
  const MatDesc* apply;        // non-null: weight step of matrix z from apply[z]
  const MatDesc* mom;          // non-null: X0 is formed here, Nesterov momentum of
                               // matrix z (mom[z].grad, .momentum) and ||U||_F in
                               // the kernel, instead of read from x_in / norm2
  float beta;
  int nesterov;
  int m, n, count;
  int steps;
  float a, b, c, eps;
  int* err;                    // device error flags (bounded waits)
  const int* skip;             // halted() -> do nothing
};

// 4-byte store into the shared memory of CTA `rank` of this cluster.
__device__ __forceinline__ void st_cluster_f32(uint32_t local_addr, uint32_t rank, float v) {
  const uint32_t a = map_to_cta(local_addr, rank);
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

// 16-byte store into the shared memory of CTA `rank` of this cluster.
__device__ __forceinline__ void st_cluster_v4(uint32_t local_addr, uint32_t rank, uint4 v) {
  const uint32_t a = map_to_cta(local_addr, rank);
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// 16-byte global -> shared copy that does not pass through registers;
// src_bytes (0..16) are read, the rest of the 16 bytes is zero-filled.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void fence_async_cluster() {
  asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
}

// Offset of K-major element (row, k) in a panel (128-byte swizzle).
__device__ __forceinline__ uint32_t kmaj_off(int row, int k) {
  return static_cast<uint32_t>((k >> 6) * small_cfg::CHUNK + row * 128 + ((((k & 63) >> 3) ^ (row & 7)) << 4) +
                               (k & 7) * 2);
}
// Offset of MN-major element (k, mn) in an XC panel (mn local to the CTA's 128 columns).
__device__ __forceinline__ uint32_t mnmaj_off(int k, int mn) {
  const int kr = k & 63;
  return static_cast<uint32_t>((k >> 6) * small_cfg::CHUNK + (mn >> 6) * (small_cfg::CHUNK / 2) + kr * 128 +
                               ((((mn & 63) >> 3) ^ (kr & 7)) << 4) + (mn & 7) * 2);
}

__device__ __forceinline__ uint4 pack8(const float* v) {
  uint4 w;
  w.x = pack_bf16x2(v[0], v[1]);
  w.y = pack_bf16x2(v[2], v[3]);
  w.z = pack_bf16x2(v[4], v[5]);
  w.w = pack_bf16x2(v[6], v[7]);
  return w;
}

// Sum over the CTA's threads (valid in every thread): warp shuffles, then
// one partial per warp in red[], added in warp order.
__device__ __forceinline__ float cta_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < small_cfg::THREADS / 32; ++w) t += red[w];
  return t;
}

// One 8-column unit of wide row gi, in two halves so that several units'
// loads can be in flight: momentum_load reads the gradient and momentum of
// columns j0..j0+7 (zero past the matrix), momentum_finish forms U (the
// Nesterov look-ahead of the updated momentum) and stores the momentum.
// Wide (i, j) is the matrix's (i, j), or (j, i) when it is tall
// (transposed: the wide rows are its columns).
__device__ __forceinline__ bool unit_vec(const MatDesc& d, int m, int n, int gi, int j0) {
  return gi < m && !d.transposed && j0 + 8 <= n && (n & 7) == 0;
}
__device__ __forceinline__ int64_t unit_idx(const MatDesc& d, int m, int n, int gi, int j) {
  return d.transposed ? static_cast<int64_t>(j) * m + gi : static_cast<int64_t>(gi) * n + j;
}
__device__ __forceinline__ void momentum_load(const MatDesc& d, int m, int n, int gi, int j0, float (&g)[8],
                                              float (&b)[8]) {
  if (unit_vec(d, m, n, gi, j0)) {
    const int64_t idx = unit_idx(d, m, n, gi, j0);
    load8_grad(d.grad, d.grad_dtype, idx, g);
    const float4* bp = reinterpret_cast<const float4*>(d.momentum + idx);
    const float4 b0 = bp[0], b1 = bp[1];
    b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w; b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
    return;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const bool in = gi < m && j0 + e < n;
    const int64_t idx = unit_idx(d, m, n, gi, j0 + e);
    g[e] = in ? load1_grad(d.grad, d.grad_dtype, idx) : 0.f;
    b[e] = in ? d.momentum[idx] : 0.f;
  }
}
__device__ __forceinline__ void momentum_finish(const MatDesc& d, float beta, int nesterov, int m, int n, int gi,
                                                int j0, const float (&g)[8], float (&b)[8], float (&u)[8]) {
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    b[e] = beta * b[e] + (1.f - beta) * g[e];
    u[e] = nesterov ? (1.f - beta) * g[e] + beta * b[e] : b[e];
  }
  if (unit_vec(d, m, n, gi, j0)) {
    float4* bp = reinterpret_cast<float4*>(d.momentum + unit_idx(d, m, n, gi, j0));
    bp[0] = make_float4(b[0], b[1], b[2], b[3]);
    bp[1] = make_float4(b[4], b[5], b[6], b[7]);
    return;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e)
    if (gi < m && j0 + e < n) d.momentum[unit_idx(d, m, n, gi, j0 + e)] = b[e];
}

// X0 of this CTA from the gradient and momentum: every (row, 8-column unit)
// of its 128 wide rows, two units per thread in flight; returns the
// thread's sum of U^2.  A non-transposed matrix takes units along a row per
// warp (coalesced along the row), a transposed one units down a column.
__device__ __forceinline__ float momentum_rows(const MatDesc& d, float beta, int nesterov, int m, int n,
                                               uint32_t rank, uint8_t* XR, uint8_t* XC) {
  using namespace small_cfg;
  float ss = 0.f;
  const uint32_t xc = smem_u32(XC);
#pragma unroll 1
  for (int v0 = threadIdx.x; v0 < 128 * (MAXD / 8); v0 += 2 * THREADS) {
    float g[2][8], b[2][8], u[2][8];
    int rl[2], j0[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int v = v0 + q * THREADS;
      rl[q] = d.transposed ? (v & 127) : (v >> 5);
      j0[q] = d.transposed ? (v >> 7) * 8 : (v & 31) * 8;
      momentum_load(d, m, n, static_cast<int>(rank) * 128 + rl[q], j0[q], g[q], b[q]);
    }
#pragma unroll
    for (int q = 0; q < 2; ++q)
      momentum_finish(d, beta, nesterov, m, n, static_cast<int>(rank) * 128 + rl[q], j0[q], g[q], b[q], u[q]);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
#pragma unroll
      for (int e = 0; e < 8; ++e) ss += u[q][e] * u[q][e];
      const uint4 w = pack8(u[q]);
      const int gi = static_cast<int>(rank) * 128 + rl[q];
      *reinterpret_cast<uint4*>(XR + kmaj_off(rl[q], j0[q])) = w;
      const uint32_t off = mnmaj_off(gi, j0[q] & 127);
      const uint32_t owner = static_cast<uint32_t>(j0[q] >> 7);
      if (owner == rank) *reinterpret_cast<uint4*>(XC + off) = w;
      else st_cluster_v4(xc + off, owner, w);
    }
  }
  return ss;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(small_cfg::THREADS, 1)
    small_ns_kernel(const __grid_constant__ SmallNsArgs args) {
  using namespace small_cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* XR = smem;
  uint8_t* XC = smem + PANEL;
  uint8_t* AB = smem + 2 * PANEL;
  uint64_t* done_bar = reinterpret_cast<uint64_t*>(smem + 3 * PANEL);
  uint64_t* drain_bar = done_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* nslot = reinterpret_cast<float*>(tmem_slot + 2);   // ||U||^2 partial of CTA 0, CTA 1
  float* red = nslot + 2;                                    // block reduction, one per warp

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool issuer = rank == 0 && threadIdx.x == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int m = args.m, n = args.n;

  if (threadIdx.x == 0) {
    mbar_init(done_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(tmem_slot, 2 * ACC);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  // uniform over the grid, so both CTAs of a pair take the same branch
  const int count = halted(args.skip) ? 0 : args.count;

  const int q = warp & 3, h = warp >> 2;       // TMEM lane quarter, 128-column half
  const int il = q * 32 + lane;                 // row of this thread within the CTA
  const int gi = static_cast<int>(rank) * 128 + il;   // row of X / A / B'
  const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * 128;
  const int kx = (n + 63) & ~63, km = (m + 63) & ~63;   // K extents of the products
  constexpr uint32_t idesc_k = idesc_bf16_f32(256, 256, false);
  constexpr uint32_t idesc_mn = idesc_bf16_f32(256, 256, true);
  uint32_t nprod = 0;                           // completed products: done_bar phase

  // One product: the issuing thread runs `issue`, everyone waits for the
  // accumulator.  Returns false when the wait gave up (then nothing more is
  // issued or read, but every barrier is still passed).
  auto wait_done = [&]() -> bool {
    const bool ok = *abort_flag == 0 && mbar_wait(done_bar, nprod & 1, args.err, abort_flag);
    ++nprod;
    tc_fence_after();
    return __all_sync(0xffffffffu, ok);
  };
  auto end_phase = [&]() {
    fence_async_smem();
    fence_async_cluster();
    tc_fence_before();
    cluster_sync();
  };

  for (int z = pair; z < count; z += npairs) {
    float s;
    if (args.mom == nullptr) {
    // ---- X0 into XR (this CTA's rows) and XC (this CTA's columns), zero
    // padded: every 16-byte piece is an asynchronous copy, all in flight at
    // once (a piece past the matrix reads nothing and is zero-filled)
    const __nv_bfloat16* x0 = args.x_in + static_cast<int64_t>(z) * args.bs;
#pragma unroll 4
    for (int v = threadIdx.x; v < 128 * (MAXD / 8); v += THREADS) {
      const int r = v >> 5, c = (v & 31) * 8;                 // XR: row r, columns c..c+7
      const int gr = static_cast<int>(rank) * 128 + r;
      const bool in = gr < m && c < n;
      const uint32_t bytes = in ? static_cast<uint32_t>(min(8, n - c) * 2) : 0u;
      cp_async16(XR + kmaj_off(r, c), in ? x0 + static_cast<int64_t>(gr) * args.ld + c : x0, bytes);
    }
#pragma unroll 4
    for (int v = threadIdx.x; v < MAXD * 16; v += THREADS) {
      const int k = v >> 4, c = (v & 15) * 8;                 // XC: row k, local columns c..c+7
      const int gc = static_cast<int>(rank) * 128 + c;
      const bool in = k < m && gc < n;
      const uint32_t bytes = in ? static_cast<uint32_t>(min(8, n - gc) * 2) : 0u;
      cp_async16(XC + mnmaj_off(k, c), in ? x0 + static_cast<int64_t>(k) * args.ld + gc : x0, bytes);
    }
    s = 1.0f / (sqrtf(args.norm2[z]) + args.eps);
    cp_async_wait_all();
    end_phase();
    } else {
      // ---- momentum in the kernel: this CTA forms U for its wide rows,
      // updates their momentum, writes U (bf16) as its XR rows and, by
      // columns, into both CTAs' XC; the two CTAs' sums of U^2 meet in
      // nslot and are added in rank order on both sides
      const float ss = momentum_rows(args.mom[z], args.beta, args.nesterov, m, n, rank, XR, XC);
      const float tot = cta_sum(ss, red);
      if (threadIdx.x == 0) {
        nslot[rank] = tot;
        st_cluster_f32(smem_u32(&nslot[rank]), rank ^ 1u, tot);
      }
      end_phase();
      s = 1.0f / (sqrtf(nslot[0] + nslot[1]) + args.eps);
    }

    for (int it = 0; it < args.steps; ++it) {
      const float ag = it == 0 ? s * s : 1.0f, au = it == 0 ? s : 1.0f;
      const bool last = it == args.steps - 1;
      // ---- Gram: acc0 = X X^T (K-major X rows as both operands)
      if (warp == 0) {
        if (issuer && *abort_flag == 0) {
          tc_fence_after();
          const uint32_t xr = smem_u32(XR);
          for (int k = 0; k < kx; k += 16) {
            const uint64_t d = sdesc_kmajor_sw128(xr + (k >> 6) * CHUNK + (k & 63) * 2);
            mma_bf16_ss_pair(tmem, d, d, idesc_k, k > 0 ? 1u : 0u);
          }
          mma_commit_pair_mc(done_bar, 0x3);
        }
        // the other lanes of the issuing warp wait here rather than spin
        // on the barrier beside the issuing lane
        __syncwarp();
      }
      if (wait_done()) {
        // A = alpha X X^T, rounded to bf16, into AB (row il, columns h*128..)
#pragma unroll 1
        for (int c32 = 0; c32 < 4; ++c32) {
          uint32_t raw[32];
          tmem_ld_32x32b_x32(taddr + c32 * 32, raw);
          tmem_ld_wait();
          float v[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = ag * __uint_as_float(raw[k]);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(AB + kmaj_off(il, h * 128 + c32 * 32 + u * 8)) = pack8(v + u * 8);
        }
      }
      end_phase();
      // ---- polynomial: acc1 = A A (A symmetric: its rows are both operands)
      if (warp == 0) {
        if (issuer && *abort_flag == 0) {
          tc_fence_after();
          const uint32_t ab = smem_u32(AB);
          for (int k = 0; k < km; k += 16) {
            const uint64_t d = sdesc_kmajor_sw128(ab + (k >> 6) * CHUNK + (k & 63) * 2);
            mma_bf16_ss_pair(tmem + ACC, d, d, idesc_k, k > 0 ? 1u : 0u);
          }
          mma_commit_pair_mc(done_bar, 0x3);
        }
        // the other lanes of the issuing warp wait here rather than spin
        // on the barrier beside the issuing lane
        __syncwarp();
      }
      if (wait_done()) {
        // B' = b A + c A A + a I from the bf16 A in AB, overwritten in place
#pragma unroll 1
        for (int c32 = 0; c32 < 4; ++c32) {
          uint32_t raw[32];
          tmem_ld_32x32b_x32(taddr + ACC + c32 * 32, raw);
          tmem_ld_wait();
          const int j0 = h * 128 + c32 * 32;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4* cell = reinterpret_cast<uint4*>(AB + kmaj_off(il, j0 + u * 8));
            const uint4 w = *cell;
            float in[8], v[8];
            float2 f;
            f = unpack_bf16x2(w.x); in[0] = f.x; in[1] = f.y;
            f = unpack_bf16x2(w.y); in[2] = f.x; in[3] = f.y;
            f = unpack_bf16x2(w.z); in[4] = f.x; in[5] = f.y;
            f = unpack_bf16x2(w.w); in[6] = f.x; in[7] = f.y;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int j = j0 + u * 8 + e;
              v[e] = args.b * in[e] + args.c * __uint_as_float(raw[u * 8 + e]) + (j == gi && gi < m ? args.a : 0.0f);
            }
            *cell = pack8(v);
          }
        }
      }
      end_phase();
      // ---- update: acc0 = B' X (B' rows K-major, X columns MN-major)
      if (warp == 0) {
        if (issuer && *abort_flag == 0) {
          tc_fence_after();
          const uint32_t ab = smem_u32(AB), xc = smem_u32(XC);
          for (int k = 0; k < km; k += 16) {
            const uint64_t da = sdesc_kmajor_sw128(ab + (k >> 6) * CHUNK + (k & 63) * 2);
            const uint64_t db = sdesc_mnmajor_sw128(xc + (k >> 6) * CHUNK + (k & 63) * 128, CHUNK / 2);
            mma_bf16_ss_pair(tmem, da, db, idesc_mn, k > 0 ? 1u : 0u);
          }
          mma_commit_pair_mc(done_bar, 0x3);
        }
        // the other lanes of the issuing warp wait here rather than spin
        // on the barrier beside the issuing lane
        __syncwarp();
      }
      if (wait_done()) {
        if (!last) {
          // X' = alpha B' X in bf16: this CTA's rows into XR, and column half
          // h of them into the XC of CTA h (the peer's through DSMEM)
          const uint32_t xr = smem_u32(XR), xc = smem_u32(XC);
#pragma unroll 1
          for (int c32 = 0; c32 < 4; ++c32) {
            uint32_t raw[32];
            tmem_ld_32x32b_x32(taddr + c32 * 32, raw);
            tmem_ld_wait();
            float v[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = gi < m ? au * __uint_as_float(raw[k]) : 0.0f;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int j = h * 128 + c32 * 32 + u * 8;
              const uint4 w = pack8(v + u * 8);
              *reinterpret_cast<uint4*>(XR + kmaj_off(il, j)) = w;
              const uint32_t off = mnmaj_off(gi, j & 127);
              if (h == static_cast<int>(rank)) *reinterpret_cast<uint4*>(XC + off) = w;
              else st_cluster_v4(xc + off, static_cast<uint32_t>(h), w);
            }
          }
          (void)xr;
        } else if (args.apply == nullptr) {
          // final X, bf16, wide layout
          __nv_bfloat16* xo = args.x_out + static_cast<int64_t>(z) * args.bs;
#pragma unroll 1
          for (int c32 = 0; c32 < 4; ++c32) {
            uint32_t raw[32];
            tmem_ld_32x32b_x32(taddr + c32 * 32, raw);
            tmem_ld_wait();
            const int j0 = h * 128 + c32 * 32;
            if (gi < m && j0 < n) {
              float v[32];
#pragma unroll
              for (int k = 0; k < 32; ++k) v[k] = au * __uint_as_float(raw[k]);
              __nv_bfloat16* dst = xo + static_cast<int64_t>(gi) * args.ld + j0;
              if (j0 + 32 <= n) {
#pragma unroll
                for (int u = 0; u < 4; ++u) reinterpret_cast<uint4*>(dst)[u] = pack8(v + u * 8);
              } else {
#pragma unroll
                for (int k = 0; k < 32; ++k)
                  if (j0 + k < n) dst[k] = __float2bfloat16_rn(v[k]);
              }
            }
          }
        } else {
          // weight step from the fp32 accumulator: W <- W decay - lr scale O,
          // O = alpha B' X (W is O^T for a tall matrix)
          // The 32 weights of a chunk are all loaded before any is stored:
          // one read-modify-write after another would wait a full memory
          // round trip per element (the stores may alias the next loads as
          // far as the compiler knows).
          const MatDesc& d = args.apply[z];
#pragma unroll 1
          for (int c32 = 0; c32 < 4; ++c32) {
            uint32_t raw[32];
            tmem_ld_32x32b_x32(taddr + c32 * 32, raw);
            tmem_ld_wait();
            const int j0 = h * 128 + c32 * 32;
            if (gi < m && j0 < n) {
              float w[32];
              const bool vec = !d.transposed && j0 + 32 <= n && (d.cols & 3) == 0;
              float* row = d.weight + static_cast<int64_t>(gi) * d.cols + j0;   // !transposed
              if (vec) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                  const float4 q = reinterpret_cast<const float4*>(row)[u];
                  w[u * 4] = q.x; w[u * 4 + 1] = q.y; w[u * 4 + 2] = q.z; w[u * 4 + 3] = q.w;
                }
              } else {
#pragma unroll
                for (int k = 0; k < 32; ++k)
                  w[k] = j0 + k < n ? (d.transposed ? d.weight[static_cast<int64_t>(j0 + k) * d.cols + gi] : row[k])
                                    : 0.f;
              }
#pragma unroll
              for (int k = 0; k < 32; ++k) w[k] = w[k] * d.decay - d.lr_scale * (au * __uint_as_float(raw[k]));
              if (vec) {
#pragma unroll
                for (int u = 0; u < 8; ++u)
                  reinterpret_cast<float4*>(row)[u] = make_float4(w[u * 4], w[u * 4 + 1], w[u * 4 + 2], w[u * 4 + 3]);
              } else {
#pragma unroll
                for (int k = 0; k < 32; ++k)
                  if (j0 + k < n) {
                    if (d.transposed) d.weight[static_cast<int64_t>(j0 + k) * d.cols + gi] = w[k];
                    else row[k] = w[k];
                  }
              }
            }
          }
        }
      }
      end_phase();
    }
  }

  // ---- teardown: let an issued product drain before TMEM is released
  if (issuer && *abort_flag != 0) {
    volatile int no_abort = 0;
    mma_commit_pair_mc(drain_bar, 0x1);
    mbar_wait(drain_bar, 0, args.err, &no_abort);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 2 * ACC);
  }
}

}  // namespace muon
