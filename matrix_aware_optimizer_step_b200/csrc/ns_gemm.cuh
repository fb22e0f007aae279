// ns_gemm.cuh -- batched bf16 GEMM engine for the quintic Newton-Schulz
// iteration on sm_100a tensor cores (tcgen05 + TMEM, operands staged by TMA).
//
// One iteration on a wide bf16 X (m x n, m <= n) is three products
// ("Muon: when the LLM optimizer treats weight matrices as matrices",
// section 3, X <- a X + b (X X^T) X + c (X X^T)^2 X):
//
//   GRAM    A  = alpha * X X^T           M = N = m, K = n   symmetric
//   POLY    B  = b A + c A A             M = N = K = m      symmetric
//   UPDATE  X' = alpha * (a X + B X)     M = m, N = n, K = m
//
// The symmetric products compute only the tiles that touch the upper
// triangle and write each strictly-upper 128x128 block twice (direct and
// mirrored), so every element is written exactly once.  The fp32 sums stay in
// TMEM; each output is rounded to bf16 once, in the epilogue, after the
// polynomial terms are added.  alpha folds the Frobenius normalisation of the
// first iteration in (alpha = s^2 for GRAM, s for UPDATE, s = 1/(||U||+eps)).
//
// CTA: 192 threads.  Warp 0 issues TMA loads, warp 1 owns TMEM and issues
// tcgen05.mma from one thread, warps 2..5 run the epilogue (warp w reads
// TMEM lanes 32*(w%4) .. +31).  Tile 128 x 256 x 64, 4-stage smem ring.
#pragma once

#include "sm100_ptx.cuh"

namespace muon {

enum EpiKind : int { EPI_GRAM = 0, EPI_POLY = 1, EPI_UPDATE = 2 };

namespace gemm_cfg {
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;                 // 16 KB
constexpr int B_BYTES = BN * BK * 2;                 // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;       // 48 KB
constexpr int MN_CHUNK_BYTES = BK * 128;             // one 64-wide MN chunk of B (MN-major)
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;   // + alignment slack
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 256;
}  // namespace gemm_cfg

struct GemmArgs {
  int M, N, K;               // per-matrix extents
  int batch;                 // matrices in this launch
  int tiles_m, tiles_n;      // ceil(M/128), ceil(N/256)
  int tiles_per_mat;
  __nv_bfloat16* out;        // output, ld out_ld, batch stride out_bs (elements)
  int64_t out_ld, out_bs;
  const __nv_bfloat16* aux;  // POLY: A (same layout as out); UPDATE: X
  int64_t aux_ld, aux_bs;
  const float* norm2;        // per-matrix ||U||_F^2 (nullptr: alpha = 1)
  int alpha_pow;             // alpha = s^alpha_pow
  float eps;
  float c0, c1;              // POLY: b, c.  UPDATE: a.
  int* err;                  // device error flags
  const int* skip;           // non-null and set: do nothing (non-finite gradient)
};

// Number of 128x256 tiles per matrix that the GEMM kind computes.
__host__ __device__ inline int gemm_tiles_per_mat(int kind, int tiles_m, int tiles_n) {
  if (kind == EPI_UPDATE) return tiles_m * tiles_n;
  int t = 0;
  for (int i = 0; i < tiles_m; ++i) t += tiles_n - (i >> 1);
  return t;
}

template <int KIND, bool B_MN_MAJOR>
__global__ void __launch_bounds__(gemm_cfg::THREADS, 1)
    ns_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmArgs args) {
  using namespace gemm_cfg;
  extern __shared__ uint8_t smem_raw[];
  if (args.skip != nullptr && *args.skip) return;

  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* accum_bar = empty_bar + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- tile of this CTA ----
  const int bidx = blockIdx.x / args.tiles_per_mat;
  int t = blockIdx.x - bidx * args.tiles_per_mat;
  int ti = 0, tj = 0;
  if (KIND == EPI_UPDATE) {
    ti = t % args.tiles_m;          // row tiles fastest: CTAs in flight share X columns
    tj = t / args.tiles_m;
  } else {
    while (true) {
      const int cnt = args.tiles_n - (ti >> 1);
      if (t < cnt) { tj = (ti >> 1) + t; break; }
      t -= cnt;
      ++ti;
    }
  }
  const int nk = (args.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(accum_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (kb / STAGES) & 1;
        if (!mbar_wait(&empty_bar[s], ph ^ 1, args.err, abort_flag)) break;
        uint8_t* a_dst = smem + s * STAGE_BYTES;
        uint8_t* b_dst = a_dst + A_BYTES;
        mbar_arrive_expect_tx(&full_bar[s], STAGE_BYTES);
        tma_load_3d(a_dst, &tmA, &full_bar[s], kb * BK, ti * BM, bidx);
        if (B_MN_MAJOR) {
#pragma unroll
          for (int c = 0; c < BN / 64; ++c)
            tma_load_3d(b_dst + c * MN_CHUNK_BYTES, &tmB, &full_bar[s], tj * BN + c * 64, kb * BK,
                        bidx);
        } else {
          tma_load_3d(b_dst, &tmB, &full_bar[s], kb * BK, tj * BN, bidx);
        }
        issued = kb + 1;
      }
      if (*abort_flag) {
        // Let every copy this thread started land before the CTA exits.
        volatile int no_abort = 0;
        for (int kb = (issued > STAGES ? issued - STAGES : 0); kb < issued; ++kb)
          mbar_wait(&full_bar[kb % STAGES], (kb / STAGES) & 1, args.err, &no_abort);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, B_MN_MAJOR);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (kb / STAGES) & 1;
        if (!mbar_wait(&full_bar[s], ph, args.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + s * STAGE_BYTES);
        const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t adesc = sdesc_kmajor_sw128(a_base + kk * 32);
          const uint64_t bdesc = B_MN_MAJOR ? sdesc_mnmajor_sw128(b_base + kk * 16 * 128, MN_CHUNK_BYTES)
                                            : sdesc_kmajor_sw128(b_base + kk * 32);
          mma_bf16_ss(tmem, adesc, bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty_bar[s]);
      }
      mma_commit(accum_bar);   // arrives once every MMA above has completed
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;
    const bool ok = mbar_wait(accum_bar, 0, args.err, abort_flag);
    tc_fence_after();
    if (ok && !*abort_flag) {
      const int r = ti * BM + q * 32 + lane;          // output row of this thread
      const bool row_ok = r < args.M;
      float alpha = 1.0f;
      if (args.norm2 != nullptr) {
        const float s = 1.0f / (sqrtf(args.norm2[bidx]) + args.eps);
        alpha = (args.alpha_pow == 2) ? s * s : s;
      }
      __nv_bfloat16* out = args.out + static_cast<int64_t>(bidx) * args.out_bs;
      const __nv_bfloat16* aux =
          (KIND == EPI_GRAM) ? nullptr : args.aux + static_cast<int64_t>(bidx) * args.aux_bs;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int cb = tj * 2 + h;                     // 128-column block index
        const int col0 = cb * 128;
        if (col0 >= args.N) break;
        bool mirror = false;
        if (KIND != EPI_UPDATE) {
          if (cb < ti) continue;                       // below the diagonal: mirrored elsewhere
          mirror = cb > ti;
        }
#pragma unroll 1
        for (int c32 = 0; c32 < 4; ++c32) {
          const int cbase = col0 + c32 * 32;
          if (cbase >= args.N) break;
          uint32_t raw[32];
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + h * 128 + c32 * 32, raw);
          tmem_ld_wait();
          float v[32];
          const bool full = (cbase + 32 <= args.N);
          if (KIND == EPI_GRAM) {
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = alpha * __uint_as_float(raw[k]);
          } else {
            float in[32];
            if (row_ok && full) {
              const uint4* src = reinterpret_cast<const uint4*>(aux + static_cast<int64_t>(r) * args.aux_ld + cbase);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const uint4 w = src[u];
                float2 f;
                f = unpack_bf16x2(w.x); in[u * 8 + 0] = f.x; in[u * 8 + 1] = f.y;
                f = unpack_bf16x2(w.y); in[u * 8 + 2] = f.x; in[u * 8 + 3] = f.y;
                f = unpack_bf16x2(w.z); in[u * 8 + 4] = f.x; in[u * 8 + 5] = f.y;
                f = unpack_bf16x2(w.w); in[u * 8 + 6] = f.x; in[u * 8 + 7] = f.y;
              }
            } else {
#pragma unroll
              for (int k = 0; k < 32; ++k)
                in[k] = (row_ok && cbase + k < args.N)
                            ? __bfloat162float(aux[static_cast<int64_t>(r) * args.aux_ld + cbase + k])
                            : 0.0f;
            }
            if (KIND == EPI_POLY) {
#pragma unroll
              for (int k = 0; k < 32; ++k) v[k] = args.c0 * in[k] + args.c1 * __uint_as_float(raw[k]);
            } else {
#pragma unroll
              for (int k = 0; k < 32; ++k) v[k] = alpha * (args.c0 * in[k] + __uint_as_float(raw[k]));
            }
          }
          // direct store, row r, columns cbase .. cbase+31
          if (row_ok) {
            __nv_bfloat16* dst = out + static_cast<int64_t>(r) * args.out_ld + cbase;
            if (full) {
              uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                uint4 w;
                w.x = pack_bf16x2(v[u * 8 + 0], v[u * 8 + 1]);
                w.y = pack_bf16x2(v[u * 8 + 2], v[u * 8 + 3]);
                w.z = pack_bf16x2(v[u * 8 + 4], v[u * 8 + 5]);
                w.w = pack_bf16x2(v[u * 8 + 6], v[u * 8 + 7]);
                d4[u] = w;
              }
            } else {
#pragma unroll
              for (int k = 0; k < 32; ++k)
                if (cbase + k < args.N) dst[k] = __float2bfloat16_rn(v[k]);
            }
          }
          // mirrored store: element (r, c) also goes to (c, r)
          if (mirror && row_ok) {
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (cbase + k < args.N)
                out[static_cast<int64_t>(cbase + k) * args.out_ld + r] = __float2bfloat16_rn(v[k]);
          }
        }
      }
    }
  }

  // ---- teardown: TMEM is freed by the warp that allocated it ----
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace muon
