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
// Persistent CTAs, one per SM, stride over the tile list.  Warp 0 issues TMA
// loads into a 4-stage smem ring that runs across tile boundaries, warp 1
// owns TMEM (two 128x256 fp32 accumulators) and issues tcgen05.mma from one
// thread, warps 2..9 drain the other accumulator meanwhile: the epilogue of
// one tile overlaps the main loop of the next.  Epilogue warp w reads TMEM
// lanes 32*(w%4) .. +31 and one 128-column half of the tile; its stores are
// staged through shared memory so that global writes (direct and mirrored)
// are whole 64-byte row segments.
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
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + EPI_WARPS * 32;         // producer, MMA, 8 epilogue warps
constexpr int STG_PITCH = 80;                        // staged row: 64 B of data + 16 B pad
constexpr int STG_BYTES = 32 * STG_PITCH;            // one 32x32 bf16 block per epilogue warp
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_WARPS * STG_BYTES + BAR_BYTES + 1024;
constexpr int ACC_COLS = 256;                        // one fp32 128x256 accumulator
constexpr int TMEM_COLS = 2 * ACC_COLS;              // double-buffered
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

__device__ __forceinline__ void decode_tile(int kind, const GemmArgs& a, int t, int& bidx, int& ti,
                                            int& tj) {
  bidx = t / a.tiles_per_mat;
  t -= bidx * a.tiles_per_mat;
  if (kind == EPI_UPDATE) {
    ti = t % a.tiles_m;          // row tiles fastest: CTAs in flight share X columns
    tj = t / a.tiles_m;
    return;
  }
  ti = 0;
  while (true) {
    const int cnt = a.tiles_n - (ti >> 1);
    if (t < cnt) { tj = (ti >> 1) + t; return; }
    t -= cnt;
    ++ti;
  }
}

// Copy one staged 32x32 bf16 block (rows of STG_PITCH bytes) to global
// memory at (r0, c0): 4 lanes per row, 16 B each.
__device__ __forceinline__ void store_staged(const uint8_t* stg, __nv_bfloat16* out, int64_t ld, int r0,
                                             int c0, int rows, int cols, int lane) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int v = lane + 32 * k;
    const int row = v >> 2, c16 = v & 3;
    const int gr = r0 + row, gc = c0 + c16 * 8;
    if (gr >= rows) continue;
    const uint8_t* src = stg + row * gemm_cfg::STG_PITCH + c16 * 16;
    __nv_bfloat16* dst = out + static_cast<int64_t>(gr) * ld + gc;
    if (gc + 8 <= cols) {
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    } else {
      const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(src);
      for (int j = 0; j < 8 && gc + j < cols; ++j) dst[j] = e[j];
    }
  }
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
  uint8_t* smem_epi = smem + STAGES * STAGE_BYTES;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem_epi + EPI_WARPS * STG_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;     // accumulator ready   (MMA -> epilogue)
  uint64_t* tempty_bar = tfull_bar + 2;         // accumulator drained (epilogue -> MMA)
  uint64_t* drain_bar = tempty_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total = args.batch * args.tiles_per_mat;
  const int nk = (args.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
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
      int it = 0;
      for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
        int bidx, ti, tj;
        decode_tile(KIND, args, t, bidx, ti, tj);
        for (int kb = 0; kb < nk; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
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
          ++it;
        }
      }
      if (*abort_flag) {
        // Let every copy this thread started land before the CTA exits.
        volatile int no_abort = 0;
        for (int k = (it > STAGES ? it - STAGES : 0); k < it; ++k)
          mbar_wait(&full_bar[k % STAGES], (k / STAGES) & 1, args.err, &no_abort);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, B_MN_MAJOR);
      int it = 0, lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++lt) {
        const int acc = lt & 1;
        if (!mbar_wait(&tempty_bar[acc], ((lt >> 1) & 1) ^ 1, args.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * ACC_COLS;
        for (int kb = 0; kb < nk; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&full_bar[s], ph, args.err, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t adesc = sdesc_kmajor_sw128(a_base + kk * 32);
            const uint64_t bdesc = B_MN_MAJOR ? sdesc_mnmajor_sw128(b_base + kk * 16 * 128, MN_CHUNK_BYTES)
                                              : sdesc_kmajor_sw128(b_base + kk * 32);
            mma_bf16_ss(d_tmem, adesc, bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty_bar[s]);
          ++it;
        }
        if (ok) mma_commit(&tfull_bar[acc]);
      }
      if (*abort_flag) {
        // wait for the MMAs already issued before TMEM is released
        volatile int no_abort = 0;
        mma_commit(drain_bar);
        mbar_wait(drain_bar, 0, args.err, &no_abort);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..9) ----------------
    const int ew = warp - 2;
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int half = ew >> 2;               // 128-column half of the tile
    uint8_t* stg = smem_epi + ew * STG_BYTES;
    int lt = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++lt) {
      int bidx, ti, tj;
      decode_tile(KIND, args, t, bidx, ti, tj);
      const int acc = lt & 1;
      // warp-uniform decision: tcgen05.ld below is warp-collective
      const bool got = mbar_wait(&tfull_bar[acc], (lt >> 1) & 1, args.err, abort_flag);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int rbase = ti * BM + q * 32;
      const int r = rbase + lane;
      const bool row_ok = r < args.M;
      float alpha = 1.0f;
      if (args.norm2 != nullptr) {
        const float sc = 1.0f / (sqrtf(args.norm2[bidx]) + args.eps);
        alpha = (args.alpha_pow == 2) ? sc * sc : sc;
      }
      __nv_bfloat16* out = args.out + static_cast<int64_t>(bidx) * args.out_bs;
      const __nv_bfloat16* aux =
          (KIND == EPI_GRAM) ? nullptr : args.aux + static_cast<int64_t>(bidx) * args.aux_bs;
      const int cb = tj * 2 + half;          // 128-column block index
      const int col0 = cb * 128;
      bool active = col0 < args.N;
      bool mirror = false;
      if (KIND != EPI_UPDATE) {
        if (cb < ti) active = false;         // below the diagonal: mirrored by another tile
        mirror = cb > ti;
      }
      if (active) {
#pragma unroll 1
        for (int c32 = 0; c32 < 4; ++c32) {
          const int cbase = col0 + c32 * 32;
          if (cbase >= args.N) break;
          uint32_t raw[32];
          tmem_ld_32x32b_x32(tmem + acc * ACC_COLS + (static_cast<uint32_t>(q * 32) << 16) + half * 128 + c32 * 32,
                             raw);
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
          // direct: row `lane` of the staged block, then whole row segments out
          {
            uint4* srow = reinterpret_cast<uint4*>(stg + lane * STG_PITCH);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint4 w;
              w.x = pack_bf16x2(v[u * 8 + 0], v[u * 8 + 1]);
              w.y = pack_bf16x2(v[u * 8 + 2], v[u * 8 + 3]);
              w.z = pack_bf16x2(v[u * 8 + 4], v[u * 8 + 5]);
              w.w = pack_bf16x2(v[u * 8 + 6], v[u * 8 + 7]);
              srow[u] = w;
            }
          }
          __syncwarp();
          store_staged(stg, out, args.out_ld, rbase, cbase, args.M, args.N, lane);
          __syncwarp();
          if (mirror) {
            // transposed block: staged row k holds column cbase+k of the tile
#pragma unroll
            for (int k = 0; k < 32; ++k)
              reinterpret_cast<__nv_bfloat16*>(stg + k * STG_PITCH)[lane] = __float2bfloat16_rn(v[k]);
            __syncwarp();
            store_staged(stg, out, args.out_ld, cbase, rbase, args.N, args.M, lane);
            __syncwarp();
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[acc]);
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
