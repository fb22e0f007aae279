// ns_gemm.cuh -- batched bf16 GEMM engine for the quintic Newton-Schulz
// iteration on sm_100a tensor cores (tcgen05 + TMEM, operands staged by TMA).
//
// One iteration on a wide bf16 X (m x n, m <= n) is three products
// ("Muon: when the LLM optimizer treats weight matrices as matrices",
// section 3, X <- a X + b (X X^T) X + c (X X^T)^2 X):
//
//   GRAM    A  = alpha * X X^T           M = N = m, K = n   symmetric
//   POLY    B' = b A + c A A + a I       M = N = K = m      symmetric
//   UPDATE  X' = alpha * B' X            M = m, N = n, K = m
//   UPDATE_APPLY (the last update of an optimizer step)
//           W <- W (1 - lr wd) - lr scale * alpha * B' X, with W read and
//           written in 32x32 fp32 chunks by TMA; X' is not stored
//
// a X + B X is computed as (a I + B) X: the same product, but the update
// needs no second read of X.  Rounding a I + B to bf16 instead of B costs no
// accuracy on matrices of 16 or more: late in the iteration B's diagonal is
// near -a + 0.7, so B' has the smaller entries (bf16 emulation, 16x16 ...
// 1024x4096: lower error than rounding B; only a 5x3 matrix came out higher,
// 3.0e-2 against 2.4e-2).
//
// The symmetric products compute only the tiles that touch the upper
// triangle and write each strictly-upper 128x128 block twice (direct and
// mirrored), so every element is written exactly once.  The fp32 sums stay in
// TMEM; each output is rounded to bf16 once, in the epilogue, after the
// polynomial terms are added.  alpha folds the Frobenius normalisation of the
// first iteration in (alpha = s^2 for GRAM, s for UPDATE, s = 1/(||U||+eps)).
//
// CTA pairs.  A cluster of two CTAs on two SMs computes one 256x256 output
// tile with tcgen05.mma.cta_group::2: CTA r holds rows [128r, 128r+128) of
// the A tile and rows [128r, 128r+128) of the B tile (N side) in its own
// shared memory and receives rows [128r, 128r+128) of the accumulator in its
// own TMEM.  Per SM this halves the operand bytes per FLOP of a 128x256 tile.
// Both CTAs load their halves with TMA (no multicast) and signal the leader's
// (rank 0) "full" barrier; the leader's single MMA thread waits for both
// halves, issues the MMAs and commits to the "empty"/"accumulator ready"
// barriers of both CTAs at once; both CTAs' epilogue warps report a drained
// accumulator to the leader.
//
// Pairs are persistent (one CTA per SM) and stride over the tile list; two
// 128x256 fp32 accumulators per CTA (512 TMEM columns) let eight epilogue
// warps drain one tile while the next is computed.  Epilogue warp w reads
// TMEM lanes 32*(w%4) .. +31 and one 128-column half of the CTA's 128x256
// accumulator.  For the poly, its 32x128 slice of the epilogue input A
// arrives by TMA into a 128-byte-swizzled shared region before the
// accumulator is ready; the warp reads it, writes its output back in place
// (the swizzle keeps both conflict-free) and one lane stores the slice with
// TMA.  GRAM and UPDATE have no epilogue input: each 32x32 output chunk goes
// through one of two alternating 2 KB buffers per warp and leaves by TMA, so
// their pipelines get the shared memory a whole slice would take.  Mirrored
// blocks of the symmetric products leave through a small staging buffer as
// 64-byte row segments.  The accumulator is released to the MMA thread with
// a relaxed cluster arrive once the warp's TMEM reads have completed.
//
// Two more products serve Newton-Muon ("The Newton-Muon Optimizer", "What Is
// Newton-Muon?") and write fp32 directly from registers:
//
//   GRAM32   S = (1/N) Xt Xt^T          M = N = d, K = N tokens  symmetric
//            (Xt: bf16 activation block, transposed; bf16 products are exact
//            in fp32).  Launched with MN-major operands it reads the tokens
//            x width activation in place: A and B are both MN-major, with
//            the block's column offset added to the MN coordinate, and the
//            per-activation maps come from device memory.  For fp32
//            activations X = H + L (bf16 high and low parts) it runs over
//            K = 3N with A = [H | H | L] and B = [H | L | H] (transposed):
//            the sum H^T H + H^T L + L^T H, symmetric, but with A and B
//            different tensors (args.ab_distinct).
//   PRECOND  G' = G [S_hi; S_lo]         M = rows, N = d, K = 2d
//            (S^-1 = S_hi + S_lo split into two bf16 matrices stacked along
//            K, G's column block read twice, so the product keeps close to
//            fp32 precision; G is read in place and each matrix's operands
//            come from its own tensor maps in device memory)
//   PRECOND_MOM  the same product inside an optimizer step, with Nesterov
//            momentum in the epilogue, so G' never reaches memory: each 32x32
//            fp32 chunk of the momentum buffer comes in by TMA (one buffer
//            per warp, the next chunk requested once the store has read it),
//            is updated with the G' chunk in place and goes back by TMA; U
//            leaves by TMA as a 32x32 bf16 block of the Newton-Schulz input
//            (staged transposed for tall matrices, whose wide layout is U^T);
//            every warp stores one partial of ||U||^2 per tile
#pragma once

#include "sm100_ptx.cuh"

namespace muon {

enum EpiKind : int {
  EPI_GRAM = 0, EPI_POLY = 1, EPI_UPDATE = 2, EPI_GRAM32 = 3, EPI_PRECOND = 4, EPI_UPDATE_APPLY = 5,
  EPI_PRECOND_MOM = 6
};

namespace gemm_cfg {
constexpr int TM = 256;                              // pair tile rows (128 per CTA)
constexpr int TN = 256;                              // pair tile columns
constexpr int HM = 128;                              // rows per CTA
constexpr int HN = 128;                              // B rows (N side) per CTA
constexpr int BK = 64;
// Pipeline depth per product.  GRAM and UPDATE stage their output in 2 KB
// chunks (below) and spend the space saved on a fifth / sixth stage; the
// update also has no mirrored blocks.
__host__ __device__ constexpr int stages_for(int kind) {
  return kind == 0 ? 5 : kind == 1 ? 4 : kind == 2 ? 6 : kind == 5 ? 5 : kind == 6 ? 5 : 7;
}
// GRAM32 and PRECOND write fp32 straight from registers: no epilogue buffers,
// so their pipelines take the shared memory.
__host__ __device__ constexpr bool fp32_out(int kind) { return kind == 3 || kind == 4; }
__host__ __device__ constexpr bool precond_kind(int kind) { return kind == 4 || kind == 6; }
__host__ __device__ constexpr bool mom_out(int kind) { return kind == 6; }
// The last update of an optimizer step may apply W <- W (1 - lr wd) - lr
// scale O in its epilogue (EPI_UPDATE_APPLY): W moves through two 4 KB
// 32x32 fp32 chunk buffers per warp by TMA, and O never reaches memory.
// (A ring of three buffers refilled across tiles, with one stage fewer to
// make room, measured slower on GPT-2-small and Llama-3-8B shapes.)
constexpr int W_NBUF = 2;
__host__ __device__ constexpr bool apply_out(int kind) { return kind == 5; }
__host__ __device__ constexpr bool mirrors(int kind) { return kind == 0 || kind == 1; }
// Output leaves through two alternating 32x32 chunk buffers per warp
// (GRAM, UPDATE) instead of a whole 32x128 slice (POLY reads its input A
// into the slice and overwrites it in place).
__host__ __device__ constexpr bool chunked_out(int kind) { return kind == 0 || kind == 2; }
constexpr int A_BYTES = HM * BK * 2;                 // 16 KB
constexpr int B_BYTES = HN * BK * 2;                 // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;       // 32 KB per CTA
constexpr int MN_CHUNK_BYTES = BK * 128;             // one 64-wide MN chunk of B (MN-major)
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + EPI_WARPS * 32;         // producer, MMA, 8 epilogue warps
constexpr int EPI_BOX_BYTES = 32 * 128;              // 32 rows x 64 bf16, 128-byte swizzle
constexpr int EPI_BYTES = 2 * EPI_BOX_BYTES;         // a warp's 32x128 slice
constexpr int STG_PITCH = 64;                        // mirror staging: 32 rows x 64 B
constexpr int STG_BYTES = 32 * STG_PITCH;
constexpr int CH_BYTES = 32 * 64;                    // 32 rows x 32 bf16, 64-byte swizzle
constexpr int CH_BUFS = 2;
constexpr int WCH_BYTES = 32 * 128;                  // 32 x 32 fp32 weight chunk, 128-byte swizzle
constexpr int BAR_BYTES = 384;
// PRECOND_MOM, per warp: two momentum chunks (fp32) and two U chunks (bf16)
// One momentum chunk buffer per warp (two U buffers): the slice then leaves
// room for a fifth pipeline stage, which the product needs more than the
// epilogue needs a second buffer (its MMA thread waited for operands on 47 %
// of its cycles with four stages; 0.321 against 0.343 ms per GPT-2-small step)
constexpr int MOM_NBUF = 1;
constexpr int MOM_SLICE = MOM_NBUF * WCH_BYTES + 2 * CH_BYTES;
__host__ __device__ constexpr int smem_bytes(int kind) {
  return stages_for(kind) * STAGE_BYTES +
         EPI_WARPS * ((mom_out(kind)       ? MOM_SLICE
                       : apply_out(kind)   ? W_NBUF * WCH_BYTES
                       : chunked_out(kind) ? CH_BUFS * CH_BYTES
                       : fp32_out(kind)    ? 0
                                           : EPI_BYTES) +
                      (mirrors(kind) ? STG_BYTES : 0)) +
         BAR_BYTES + 1024;   // + alignment slack
}
// GRAM32 sums a long K (thousands of tokens): the tensor cores accumulate
// K in chunks of this many 64-deep blocks into alternating accumulators and
// the epilogue adds the chunks in fp32 registers, so no fp32 sum in TMEM
// runs over more than 4 x 16 = 64 MMA accumulation steps.
constexpr int G32_CHUNK_KB = 4;
__host__ __device__ constexpr int chunk_kb(int kind) { return kind == 3 ? G32_CHUNK_KB : 1 << 30; }
// full + empty per stage (at most 7), two tfull, two tempty, drain, the aux
// barriers, then the TMEM slot and the abort flag
static_assert((2 * 7 + 5 + W_NBUF * EPI_WARPS) * 8 + 8 <= BAR_BYTES, "barrier area");
constexpr int ACC_COLS = 256;                        // one fp32 128x256 accumulator per CTA
constexpr int TMEM_COLS = 2 * ACC_COLS;              // double-buffered
static_assert(smem_bytes(0) <= 232448 && smem_bytes(1) <= 232448 && smem_bytes(2) <= 232448 &&
                  smem_bytes(3) <= 232448 && smem_bytes(4) <= 232448 && smem_bytes(5) <= 232448 &&
                  smem_bytes(6) <= 232448,
              "shared memory per block");
}  // namespace gemm_cfg

// One batched problem of a launch: `batch` equal-shape matrices.
struct GemmProblem {
  int M, N, K;               // per-matrix extents
  int batch;                 // matrices
  int tiles_m, tiles_n;      // ceil(M/256), ceil(N/256)
  int tiles_per_mat;
  int tile_start;            // first tile of this problem in the launch
  __nv_bfloat16* out;        // output, ld out_ld, batch stride out_bs (elements)
  int64_t out_ld, out_bs;
  const float* norm2;        // per-matrix ||U||_F^2 (nullptr: alpha = 1)
  // fp32 output (GRAM32, PRECOND): element (r, c) of matrix z at
  // out32[z * out32_bs + r * out32_ld + c]; PRECOND: z = bidx / nblocks and
  // c is offset by (bidx % nblocks) * N
  float* out32;
  int64_t out32_ld, out32_bs;
  int nblocks;
  float scale;               // GRAM32 / PRECOND: result = scale * sum
  int apply_base;            // UPDATE_APPLY: first ApplyDesc of this problem's matrices
                             // PRECOND_MOM: first MomDesc of this problem's matrices
  int pmap_base;             // PRECOND: first PrecondMaps of this problem's matrices
};

// Per matrix of a fused update + apply: the fp32 weight as a TMA tensor
// (rows x cols, box 32 x 32, 128-byte swizzle), its step scalars and its
// orientation (transposed: rows > cols, so the wide X' is W's transpose).
struct alignas(64) ApplyDesc {
  CUtensorMap w;
  float lr_scale;            // lr * shape scale
  float decay;               // 1 - lr * wd
  int transposed;
  int pad;
};

// Per matrix of a preconditioning product with momentum (PRECOND_MOM): its
// fp32 momentum buffer (rows x cols, box 32 x 32, 128-byte swizzle), its
// Newton-Schulz input in the wide layout (bf16, box 32 x 32, 64-byte
// swizzle), where its partials of ||U||^2 go, and its orientation.
struct alignas(64) MomDesc {
  CUtensorMap mom;
  CUtensorMap x;
  float* partials;
  int transposed;
  int pad;
};

// Per matrix of a preconditioning product: its bf16 gradient read in place
// (cols x rows, box 64 x 128) and the hi/lo stacks of its S^-1 (d x 2d x
// nb, box 64 x 64, one stack per column block; matrices that share an S^-1
// share the stacks).
struct alignas(64) PrecondMaps {
  CUtensorMap a;
  CUtensorMap b;
};

// A launch covers up to MAX_PROBLEMS problems of one product kind (the shape
// runs of a chunk); their tensor maps travel in parameter space.
constexpr int MAX_PROBLEMS = 4;

struct GemmArgs {
  int nprob;
  int total;                 // tiles over all problems
  GemmProblem p[MAX_PROBLEMS];
  int alpha_pow;             // alpha = s^alpha_pow
  float eps;
  float c0, c1, c2;          // POLY: b, c, and a (added on the diagonal)
  int* err;                  // device error flags
  const int* skip;           // the context's device flags: halted() -> do nothing
  int reverse;               // walk the tile list from its end (see run_newton_schulz)
  const ApplyDesc* apply;    // UPDATE_APPLY: per-matrix weights (device memory)
  const PrecondMaps* pmaps;  // PRECOND: per-matrix operand maps (device memory)
  const MomDesc* momd;       // PRECOND_MOM: per-matrix momentum and output (device memory)
  float beta;                // PRECOND_MOM: momentum coefficient
  int nesterov;              // PRECOND_MOM: U = (1 - beta) G' + beta buf, else buf
  int ab_distinct;           // GRAM32 of split fp32 activations: A and B are
                             // different tensors, so a diagonal tile loads both
  int selftest;              // failure-detection self test: the MMA thread
                             // waits for the operands but never issues or
                             // commits, so every role's bounded wait runs out
};

// Per problem: A operand rows (box 64 x 128), B operand (K-major box 64 x 128
// rows, or MN-major box 64 x 64), epilogue input (box 64 x 32), output (box
// 64 x 32).
struct GemmMaps {
  CUtensorMap a[MAX_PROBLEMS], b[MAX_PROBLEMS], aux[MAX_PROBLEMS], out[MAX_PROBLEMS];
};

// Launches whose operand tensor maps are per matrix in device memory
// (args.pmaps) rather than per problem in parameter space.
__host__ __device__ constexpr bool device_maps(int kind, bool b_mn_major) {
  return gemm_cfg::precond_kind(kind) || (kind == EPI_GRAM32 && b_mn_major);
}

__host__ __device__ constexpr bool symmetric_kind(int kind) {
  return kind == EPI_GRAM || kind == EPI_POLY || kind == EPI_GRAM32;
}

// Number of 256x256 pair tiles per matrix that the GEMM kind computes.
__host__ __device__ inline int gemm_tiles_per_mat(int kind, int tiles_m, int tiles_n) {
  if (!symmetric_kind(kind)) return tiles_m * tiles_n;
  return tiles_m * (tiles_m + 1) / 2;     // upper triangle of 256-blocks (tiles_n == tiles_m)
}

__device__ __forceinline__ void decode_tile(int kind, const GemmArgs& a, int t, int& pi, int& bidx, int& ti,
                                            int& tj) {
  if (a.reverse) t = a.total - 1 - t;
  pi = 0;
  while (pi + 1 < a.nprob && a.p[pi + 1].tile_start <= t) ++pi;
  const GemmProblem& P = a.p[pi];
  t -= P.tile_start;
  bidx = t / P.tiles_per_mat;
  t -= bidx * P.tiles_per_mat;
  if (!symmetric_kind(kind)) {
    ti = t % P.tiles_m;          // row tiles fastest: pairs in flight share X columns
    tj = t / P.tiles_m;
    return;
  }
  ti = 0;
  while (true) {
    const int cnt = P.tiles_n - ti;
    if (t < cnt) { tj = ti + t; return; }
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

// Launched in clusters of two CTAs.
template <int KIND, bool B_MN_MAJOR>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(gemm_cfg::THREADS, 1)
    ns_gemm_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmArgs args) {
  using namespace gemm_cfg;
  constexpr int STAGES = stages_for(KIND);
  // GRAM32 with MN-major operands reads the activations in place: A is
  // MN-major too, and both operands' maps come from args.pmaps
  constexpr bool A_MN = KIND == EPI_GRAM32 && B_MN_MAJOR;
  extern __shared__ uint8_t smem_raw[];

  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* smem_epi = smem + STAGES * STAGE_BYTES;             // 1024-aligned slices
  constexpr int SLICE = mom_out(KIND) ? MOM_SLICE : apply_out(KIND) ? W_NBUF * WCH_BYTES
                        : chunked_out(KIND) ? CH_BUFS * CH_BYTES
                        : fp32_out(KIND)  ? 0 : EPI_BYTES;
  uint8_t* smem_stg = smem_epi + EPI_WARPS * SLICE;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem_stg + (mirrors(KIND) ? EPI_WARPS * STG_BYTES : 0));
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;     // accumulator ready   (leader MMA -> both epilogues)
  uint64_t* tempty_bar = tfull_bar + 2;         // accumulator drained (both epilogues -> leader MMA)
  uint64_t* drain_bar = tempty_bar + 2;
  uint64_t* aux_bar = drain_bar + 1;            // W_NBUF per epilogue warp (POLY uses the first)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(aux_bar + W_NBUF * EPI_WARPS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();      // 0: leader of the pair
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 2 * EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
    for (int w = 0; w < W_NBUF * EPI_WARPS; ++w) mbar_init(&aux_bar[w], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0 && !device_maps(KIND, B_MN_MAJOR)) {
    for (int p = 0; p < args.nprob; ++p) {
      prefetch_tensormap(&maps.a[p]);
      prefetch_tensormap(&maps.b[p]);
      prefetch_tensormap(&maps.out[p]);
      if (KIND == EPI_POLY) prefetch_tensormap(&maps.aux[p]);
    }
  }
  tc_fence_before();
  cluster_sync();              // both CTAs' barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // everything above touches only shared memory, TMEM and the parameter
  // space, so it runs before the wait for the previous kernel
  pdl_wait();
  // a non-finite gradient or an earlier device error (uniform over the grid)
  // leaves an empty tile list
  const int total = halted(args.skip) ? 0 : args.total;

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs load their halves) ----------------
    if (lane == 0) {
      const uint32_t full0 = map_to_cta(smem_u32(full_bar), 0);   // leader's full_bar[0]
      int it = 0;
      for (int t = pair; t < total && !*abort_flag; t += npairs) {
        int pi, bidx, ti, tj;
        decode_tile(KIND, args, t, pi, bidx, ti, tj);
        const CUtensorMap* tmA = &maps.a[pi];
        const CUtensorMap* tmB = &maps.b[pi];
        int za = bidx, zb = bidx;              // depth coordinates of the A and B loads
        int xoff = 0;                          // MN offset of both operands (GRAM32 direct)
        if (precond_kind(KIND)) {
          // tile bidx: column block bidx % nblocks of matrix bidx / nblocks
          const int nbk = args.p[pi].nblocks;
          const PrecondMaps& pm = args.pmaps[args.p[pi].pmap_base + bidx / nbk];
          tmA = &pm.a;
          tmB = &pm.b;
          za = 0;
          zb = bidx % nbk;
        } else if (A_MN) {
          // tile bidx: column block bidx % nblocks of activation bidx / nblocks,
          // both operands read from the tokens x width activation itself
          const int nbk = args.p[pi].nblocks;
          const PrecondMaps& pm = args.pmaps[args.p[pi].pmap_base + bidx / nbk];
          tmA = tmB = &pm.a;
          za = zb = 0;
          xoff = (bidx % nbk) * args.p[pi].N;
        }
        const int nk = (args.p[pi].K + BK - 1) / BK;
        // diagonal tile of a symmetric product: each CTA's B rows are its A
        // rows, so only A is loaded and the MMA reads it for both operands
        const bool diag = symmetric_kind(KIND) && ti == tj && !args.ab_distinct;
        for (int kb = 0; kb < nk; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&empty_bar[s], ph ^ 1, args.err, abort_flag)) break;
          uint8_t* a_dst = smem + s * STAGE_BYTES;
          uint8_t* b_dst = a_dst + A_BYTES;
          const uint32_t fb = full0 + s * 8;
          if (leader) mbar_arrive_expect_tx(&full_bar[s], diag ? 2 * A_BYTES : 2 * STAGE_BYTES);
          if (precond_kind(KIND)) {
            // A: the gradient's column block zb, read twice along K (against
            // S_hi, then S_lo)
            const int d = args.p[pi].N;
            int kx = kb * BK;
            if (kx >= d) kx -= d;
            tma_load_3d_pair(a_dst, tmA, fb, zb * d + kx, ti * TM + rank * HM, za);
          } else if (A_MN) {
#pragma unroll
            for (int c = 0; c < HM / 64; ++c)
              tma_load_3d_pair(a_dst + c * MN_CHUNK_BYTES, tmA, fb, xoff + ti * TM + rank * HM + c * 64, kb * BK, za);
          } else {
            tma_load_3d_pair(a_dst, tmA, fb, kb * BK, ti * TM + rank * HM, za);
          }
          // a diagonal tile's B is its A (expect_tx above counts A only)
          if (B_MN_MAJOR && !diag) {
#pragma unroll
            for (int c = 0; c < HN / 64; ++c)
              tma_load_3d_pair(b_dst + c * MN_CHUNK_BYTES, tmB, fb, xoff + tj * TN + rank * HN + c * 64, kb * BK, zb);
          } else if (!diag) {
            tma_load_3d_pair(b_dst, tmB, fb, kb * BK, tj * TN + rank * HN, zb);
          }
          ++it;
        }
      }
      if (*abort_flag && leader) {
        // Let every copy that signals this CTA's barriers land before exit.
        volatile int no_abort = 0;
        for (int k = (it > STAGES ? it - STAGES : 0); k < it; ++k)
          mbar_wait(&full_bar[k % STAGES], (k / STAGES) & 1, args.err, &no_abort);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader CTA only) ----------------
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(TM, TN, B_MN_MAJOR, A_MN);
      constexpr int CHUNK = chunk_kb(KIND);
      int it = 0, la = 0;                   // stages consumed, accumulators filled
      bool ok = true;
      for (int t = pair; t < total && ok && args.selftest; t += npairs) {
        // self test: take the operand stages as they land, issue nothing
        const int nk = (args.p[0].K + BK - 1) / BK;
        for (int kb = 0; kb < nk; ++kb, ++it)
          if (!mbar_wait(&full_bar[it % STAGES], (it / STAGES) & 1, args.err, abort_flag)) { ok = false; break; }
      }
      for (int t = pair; t < total && ok && !args.selftest; t += npairs) {
        int pi, bidx, ti, tj;
        decode_tile(KIND, args, t, pi, bidx, ti, tj);
        const int nk = (args.p[pi].K + BK - 1) / BK;
        const bool diag = symmetric_kind(KIND) && ti == tj && !args.ab_distinct;
        // one accumulator per K chunk (the whole K except for GRAM32)
        for (int k0 = 0; k0 < nk && ok; k0 += CHUNK, ++la) {
          const int acc = la & 1;
          if (!mbar_wait(&tempty_bar[acc], ((la >> 1) & 1) ^ 1, args.err, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem + acc * ACC_COLS;
          const int k1 = min(nk, k0 + CHUNK);
          for (int kb = k0; kb < k1; ++kb) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!mbar_wait(&full_bar[s], ph, args.err, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a_base = smem_u32(smem + s * STAGE_BYTES);
            const uint32_t b_base = diag ? a_base : a_base + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t adesc = A_MN ? sdesc_mnmajor_sw128(a_base + kk * 16 * 128, MN_CHUNK_BYTES)
                                          : sdesc_kmajor_sw128(a_base + kk * 32);
              const uint64_t bdesc = B_MN_MAJOR ? sdesc_mnmajor_sw128(b_base + kk * 16 * 128, MN_CHUNK_BYTES)
                                                : sdesc_kmajor_sw128(b_base + kk * 32);
              mma_bf16_ss_pair(d_tmem, adesc, bdesc, idesc, (kb > k0 || kk > 0) ? 1u : 0u);
            }
            mma_commit_pair_mc(&empty_bar[s], 0x3);
            ++it;
          }
          if (ok) mma_commit_pair_mc(&tfull_bar[acc], 0x3);
        }
      }
      if (*abort_flag) {
        // wait for the MMAs already issued before TMEM is released
        volatile int no_abort = 0;
        mma_commit_pair_mc(drain_bar, 0x1);
        mbar_wait(drain_bar, 0, args.err, &no_abort);
      }
    }
    __syncwarp();
  } else if constexpr (KIND == EPI_GRAM32) {
    // ---------------- GRAM32 epilogue: K chunks summed in registers ----------------
    const int ew = warp - 2;
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int half = ew >> 2;               // 128-column half of the tile
    const uint32_t tempty0 = map_to_cta(smem_u32(tempty_bar), 0);
    int la = 0;
    for (int t = pair; t < total; t += npairs) {
      int pi, bidx, ti, tj;
      decode_tile(KIND, args, t, pi, bidx, ti, tj);
      const GemmProblem& P = args.p[pi];
      const int rb = ti * 2 + static_cast<int>(rank);   // 128-row block index of this CTA
      const int rbase = rb * HM + q * 32;
      const int cb = tj * 2 + half;          // 128-column block index
      const int col0 = cb * 128;
      // below the diagonal: mirrored by another block
      const bool active = col0 < P.N && rbase < P.M && cb >= rb;
      const bool mirror = cb > rb;
      const int nk = (P.K + BK - 1) / BK;
      float run[4][32];
#pragma unroll
      for (int c32 = 0; c32 < 4; ++c32)
#pragma unroll
        for (int k = 0; k < 32; ++k) run[c32][k] = 0.f;
      bool ok = true;
      for (int k0 = 0; k0 < nk; k0 += G32_CHUNK_KB, ++la) {
        const int acc = la & 1;
        // warp-uniform decision: tcgen05.ld below is warp-collective
        const bool got = mbar_wait(&tfull_bar[acc], (la >> 1) & 1, args.err, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tc_fence_after();
        if (active) {
          // eight columns at a time: the 128 running sums already hold most
          // of the registers a thread may have
#pragma unroll
          for (int c8 = 0; c8 < 16; ++c8) {
            uint32_t raw[8];
            tmem_ld_32x32b_x8(tmem + acc * ACC_COLS + (static_cast<uint32_t>(q * 32) << 16) + half * 128 + c8 * 8,
                              raw);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 8; ++k) run[c8 >> 2][(c8 & 3) * 8 + k] += __uint_as_float(raw[k]);
          }
        }
        // this warp's reads of the chunk completed (tcgen05.wait::ld)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_relaxed(tempty0 + acc * 8);   // leader's tempty_bar[acc]
      }
      if (!ok) break;
      const int r = rbase + lane;
      if (active && r < P.M) {
        const int64_t zoff = static_cast<int64_t>(bidx) * P.out32_bs;
#pragma unroll
        for (int c32 = 0; c32 < 4; ++c32) {
          const int cbase = col0 + c32 * 32;
          if (cbase < P.N) {
            float* v = run[c32];
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] *= P.scale;
            float* dst = P.out32 + zoff + static_cast<int64_t>(r) * P.out32_ld + cbase;
            if (cbase + 32 <= P.N && (P.out32_ld & 3) == 0) {
#pragma unroll
              for (int u = 0; u < 8; ++u)
                reinterpret_cast<float4*>(dst)[u] = make_float4(v[u * 4], v[u * 4 + 1], v[u * 4 + 2], v[u * 4 + 3]);
            } else {
              for (int k = 0; k < 32 && cbase + k < P.N; ++k) dst[k] = v[k];
            }
            if (mirror) {
              // (r, c) also goes to (c, r): lanes write consecutive r
#pragma unroll
              for (int k = 0; k < 32; ++k)
                if (cbase + k < P.N) P.out32[zoff + static_cast<int64_t>(cbase + k) * P.out32_ld + r] = v[k];
            }
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..9, both CTAs) ----------------
    const int ew = warp - 2;
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int half = ew >> 2;               // 128-column half of the tile
    uint8_t* slice = smem_epi + ew * SLICE;
    uint32_t wph = 0;                       // UPDATE_APPLY: phase bit per weight buffer (bits 0, 1)
    uint32_t wpend = 0;                     // UPDATE_APPLY: weight loads in flight per buffer
    uint32_t nch = 0;                       // output chunks stored so far (buffer = nch & 1)
    uint8_t* stg = smem_stg + ew * STG_BYTES;
    const uint32_t tempty0 = map_to_cta(smem_u32(tempty_bar), 0);
    uint32_t aux_phase = 0;
    bool aux_pending = false;
    int lt = 0;
    for (int t = pair; t < total; t += npairs, ++lt) {
      int pi, bidx, ti, tj;
      decode_tile(KIND, args, t, pi, bidx, ti, tj);
      const GemmProblem& P = args.p[pi];
      const CUtensorMap* tmAux = &maps.aux[pi];
      const CUtensorMap* tmOut = &maps.out[pi];
      const int acc = lt & 1;
      const int rb = ti * 2 + static_cast<int>(rank);   // 128-row block index of this CTA
      const int rbase = rb * HM + q * 32;
      const int cb = tj * 2 + half;          // 128-column block index
      const int col0 = cb * 128;
      bool active = col0 < P.N && rbase < P.M;
      bool mirror = false;
      if (symmetric_kind(KIND)) {
        if (cb < rb) active = false;         // below the diagonal: mirrored by another tile
        mirror = cb > rb;
      }
      const bool two_boxes = col0 + 64 < P.N;
      // the slice is free once the previous tile's TMA store has read it;
      // then fetch this tile's epilogue input into it
      if constexpr (apply_out(KIND)) {
        // weight chunks 0 and 1 of this tile into the two buffers, once the
        // previous tile's stores have read them
        if (lane == 0 && active) {
          bulk_wait_group_read0();
          const ApplyDesc& ad = args.apply[P.apply_base + bidx];
          for (int c = 0; c < 2 && col0 + c * 32 < P.N; ++c) {
            const int cb = col0 + c * 32;
            mbar_arrive_expect_tx(&aux_bar[2 * ew + c], WCH_BYTES);
            if (ad.transposed) tma_load_3d(slice + c * WCH_BYTES, &ad.w, &aux_bar[2 * ew + c], rbase, cb, 0);
            else tma_load_3d(slice + c * WCH_BYTES, &ad.w, &aux_bar[2 * ew + c], cb, rbase, 0);
            wpend |= 1u << c;
          }
        }
      }
      if constexpr (mom_out(KIND)) {
        // momentum chunks 0 and 1 of this tile into the two buffers, once the
        // previous tile's stores have read them
        if (lane == 0 && active) {
          bulk_wait_group_read0();
          const int z = bidx / P.nblocks, blk = bidx % P.nblocks;
          const MomDesc& md = args.momd[P.apply_base + z];
          for (int c = 0; c < MOM_NBUF && col0 + c * 32 < P.N; ++c) {
            mbar_arrive_expect_tx(&aux_bar[2 * ew + c], WCH_BYTES);
            tma_load_3d(slice + c * WCH_BYTES, &md.mom, &aux_bar[2 * ew + c], blk * P.N + col0 + c * 32, rbase, 0);
            wpend |= 1u << c;
          }
        }
      }
      if (lane == 0 && KIND == EPI_POLY) {
        bulk_wait_group_read0();
        if (active) {
          mbar_arrive_expect_tx(&aux_bar[ew], EPI_BYTES);
          tma_load_3d(slice, tmAux, &aux_bar[ew], col0, rbase, bidx);
          tma_load_3d(slice + EPI_BOX_BYTES, tmAux, &aux_bar[ew], col0 + 64, rbase, bidx);
        }
      }
      if (KIND == EPI_POLY && active) aux_pending = true;
      __syncwarp();
      // warp-uniform decision: tcgen05.ld below is warp-collective
      const bool got = mbar_wait(&tfull_bar[acc], (lt >> 1) & 1, args.err, abort_flag);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      if (active && KIND == EPI_POLY) {
        const bool ok = mbar_wait(&aux_bar[ew], aux_phase, args.err, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
        aux_phase ^= 1;
        aux_pending = false;
      }
      float ss_tile = 0.f;                   // PRECOND_MOM: this warp's share of ||U||^2
      if (active) {
        float alpha = 1.0f;
        if (P.norm2 != nullptr) {
          const float sc = 1.0f / (sqrtf(P.norm2[bidx]) + args.eps);
          alpha = (args.alpha_pow == 2) ? sc * sc : sc;
        }
        __nv_bfloat16* out = P.out + static_cast<int64_t>(bidx) * P.out_bs;
#pragma unroll 1
        for (int c32 = 0; c32 < 4; ++c32) {
          const int cbase = col0 + c32 * 32;
          if (cbase >= P.N) break;
          uint32_t raw[32];
          tmem_ld_32x32b_x32(tmem + acc * ACC_COLS + (static_cast<uint32_t>(q * 32) << 16) + half * 128 + c32 * 32,
                             raw);
          tmem_ld_wait();
          if constexpr (KIND == EPI_GRAM32 || KIND == EPI_PRECOND) {
            // fp32 result straight to global memory
            const int r = rbase + lane;
            int64_t zoff = static_cast<int64_t>(bidx) * P.out32_bs;
            int coff = 0;
            if (KIND == EPI_PRECOND) {
              zoff = static_cast<int64_t>(bidx / P.nblocks) * P.out32_bs;
              coff = (bidx % P.nblocks) * P.N;
            }
            float v[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = P.scale * __uint_as_float(raw[k]);
            if (r < P.M) {
              float* dst = P.out32 + zoff + static_cast<int64_t>(r) * P.out32_ld + coff + cbase;
              if (cbase + 32 <= P.N && ((P.out32_ld | coff) & 3) == 0) {
#pragma unroll
                for (int u = 0; u < 8; ++u)
                  reinterpret_cast<float4*>(dst)[u] = make_float4(v[u * 4], v[u * 4 + 1], v[u * 4 + 2], v[u * 4 + 3]);
              } else {
                for (int k = 0; k < 32 && cbase + k < P.N; ++k) dst[k] = v[k];
              }
              if (KIND == EPI_GRAM32 && mirror) {
                // (r, c) also goes to (c, r): lanes write consecutive r
#pragma unroll
                for (int k = 0; k < 32; ++k)
                  if (cbase + k < P.N) P.out32[zoff + static_cast<int64_t>(cbase + k) * P.out32_ld + r] = v[k];
              }
            }
          } else if constexpr (mom_out(KIND)) {
            // G' chunk (row `lane`, 32 columns of column block blk of matrix
            // z): momentum updated in its buffer and stored back, U staged
            // as bf16 and stored into the Newton-Schulz input
            const int z = bidx / P.nblocks, blk = bidx % P.nblocks;
            const MomDesc& md = args.momd[P.apply_base + z];
            const int wb = c32 % MOM_NBUF;
            uint8_t* wbuf = slice + wb * WCH_BYTES;
            // lane 0 issued the load; all lanes wait on its barrier
            const bool okw = mbar_wait(&aux_bar[2 * ew + wb], (wph >> wb) & 1u, args.err, abort_flag);
            if (!__all_sync(0xffffffffu, okw)) break;
            wph ^= 1u << wb;
            wpend &= ~(1u << wb);
            const int cg = blk * P.N + cbase;          // column in the whole matrix
            const float beta = args.beta;
            float u[32];
            // row `lane` of the chunk: 16-byte unit v at unit v ^ (lane % 8)
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              float4* pb = reinterpret_cast<float4*>(wbuf + lane * 128 + ((v ^ (lane & 7)) << 4));
              const float4 b4 = *pb;
              float b[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float g = P.scale * __uint_as_float(raw[v * 4 + e]);
                b[e] = beta * b[e] + (1.f - beta) * g;
                u[v * 4 + e] = args.nesterov ? (1.f - beta) * g + beta * b[e] : b[e];
              }
              *pb = make_float4(b[0], b[1], b[2], b[3]);
            }
            if (rbase + lane < P.M) {
#pragma unroll
              for (int k = 0; k < 32; ++k) ss_tile += u[k] * u[k];
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&md.mom, wbuf, cg, rbase, 0);   // rows past the matrix are clipped
              bulk_commit_group();
            }
            // U buffer wb: the store that last read it (two chunks ago) is
            // at most the fourth most recent group
            uint8_t* ubuf = slice + MOM_NBUF * WCH_BYTES + (c32 & 1) * CH_BYTES;
            if (lane == 0) bulk_wait_group_read3();
            __syncwarp();
            if (!md.transposed) {
              // row `lane`: 16-byte unit v at unit v ^ ((lane / 2) % 4) (64-byte swizzle)
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                uint4 w;
                w.x = pack_bf16x2(u[v * 8 + 0], u[v * 8 + 1]);
                w.y = pack_bf16x2(u[v * 8 + 2], u[v * 8 + 3]);
                w.z = pack_bf16x2(u[v * 8 + 4], u[v * 8 + 5]);
                w.w = pack_bf16x2(u[v * 8 + 6], u[v * 8 + 7]);
                *reinterpret_cast<uint4*>(ubuf + lane * 64 + ((v ^ ((lane >> 1) & 3)) << 4)) = w;
              }
            } else {
              // the wide layout is U^T: buffer row k is column cg + k, the
              // lanes' rows side by side (element `lane` of unit lane / 8)
#pragma unroll
              for (int k = 0; k < 32; ++k)
                *reinterpret_cast<__nv_bfloat16*>(ubuf + k * 64 + ((((lane >> 3) ^ ((k >> 1) & 3)) & 3) << 4) +
                                                  (lane & 7) * 2) = __float2bfloat16_rn(u[k]);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (!md.transposed) tma_store_3d(&md.x, ubuf, cg, rbase, 0);
              else tma_store_3d(&md.x, ubuf, rbase, cg, 0);
              bulk_commit_group();
              // momentum chunk c32 + MOM_NBUF into this buffer once its store has read it
              const int cn = cbase + 32 * MOM_NBUF;
              if (c32 + MOM_NBUF < 4 && cn < P.N) {
                bulk_wait_group_read1();
                mbar_arrive_expect_tx(&aux_bar[2 * ew + wb], WCH_BYTES);
                tma_load_3d(wbuf, &md.mom, &aux_bar[2 * ew + wb], blk * P.N + cn, rbase, 0);
                wpend |= 1u << wb;
              }
            }
            wpend = __shfl_sync(0xffffffffu, wpend, 0);
          } else if constexpr (apply_out(KIND)) {
            const ApplyDesc& ad = args.apply[P.apply_base + bidx];
            const int wb = c32 & 1;
            uint8_t* wbuf = slice + wb * WCH_BYTES;
            // lane 0 issued the load; all lanes wait on its barrier
            const bool okw = mbar_wait(&aux_bar[2 * ew + wb], (wph >> wb) & 1u, args.err, abort_flag);
            if (!__all_sync(0xffffffffu, okw)) break;
            wph ^= 1u << wb;
            wpend &= ~(1u << wb);
            const float dec = ad.decay, lrs = ad.lr_scale;
            if (!ad.transposed) {
              // row `lane` of the chunk: 16-byte unit u at unit u ^ (lane % 8)
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                float4* pw = reinterpret_cast<float4*>(wbuf + lane * 128 + ((u ^ (lane & 7)) << 4));
                float4 w = *pw;
                w.x = w.x * dec - lrs * (alpha * __uint_as_float(raw[u * 4 + 0]));
                w.y = w.y * dec - lrs * (alpha * __uint_as_float(raw[u * 4 + 1]));
                w.z = w.z * dec - lrs * (alpha * __uint_as_float(raw[u * 4 + 2]));
                w.w = w.w * dec - lrs * (alpha * __uint_as_float(raw[u * 4 + 3]));
                *pw = w;
              }
            } else {
              // W is X'^T: element k of this lane's row is W[cbase + k][rbase + lane],
              // row k of the chunk, column `lane`
#pragma unroll
              for (int k = 0; k < 32; ++k) {
                float* pw = reinterpret_cast<float*>(wbuf + k * 128 + ((((lane >> 2) ^ k) & 7) << 4) + (lane & 3) * 4);
                *pw = *pw * dec - lrs * (alpha * __uint_as_float(raw[k]));
              }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (ad.transposed) tma_store_3d(&ad.w, wbuf, rbase, cbase, 0);
              else tma_store_3d(&ad.w, wbuf, cbase, rbase, 0);
              bulk_commit_group();
              // chunk c32 + 2 into this buffer once the store has read it
              const int cn = cbase + 64;
              if (c32 + 2 < 4 && cn < P.N) {
                bulk_wait_group_read0();
                mbar_arrive_expect_tx(&aux_bar[2 * ew + wb], WCH_BYTES);
                if (ad.transposed) tma_load_3d(wbuf, &ad.w, &aux_bar[2 * ew + wb], rbase, cn, 0);
                else tma_load_3d(wbuf, &ad.w, &aux_bar[2 * ew + wb], cn, rbase, 0);
                wpend |= 1u << wb;
              }
            }
            wpend = __shfl_sync(0xffffffffu, wpend, 0);
          } else if constexpr (chunked_out(KIND)) {
            float v[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = alpha * __uint_as_float(raw[k]);
            // the store that last read this buffer (two chunks ago) is done with it
            uint8_t* buf = slice + (nch & 1) * CH_BYTES;
            if (lane == 0) bulk_wait_group_read1();
            __syncwarp();
            // row `lane`: 16-byte unit u at unit u ^ ((lane / 2) % 4) (64-byte swizzle)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint4 w;
              w.x = pack_bf16x2(v[u * 8 + 0], v[u * 8 + 1]);
              w.y = pack_bf16x2(v[u * 8 + 2], v[u * 8 + 3]);
              w.z = pack_bf16x2(v[u * 8 + 4], v[u * 8 + 5]);
              w.w = pack_bf16x2(v[u * 8 + 6], v[u * 8 + 7]);
              *reinterpret_cast<uint4*>(buf + lane * 64 + ((u ^ ((lane >> 1) & 3)) << 4)) = w;
            }
            if (mirror) {
#pragma unroll
              for (int k = 0; k < 32; ++k)
                reinterpret_cast<__nv_bfloat16*>(stg + k * STG_PITCH)[lane] = __float2bfloat16_rn(v[k]);
              __syncwarp();
              store_staged(stg, out, P.out_ld, cbase, rbase, P.N, P.M, lane);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(tmOut, buf, cbase, rbase, bidx);
              bulk_commit_group();
            }
            ++nch;
          } else {
          // this thread's row `lane`, 4 x 16 B at columns c32*32 + u*8 of the slice
          uint4* cell[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int cc = c32 * 32 + u * 8;
            const int j = (cc & 63) >> 3;
            cell[u] = reinterpret_cast<uint4*>(slice + (cc >> 6) * EPI_BOX_BYTES + lane * 128 +
                                               ((j ^ (lane & 7)) << 4));
          }
          float v[32];
          if (KIND != EPI_POLY) {
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = alpha * __uint_as_float(raw[k]);
          } else {
            // B' = b A + c A^2 + a I: the diagonal element of this row, if it
            // falls in this chunk, is column rbase + lane
            const int dk = rbase + lane - cbase;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint4 w = *cell[u];
              float in[8];
              float2 f;
              f = unpack_bf16x2(w.x); in[0] = f.x; in[1] = f.y;
              f = unpack_bf16x2(w.y); in[2] = f.x; in[3] = f.y;
              f = unpack_bf16x2(w.z); in[4] = f.x; in[5] = f.y;
              f = unpack_bf16x2(w.w); in[6] = f.x; in[7] = f.y;
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float a = __uint_as_float(raw[u * 8 + e]);
                v[u * 8 + e] = args.c0 * in[e] + args.c1 * a + (u * 8 + e == dk ? args.c2 : 0.0f);
              }
            }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 w;
            w.x = pack_bf16x2(v[u * 8 + 0], v[u * 8 + 1]);
            w.y = pack_bf16x2(v[u * 8 + 2], v[u * 8 + 3]);
            w.z = pack_bf16x2(v[u * 8 + 4], v[u * 8 + 5]);
            w.w = pack_bf16x2(v[u * 8 + 6], v[u * 8 + 7]);
            *cell[u] = w;
          }
          if (mirror) {
            // transposed block: staged row k holds column cbase+k of the tile
#pragma unroll
            for (int k = 0; k < 32; ++k)
              reinterpret_cast<__nv_bfloat16*>(stg + k * STG_PITCH)[lane] = __float2bfloat16_rn(v[k]);
            __syncwarp();
            store_staged(stg, out, P.out_ld, cbase, rbase, P.N, P.M, lane);
            __syncwarp();
          }
          }
        }
        // the slice now holds the output: make it visible to the TMA unit, store it
        fence_async_smem();
        __syncwarp();
        if (lane == 0 && KIND == EPI_POLY) {
          tma_store_3d(tmOut, slice, col0, rbase, bidx);
          if (two_boxes) tma_store_3d(tmOut, slice + EPI_BOX_BYTES, col0 + 64, rbase, bidx);
          bulk_commit_group();
        }
      }
      if constexpr (mom_out(KIND)) {
        // one partial of ||U||^2 per (tile, CTA, warp), zero when the warp's
        // rows or columns lie outside the matrix; the norm kernel adds a
        // matrix's partials in this fixed order
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss_tile += __shfl_xor_sync(0xffffffffu, ss_tile, o);
        if (lane == 0) {
          const int z = bidx / P.nblocks, blk = bidx % P.nblocks;
          args.momd[P.apply_base + z].partials[((static_cast<int64_t>(blk) * P.tiles_m + ti) * P.tiles_n + tj) *
                                                   (2 * EPI_WARPS) + static_cast<int>(rank) * EPI_WARPS + ew] = ss_tile;
        }
      }
      // this warp's tcgen05.ld reads of the accumulator have completed
      // (tcgen05.wait::ld); the MMA may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(tempty0 + acc * 8);   // leader's tempty_bar[acc]
    }
    if (lane == 0) {
      if (aux_pending) {
        volatile int no_abort = 0;
        mbar_wait(&aux_bar[ew], aux_phase, args.err, &no_abort);   // let the copy land
      }
      for (int b = 0; b < 2; ++b)
        if (wpend & (1u << b)) {
          volatile int no_abort = 0;
          mbar_wait(&aux_bar[2 * ew + b], (wph >> b) & 1u, args.err, &no_abort);
        }
      bulk_wait_group0();
    }
    __syncwarp();
  }

  // ---- teardown: both CTAs done with each other's barriers and smem, then
  // TMEM is freed by the warp that allocated it ----
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

}  // namespace muon
