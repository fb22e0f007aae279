// muon_abi.cu -- host side of the library: argument checks, the grouping
// scheduler, workspace planning, TMA descriptor encoding, kernel launches
// and the extern "C" entry points declared in include/muon.h.
//
// Scheduling.  Every hidden weight is handled in its wide orientation
// (m = min(rows, cols) rows, n = max columns; a tall matrix is transposed by
// the momentum kernel on its way into the workspace).  Matrices of one wide
// shape form a run; each Newton-Schulz product of a run is ONE batched launch
// whose tile list covers every matrix of the run, so small layers fill the
// 148 SMs together.  When a caller-bounded workspace cannot hold everything,
// the matrices are processed in chunks that fit.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/muon.h"
#include "elementwise.cuh"
#include "newton.cuh"
#include "ns_gemm.cuh"
#include "small_ns.cuh"

using namespace muon;

struct muon_ctx {
  int device = 0;
  size_t ws_cap = 0;            // 0: grow on demand
  void* ws_own = nullptr;
  size_t ws_own_bytes = 0;
  void* ws_user = nullptr;
  size_t ws_user_bytes = 0;
  void* dtable = nullptr;       // device descriptor table
  size_t dtable_bytes = 0;
  void* htable[2] = {nullptr, nullptr};   // pinned staging, double-buffered
  size_t htable_bytes[2] = {0, 0};
  cudaEvent_t hevent[2] = {nullptr, nullptr};
  int hslot = 0;
  int* dflags = nullptr;        // [0] error bits, [1] non-finite, [2..] spare
  uint64_t launches = 0;
  cudaStream_t last_stream = nullptr;
  std::string err;
  // profiler: event pairs per kernel class, recycled through a pool
  bool prof = false;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> prof_pending[MUON_K_COUNT];
  std::vector<cudaEvent_t> prof_pool;
  double prof_ms[MUON_K_COUNT] = {};
  uint64_t prof_n[MUON_K_COUNT] = {};
};

namespace {

// ---------------------------------------------------------------------------
// errors
// ---------------------------------------------------------------------------
muon_status fail(muon_ctx* ctx, muon_status st, const char* fmt, ...) {
  if (ctx) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    ctx->err = buf;
  }
  return st;
}

#define CUDA_TRY(ctx, expr)                                                                    \
  do {                                                                                         \
    cudaError_t e_ = (expr);                                                                   \
    if (e_ != cudaSuccess)                                                                     \
      return fail((ctx), MUON_ERR_CUDA, "%s failed: %s (%s:%d)", #expr, cudaGetErrorString(e_), \
                  __FILE__, __LINE__);                                                         \
  } while (0)

// ---------------------------------------------------------------------------
// TMA descriptors through the driver entry point (no link against libcuda)
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// bf16 tensor [batch][rows][ld] viewed as (cols, rows, batch), 128-byte swizzle.
bool encode_bf16_3d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t batch,
                    uint64_t ld, uint32_t box_cols, uint32_t box_rows,
                    CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {cols, rows, batch};
  cuuint64_t strides[2] = {ld * 2, rows * ld * 2};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 tensor of `batch` matrices rows x ld, `zstride` elements apart,
// viewed as (cols, rows, batch), 128-byte swizzle.
bool encode_bf16_3d_strided(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t batch,
                            uint64_t ld, uint64_t zstride, uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {cols, rows, batch};
  cuuint64_t strides[2] = {ld * 2, zstride * 2};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 matrix rows x cols (row pitch cols) viewed as (cols, rows, 1): 32 x 32
// boxes, 128-byte swizzle (a box row is 128 bytes).
bool encode_f32_matrix(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {cols, rows, 1};
  cuuint64_t strides[2] = {cols * 4, rows * cols * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------
inline int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }
inline int64_t cdiv(int64_t x, int64_t a) { return (x + a - 1) / a; }

float shape_scale(int64_t rows, int64_t cols, int mode) {
  switch (mode) {
    case MUON_SCALE_ORIGINAL: return std::sqrt(std::max(1.0, double(rows) / double(cols)));
    case MUON_SCALE_MATCH_RMS_ADAMW: return float(0.2 * std::sqrt(double(std::max(rows, cols))));
    default: return 1.0f;
  }
}

// Multiprocessor count of a device (cached).
int device_sms(int device) {
  static int sms[64] = {};
  const int dev = device & 63;
  if (sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0) n = 148;
    sms[dev] = n;
  }
  return sms[dev];
}

// Elementwise launches over descriptors d[0..n) whose tile_start fields are
// set: each launch covers up to MAX_SEGS segments of equal-shape matrices.
// The segment table counts tiles from the launch's first block (tile_base)
// in 32 bits; a launch is one grid, at most 2^31 - 1 blocks, and every
// tensor the library takes fits in device memory, far below 2^31 tiles of
// 4096 elements.
struct SegLaunch {
  SegTable t;
  int64_t tile_base;
  int64_t tiles;
};

inline int64_t desc_tiles(const MatDesc& d) { return ((d.rows + EW_TILE - 1) / EW_TILE) * d.tiles_c; }

std::vector<SegLaunch> build_seg_launches(const MatDesc* d, int n) {
  std::vector<SegLaunch> out;
  SegLaunch cur{};
  auto close = [&](int64_t end_tile) {
    cur.tiles = end_tile - cur.tile_base;
    out.push_back(cur);
    cur = SegLaunch{};
  };
  for (int i = 0; i < n; ++i) {
    const bool fresh = i == 0 || d[i].rows != d[i - 1].rows || d[i].cols != d[i - 1].cols;
    if (!fresh) continue;
    if (cur.t.n == MAX_SEGS) close(d[i].tile_start);
    if (cur.t.n == 0) cur.tile_base = d[i].tile_start;
    const int s = cur.t.n++;
    cur.t.first_mat[s] = i;
    cur.t.tile_start[s] = static_cast<uint32_t>(d[i].tile_start - cur.tile_base);
    cur.t.tiles_per_mat[s] = static_cast<uint32_t>(desc_tiles(d[i]));
  }
  if (n > 0) close(d[n - 1].tile_start + desc_tiles(d[n - 1]));
  return out;
}

// One matrix after validation, in scheduling order.
struct Item {
  int64_t rows, cols, m, n;
  bool transposed;
  int grad_dtype;
  const void* grad;
  float* weight;
  float* momentum;
  float* update_out;
  const float* precond;
  int precond_blocks;
  const void* precond_split = nullptr;   // caller's bf16 hi/lo split of precond (muon_step)
};

// A run of matrices sharing one wide shape, inside one chunk.
struct Run {
  int64_t m, n, ld_n, ld_m;
  int first, count;              // item range
  size_t off_x0, off_x1, off_a, off_b;
};

struct Chunk {
  int first, count;              // item range
  size_t off_norm;               // count floats, then per-tile partials
  size_t off_partials;
  size_t off_pgrad;              // preconditioned gradients (fp32), if any
  size_t off_fparts;             // partials of ||U||^2 from the preconditioning epilogue
  bool tc_pre;                   // preconditioning on the tensor-core engine
  size_t off_sst;                // S^-1 hi/lo stacks (tensor-core preconditioning)
  std::vector<Run> runs;
  size_t bytes;
};

// Tensor-core preconditioning needs block widths that are whole 64-wide
// K blocks (the hi/lo halves of K must not share one).
inline bool tc_precond_ok(const Item& it) { return (it.cols / it.precond_blocks) % 64 == 0; }
inline size_t sst_bytes(const Item& it) {
  const size_t d = size_t(it.cols / it.precond_blocks);
  return size_t(it.precond_blocks) * 2 * d * d * 2;
}
// Partials of ||U||^2 that the preconditioning product writes when it applies
// the momentum itself: one per (256 x 256 pair tile, CTA, epilogue warp).
inline int64_t fused_parts(const Item& it) {
  const int64_t d = it.cols / it.precond_blocks;
  return int64_t(it.precond_blocks) * cdiv(it.rows, gemm_cfg::TM) * cdiv(d, gemm_cfg::TN) * 2 * gemm_cfg::EPI_WARPS;
}

constexpr size_t kAlign = 256;

// Lay the chunk out in workspace; returns its total bytes.
size_t layout_chunk(Chunk& c, const std::vector<Item>& items) {
  size_t off = 0;
  c.off_norm = off;
  off += round_up(c.count * sizeof(float), kAlign);
  c.off_partials = off;
  int64_t tiles = 0;
  for (int i = c.first; i < c.first + c.count; ++i)
    tiles += cdiv(items[i].rows, EW_TILE) * cdiv(items[i].cols, EW_TILE);
  off += round_up(size_t(tiles) * sizeof(float), kAlign);
  c.off_fparts = off;
  int64_t fparts = 0;
  for (int i = c.first; i < c.first + c.count; ++i)
    if (items[i].precond) fparts += fused_parts(items[i]);
  off += round_up(size_t(fparts) * sizeof(float), kAlign);
  c.off_pgrad = off;
  bool any_pre = false;
  c.tc_pre = true;
  for (int i = c.first; i < c.first + c.count; ++i)
    if (items[i].precond) {
      off += round_up(size_t(items[i].rows) * items[i].cols * 4, kAlign);
      any_pre = true;
      c.tc_pre = c.tc_pre && tc_precond_ok(items[i]);
    }
  c.tc_pre = c.tc_pre && any_pre;
  c.off_sst = off;
  if (c.tc_pre) {
    size_t t = 0;
    for (int i = c.first; i < c.first + c.count; ++i)
      if (items[i].precond) t += round_up(sst_bytes(items[i]), kAlign);
    off += t;
  }
  c.runs.clear();
  int i = c.first;
  while (i < c.first + c.count) {
    Run r{};
    r.m = items[i].m;
    r.n = items[i].n;
    r.ld_n = round_up(r.n, 8);
    r.ld_m = round_up(r.m, 8);
    r.first = i;
    int j = i;
    while (j < c.first + c.count && items[j].m == r.m && items[j].n == r.n) ++j;
    r.count = j - i;
    const size_t xb = round_up(size_t(r.count) * r.m * r.ld_n * 2, kAlign);
    const size_t ab = round_up(size_t(r.count) * r.m * r.ld_m * 2, kAlign);
    r.off_x0 = off; off += xb;
    r.off_x1 = off; off += xb;
    r.off_a = off; off += ab;
    r.off_b = off; off += ab;
    c.runs.push_back(r);
    i = j;
  }
  c.bytes = off;
  return off;
}

// Split items into chunks whose layout fits `cap` bytes (cap == 0: one chunk).
bool plan_chunks(const std::vector<Item>& items, size_t cap, std::vector<Chunk>& out) {
  out.clear();
  int i = 0;
  const int n = int(items.size());
  while (i < n) {
    Chunk c{};
    c.first = i;
    c.count = cap == 0 ? n - i : 1;
    if (cap != 0 && layout_chunk(c, items) > cap) return false;
    // grow greedily
    while (i + c.count < n) {
      Chunk t = c;
      t.count = c.count + 1;
      if (cap != 0 && layout_chunk(t, items) > cap) break;
      c.count = t.count;
    }
    layout_chunk(c, items);
    out.push_back(c);
    i += c.count;
  }
  return true;
}

// ---------------------------------------------------------------------------
// context resources
// ---------------------------------------------------------------------------
muon_status ensure_workspace(muon_ctx* ctx, size_t need, void** base) {
  if (ctx->ws_user) {
    if (need > ctx->ws_user_bytes)
      return fail(ctx, MUON_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed",
                  ctx->ws_user_bytes, need);
    *base = ctx->ws_user;
    return MUON_OK;
  }
  if (need > ctx->ws_own_bytes) {
    if (ctx->ws_cap != 0)
      return fail(ctx, MUON_ERR_WORKSPACE, "workspace cap %zu < %zu", ctx->ws_cap, need);
    if (ctx->ws_own) {
      CUDA_TRY(ctx, cudaDeviceSynchronize());
      CUDA_TRY(ctx, cudaFree(ctx->ws_own));
      ctx->ws_own = nullptr;
      ctx->ws_own_bytes = 0;
    }
    const size_t grow = round_up(need, size_t(1) << 20);
    CUDA_TRY(ctx, cudaMalloc(&ctx->ws_own, grow));
    ctx->ws_own_bytes = grow;
  }
  *base = ctx->ws_own;
  return MUON_OK;
}

size_t ws_limit(const muon_ctx* ctx) {
  if (ctx->ws_user) return ctx->ws_user_bytes;
  return ctx->ws_cap;   // 0 = unbounded
}

// Copy `bytes` of host data to the device table through pinned staging.
muon_status upload_table(muon_ctx* ctx, const void* data, size_t bytes, cudaStream_t st, void** dptr) {
  if (bytes > ctx->dtable_bytes) {
    if (ctx->dtable) {
      CUDA_TRY(ctx, cudaDeviceSynchronize());
      CUDA_TRY(ctx, cudaFree(ctx->dtable));
      ctx->dtable = nullptr;
    }
    const size_t nb = round_up(std::max<size_t>(bytes, 1 << 16), 1 << 16);
    CUDA_TRY(ctx, cudaMalloc(&ctx->dtable, nb));
    ctx->dtable_bytes = nb;
  }
  const int s = ctx->hslot;
  ctx->hslot ^= 1;
  CUDA_TRY(ctx, cudaEventSynchronize(ctx->hevent[s]));   // previous copy from this slot done
  if (bytes > ctx->htable_bytes[s]) {
    if (ctx->htable[s]) CUDA_TRY(ctx, cudaFreeHost(ctx->htable[s]));
    ctx->htable[s] = nullptr;
    const size_t nb = round_up(std::max<size_t>(bytes, 1 << 16), 1 << 16);
    CUDA_TRY(ctx, cudaMallocHost(&ctx->htable[s], nb));
    ctx->htable_bytes[s] = nb;
  }
  std::memcpy(ctx->htable[s], data, bytes);
  CUDA_TRY(ctx, cudaMemcpyAsync(ctx->dtable, ctx->htable[s], bytes, cudaMemcpyHostToDevice, st));
  CUDA_TRY(ctx, cudaEventRecord(ctx->hevent[s], st));
  *dptr = ctx->dtable;
  return MUON_OK;
}

// Profiler brackets: begin records an event before the launch, end after it.
cudaEvent_t prof_event(muon_ctx* ctx) {
  if (!ctx->prof_pool.empty()) {
    cudaEvent_t e = ctx->prof_pool.back();
    ctx->prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

struct ProfScope {
  muon_ctx* ctx;
  int kind;
  cudaStream_t st;
  cudaEvent_t a = nullptr;
  ProfScope(muon_ctx* c, int k, cudaStream_t s) : ctx(c), kind(k), st(s) {
    if (ctx->prof) {
      a = prof_event(ctx);
      cudaEventRecord(a, st);
    }
  }
  ~ProfScope() {
    if (a) {
      cudaEvent_t b = prof_event(ctx);
      cudaEventRecord(b, st);
      ctx->prof_pending[kind].push_back({a, b});
    }
  }
};

muon_status set_device(muon_ctx* ctx) {
  CUDA_TRY(ctx, cudaSetDevice(ctx->device));
  return MUON_OK;
}

// ---------------------------------------------------------------------------
// launches
// ---------------------------------------------------------------------------
// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel in the stream drains; every kernel launched this
// way calls pdl_wait() before its first global-memory access.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int KIND, bool BMN>
cudaError_t launch_gemm(muon_ctx* ctx, const GemmMaps& maps, const GemmArgs& g, cudaStream_t st) {
  static bool attr_done[64] = {};
  static int max_pairs[64] = {};
  const int dev = ctx->device & 63;
  if (!attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(ns_gemm_kernel<KIND, BMN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         gemm_cfg::smem_bytes(KIND));
    if (e != cudaSuccess) return e;
    // how many CTA pairs can be resident at once (one CTA per SM)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (device_sms(ctx->device) / 2));
    cfg.blockDim = dim3(gemm_cfg::THREADS);
    cfg.dynamicSmemBytes = gemm_cfg::smem_bytes(KIND);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, ns_gemm_kernel<KIND, BMN>, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = device_sms(ctx->device) / 2;
    }
    max_pairs[dev] = n;
    attr_done[dev] = true;
  }
  if (g.total <= 0) return cudaSuccess;
  const int pairs = std::min(g.total, max_pairs[dev]);   // persistent pairs
  const cudaError_t e = launch_pdl(ns_gemm_kernel<KIND, BMN>, dim3(unsigned(2 * pairs)), dim3(gemm_cfg::THREADS),
                                   size_t(gemm_cfg::smem_bytes(KIND)), st, maps, g);
  ctx->launches++;
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Device buffers and tensor maps of one shape run.
struct RunMaps {
  __nv_bfloat16 *x[2], *A, *B;
  CUtensorMap x_r128[2], x_mn[2], x_r32[2], a_r128, a_r32, b_r128, b_r32;
  CUtensorMap x_c32[2], a_c32;   // 32 x 32 output chunks, 64-byte swizzle
};

bool encode_run(uint8_t* ws, const Run& r, RunMaps& mp) {
  mp.x[0] = reinterpret_cast<__nv_bfloat16*>(ws + r.off_x0);
  mp.x[1] = reinterpret_cast<__nv_bfloat16*>(ws + r.off_x1);
  mp.A = reinterpret_cast<__nv_bfloat16*>(ws + r.off_a);
  mp.B = reinterpret_cast<__nv_bfloat16*>(ws + r.off_b);
  bool ok = true;
  for (int k = 0; k < 2; ++k) {
    ok &= encode_bf16_3d(&mp.x_r128[k], mp.x[k], r.n, r.m, r.count, r.ld_n, 64, 128);
    ok &= encode_bf16_3d(&mp.x_mn[k], mp.x[k], r.n, r.m, r.count, r.ld_n, 64, 64);
    ok &= encode_bf16_3d(&mp.x_r32[k], mp.x[k], r.n, r.m, r.count, r.ld_n, 64, 32);
    ok &= encode_bf16_3d(&mp.x_c32[k], mp.x[k], r.n, r.m, r.count, r.ld_n, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  ok &= encode_bf16_3d(&mp.a_c32, mp.A, r.m, r.m, r.count, r.ld_m, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  ok &= encode_bf16_3d(&mp.a_r128, mp.A, r.m, r.m, r.count, r.ld_m, 64, 128);
  ok &= encode_bf16_3d(&mp.a_r32, mp.A, r.m, r.m, r.count, r.ld_m, 64, 32);
  ok &= encode_bf16_3d(&mp.b_r128, mp.B, r.m, r.m, r.count, r.ld_m, 64, 128);
  ok &= encode_bf16_3d(&mp.b_r32, mp.B, r.m, r.m, r.count, r.ld_m, 64, 32);
  return ok;
}

// Runs whose wide shape fits one CTA pair go through small_ns_kernel: all
// iterations in one launch.
inline bool small_run(const Run& r) { return r.m <= small_cfg::MAXD && r.n <= small_cfg::MAXD; }

// All ns_steps iterations of the matrices of one small run in one launch;
// the last update stores the final X at x[ns_steps % 2], or applies the
// weight step of matrix k from mdesc[k] when mdesc is given; with mom, the
// kernel also forms X0 itself (Nesterov momentum of matrix k from mom[k] and
// the Frobenius norm), so the run needs no other launch.
muon_status run_small_ns(muon_ctx* ctx, uint8_t* ws, const Run& r, const float* norm2, const muon_hparams* hp,
                         const int* skip, cudaStream_t st, const MatDesc* mdesc, const MatDesc* mom) {
  static bool attr_done[64] = {};
  static int max_pairs[64] = {};
  const int dev = ctx->device & 63;
  if (!attr_done[dev]) {
    CUDA_TRY(ctx, cudaFuncSetAttribute(small_ns_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       small_cfg::SMEM));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (device_sms(ctx->device) / 2));
    cfg.blockDim = dim3(small_cfg::THREADS);
    cfg.dynamicSmemBytes = small_cfg::SMEM;
    int np = 0;
    if (cudaOccupancyMaxActiveClusters(&np, small_ns_kernel, &cfg) != cudaSuccess || np <= 0) {
      cudaGetLastError();
      np = device_sms(ctx->device) / 2;
    }
    max_pairs[dev] = np;
    attr_done[dev] = true;
  }
  if (hp->ns_steps < 1 || r.count < 1) return MUON_OK;
  SmallNsArgs a{};
  a.x_in = reinterpret_cast<const __nv_bfloat16*>(ws + r.off_x0);
  a.x_out = reinterpret_cast<__nv_bfloat16*>(ws + (hp->ns_steps % 2 ? r.off_x1 : r.off_x0));
  a.ld = r.ld_n;
  a.bs = r.m * r.ld_n;
  a.norm2 = norm2;
  a.apply = mdesc;
  a.mom = mom;
  a.beta = hp->momentum;
  a.nesterov = hp->nesterov;
  a.m = int(r.m);
  a.n = int(r.n);
  a.count = r.count;
  a.steps = hp->ns_steps;
  a.a = hp->ns_a;
  a.b = hp->ns_b;
  a.c = hp->ns_c;
  a.eps = hp->eps;
  a.err = ctx->dflags;
  a.skip = skip;
  const int pairs = std::min(r.count, max_pairs[dev]);
  ProfScope ps(ctx, MUON_K_NS_SMALL, st);
  CUDA_TRY(ctx, launch_pdl(small_ns_kernel, dim3(unsigned(2 * pairs)), dim3(small_cfg::THREADS),
                           size_t(small_cfg::SMEM), st, a));
  ctx->launches++;
  CUDA_TRY(ctx, cudaGetLastError());
  return MUON_OK;
}

// ns_steps quintic iterations on the runs of one chunk (X of each run starts
// in its x0; after the call it is in x[ns_steps % 2]).  norm2s[j] is run j's
// per-matrix ||U||^2.  Runs that fit one CTA pair take one small_ns_kernel
// launch each; for the others each product of an iteration is one launch
// over up to MAX_PROBLEMS runs.  When run_apply is given the last product
// applies the weight step (run_mdesc[j]: the per-matrix descriptors of run
// j).  small_mom: the small kernel also runs the momentum of its matrices
// (their X0 and norm are not in the workspace).
muon_status run_newton_schulz(muon_ctx* ctx, uint8_t* ws, const Run* all_runs, int nall,
                              const float* const* all_norm2s, const muon_hparams* hp, const int* skip,
                              cudaStream_t st, const ApplyDesc* const* all_apply = nullptr,
                              const MatDesc* const* run_mdesc = nullptr, bool small_mom = false) {
  std::vector<Run> big;
  std::vector<const float*> big_norm2;
  std::vector<const ApplyDesc*> big_apply;
  for (int j = 0; j < nall; ++j) {
    if (small_run(all_runs[j])) {
      muon_status s = run_small_ns(ctx, ws, all_runs[j], all_norm2s[j], hp, skip, st,
                                   all_apply != nullptr && run_mdesc != nullptr ? run_mdesc[j] : nullptr,
                                   small_mom && run_mdesc != nullptr ? run_mdesc[j] : nullptr);
      if (s != MUON_OK) return s;
    } else {
      big.push_back(all_runs[j]);
      big_norm2.push_back(all_norm2s[j]);
      big_apply.push_back(all_apply != nullptr ? all_apply[j] : nullptr);
    }
  }
  const Run* runs = big.data();
  const int nruns = int(big.size());
  const float* const* norm2s = big_norm2.data();
  const ApplyDesc* const* run_apply = all_apply != nullptr ? big_apply.data() : nullptr;
  std::vector<RunMaps> mp(nruns);
  for (int j = 0; j < nruns; ++j)
    if (!encode_run(ws, runs[j], mp[j]))
      return fail(ctx, MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed (run %lldx%lld)", (long long)runs[j].m,
                  (long long)runs[j].n);
  // Successive products walk their tile lists in opposite directions, so
  // each launch starts on the matrices the previous one wrote last, which
  // are still in L2 (the first Gram starts where the momentum pass ended).
  int launch_no = 0;
  for (int b0 = 0; b0 < nruns; b0 += MAX_PROBLEMS) {
    const int nb = std::min(MAX_PROBLEMS, nruns - b0);
    int cur = 0;
    for (int it = 0; it < hp->ns_steps; ++it) {
      const bool first = (it == 0);
      for (int kind = EPI_GRAM; kind <= EPI_UPDATE; ++kind) {
        GemmMaps maps;
        GemmArgs g{};
        g.nprob = nb;
        g.eps = hp->eps;
        g.err = ctx->dflags;
        g.skip = skip;
        g.alpha_pow = kind == EPI_GRAM ? 2 : 1;
        g.c0 = hp->ns_b;
        g.c1 = hp->ns_c;
        g.c2 = hp->ns_a;
        g.reverse = (launch_no++ & 1) ^ 1;
        // the last update applies the weight step itself when every run of
        // the launch has its per-matrix weight descriptors
        bool fuse = kind == EPI_UPDATE && it == hp->ns_steps - 1 && run_apply != nullptr;
        for (int j = 0; fuse && j < nb; ++j) fuse = run_apply[b0 + j] != nullptr;
        if (fuse) g.apply = run_apply[b0];
        int tile = 0;
        for (int j = 0; j < nb; ++j) {
          const Run& r = runs[b0 + j];
          const RunMaps& m = mp[b0 + j];
          GemmProblem& P = g.p[j];
          const int tm = int(cdiv(r.m, gemm_cfg::TM));
          P.batch = r.count;
          P.tiles_m = tm;
          P.tile_start = tile;
          if (kind == EPI_GRAM) {          // A = alpha X X^T
            P.M = int(r.m); P.N = int(r.m); P.K = int(r.n);
            P.tiles_n = tm;
            P.out = m.A; P.out_ld = r.ld_m; P.out_bs = r.m * r.ld_m;
            P.norm2 = first ? norm2s[b0 + j] : nullptr;
            maps.a[j] = m.x_r128[cur]; maps.b[j] = m.x_r128[cur]; maps.aux[j] = m.a_r32; maps.out[j] = m.a_c32;
          } else if (kind == EPI_POLY) {   // B' = b A + c A A + a I
            P.M = int(r.m); P.N = int(r.m); P.K = int(r.m);
            P.tiles_n = tm;
            P.out = m.B; P.out_ld = r.ld_m; P.out_bs = r.m * r.ld_m;
            P.norm2 = nullptr;
            maps.a[j] = m.a_r128; maps.b[j] = m.a_r128; maps.aux[j] = m.a_r32; maps.out[j] = m.b_r32;
          } else {                         // X' = alpha B' X  (= alpha (a X + B X))
            P.M = int(r.m); P.N = int(r.n); P.K = int(r.m);
            P.tiles_n = int(cdiv(r.n, gemm_cfg::TN));
            P.out = m.x[cur ^ 1]; P.out_ld = r.ld_n; P.out_bs = r.m * r.ld_n;
            P.norm2 = first ? norm2s[b0 + j] : nullptr;
            maps.a[j] = m.b_r128; maps.b[j] = m.x_mn[cur]; maps.aux[j] = m.x_r32[cur ^ 1]; maps.out[j] = m.x_c32[cur ^ 1];
            if (fuse) P.apply_base = int(run_apply[b0 + j] - run_apply[b0]);
          }
          P.tiles_per_mat = gemm_tiles_per_mat(kind, P.tiles_m, P.tiles_n);
          const int64_t tt = int64_t(tile) + int64_t(P.batch) * P.tiles_per_mat;
          if (tt > INT32_MAX) return fail(ctx, MUON_ERR_UNSUPPORTED, "too many tiles in one launch");
          tile = int(tt);
        }
        g.total = tile;
        if (kind == EPI_GRAM) {
          ProfScope ps(ctx, MUON_K_GRAM, st);
          CUDA_TRY(ctx, (launch_gemm<EPI_GRAM, false>(ctx, maps, g, st)));
        } else if (kind == EPI_POLY) {
          ProfScope ps(ctx, MUON_K_POLY, st);
          CUDA_TRY(ctx, (launch_gemm<EPI_POLY, false>(ctx, maps, g, st)));
        } else if (fuse) {
          ProfScope ps(ctx, MUON_K_UPDATE_APPLY, st);
          CUDA_TRY(ctx, (launch_gemm<EPI_UPDATE_APPLY, true>(ctx, maps, g, st)));
        } else {
          ProfScope ps(ctx, MUON_K_UPDATE, st);
          CUDA_TRY(ctx, (launch_gemm<EPI_UPDATE, true>(ctx, maps, g, st)));
        }
      }
      cur ^= 1;
    }
  }
  return MUON_OK;
}

// Matrices of one shape preconditioned on the tensor cores as one batched
// problem: `count` matrices whose operand maps are consecutive PrecondMaps
// from pmap_base on, fp32 results consecutive in pg (pg_stride floats
// apart).
struct PreProblem {
  int64_t rows, cols;
  int nb, d, count, last;
  int pmap_base;
  float* pg;
  int64_t pg_stride;
  int fused;                 // momentum in the epilogue (PRECOND_MOM); pg unused
  int momd_base;             // fused: MomDesc of the problem's first matrix
};

// Operand maps of one preconditioned matrix: its gradient in place and the
// hi/lo stacks of its S^-1 at sst.
bool encode_precond_maps(PrecondMaps* pm, const void* grad, int64_t rows, int64_t cols, int nb, int d,
                         const __nv_bfloat16* sst) {
  bool ok = encode_bf16_3d(&pm->a, grad, cols, rows, 1, cols, 64, 128);
  ok &= encode_bf16_3d(&pm->b, sst, d, 2 * int64_t(d), nb, d, 64, 64);
  return ok;
}

// G' = G [S_hi; S_lo] for every problem, up to MAX_PROBLEMS per launch;
// pmaps is the device copy of the PrecondMaps table.  Fused problems (inside
// a step) apply the momentum in the epilogue instead of writing G' (their
// matrices' MomDescs start at momd + momd_base); consecutive problems of one
// kind share a launch.
muon_status run_precondition(muon_ctx* ctx, const std::vector<PreProblem>& probs, const PrecondMaps* pmaps,
                             const int* skip, cudaStream_t st, const MomDesc* momd = nullptr, float beta = 0.f,
                             int nesterov = 0) {
  size_t b0 = 0;
  while (b0 < probs.size()) {
    const int fused = probs[b0].fused;
    int nb = 0;
    while (nb < MAX_PROBLEMS && b0 + nb < probs.size() && probs[b0 + nb].fused == fused) ++nb;
    GemmMaps maps{};           // unused: the operands' maps are in pmaps
    GemmArgs g{};
    g.nprob = nb;
    g.err = ctx->dflags;
    g.skip = skip;
    g.pmaps = pmaps;
    g.momd = momd;
    g.beta = beta;
    g.nesterov = nesterov;
    int tile = 0;
    for (int j = 0; j < nb; ++j) {
      const PreProblem& q = probs[b0 + j];
      GemmProblem& P = g.p[j];
      P.M = int(q.rows); P.N = q.d; P.K = 2 * q.d;
      P.batch = q.count * q.nb;
      P.tiles_m = int(cdiv(q.rows, gemm_cfg::TM));
      P.tiles_n = int(cdiv(q.d, gemm_cfg::TN));
      P.tiles_per_mat = gemm_tiles_per_mat(EPI_PRECOND, P.tiles_m, P.tiles_n);
      P.tile_start = tile;
      P.out32 = q.pg; P.out32_ld = q.cols; P.out32_bs = q.pg_stride;
      P.nblocks = q.nb;
      P.scale = 1.0f;
      P.pmap_base = q.pmap_base;
      P.apply_base = q.momd_base;
      const int64_t tt = int64_t(tile) + int64_t(P.batch) * P.tiles_per_mat;
      if (tt > INT32_MAX) return fail(ctx, MUON_ERR_UNSUPPORTED, "too many tiles in one launch");
      tile = int(tt);
    }
    g.total = tile;
    if (fused) CUDA_TRY(ctx, (launch_gemm<EPI_PRECOND_MOM, true>(ctx, maps, g, st)));
    else CUDA_TRY(ctx, (launch_gemm<EPI_PRECOND, true>(ctx, maps, g, st)));
    b0 += nb;
  }
  return MUON_OK;
}

// The S^-1 hi/lo stacks of a launch, one per distinct (S^-1, nb, d): the
// staging pass splits each once, however many matrices share it.
struct StackKey {
  const float* s_inv;
  int nb, d;
  bool operator<(const StackKey& o) const {
    return s_inv != o.s_inv ? s_inv < o.s_inv : nb != o.nb ? nb < o.nb : d < o.d;
  }
};

// Newton-Muon preconditioning on its own: update_out[i] = G_i S^-1 in fp32.
// Matrices whose block width is a multiple of 64 go through the tensor-core
// engine (S^-1 hi/lo stacks staged in workspace, in batches that fit it;
// each matrix its own problem, since the outputs are the caller's); the rest
// through the plain fp32 tile kernel, which writes the caller's buffers
// directly.
muon_status run_precondition_items(muon_ctx* ctx, const std::vector<Item>& items, cudaStream_t st) {
  if (items.empty()) return MUON_OK;
  const size_t limit = ws_limit(ctx);
  std::vector<PrepDesc> prep;               // one per distinct stack of a batch
  std::vector<PrecondMaps> pmaps;           // one per tensor-core matrix
  std::vector<size_t> pm_sst;               // workspace offset of its stacks
  std::vector<PreProblem> probs;
  std::vector<int> batch_prep, batch_prob;  // first prep / problem index of each batch
  std::vector<PrecondDesc> pdescs;
  std::map<StackKey, size_t> stacks;        // this batch's stacks
  int64_t ptiles = 0;
  size_t cur = 0, need = 0;
  for (const Item& it : items) {
    if (tc_precond_ok(it)) {
      const int d = int(it.cols / it.precond_blocks);
      const StackKey key{it.precond, it.precond_blocks, d};
      const size_t sb = round_up(sst_bytes(it), kAlign);
      if (limit != 0 && sb > limit)
        return fail(ctx, MUON_ERR_WORKSPACE, "one matrix needs %zu bytes of workspace, %zu available", sb, limit);
      const bool have = !batch_prep.empty() && stacks.count(key) != 0;
      if (batch_prep.empty() || (!have && limit != 0 && cur + sb > limit)) {
        batch_prep.push_back(int(prep.size()));
        batch_prob.push_back(int(probs.size()));
        stacks.clear();
        cur = 0;
      }
      auto f = stacks.find(key);
      if (f == stacks.end()) {
        f = stacks.emplace(key, cur).first;
        PrepDesc pd{};
        pd.s_inv = it.precond;
        pd.sst = reinterpret_cast<__nv_bfloat16*>(cur);     // offset; rebased below
        pd.nb = it.precond_blocks;
        pd.d = d;
        prep.push_back(pd);
        cur += sb;
        need = std::max(need, cur);
      }
      PreProblem q{};
      q.rows = it.rows; q.cols = it.cols; q.nb = it.precond_blocks; q.d = d; q.count = 1;
      q.pmap_base = int(pmaps.size());
      q.pg = it.update_out; q.pg_stride = it.rows * it.cols;
      probs.push_back(q);
      pmaps.push_back(PrecondMaps{});
      pm_sst.push_back(f->second);
    } else {
      PrecondDesc p{};
      p.grad = static_cast<const __nv_bfloat16*>(it.grad);
      p.s_inv = it.precond;
      p.out = it.update_out;
      p.rows = it.rows;
      p.cols = it.cols;
      p.d = it.cols / it.precond_blocks;
      p.tiles_r = int(cdiv(it.rows, PRE_BM));
      p.tiles_c = int(cdiv(p.d, PRE_BN));
      p.tile_start = ptiles;
      ptiles += int64_t(p.tiles_r) * p.tiles_c * it.precond_blocks;
      pdescs.push_back(p);
    }
  }
  if (ptiles > INT32_MAX) return fail(ctx, MUON_ERR_UNSUPPORTED, "too many precondition tiles in one launch");
  uint8_t* ws = nullptr;
  if (need > 0) {
    void* wsv = nullptr;
    muon_status s = ensure_workspace(ctx, need, &wsv);
    if (s != MUON_OK) return s;
    ws = static_cast<uint8_t*>(wsv);
  }
  for (PrepDesc& pd : prep) pd.sst = reinterpret_cast<__nv_bfloat16*>(ws + reinterpret_cast<uintptr_t>(pd.sst));
  {
    size_t k = 0;
    for (const Item& it : items) {
      if (!tc_precond_ok(it)) continue;
      if (!encode_precond_maps(&pmaps[k], it.grad, it.rows, it.cols, it.precond_blocks,
                               int(it.cols / it.precond_blocks),
                               reinterpret_cast<const __nv_bfloat16*>(ws + pm_sst[k])))
        return fail(ctx, MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed (precondition)");
      ++k;
    }
  }
  const size_t prep_bytes = round_up(prep.size() * sizeof(PrepDesc), kAlign);
  const size_t pm_off = prep_bytes;
  const size_t pm_bytes = round_up(pmaps.size() * sizeof(PrecondMaps), kAlign);
  std::vector<uint8_t> table(pm_off + pm_bytes + pdescs.size() * sizeof(PrecondDesc));
  if (!prep.empty()) std::memcpy(table.data(), prep.data(), prep.size() * sizeof(PrepDesc));
  if (!pmaps.empty()) std::memcpy(table.data() + pm_off, pmaps.data(), pmaps.size() * sizeof(PrecondMaps));
  if (!pdescs.empty())
    std::memcpy(table.data() + pm_off + pm_bytes, pdescs.data(), pdescs.size() * sizeof(PrecondDesc));
  void* dtab = nullptr;
  muon_status s = upload_table(ctx, table.data(), table.size(), st, &dtab);
  if (s != MUON_OK) return s;
  const PrepDesc* dprep = static_cast<const PrepDesc*>(dtab);
  const PrecondMaps* dpm = reinterpret_cast<const PrecondMaps*>(static_cast<uint8_t*>(dtab) + pm_off);
  const PrecondDesc* dpdesc = reinterpret_cast<const PrecondDesc*>(static_cast<uint8_t*>(dtab) + pm_off + pm_bytes);
  ProfScope ps(ctx, MUON_K_PRECONDITION, st);
  for (size_t b = 0; b < batch_prep.size(); ++b) {
    const int p0 = batch_prep[b];
    const int p1 = b + 1 < batch_prep.size() ? batch_prep[b + 1] : int(prep.size());
    const int q0 = batch_prob[b];
    const int q1 = b + 1 < batch_prob.size() ? batch_prob[b + 1] : int(probs.size());
    int64_t most = 0;
    for (int k = p0; k < p1; ++k) most = std::max<int64_t>(most, int64_t(prep[k].nb) * prep[k].d * prep[k].d);
    const dim3 grid(unsigned(std::max<int64_t>(1, std::min<int64_t>(cdiv(most, 256 * 8), 512))), unsigned(p1 - p0));
    launch_pdl(precond_prep_kernel, grid, dim3(256), size_t(0), st, dprep + p0);
    ctx->launches++;
    CUDA_TRY(ctx, cudaGetLastError());
    s = run_precondition(ctx, std::vector<PreProblem>(probs.begin() + q0, probs.begin() + q1), dpm, ctx->dflags,
                         st);
    if (s != MUON_OK) return s;
  }
  if (!pdescs.empty()) {
    launch_pdl(precond_kernel, dim3(unsigned(ptiles)), dim3(PRE_THREADS), size_t(0), st, dpdesc,
               int(pdescs.size()), static_cast<const int*>(ctx->dflags));
    ctx->launches++;
    CUDA_TRY(ctx, cudaGetLastError());
  }
  return MUON_OK;
}

muon_status check_hparams(muon_ctx* ctx, const muon_hparams* hp) {
  if (!hp) return fail(ctx, MUON_ERR_INVALID_ARG, "hparams is NULL");
  if (hp->ns_steps < 0 || hp->ns_steps > 100)
    return fail(ctx, MUON_ERR_INVALID_ARG, "ns_steps %d out of [0, 100]", hp->ns_steps);
  if (!(hp->momentum >= 0.f && hp->momentum < 1.f))
    return fail(ctx, MUON_ERR_INVALID_ARG, "momentum %g out of [0, 1)", hp->momentum);
  if (!(hp->eps > 0.f)) return fail(ctx, MUON_ERR_INVALID_ARG, "eps must be > 0");
  if (!std::isfinite(hp->lr) || !std::isfinite(hp->weight_decay) || !std::isfinite(hp->ns_a) ||
      !std::isfinite(hp->ns_b) || !std::isfinite(hp->ns_c))
    return fail(ctx, MUON_ERR_INVALID_ARG, "non-finite hyper-parameter");
  if (hp->scale_mode < 0 || hp->scale_mode > 2)
    return fail(ctx, MUON_ERR_INVALID_ARG, "scale_mode %d unknown", hp->scale_mode);
  return MUON_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Validate groups and flatten them into items sorted by wide shape.
muon_status collect_items(muon_ctx* ctx, const muon_group* groups, int32_t ngroups, std::vector<Item>& items,
                          bool for_step) {
  items.clear();
  if (ngroups < 0) return fail(ctx, MUON_ERR_INVALID_ARG, "ngroups < 0");
  if (ngroups > 0 && !groups) return fail(ctx, MUON_ERR_INVALID_ARG, "groups is NULL");
  for (int gi = 0; gi < ngroups; ++gi) {
    const muon_group& g = groups[gi];
    if (g.rows < 1 || g.cols < 1)
      return fail(ctx, MUON_ERR_INVALID_ARG, "group %d: shape %lldx%lld", gi, (long long)g.rows, (long long)g.cols);
    if (g.rows > (int64_t(1) << 20) || g.cols > (int64_t(1) << 20) || std::min(g.rows, g.cols) > 32768)
      return fail(ctx, MUON_ERR_UNSUPPORTED, "group %d: shape %lldx%lld beyond the supported range", gi,
                  (long long)g.rows, (long long)g.cols);
    if (g.count < 0) return fail(ctx, MUON_ERR_INVALID_ARG, "group %d: count < 0", gi);
    if (g.count == 0) continue;
    if (g.grad_dtype != MUON_F32 && g.grad_dtype != MUON_BF16)
      return fail(ctx, MUON_ERR_INVALID_ARG, "group %d: grad_dtype %d", gi, g.grad_dtype);
    if (!g.grads || (for_step && (!g.weights || !g.momentum)))
      return fail(ctx, MUON_ERR_INVALID_ARG, "group %d: NULL pointer array", gi);
    if (g.precond) {
      if (g.precond_blocks < 1 || g.cols % g.precond_blocks != 0)
        return fail(ctx, MUON_ERR_INVALID_ARG, "group %d: precond_blocks %d does not divide cols", gi,
                    g.precond_blocks);
      if (g.grad_dtype != MUON_BF16)
        return fail(ctx, MUON_ERR_UNSUPPORTED, "group %d: preconditioning needs bf16 gradients", gi);
      if ((g.cols / g.precond_blocks) % 8 != 0)
        return fail(ctx, MUON_ERR_UNSUPPORTED, "group %d: preconditioner block width must be a multiple of 8", gi);
    }
    for (int k = 0; k < g.count; ++k) {
      Item it{};
      it.rows = g.rows;
      it.cols = g.cols;
      it.transposed = g.rows > g.cols;
      it.m = std::min(g.rows, g.cols);
      it.n = std::max(g.rows, g.cols);
      it.grad_dtype = g.grad_dtype;
      it.grad = g.grads[k];
      it.weight = for_step ? g.weights[k] : nullptr;
      it.momentum = for_step ? g.momentum[k] : nullptr;
      it.update_out = g.update_out ? g.update_out[k] : nullptr;
      it.precond = g.precond ? g.precond[k] : nullptr;
      it.precond_blocks = g.precond ? g.precond_blocks : 0;
      it.precond_split = (for_step && g.precond && g.precond_split) ? g.precond_split[k] : nullptr;
      if (!it.grad || (for_step && (!it.weight || !it.momentum)) || (g.precond && !it.precond) ||
          (g.update_out && !it.update_out))
        return fail(ctx, MUON_ERR_INVALID_ARG, "group %d matrix %d: NULL tensor pointer", gi, k);
      if (!aligned16(it.grad) || (it.weight && !aligned16(it.weight)) || (it.momentum && !aligned16(it.momentum)) ||
          (it.update_out && !aligned16(it.update_out)) || (it.precond && !aligned16(it.precond)) ||
          (it.precond_split && !aligned16(it.precond_split)))
        return fail(ctx, MUON_ERR_INVALID_ARG, "group %d matrix %d: tensor not 16-byte aligned", gi, k);
      items.push_back(it);
    }
  }
  // wide shapes largest first, matrices that fit one CTA pair (their whole
  // step runs in small_ns_kernel) after all others
  std::stable_sort(items.begin(), items.end(), [](const Item& a, const Item& b) {
    const bool sa = a.n <= small_cfg::MAXD, sb = b.n <= small_cfg::MAXD;
    if (sa != sb) return sb;
    return a.m != b.m ? a.m > b.m : a.n > b.n;
  });
  return MUON_OK;
}

// The full pipeline over validated items.  mode 0: Muon step.  mode 1:
// Newton-Schulz only (grad = input, update_out = output).
muon_status run_items(muon_ctx* ctx, const std::vector<Item>& items, const muon_hparams* hp, int mode,
                      cudaStream_t st) {
  if (items.empty()) return MUON_OK;
  std::vector<Chunk> chunks;
  if (!plan_chunks(items, ws_limit(ctx), chunks))
    return fail(ctx, MUON_ERR_WORKSPACE, "one matrix needs more workspace than the %zu bytes available",
                ws_limit(ctx));
  size_t need = 0;
  for (auto& c : chunks) need = std::max(need, c.bytes);
  void* wsv = nullptr;
  muon_status s = ensure_workspace(ctx, need, &wsv);
  if (s != MUON_OK) return s;
  uint8_t* ws = static_cast<uint8_t*>(wsv);

  // Descriptor table: all chunks' MatDescs (the device copy is read by
  // kernels in stream order, so one upload per call suffices), then the
  // Newton-Muon precondition descriptors.
  std::vector<MatDesc> descs(items.size());
  std::vector<PrecondDesc> pdescs;
  std::vector<int64_t> chunk_tiles(chunks.size(), 0);
  std::vector<int> chunk_pbegin(chunks.size(), 0), chunk_pcount(chunks.size(), 0);
  std::vector<int64_t> chunk_ptiles(chunks.size(), 0);
  // tensor-core preconditioning: staging descriptors (one per distinct S^-1
  // stack of a chunk), per-matrix operand maps and batched problems
  std::vector<PrepDesc> prep;
  std::vector<PrecondMaps> pmaps;
  std::vector<int> chunk_prep_begin(chunks.size(), 0), chunk_prep_count(chunks.size(), 0);
  std::vector<std::vector<PreProblem>> chunk_pprob(chunks.size());
  // per matrix whose momentum the preconditioning product applies
  std::vector<MomDesc> momds;
  const bool check = mode == 0 && hp->check_finite;
  // the small-matrix kernel forms its matrices' X0 from the momentum itself
  const bool small_mom = mode == 0 && hp->ns_steps >= 1;
  for (size_t ci = 0; ci < chunks.size(); ++ci) {
    Chunk& c = chunks[ci];
    int64_t tiles = 0;
    size_t pg_off = c.off_pgrad;
    size_t sst_off = c.off_sst;
    int64_t fp_off = 0;                       // fused partials used so far
    std::map<StackKey, const __nv_bfloat16*> stacks;
    chunk_pbegin[ci] = int(pdescs.size());
    chunk_prep_begin[ci] = int(prep.size());
    int64_t ptiles = 0;
    for (const Run& r : c.runs) {
      for (int k = 0; k < r.count; ++k) {
        const int idx = r.first + k;
        const Item& it = items[idx];
        MatDesc& d = descs[idx];
        d.grad = it.grad;
        d.grad_dtype = it.grad_dtype;
        // in a step, the tensor-core preconditioning applies the momentum in
        // its epilogue (the small-matrix kernel forms its own)
        const bool fused = it.precond && c.tc_pre && mode == 0 && !small_run(r);
        if (it.precond && c.tc_pre) {
          float* pg = reinterpret_cast<float*>(ws + pg_off);
          const size_t pg_bytes = round_up(size_t(it.rows) * it.cols * 4, kAlign);
          pg_off += pg_bytes;
          const int dd = int(it.cols / it.precond_blocks);
          // the caller's split from the refresh, else one split per distinct
          // S^-1 of the chunk, staged in workspace
          const __nv_bfloat16* sst = static_cast<const __nv_bfloat16*>(it.precond_split);
          if (sst == nullptr) {
            const StackKey key{it.precond, it.precond_blocks, dd};
            auto f = stacks.find(key);
            if (f == stacks.end()) {
              PrepDesc pd{};
              pd.s_inv = it.precond;
              pd.sst = reinterpret_cast<__nv_bfloat16*>(ws + sst_off);
              pd.nb = it.precond_blocks;
              pd.d = dd;
              sst_off += round_up(sst_bytes(it), kAlign);
              prep.push_back(pd);
              f = stacks.emplace(key, pd.sst).first;
            }
            sst = f->second;
          }
          PrecondMaps pm{};
          if (!encode_precond_maps(&pm, it.grad, it.rows, it.cols, it.precond_blocks, dd, sst))
            return fail(ctx, MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed (precondition)");
          pmaps.push_back(pm);
          std::vector<PreProblem>& pp = chunk_pprob[ci];
          if (!pp.empty() && pp.back().rows == it.rows && pp.back().cols == it.cols &&
              pp.back().nb == it.precond_blocks && pp.back().last == idx - 1 && pp.back().fused == int(fused)) {
            pp.back().count++;
            pp.back().last = idx;
          } else {
            PreProblem q{};
            q.rows = it.rows; q.cols = it.cols; q.nb = it.precond_blocks; q.d = dd; q.count = 1; q.last = idx;
            q.pmap_base = int(pmaps.size()) - 1;
            q.pg = pg; q.pg_stride = int64_t(pg_bytes / 4);
            q.fused = fused ? 1 : 0;
            q.momd_base = int(momds.size());       // this matrix's MomDesc, pushed below
            pp.push_back(q);
          }
          d.grad = pg;
          d.grad_dtype = MUON_F32;
        } else if (it.precond) {
          float* pg = reinterpret_cast<float*>(ws + pg_off);
          pg_off += round_up(size_t(it.rows) * it.cols * 4, kAlign);
          PrecondDesc p{};
          p.grad = static_cast<const __nv_bfloat16*>(it.grad);
          p.s_inv = it.precond;
          p.out = pg;
          p.rows = it.rows;
          p.cols = it.cols;
          p.d = it.cols / it.precond_blocks;
          p.tiles_r = int(cdiv(it.rows, PRE_BM));
          p.tiles_c = int(cdiv(p.d, PRE_BN));
          p.tile_start = ptiles;
          ptiles += int64_t(p.tiles_r) * p.tiles_c * it.precond_blocks;
          pdescs.push_back(p);
          d.grad = pg;
          d.grad_dtype = MUON_F32;
        }
        d.weight = it.weight;
        d.momentum = it.momentum;
        d.update_out = it.update_out;
        d.x_in = reinterpret_cast<__nv_bfloat16*>(ws + r.off_x0) + int64_t(k) * r.m * r.ld_n;
        const int final_buf = hp->ns_steps % 2;
        d.x_out = reinterpret_cast<__nv_bfloat16*>(ws + (final_buf ? r.off_x1 : r.off_x0)) +
                  int64_t(k) * r.m * r.ld_n;
        d.norm2 = reinterpret_cast<float*>(ws + c.off_norm) + (idx - c.first);
        d.partials = reinterpret_cast<float*>(ws + c.off_partials);
        d.nparts = 0;
        d.rows = it.rows;
        d.cols = it.cols;
        d.ld = r.ld_n;
        d.tile_start = tiles;
        d.tiles_c = int(cdiv(it.cols, EW_TILE));
        d.transposed = it.transposed ? 1 : 0;
        const float scale = shape_scale(it.rows, it.cols, hp->scale_mode);
        d.lr_scale = hp->lr * scale;
        d.decay = 1.0f - hp->lr * hp->weight_decay;
        tiles += cdiv(it.rows, EW_TILE) * d.tiles_c;
        if (fused) {
          d.nparts = int32_t(fused_parts(it));
          d.partials = reinterpret_cast<float*>(ws + c.off_fparts) + fp_off;
          fp_off += d.nparts;
          MomDesc md{};
          bool ok = encode_f32_matrix(&md.mom, it.momentum, uint64_t(it.cols), uint64_t(it.rows));
          ok &= encode_bf16_3d(&md.x, d.x_in, uint64_t(r.n), uint64_t(r.m), 1, uint64_t(r.ld_n), 32, 32,
                               CU_TENSOR_MAP_SWIZZLE_64B);
          if (!ok) return fail(ctx, MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed (momentum)");
          md.partials = d.partials;
          md.transposed = it.transposed ? 1 : 0;
          momds.push_back(md);
        }
      }
    }
    chunk_tiles[ci] = tiles;
    chunk_pcount[ci] = int(pdescs.size()) - chunk_pbegin[ci];
    chunk_ptiles[ci] = ptiles;
    chunk_prep_count[ci] = int(prep.size()) - chunk_prep_begin[ci];
  }
  // The last Newton-Schulz product applies the weight step itself (no apply
  // pass, O never reaches memory) for every chunk whose matrices TMA can
  // reach as fp32 rows x cols (row pitch a multiple of 16 bytes) and that
  // asks for no update_out.  One ApplyDesc per matrix, in run order.
  std::vector<ApplyDesc> adescs;
  std::vector<std::vector<int64_t>> run_apply_idx(chunks.size());
  std::vector<char> chunk_fused(chunks.size(), 0);
  if (mode == 0 && hp->ns_steps >= 1) {
    for (size_t ci = 0; ci < chunks.size(); ++ci) {
      const Chunk& c = chunks[ci];
      bool ok = true;
      for (int i = c.first; i < c.first + c.count && ok; ++i)
        ok = items[i].update_out == nullptr && items[i].cols % 4 == 0;
      const size_t a0 = adescs.size();
      std::vector<int64_t> idx;
      for (size_t j = 0; ok && j < c.runs.size(); ++j) {
        const Run& r = c.runs[j];
        idx.push_back(int64_t(adescs.size()));
        for (int k = 0; ok && k < r.count; ++k) {
          const Item& it = items[r.first + k];
          ApplyDesc ad{};
          ok = encode_f32_matrix(&ad.w, it.weight, uint64_t(it.cols), uint64_t(it.rows));
          ad.lr_scale = hp->lr * shape_scale(it.rows, it.cols, hp->scale_mode);
          ad.decay = 1.0f - hp->lr * hp->weight_decay;
          ad.transposed = it.transposed ? 1 : 0;
          adescs.push_back(ad);
        }
      }
      if (!ok) {
        adescs.resize(a0);
        continue;
      }
      run_apply_idx[ci] = idx;
      chunk_fused[ci] = 1;
    }
  }
  const size_t mat_bytes = round_up(descs.size() * sizeof(MatDesc), kAlign);
  const size_t pd_bytes = round_up(pdescs.size() * sizeof(PrecondDesc), kAlign);
  const size_t ap_off = round_up(mat_bytes + pd_bytes + prep.size() * sizeof(PrepDesc), kAlign);
  const size_t pm_off = round_up(ap_off + adescs.size() * sizeof(ApplyDesc), kAlign);
  const size_t md_off = round_up(pm_off + pmaps.size() * sizeof(PrecondMaps), kAlign);
  std::vector<uint8_t> table(md_off + momds.size() * sizeof(MomDesc));
  std::memcpy(table.data(), descs.data(), descs.size() * sizeof(MatDesc));
  if (!pdescs.empty()) std::memcpy(table.data() + mat_bytes, pdescs.data(), pdescs.size() * sizeof(PrecondDesc));
  if (!prep.empty()) std::memcpy(table.data() + mat_bytes + pd_bytes, prep.data(), prep.size() * sizeof(PrepDesc));
  if (!adescs.empty()) std::memcpy(table.data() + ap_off, adescs.data(), adescs.size() * sizeof(ApplyDesc));
  if (!pmaps.empty()) std::memcpy(table.data() + pm_off, pmaps.data(), pmaps.size() * sizeof(PrecondMaps));
  if (!momds.empty()) std::memcpy(table.data() + md_off, momds.data(), momds.size() * sizeof(MomDesc));
  void* dtab = nullptr;
  s = upload_table(ctx, table.data(), table.size(), st, &dtab);
  if (s != MUON_OK) return s;
  const MatDesc* ddesc = static_cast<const MatDesc*>(dtab);
  const PrecondDesc* dpdesc = reinterpret_cast<const PrecondDesc*>(static_cast<uint8_t*>(dtab) + mat_bytes);
  const PrepDesc* dprep = reinterpret_cast<const PrepDesc*>(static_cast<uint8_t*>(dtab) + mat_bytes + pd_bytes);

  // Every kernel of the step gets the context's flags and does nothing once
  // an error bit (an earlier bounded wait that gave up, a second moment that
  // was not positive definite) or this step's non-finite flag is set.
  const int* skip = ctx->dflags;
  if (check) {
    CUDA_TRY(ctx, cudaMemsetAsync(ctx->dflags + 1, 0, sizeof(int), st));
    int64_t tiles = 0;
    for (size_t i = 0; i < items.size(); ++i) tiles += cdiv(items[i].rows, EW_TILE) * cdiv(items[i].cols, EW_TILE);
    // finite_kernel reads the caller's gradients: give it a table with those
    std::vector<MatDesc> raw(descs);
    int64_t t = 0;
    for (size_t i = 0; i < items.size(); ++i) {
      raw[i].grad = items[i].grad;
      raw[i].grad_dtype = items[i].grad_dtype;
      raw[i].tile_start = t;
      t += cdiv(items[i].rows, EW_TILE) * cdiv(items[i].cols, EW_TILE);
    }
    // second table region after the main one
    const size_t off = round_up(table.size(), kAlign);
    std::vector<uint8_t> both(off + raw.size() * sizeof(MatDesc));
    std::memcpy(both.data(), table.data(), table.size());
    std::memcpy(both.data() + off, raw.data(), raw.size() * sizeof(MatDesc));
    s = upload_table(ctx, both.data(), both.size(), st, &dtab);
    if (s != MUON_OK) return s;
    ddesc = static_cast<const MatDesc*>(dtab);
    dpdesc = reinterpret_cast<const PrecondDesc*>(static_cast<uint8_t*>(dtab) + mat_bytes);
    dprep = reinterpret_cast<const PrepDesc*>(static_cast<uint8_t*>(dtab) + mat_bytes + pd_bytes);
    const MatDesc* draw = reinterpret_cast<const MatDesc*>(static_cast<uint8_t*>(dtab) + off);
    {
      ProfScope ps(ctx, MUON_K_OTHER, st);
      for (const SegLaunch& L : build_seg_launches(raw.data(), int(raw.size()))) {
      launch_pdl(finite_kernel, dim3(unsigned(L.tiles)), dim3(EW_THREADS), size_t(0), st,
                 draw, L.t, ctx->dflags + 1);
      ctx->launches++;
    }
    }
    CUDA_TRY(ctx, cudaGetLastError());
  }

  for (size_t ci = 0; ci < chunks.size(); ++ci) {
    const Chunk& c = chunks[ci];
    float* norm2 = reinterpret_cast<float*>(ws + c.off_norm);
    if (!chunk_pprob[ci].empty()) {
      ProfScope ps(ctx, MUON_K_PRECONDITION, st);
      // split each distinct S^-1 the caller gave no split for
      if (chunk_prep_count[ci] > 0) {
        int64_t most = 0;
        for (int k = 0; k < chunk_prep_count[ci]; ++k) {
          const PrepDesc& pd = prep[chunk_prep_begin[ci] + k];
          most = std::max<int64_t>(most, int64_t(pd.nb) * pd.d * pd.d);
        }
        const dim3 grid(unsigned(std::max<int64_t>(1, std::min<int64_t>(cdiv(most, 256 * 8), 512))),
                        unsigned(chunk_prep_count[ci]));
        launch_pdl(precond_prep_kernel, grid, dim3(256), size_t(0), st, dprep + chunk_prep_begin[ci]);
        ctx->launches++;
        CUDA_TRY(ctx, cudaGetLastError());
      }
      s = run_precondition(ctx, chunk_pprob[ci],
                           reinterpret_cast<const PrecondMaps*>(static_cast<uint8_t*>(dtab) + pm_off), skip, st,
                           reinterpret_cast<const MomDesc*>(static_cast<uint8_t*>(dtab) + md_off), hp->momentum,
                           hp->nesterov);
      if (s != MUON_OK) return s;
    }
    if (chunk_pcount[ci] > 0) {
      ProfScope ps(ctx, MUON_K_PRECONDITION, st);
      launch_pdl(precond_kernel, dim3(unsigned(chunk_ptiles[ci])), dim3(PRE_THREADS), size_t(0), st,
          dpdesc + chunk_pbegin[ci], chunk_pcount[ci], skip);
      ctx->launches++;
      CUDA_TRY(ctx, cudaGetLastError());
    }
    const std::vector<SegLaunch> segl = build_seg_launches(descs.data() + c.first, c.count);
    // In a step with at least one iteration the small-matrix kernel runs the
    // momentum of its own matrices (they sort last in the chunk), so the
    // momentum launches cover only the items before them.
    int n_mom = c.count;
    if (small_mom)
      for (const Run& r : c.runs)
        if (small_run(r)) n_mom = std::min(n_mom, r.first - c.first);
    if (n_mom > 0) {
      // matrices whose momentum the preconditioning product applied are
      // skipped by the momentum kernel; when that is all of them, it is not
      // launched and only their norms are reduced
      bool all_fused = true;
      for (int i = c.first; i < c.first + n_mom && all_fused; ++i) all_fused = descs[i].nparts > 0;
      ProfScope ps(ctx, MUON_K_MOMENTUM, st);
      if (!all_fused) {
        const std::vector<SegLaunch> segm = build_seg_launches(descs.data() + c.first, n_mom);
        for (const SegLaunch& L : segm) {
          if (mode == 0)
            launch_pdl(momentum_kernel<0>, dim3(unsigned(L.tiles)), dim3(MOM_THREADS), size_t(0), st,
                ddesc + c.first, L.t, L.tile_base, hp->momentum, hp->nesterov, skip);
          else
            launch_pdl(momentum_kernel<1>, dim3(unsigned(L.tiles)), dim3(MOM_THREADS), size_t(0), st,
                ddesc + c.first, L.t, L.tile_base, 0.f, 0, skip);
        }
        ctx->launches += segm.size();
      }
      launch_pdl(norm_reduce_kernel, dim3(unsigned(n_mom)), dim3(EW_THREADS), size_t(0), st, ddesc + c.first, skip);
      ctx->launches += 1;
    }
    CUDA_TRY(ctx, cudaGetLastError());
    {
      std::vector<const float*> n2(c.runs.size());
      for (size_t j = 0; j < c.runs.size(); ++j) n2[j] = norm2 + (c.runs[j].first - c.first);
      std::vector<const ApplyDesc*> ra;
      std::vector<const MatDesc*> rm;
      for (const Run& r : c.runs) rm.push_back(ddesc + r.first);
      if (chunk_fused[ci]) {
        const ApplyDesc* dapply = reinterpret_cast<const ApplyDesc*>(static_cast<uint8_t*>(dtab) + ap_off);
        for (int64_t k : run_apply_idx[ci]) ra.push_back(dapply + k);
      }
      s = run_newton_schulz(ctx, ws, c.runs.data(), int(c.runs.size()), n2.data(), hp, skip, st,
                            chunk_fused[ci] ? ra.data() : nullptr, rm.data(), small_mom);
      if (s != MUON_OK) return s;
    }
    if (!chunk_fused[ci]) {
      ProfScope ps(ctx, MUON_K_APPLY, st);
      for (const SegLaunch& L : segl) {
        if (mode == 0)
          launch_pdl(apply_kernel<0>, dim3(unsigned(L.tiles)), dim3(EW_THREADS), size_t(0), st,
              ddesc + c.first, L.t, hp->ns_steps == 0, hp->eps, skip);
        else
          launch_pdl(apply_kernel<1>, dim3(unsigned(L.tiles)), dim3(EW_THREADS), size_t(0), st,
              ddesc + c.first, L.t, hp->ns_steps == 0, hp->eps, skip);
      }
      ctx->launches += segl.size();
    }
    CUDA_TRY(ctx, cudaGetLastError());
  }

  if (check) {
    int flag = 0;
    CUDA_TRY(ctx, cudaMemcpyAsync(&flag, ctx->dflags + 1, sizeof(int), cudaMemcpyDeviceToHost, st));
    CUDA_TRY(ctx, cudaStreamSynchronize(st));
    if (flag) {
      // the flag only halts this step's kernels: clear it for the next call
      CUDA_TRY(ctx, cudaMemsetAsync(ctx->dflags + 1, 0, sizeof(int), st));
      CUDA_TRY(ctx, cudaStreamSynchronize(st));
      return fail(ctx, MUON_ERR_NONFINITE, "a gradient holds NaN or Inf; nothing was updated");
    }
  }
  return MUON_OK;
}

// ---------------------------------------------------------------------------
// Scratch for muon_orthogonalize_noalloc: a fixed device array that is part of
// the module, so that entry point never asks the CUDA allocator for memory.
// Every GPU that loads this library holds these bytes until the process exits.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;   // 32 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on `device`.  In host code the array's
// name only stands for the symbol; the usable address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
muon_status noalloc_scratch_address(int device, uint8_t** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  if (device < 0 || device >= 64) return MUON_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[device] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MUON_ERR_CUDA;
    addr[device] = p;
  }
  *out = static_cast<uint8_t*>(addr[device]);
  return MUON_OK;
}

}  // namespace

// ===========================================================================
// extern "C"
// ===========================================================================
// Failure detection without a fault: one thread waits on an mbarrier that
// nothing completes.  The bounded wait gives up after its limit (2 s of
// %globaltimer), records kDevErrTimeout in the context's flags and the
// kernel returns, leaving the context usable.
__global__ void selftest_wait_kernel(int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, err, &abort_flag);
}

// muon_orthogonalize_noalloc set-up: the matrix descriptor arrives as a
// kernel parameter and is stored where the kernels read it; the flags of the
// previous call are cleared.
__global__ void noalloc_setup_kernel(const __grid_constant__ MatDesc d, MatDesc* dst, int* flags) {
  if (threadIdx.x == 0) *dst = d;
  if (threadIdx.x < 4) flags[threadIdx.x] = 0;
}

// muon_orthogonalize_noalloc epilogue: when a bounded wait gave up during the
// call (flags[0] set), the output is filled with NaN, so a caller that cannot
// query the library's flags still sees that the result is not valid.
__global__ void noalloc_poison_kernel(const int* flags, float* out, int64_t n) {
  if (flags[0] == 0) return;
  const float nan = __int_as_float(0x7fffffff);
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
    out[i] = nan;
}

extern "C" {

void muon_default_hparams(muon_hparams* hp) {
  if (!hp) return;
  hp->lr = 0.02f;
  hp->momentum = 0.95f;
  hp->weight_decay = 0.01f;
  hp->eps = 1e-7f;
  hp->ns_a = 3.4445f;
  hp->ns_b = -4.7750f;
  hp->ns_c = 2.0315f;
  hp->nesterov = 1;
  hp->ns_steps = 5;
  hp->scale_mode = MUON_SCALE_ORIGINAL;
  hp->check_finite = 0;
}

void muon_default_adamw_hparams(muon_adamw_hparams* hp) {
  if (!hp) return;
  hp->lr = 3e-4f;
  hp->beta1 = 0.9f;
  hp->beta2 = 0.95f;
  hp->eps = 1e-8f;
  hp->weight_decay = 0.01f;
}

const char* muon_status_string(muon_status s) {
  switch (s) {
    case MUON_OK: return "MUON_OK";
    case MUON_ERR_INVALID_ARG: return "MUON_ERR_INVALID_ARG";
    case MUON_ERR_UNSUPPORTED: return "MUON_ERR_UNSUPPORTED";
    case MUON_ERR_WORKSPACE: return "MUON_ERR_WORKSPACE";
    case MUON_ERR_CUDA: return "MUON_ERR_CUDA";
    case MUON_ERR_NONFINITE: return "MUON_ERR_NONFINITE";
    case MUON_ERR_TIMEOUT: return "MUON_ERR_TIMEOUT";
  }
  return "unknown muon_status";
}

muon_status muon_init(muon_ctx** out, int device, size_t workspace_bytes) {
  if (!out) return MUON_ERR_INVALID_ARG;
  *out = nullptr;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) return MUON_ERR_INVALID_ARG;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return MUON_ERR_CUDA;
  if (prop.major != 10 || prop.minor != 0) return MUON_ERR_UNSUPPORTED;   // built for sm_100a only
  if (encode_fn() == nullptr) return MUON_ERR_CUDA;
  muon_ctx* ctx = new muon_ctx();
  ctx->device = device;
  ctx->ws_cap = workspace_bytes;
  auto bail = [&](muon_status s) { muon_destroy(ctx); return s; };
  if (cudaSetDevice(device) != cudaSuccess) return bail(MUON_ERR_CUDA);
  if (cudaMalloc(&ctx->dflags, 16 * sizeof(int)) != cudaSuccess) return bail(MUON_ERR_CUDA);
  if (cudaMemset(ctx->dflags, 0, 16 * sizeof(int)) != cudaSuccess) return bail(MUON_ERR_CUDA);
  for (int k = 0; k < 2; ++k)
    if (cudaEventCreateWithFlags(&ctx->hevent[k], cudaEventDisableTiming) != cudaSuccess) return bail(MUON_ERR_CUDA);
  if (workspace_bytes != 0) {
    if (cudaMalloc(&ctx->ws_own, workspace_bytes) != cudaSuccess) return bail(MUON_ERR_CUDA);
    ctx->ws_own_bytes = workspace_bytes;
  }
  *out = ctx;
  return MUON_OK;
}

void muon_destroy(muon_ctx* ctx) {
  if (!ctx) return;
  cudaSetDevice(ctx->device);
  cudaDeviceSynchronize();
  if (ctx->ws_own) cudaFree(ctx->ws_own);
  if (ctx->dtable) cudaFree(ctx->dtable);
  for (int k = 0; k < 2; ++k) {
    if (ctx->htable[k]) cudaFreeHost(ctx->htable[k]);
    if (ctx->hevent[k]) cudaEventDestroy(ctx->hevent[k]);
  }
  if (ctx->dflags) cudaFree(ctx->dflags);
  for (int k = 0; k < MUON_K_COUNT; ++k)
    for (auto& pr : ctx->prof_pending[k]) {
      cudaEventDestroy(pr.first);
      cudaEventDestroy(pr.second);
    }
  for (auto e : ctx->prof_pool) cudaEventDestroy(e);
  delete ctx;
}

const char* muon_last_error(const muon_ctx* ctx) { return ctx ? ctx->err.c_str() : "NULL context"; }

muon_status muon_query_workspace(const muon_group* groups, int32_t ngroups, size_t* bytes) {
  if (!bytes) return MUON_ERR_INVALID_ARG;
  std::vector<Item> items;
  muon_status s = collect_items(nullptr, groups, ngroups, items, false);
  if (s != MUON_OK) return s;
  std::vector<Chunk> chunks;
  plan_chunks(items, 0, chunks);
  *bytes = chunks.empty() ? 0 : chunks[0].bytes;
  return MUON_OK;
}

muon_status muon_set_workspace(muon_ctx* ctx, void* ptr, size_t bytes) {
  if (!ctx) return MUON_ERR_INVALID_ARG;
  if (ptr && (reinterpret_cast<uintptr_t>(ptr) & 255))
    return fail(ctx, MUON_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  ctx->ws_user = ptr;
  ctx->ws_user_bytes = ptr ? bytes : 0;
  return MUON_OK;
}

muon_status muon_step(muon_ctx* ctx, const muon_group* groups, int32_t ngroups, const muon_hparams* hp,
                      void* stream) {
  if (!ctx) return MUON_ERR_INVALID_ARG;
  muon_status s = check_hparams(ctx, hp);
  if (s != MUON_OK) return s;
  std::vector<Item> items;
  s = collect_items(ctx, groups, ngroups, items, true);
  if (s != MUON_OK) return s;
  s = set_device(ctx);
  if (s != MUON_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ctx->last_stream = st;
  CUDA_TRY(ctx, cudaGetLastError());
  return run_items(ctx, items, hp, 0, st);
}

muon_status muon_orthogonalize(muon_ctx* ctx, const muon_ns_group* groups, int32_t ngroups,
                               const muon_hparams* hp, void* stream) {
  if (!ctx) return MUON_ERR_INVALID_ARG;
  muon_status s = check_hparams(ctx, hp);
  if (s != MUON_OK) return s;
  if (ngroups < 0 || (ngroups > 0 && !groups)) return fail(ctx, MUON_ERR_INVALID_ARG, "bad groups");
  std::vector<muon_group> gs(ngroups);
  for (int i = 0; i < ngroups; ++i) {
    gs[i] = muon_group{};
    gs[i].rows = groups[i].rows;
    gs[i].cols = groups[i].cols;
    gs[i].count = groups[i].count;
    gs[i].grad_dtype = groups[i].in_dtype;
    gs[i].grads = groups[i].inputs;
    gs[i].update_out = groups[i].outputs;
    if (groups[i].count > 0 && !groups[i].outputs)
      return fail(ctx, MUON_ERR_INVALID_ARG, "group %d: outputs is NULL", i);
  }
  std::vector<Item> items;
  s = collect_items(ctx, gs.data(), ngroups, items, false);
  if (s != MUON_OK) return s;
  s = set_device(ctx);
  if (s != MUON_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ctx->last_stream = st;
  CUDA_TRY(ctx, cudaGetLastError());
  return run_items(ctx, items, hp, 1, st);
}

muon_status muon_newton_precondition(muon_ctx* ctx, const muon_group* groups, int32_t ngroups, void* stream) {
  if (!ctx) return MUON_ERR_INVALID_ARG;
  if (ngroups < 0 || (ngroups > 0 && !groups)) return fail(ctx, MUON_ERR_INVALID_ARG, "bad groups");
  for (int i = 0; i < ngroups; ++i) {
    if (groups[i].count <= 0) continue;
    if (!groups[i].precond) return fail(ctx, MUON_ERR_INVALID_ARG, "group %d: precond is NULL", i);
    if (!groups[i].update_out) return fail(ctx, MUON_ERR_INVALID_ARG, "group %d: update_out is NULL", i);
  }
  std::vector<Item> items;
  muon_status s = collect_items(ctx, groups, ngroups, items, false);
  if (s != MUON_OK) return s;
  s = set_device(ctx);
  if (s != MUON_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ctx->last_stream = st;
  CUDA_TRY(ctx, cudaGetLastError());
  return run_precondition_items(ctx, items, st);
}

muon_status muon_adamw_step(muon_ctx* ctx, const muon_adamw_tensor* tensors, int32_t n,
                            const muon_adamw_hparams* hp, int64_t step, void* stream) {
  if (!ctx) return MUON_ERR_INVALID_ARG;
  if (!hp) return fail(ctx, MUON_ERR_INVALID_ARG, "hparams is NULL");
  if (n < 0 || (n > 0 && !tensors)) return fail(ctx, MUON_ERR_INVALID_ARG, "bad tensor list");
  if (step < 1) return fail(ctx, MUON_ERR_INVALID_ARG, "step counts from 1");
  if (!(hp->beta1 >= 0.f && hp->beta1 < 1.f && hp->beta2 >= 0.f && hp->beta2 < 1.f && hp->eps > 0.f))
    return fail(ctx, MUON_ERR_INVALID_ARG, "betas must lie in [0,1), eps > 0");
  std::vector<AdamDesc> descs;
  int64_t chunks = 0;
  for (int i = 0; i < n; ++i) {
    const muon_adamw_tensor& t = tensors[i];
    if (t.numel < 0) return fail(ctx, MUON_ERR_INVALID_ARG, "tensor %d: numel < 0", i);
    if (t.numel == 0) continue;
    if (!t.param || !t.grad || !t.exp_avg || !t.exp_avg_sq)
      return fail(ctx, MUON_ERR_INVALID_ARG, "tensor %d: NULL pointer", i);
    if (t.grad_dtype != MUON_F32 && t.grad_dtype != MUON_BF16)
      return fail(ctx, MUON_ERR_INVALID_ARG, "tensor %d: grad_dtype %d", i, t.grad_dtype);
    AdamDesc d{};
    d.param = t.param;
    d.grad = t.grad;
    d.m = t.exp_avg;
    d.v = t.exp_avg_sq;
    d.numel = t.numel;
    d.grad_dtype = t.grad_dtype;
    d.chunk_start = chunks;
    chunks += cdiv(t.numel, ADAM_CHUNK);
    descs.push_back(d);
  }
  if (descs.empty()) return MUON_OK;
  muon_status s = set_device(ctx);
  if (s != MUON_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ctx->last_stream = st;
  CUDA_TRY(ctx, cudaGetLastError());
  void* dtab = nullptr;
  s = upload_table(ctx, descs.data(), descs.size() * sizeof(AdamDesc), st, &dtab);
  if (s != MUON_OK) return s;
  AdamScalars sc;
  sc.lr = hp->lr;
  sc.beta1 = hp->beta1;
  sc.beta2 = hp->beta2;
  sc.eps = hp->eps;
  sc.decay = 1.0f - hp->lr * hp->weight_decay;
  sc.bc1 = float(1.0 - std::pow(double(hp->beta1), double(step)));
  sc.bc2_sqrt = float(std::sqrt(1.0 - std::pow(double(hp->beta2), double(step))));
  {
    ProfScope ps(ctx, MUON_K_ADAMW, st);
    launch_pdl(adamw_kernel, dim3(unsigned(chunks)), dim3(EW_THREADS), size_t(0), st,
        static_cast<const AdamDesc*>(dtab), int(descs.size()), sc, static_cast<const int*>(ctx->dflags));
  }
  ctx->launches++;
  CUDA_TRY(ctx, cudaGetLastError());
  return MUON_OK;
}

muon_status muon_newton_refresh(muon_ctx* ctx, const muon_act_desc* acts, int32_t n, float damping,
                                void* stream) {
  if (!ctx) return MUON_ERR_INVALID_ARG;
  if (n < 0 || (n > 0 && !acts)) return fail(ctx, MUON_ERR_INVALID_ARG, "bad activation list");
  if (!(damping >= 0.f) || !std::isfinite(damping)) return fail(ctx, MUON_ERR_INVALID_ARG, "damping must be >= 0");
  // Per d-wide activation block: the fp32 second moment S (then its
  // Cholesky factor) and the output S^-1.  When every bf16 activation's
  // width and block width is a multiple of 8 elements (16 bytes, the TMA
  // coordinate granule) the second-moment product reads the bf16
  // activations in place; otherwise each bf16 block is first copied
  // transposed (d x tokens bf16).  An fp32 activation block is split into
  // bf16 high and low parts, laid out as the two operands of one product
  // over 3 x tokens (act_split_kernel).
  struct GramProb {
    int64_t tokens, d, ldt;
    int count, nb, pmap_base;
    int mode;                  // 0: transposed bf16 copy, 1: bf16 in place, 2: split fp32
    size_t xt_off, xb_off, s_off;
    int64_t s_stride;          // floats between consecutive blocks' S
  };
  bool direct = true;
  for (int i = 0; i < n; ++i)
    if (acts[i].act_dtype == MUON_BF16)
      direct = direct && acts[i].nblocks >= 1 && acts[i].width % 8 == 0 && (acts[i].width / acts[i].nblocks) % 8 == 0;
  std::vector<ActBlock> ab;
  std::vector<ActSplitBlock> sbk;
  std::vector<CholDesc> cd;
  std::vector<GramProb> gp;
  size_t s_total = 0, xt_total = 0;
  int max_d = 0;
  int64_t max_tiles = 0, max_split_tiles = 0;
  std::vector<PrepDesc> splits;     // S^-1 to split into the caller's hi/lo stacks
  // activations of one (dtype, tokens, d, nblocks) next to each other, so
  // each shape is one batched problem of the second-moment product
  std::vector<int> order(n);
  for (int i = 0; i < n; ++i) order[i] = i;
  auto key = [&](int i) {
    const int64_t nb = acts[i].nblocks >= 1 ? acts[i].nblocks : 1;
    return std::make_tuple(acts[i].act_dtype, acts[i].tokens, acts[i].width / nb, acts[i].nblocks);
  };
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return key(x) < key(y); });
  for (int oi = 0; oi < n; ++oi) {
    const int i = order[oi];
    const muon_act_desc& a = acts[i];
    if (!a.acts || !a.s_inv) return fail(ctx, MUON_ERR_INVALID_ARG, "activation %d: NULL pointer", i);
    if (a.act_dtype != MUON_BF16 && a.act_dtype != MUON_F32)
      return fail(ctx, MUON_ERR_INVALID_ARG, "activation %d: act_dtype %d", i, a.act_dtype);
    if (a.tokens < 1 || a.width < 1 || a.nblocks < 1 || a.width % a.nblocks != 0)
      return fail(ctx, MUON_ERR_INVALID_ARG, "activation %d: bad shape", i);
    const int64_t d = a.width / a.nblocks;
    if (d > CHOL_MAX_D)
      return fail(ctx, MUON_ERR_UNSUPPORTED, "activation %d: block width %lld > %d", i, (long long)d, CHOL_MAX_D);
    if (!aligned16(a.acts) || !aligned16(a.s_inv) || (a.s_inv_split && !aligned16(a.s_inv_split)))
      return fail(ctx, MUON_ERR_INVALID_ARG, "activation %d: not 16-byte aligned", i);
    if (a.s_inv_split) {
      PrepDesc pd{};
      pd.s_inv = a.s_inv;
      pd.sst = static_cast<__nv_bfloat16*>(a.s_inv_split);
      pd.nb = a.nblocks;
      pd.d = int(d);
      splits.push_back(pd);
    }
    const bool split = a.act_dtype == MUON_F32;
    if (split && 3 * a.tokens > INT32_MAX)
      return fail(ctx, MUON_ERR_UNSUPPORTED, "activation %d: too many tokens", i);
    const int mode = split ? 2 : direct ? 1 : 0;
    // K extent of the operands: tokens, or three segments of tokens (split)
    const int64_t ldt = round_up(split ? 3 * a.tokens : a.tokens, 8);
    // each block's S starts 256-byte aligned, whatever d is (the Cholesky
    // kernels take 16-byte vector paths when d is a multiple of 4)
    const size_t s_bytes = round_up(size_t(d) * d * 4, kAlign);
    const size_t op_bytes = round_up(size_t(d) * ldt * 2, kAlign);
    for (int b = 0; b < a.nblocks; ++b) {
      size_t xa_off = xt_total, xb_off = xt_total;
      if (split) {
        ActSplitBlock x{};
        x.acts = static_cast<const float*>(a.acts);
        xb_off = xt_total + op_bytes;
        x.xa = reinterpret_cast<__nv_bfloat16*>(xa_off);   // offsets, rebased below
        x.xb = reinterpret_cast<__nv_bfloat16*>(xb_off);
        x.tokens = a.tokens;
        x.width = a.width;
        x.col0 = b * d;
        x.d = d;
        x.ld3 = ldt;
        sbk.push_back(x);
        xt_total += 2 * op_bytes;
        max_split_tiles = std::max<int64_t>(max_split_tiles, cdiv(a.tokens, TPOSE_T) * cdiv(d, TPOSE_T));
      } else if (!direct) {
        ActBlock x{};
        x.acts = static_cast<const __nv_bfloat16*>(a.acts);
        x.xt = reinterpret_cast<__nv_bfloat16*>(xa_off);    // offset, rebased below
        x.tokens = a.tokens;
        x.width = a.width;
        x.col0 = b * d;
        x.d = d;
        x.ldt = ldt;
        ab.push_back(x);
        xt_total += op_bytes;
        max_tiles = std::max<int64_t>(max_tiles, cdiv(a.tokens, TPOSE_T) * cdiv(d, TPOSE_T));
      }
      CholDesc c{};
      c.a = reinterpret_cast<float*>(s_total);               // offset, rebased below
      c.inv = a.s_inv + size_t(b) * d * d;
      c.d = int(d);
      cd.push_back(c);
      // consecutive blocks of one problem sit op_bytes (or 2 op_bytes) apart
      // in the operand region and s_bytes apart in the S region
      if (!gp.empty() && gp.back().mode == mode && gp.back().tokens == a.tokens && gp.back().d == d &&
          (mode != 1 || gp.back().nb == a.nblocks)) {
        gp.back().count++;
      } else {
        gp.push_back(GramProb{a.tokens, d, ldt, 1, a.nblocks, oi, mode, xa_off, xb_off, s_total,
                              int64_t(s_bytes / 4)});
      }
      s_total += s_bytes;
      max_d = std::max(max_d, int(d));
    }
  }
  if (cd.empty()) return MUON_OK;
  if (cd.size() > 65535) return fail(ctx, MUON_ERR_UNSUPPORTED, "more than 65535 activation blocks");
  muon_status s = set_device(ctx);
  if (s != MUON_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ctx->last_stream = st;
  CUDA_TRY(ctx, cudaGetLastError());
  const size_t s_region = round_up(s_total, kAlign);
  void* wsv = nullptr;
  // S / L per block, then the recursive L^-1's T per block (same layout),
  // then the transposed or split activation copies
  s = ensure_workspace(ctx, 2 * s_region + xt_total, &wsv);
  if (s != MUON_OK) return s;
  uint8_t* ws = static_cast<uint8_t*>(wsv);
  uint8_t* xt_base = ws + 2 * s_region;
  for (auto& x : ab) x.xt = reinterpret_cast<__nv_bfloat16*>(xt_base + reinterpret_cast<size_t>(x.xt));
  for (auto& x : sbk) {
    x.xa = reinterpret_cast<__nv_bfloat16*>(xt_base + reinterpret_cast<size_t>(x.xa));
    x.xb = reinterpret_cast<__nv_bfloat16*>(xt_base + reinterpret_cast<size_t>(x.xb));
  }
  for (auto& c : cd) {
    c.t = reinterpret_cast<float*>(ws + s_region + reinterpret_cast<size_t>(c.a));
    c.a = reinterpret_cast<float*>(ws + reinterpret_cast<size_t>(c.a));
  }
  // in place: one map per bf16 activation over its whole tokens x width
  // matrix, in the sorted order (fp32 activations leave their slot unused)
  std::vector<PrecondMaps> pmaps(direct ? n : 0);
  for (int oi = 0; direct && oi < n; ++oi) {
    const muon_act_desc& a = acts[order[oi]];
    if (a.act_dtype != MUON_BF16) continue;
    if (!encode_bf16_3d(&pmaps[oi].a, a.acts, a.width, a.tokens, 1, a.width, 64, 64))
      return fail(ctx, MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed (second moment)");
  }
  const size_t ab_bytes = round_up(ab.size() * sizeof(ActBlock), kAlign);
  const size_t sb_off = round_up(ab_bytes + cd.size() * sizeof(CholDesc), kAlign);
  const size_t pm_off = round_up(sb_off + sbk.size() * sizeof(ActSplitBlock), kAlign);
  const size_t sp_off = round_up(pm_off + pmaps.size() * sizeof(PrecondMaps), kAlign);
  std::vector<uint8_t> table(sp_off + splits.size() * sizeof(PrepDesc));
  if (!ab.empty()) std::memcpy(table.data(), ab.data(), ab.size() * sizeof(ActBlock));
  std::memcpy(table.data() + ab_bytes, cd.data(), cd.size() * sizeof(CholDesc));
  if (!sbk.empty()) std::memcpy(table.data() + sb_off, sbk.data(), sbk.size() * sizeof(ActSplitBlock));
  if (!pmaps.empty()) std::memcpy(table.data() + pm_off, pmaps.data(), pmaps.size() * sizeof(PrecondMaps));
  if (!splits.empty()) std::memcpy(table.data() + sp_off, splits.data(), splits.size() * sizeof(PrepDesc));
  void* dtab = nullptr;
  s = upload_table(ctx, table.data(), table.size(), st, &dtab);
  if (s != MUON_OK) return s;
  const ActBlock* dab = static_cast<const ActBlock*>(dtab);
  const CholDesc* dc = reinterpret_cast<const CholDesc*>(static_cast<uint8_t*>(dtab) + ab_bytes);
  const ActSplitBlock* dsb = reinterpret_cast<const ActSplitBlock*>(static_cast<uint8_t*>(dtab) + sb_off);
  // after S^-1 is written: the hi/lo splits the caller asked for
  auto emit_splits = [&]() -> muon_status {
    if (splits.empty()) return MUON_OK;
    int64_t most = 0;
    for (const PrepDesc& pd : splits) most = std::max<int64_t>(most, int64_t(pd.nb) * pd.d * pd.d);
    const dim3 grid(unsigned(std::max<int64_t>(1, std::min<int64_t>(cdiv(most, 256 * 8), 512))),
                    unsigned(splits.size()));
    launch_pdl(precond_prep_kernel, grid, dim3(256), size_t(0), st,
               reinterpret_cast<const PrepDesc*>(static_cast<uint8_t*>(dtab) + sp_off));
    ctx->launches++;
    CUDA_TRY(ctx, cudaGetLastError());
    return MUON_OK;
  };
  ProfScope ps(ctx, MUON_K_NEWTON_REFRESH, st);
  if (!ab.empty()) {
    launch_pdl(act_transpose_kernel, dim3(unsigned(max_tiles), unsigned(ab.size())), dim3(256), size_t(0), st, dab);
    ctx->launches++;
    CUDA_TRY(ctx, cudaGetLastError());
  }
  if (!sbk.empty()) {
    launch_pdl(act_split_kernel, dim3(unsigned(max_split_tiles), unsigned(sbk.size())), dim3(256), size_t(0), st,
               dsb);
    ctx->launches++;
    CUDA_TRY(ctx, cudaGetLastError());
  }
  // S = Xt Xt^T / tokens on the tensor cores, up to MAX_PROBLEMS problems
  // of one operand mode per launch
  for (size_t b0 = 0; b0 < gp.size();) {
    const int mode = gp[b0].mode;
    int nb = 0;
    while (nb < MAX_PROBLEMS && b0 + nb < gp.size() && gp[b0 + nb].mode == mode) ++nb;
    GemmMaps maps{};
    GemmArgs g{};
    g.nprob = nb;
    g.err = ctx->dflags;
    g.ab_distinct = mode == 2;
    if (mode == 1) g.pmaps = reinterpret_cast<const PrecondMaps*>(static_cast<uint8_t*>(dtab) + pm_off);
    int tile = 0;
    for (int j = 0; j < nb; ++j) {
      const GramProb& q = gp[b0 + j];
      const int64_t kx = mode == 2 ? 3 * q.tokens : q.tokens;   // K extent
      if (mode != 1) {
        // consecutive blocks of the problem: one (or, split, two) operand
        // copies apart
        const uint64_t zstride = (mode == 2 ? 2 : 1) * round_up(size_t(q.d) * q.ldt * 2, kAlign) / 2;
        bool ok = encode_bf16_3d_strided(&maps.a[j], xt_base + q.xt_off, kx, q.d, q.count, q.ldt, zstride, 64, 128);
        if (mode == 2)
          ok &= encode_bf16_3d_strided(&maps.b[j], xt_base + q.xb_off, kx, q.d, q.count, q.ldt, zstride, 64, 128);
        else
          maps.b[j] = maps.a[j];
        if (!ok) return fail(ctx, MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed (second moment)");
        maps.aux[j] = maps.a[j];
        maps.out[j] = maps.a[j];
      }
      GemmProblem& P = g.p[j];
      P.M = int(q.d); P.N = int(q.d); P.K = int(kx);
      P.batch = q.count;
      P.tiles_m = P.tiles_n = int(cdiv(q.d, gemm_cfg::TM));
      P.tiles_per_mat = gemm_tiles_per_mat(EPI_GRAM32, P.tiles_m, P.tiles_n);
      P.tile_start = tile;
      P.out32 = reinterpret_cast<float*>(ws + q.s_off);
      P.out32_ld = q.d;
      P.out32_bs = q.s_stride;
      P.nblocks = mode == 1 ? q.nb : 1;
      P.pmap_base = q.pmap_base;
      P.scale = 1.0f / float(q.tokens);
      const int64_t tt = int64_t(tile) + int64_t(P.batch) * P.tiles_per_mat;
      if (tt > INT32_MAX) return fail(ctx, MUON_ERR_UNSUPPORTED, "too many tiles in one launch");
      tile = int(tt);
    }
    g.total = tile;
    if (mode == 1) CUDA_TRY(ctx, (launch_gemm<EPI_GRAM32, true>(ctx, maps, g, st)));
    else CUDA_TRY(ctx, (launch_gemm<EPI_GRAM32, false>(ctx, maps, g, st)));
    b0 += nb;
  }
  if (max_d <= CHOL_BLOCKED_MAX_D) {
    // blocked factorisation, panels of 32: panel, then trailing update
    for (int p0 = 0; p0 < max_d; p0 += CB) {
      const int rest = max_d - p0 - CB;                   // trailing rows of the largest matrix
      const unsigned chunks = unsigned(std::max<int64_t>(1, cdiv(std::max(rest, 0), CPR)));
      launch_pdl(chol_panel_kernel, dim3(chunks, unsigned(cd.size())), dim3(CP_THREADS), size_t(0), st,
          dc, p0, damping, ctx->dflags);
      ctx->launches++;
      CUDA_TRY(ctx, cudaGetLastError());
      if (rest > 0) {
        const int nt = int(cdiv(rest, CU_T));
        launch_pdl(chol_update_kernel, dim3(unsigned(nt * (nt + 1) / 2), unsigned(cd.size())), dim3(CP_THREADS),
                   size_t(0), st, dc, p0);
        ctx->launches++;
        CUDA_TRY(ctx, cudaGetLastError());
      }
    }
    // L^-1 into the output buffers (diagonal-block inverses, then doubling
    // levels of two products each), then S^-1 = L^-T L^-1 into the scratch
    // that held L, then copied out
    launch_pdl(linv_init_kernel, dim3(unsigned(cdiv(max_d, 64)), unsigned(cd.size())), dim3(256), size_t(0), st,
               dc);
    ctx->launches++;
    CUDA_TRY(ctx, cudaGetLastError());
    for (int sl = CB; sl < max_d; sl *= 2) {
      const int64_t tiles = cdiv(sl, LV_T);
      const int64_t pairs = cdiv(max_d - sl, 2 * int64_t(sl));
      for (int mode = 0; mode < 2; ++mode) {
        launch_pdl(linv_level_kernel, dim3(unsigned(pairs * tiles * tiles), unsigned(cd.size())), dim3(LV_THREADS),
                   size_t(0), st, dc, sl, mode);
        ctx->launches++;
        CUDA_TRY(ctx, cudaGetLastError());
      }
    }
    const int nt = int(cdiv(max_d, SIP_T));
    launch_pdl(spd_inverse_product_kernel, dim3(unsigned(nt * (nt + 1) / 2), unsigned(cd.size())),
               dim3(SIP_THREADS), size_t(0), st, dc);
    ctx->launches++;
    CUDA_TRY(ctx, cudaGetLastError());
    const int64_t most = int64_t(max_d) * max_d;
    launch_pdl(copy_inverse_kernel, dim3(unsigned(std::min<int64_t>(cdiv(most, 4 * 256), 1024)), unsigned(cd.size())),
               dim3(256), size_t(0), st, dc);
    ctx->launches++;
    CUDA_TRY(ctx, cudaGetLastError());
    return emit_splits();
  }
  cholesky_kernel<<<unsigned(cd.size()), CHOL_THREADS, 0, st>>>(dc, damping, ctx->dflags);
  ctx->launches++;
  CUDA_TRY(ctx, cudaGetLastError());
  const int parts = int(cdiv(max_d, SOLVE_ROWS_PER_BLOCK));
  chol_solve_kernel<<<unsigned(cd.size() * parts), SOLVE_THREADS, 0, st>>>(dc, parts);
  ctx->launches++;
  CUDA_TRY(ctx, cudaGetLastError());
  return emit_splits();
}

muon_status muon_check_device(muon_ctx* ctx) {
  if (!ctx) return MUON_ERR_INVALID_ARG;
  muon_status s = set_device(ctx);
  if (s != MUON_OK) return s;
  CUDA_TRY(ctx, cudaDeviceSynchronize());
  int flags = 0;
  CUDA_TRY(ctx, cudaMemcpy(&flags, ctx->dflags, sizeof(int), cudaMemcpyDeviceToHost));
  if (flags) {
    CUDA_TRY(ctx, cudaMemset(ctx->dflags, 0, sizeof(int)));
    if (flags & kDevErrTimeout) return fail(ctx, MUON_ERR_TIMEOUT, "a device-side wait gave up (flags 0x%x)", flags);
    if (flags & kDevErrNotSPD)
      return fail(ctx, MUON_ERR_INVALID_ARG, "a second moment was not positive definite (flags 0x%x)", flags);
    return fail(ctx, MUON_ERR_CUDA, "device error flags 0x%x", flags);
  }
  return MUON_OK;
}

muon_status muon_selftest_wait(muon_ctx* ctx, void* stream) {
  if (!ctx) return MUON_ERR_INVALID_ARG;
  muon_status s = set_device(ctx);
  if (s != MUON_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ctx->last_stream = st;
  CUDA_TRY(ctx, cudaGetLastError());
  selftest_wait_kernel<<<1, 32, 0, st>>>(ctx->dflags);
  ctx->launches++;
  CUDA_TRY(ctx, cudaGetLastError());
  return MUON_OK;
}

muon_status muon_selftest_gemm(muon_ctx* ctx, void* stream) {
  if (!ctx) return MUON_ERR_INVALID_ARG;
  muon_status s = set_device(ctx);
  if (s != MUON_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ctx->last_stream = st;
  CUDA_TRY(ctx, cudaGetLastError());
  // One Gram tile of a zero 256 x 640 X: ten K blocks, more than the
  // pipeline holds, so the producer also waits for a stage the MMA thread
  // never releases.
  constexpr int m = 256, n = 640;
  const size_t xb = size_t(m) * n * 2, ab = size_t(m) * m * 2;
  void* wsv = nullptr;
  s = ensure_workspace(ctx, xb + ab, &wsv);
  if (s != MUON_OK) return s;
  uint8_t* ws = static_cast<uint8_t*>(wsv);
  CUDA_TRY(ctx, cudaMemsetAsync(ws, 0, xb + ab, st));
  GemmMaps maps{};
  bool ok = encode_bf16_3d(&maps.a[0], ws, n, m, 1, n, 64, 128);
  maps.b[0] = maps.a[0];
  ok &= encode_bf16_3d(&maps.out[0], ws + xb, m, m, 1, m, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  ok &= encode_bf16_3d(&maps.aux[0], ws + xb, m, m, 1, m, 64, 32);
  if (!ok) return fail(ctx, MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed (self test)");
  GemmArgs g{};
  g.nprob = 1;
  g.total = 1;
  GemmProblem& P = g.p[0];
  P.M = m; P.N = m; P.K = n;
  P.batch = 1;
  P.tiles_m = P.tiles_n = 1;
  P.tiles_per_mat = 1;
  P.out = reinterpret_cast<__nv_bfloat16*>(ws + xb);
  P.out_ld = m;
  P.out_bs = int64_t(m) * m;
  g.alpha_pow = 2;
  g.eps = 1e-7f;
  g.err = ctx->dflags;
  g.skip = nullptr;          // runs whatever the flags hold
  g.selftest = 1;
  CUDA_TRY(ctx, (launch_gemm<EPI_GRAM, false>(ctx, maps, g, st)));
  return MUON_OK;
}

uint64_t muon_launch_count(const muon_ctx* ctx) { return ctx ? ctx->launches : 0; }

muon_status muon_partition(const int64_t* rows, const int64_t* cols, int32_t n, int32_t world, int32_t* owner) {
  if (n < 0 || world < 1 || (n > 0 && (!rows || !cols || !owner))) return MUON_ERR_INVALID_ARG;
  std::vector<std::pair<double, int>> cost(n);
  for (int i = 0; i < n; ++i) {
    if (rows[i] < 1 || cols[i] < 1) return MUON_ERR_INVALID_ARG;
    const double m = double(std::min(rows[i], cols[i])), nn = double(std::max(rows[i], cols[i]));
    cost[i] = {5.0 * (4.0 * m * m * nn + 2.0 * m * m * m) + 5600.0 * double(rows[i]) * double(cols[i]), i};
  }
  std::stable_sort(cost.begin(), cost.end(), [](const std::pair<double, int>& a, const std::pair<double, int>& b) {
    return a.first > b.first;
  });
  std::vector<double> load(world, 0.0);
  for (const auto& c : cost) {
    int best = 0;
    for (int r = 1; r < world; ++r)
      if (load[r] < load[best]) best = r;
    load[best] += c.first;
    owner[c.second] = best;
  }
  return MUON_OK;
}

muon_status muon_profile_enable(muon_ctx* ctx, int enable) {
  if (!ctx) return MUON_ERR_INVALID_ARG;
  ctx->prof = enable != 0;
  return MUON_OK;
}

muon_status muon_profile_read(muon_ctx* ctx, muon_kernel_times* out) {
  if (!ctx || !out) return MUON_ERR_INVALID_ARG;
  muon_status s = set_device(ctx);
  if (s != MUON_OK) return s;
  for (int k = 0; k < MUON_K_COUNT; ++k) {
    for (auto& pr : ctx->prof_pending[k]) {
      CUDA_TRY(ctx, cudaEventSynchronize(pr.second));
      float ms = 0.f;
      CUDA_TRY(ctx, cudaEventElapsedTime(&ms, pr.first, pr.second));
      ctx->prof_ms[k] += ms;
      ctx->prof_n[k] += 1;
      ctx->prof_pool.push_back(pr.first);
      ctx->prof_pool.push_back(pr.second);
    }
    ctx->prof_pending[k].clear();
    out->ms[k] = ctx->prof_ms[k];
    out->launches[k] = ctx->prof_n[k];
    ctx->prof_ms[k] = 0.0;
    ctx->prof_n[k] = 0;
  }
  return MUON_OK;
}

// Newton-Schulz of one matrix without any device allocation: all scratch
// lives in g_noalloc_scratch (see include/muon.h for the contract).
muon_status muon_orthogonalize_noalloc(const void* input, int32_t in_dtype, int64_t rows, int64_t cols,
                                       float* output, const muon_hparams* hp, void* stream) {
  if (!input || !output || !hp) return MUON_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1) return MUON_ERR_INVALID_ARG;
  if (in_dtype != MUON_F32 && in_dtype != MUON_BF16) return MUON_ERR_INVALID_ARG;
  if (!aligned16(input) || !aligned16(output)) return MUON_ERR_INVALID_ARG;
  muon_ctx tmp;   // host-side bookkeeping only; no device resources
  muon_status s = check_hparams(&tmp, hp);
  if (s != MUON_OK) return s;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return MUON_ERR_CUDA;
  uint8_t* base = nullptr;
  s = noalloc_scratch_address(device, &base);
  if (s != MUON_OK) return s;
  tmp.device = device;

  // Layout: flags | descriptor | norm | partials | X0 | X1 | A | B
  Item it{};
  it.rows = rows;
  it.cols = cols;
  it.transposed = rows > cols;
  it.m = std::min(rows, cols);
  it.n = std::max(rows, cols);
  it.grad_dtype = in_dtype;
  it.grad = input;
  it.update_out = output;
  std::vector<Item> items(1, it);
  Chunk c{};
  c.first = 0;
  c.count = 1;
  const size_t body = layout_chunk(c, items);
  const size_t head = 2 * kAlign;   // flags, descriptor
  if (head + body > kNoAllocScratchBytes) return MUON_ERR_WORKSPACE;
  int* flags = reinterpret_cast<int*>(base);
  MatDesc* ddesc = reinterpret_cast<MatDesc*>(base + kAlign);
  uint8_t* ws = base + head;
  const Run& r = c.runs[0];

  MatDesc d{};
  d.grad = input;
  d.grad_dtype = in_dtype;
  d.update_out = output;
  d.x_in = reinterpret_cast<__nv_bfloat16*>(ws + r.off_x0);
  d.x_out = reinterpret_cast<__nv_bfloat16*>(ws + ((hp->ns_steps % 2) ? r.off_x1 : r.off_x0));
  d.norm2 = reinterpret_cast<float*>(ws + c.off_norm);
  d.partials = reinterpret_cast<float*>(ws + c.off_partials);
  d.rows = rows;
  d.cols = cols;
  d.ld = r.ld_n;
  d.tile_start = 0;
  d.tiles_c = int(cdiv(cols, EW_TILE));
  d.transposed = it.transposed ? 1 : 0;
  const int64_t tiles = cdiv(rows, EW_TILE) * d.tiles_c;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The descriptor travels as a kernel parameter and is stored into the
  // scratch array on the device, together with zeroed flags (a previous
  // call leaves its values behind; everything else is fully overwritten
  // before it is read), so the call makes no host-to-device copy.
  noalloc_setup_kernel<<<1, 32, 0, st>>>(d, ddesc, flags);
  const std::vector<SegLaunch> segl = build_seg_launches(&d, 1);
  momentum_kernel<1><<<unsigned(tiles), MOM_THREADS, 0, st>>>(ddesc, segl[0].t, 0, 0.f, 0, flags);
  norm_reduce_kernel<<<1, EW_THREADS, 0, st>>>(ddesc, flags);
  if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  tmp.dflags = flags;
  const float* n2 = d.norm2;
  // a product whose bounded wait gives up raises flags[0]; the later
  // products and the export then do nothing, and the output is poisoned
  s = run_newton_schulz(&tmp, ws, &r, 1, &n2, hp, flags, st);
  tmp.dflags = nullptr;
  if (s != MUON_OK) return s;
  apply_kernel<1><<<unsigned(tiles), EW_THREADS, 0, st>>>(ddesc, segl[0].t, hp->ns_steps == 0, hp->eps,
                                                          flags);
  const int64_t n = rows * cols;
  noalloc_poison_kernel<<<unsigned(std::min<int64_t>(cdiv(n, 256), 1024)), 256, 0, st>>>(flags, output, n);
  if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  return MUON_OK;
}

}  // extern "C"
