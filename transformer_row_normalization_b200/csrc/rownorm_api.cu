// C ABI of librownorm.so: argument validation, launch planning and dispatch.
// The operations and conventions are documented in include/rownorm.h.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "rownorm.h"
#include "rownorm_kernels.cuh"
#include "rownorm_launch.h"
#include "rownorm_ring.cuh"

namespace {

thread_local char g_last_error[512] = "";
// Testing controls, process-wide: set by rn_set_grid_override /
// rn_set_path_override from any thread while other threads plan launches.
std::atomic<int> g_grid_override{0};
std::atomic<int> g_path_override{0};  // 0 automatic, 1 register, 2 ring, 3 register + prefetch
std::atomic<int> g_ring_wait_test{0};  // 1: ring stages never complete (bounded-wait test)

int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return status;
}

int elem_size(int dtype) { return dtype == RN_F32 ? 4 : 2; }

// Rows in blocks of inner_rows (row r at (r / inner) * outer + (r % inner) *
// row_stride) when there is more than one block; else one row stride.
bool two_level(const rn_view* v) { return v->inner_rows > 0 && v->rows > v->inner_rows; }

// Element offset of the start of row r.
int64_t row_start(const rn_view* v, int64_t r) {
  if (!two_level(v)) return r * v->row_stride;
  return (r / v->inner_rows) * v->outer_stride + (r % v->inner_rows) * v->row_stride;
}

// Start of the last row (the furthest, since blocks do not overlap).
int64_t last_row_start(const rn_view* v) { return v->rows > 0 ? row_start(v, v->rows - 1) : 0; }

// rows == 0 views are valid (they enqueue nothing); the checks below still
// run so that malformed descriptors are reported consistently.
int check_view(const rn_view* v, const char* name) {
  if (!v) return fail(RN_ERR_NULL, "%s: view pointer is NULL", name);
  if (v->dtype != RN_F32 && v->dtype != RN_BF16)
    return fail(RN_ERR_DTYPE, "%s: unknown dtype %d", name, (int)v->dtype);
  if (v->rows < 0) return fail(RN_ERR_SHAPE, "%s: rows %lld < 0", name, (long long)v->rows);
  if (v->dim < 1) return fail(RN_ERR_SHAPE, "%s: dim %lld < 1", name, (long long)v->dim);
  const int64_t inner = two_level(v) ? v->inner_rows : v->rows;  // rows of one stride
  if (inner > 1 && v->row_stride < v->dim)
    return fail(RN_ERR_SHAPE, "%s: row_stride %lld < dim %lld", name,
                (long long)v->row_stride, (long long)v->dim);
  if (v->inner_rows < 0 || v->inner_rows > INT32_MAX)
    return fail(RN_ERR_SHAPE, "%s: inner_rows %lld outside [0, 2^31)", name,
                (long long)v->inner_rows);
  const int es = elem_size(v->dtype);
  if (inner > 1) {
    const int64_t limit = (INT64_MAX / es - v->dim) / (inner - 1);
    if (v->row_stride > limit) return fail(RN_ERR_SHAPE, "%s: extent overflows", name);
  }
  if (two_level(v)) {
    // blocks must not overlap: the next block starts past this block's rows
    const int64_t block = (v->inner_rows - 1) * v->row_stride + v->dim;
    if (v->outer_stride < block)
      return fail(RN_ERR_SHAPE, "%s: outer_stride %lld < one block (%lld)", name,
                  (long long)v->outer_stride, (long long)block);
    const int64_t blocks = (v->rows - 1) / v->inner_rows;
    if (v->outer_stride > (INT64_MAX / es - block) / blocks)
      return fail(RN_ERR_SHAPE, "%s: extent overflows", name);
  }
  if (v->rows > 0 && !v->data) return fail(RN_ERR_NULL, "%s: data is NULL", name);
  if (reinterpret_cast<uintptr_t>(v->data) % es)
    return fail(RN_ERR_ALIGN, "%s: data not aligned to its %d-byte element", name, es);
  if (v->dim > RN_MAX_DIM_STREAM)
    return fail(RN_ERR_UNSUPPORTED, "%s: dim %lld above the supported maximum %lld", name,
                (long long)v->dim, (long long)RN_MAX_DIM_STREAM);
  return RN_OK;
}

int check_vector(const void* p, int dtype, const char* name) {
  if (p && reinterpret_cast<uintptr_t>(p) % elem_size(dtype))
    return fail(RN_ERR_ALIGN, "%s: not aligned to its element size", name);
  return RN_OK;
}

struct Span {
  uintptr_t lo, hi;  // [lo, hi)
};

Span span_of(const rn_view* v) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(v->data);
  if (v->rows == 0) return {lo, lo};
  const int64_t n = last_row_start(v) + v->dim;
  return {lo, lo + static_cast<uintptr_t>(n) * elem_size(v->dtype)};
}

Span span_of_vector(const void* p, int64_t dim, int dtype) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return {lo, p ? lo + static_cast<uintptr_t>(dim) * elem_size(dtype) : lo};
}

bool intersects(Span a, Span b) { return a.lo < b.hi && b.lo < a.hi && a.lo != a.hi && b.lo != b.hi; }

// Whether two views can share an element. Beyond their spans: views laid out
// in blocks with one common block stride (head rows of one packed buffer,
// e.g. the q and k heads of a QKV projection) repeat with that period, so
// their rows are disjoint when, within one period, each block's footprint
// fits and misses the other's.
bool views_overlap(const rn_view* a, const rn_view* b) {
  if (!intersects(span_of(a), span_of(b))) return false;
  if (!two_level(a) || !two_level(b) || a->outer_stride != b->outer_stride ||
      a->dtype != b->dtype)
    return true;
  const int es = elem_size(a->dtype);
  const intptr_t bytes = reinterpret_cast<intptr_t>(b->data) -
                         reinterpret_cast<intptr_t>(a->data);
  if (bytes % es) return true;
  const int64_t o = a->outer_stride;
  const int64_t la = (a->inner_rows - 1) * a->row_stride + a->dim;  // block footprints
  const int64_t lb = (b->inner_rows - 1) * b->row_stride + b->dim;
  int64_t beta = (int64_t)(bytes / es) % o;  // b's block start within a's period
  if (beta < 0) beta += o;
  return !(la <= o && lb <= o && beta >= la && beta + lb <= o);
}

bool same_view(const rn_view* a, const rn_view* b) {
  if (a->data != b->data || two_level(a) != two_level(b)) return false;
  if (a->rows <= 1) return true;
  if (!two_level(a)) return a->row_stride == b->row_stride;
  return a->row_stride == b->row_stride && a->inner_rows == b->inner_rows &&
         a->outer_stride == b->outer_stride;
}

// An output may be its own input exactly, and must not touch anything else.
int check_output(const rn_view* y, const rn_view* x_own, const rn_view* const* others,
                 int n_others, const void* const* vecs, const int64_t* vec_dims,
                 int n_vecs, const char* name) {
  const Span sy = span_of(y);
  if (views_overlap(y, x_own) && !same_view(y, x_own))
    return fail(RN_ERR_OVERLAP, "%s partially overlaps its input", name);
  for (int i = 0; i < n_others; ++i)
    if (views_overlap(y, others[i]))
      return fail(RN_ERR_OVERLAP, "%s overlaps another argument", name);
  for (int i = 0; i < n_vecs; ++i)
    if (vecs[i] && intersects(sy, span_of_vector(vecs[i], vec_dims[i], y->dtype)))
      return fail(RN_ERR_OVERLAP, "%s overlaps a weight/bias vector", name);
  return RN_OK;
}

int check_eps(float eps) {
  if (!(eps >= 0.0f) || !std::isfinite(eps))
    return fail(RN_ERR_EPS, "eps must be finite and >= 0 (got %g)", (double)eps);
  return RN_OK;
}

int check_pair(const rn_view* x, const rn_view* y, const char* xn, const char* yn) {
  if (x->dtype != y->dtype) return fail(RN_ERR_DTYPE, "%s and %s differ in dtype", xn, yn);
  if (x->rows != y->rows || x->dim != y->dim)
    return fail(RN_ERR_SHAPE, "%s [%lld, %lld] and %s [%lld, %lld] differ", xn,
                (long long)x->rows, (long long)x->dim, yn, (long long)y->rows,
                (long long)y->dim);
  return RN_OK;
}

// ---------------------------------------------------------------------------
// planning

// Every row of v starts at the same 16-byte phase as v's first row.
bool strides_aligned(const rn_view* v) {
  const int es = elem_size(v->dtype);
  const int64_t inner = two_level(v) ? v->inner_rows : v->rows;
  if (inner > 1 && (v->row_stride * es) % 16) return false;
  if (two_level(v) && (v->outer_stride * es) % 16) return false;
  return true;
}

// Every row of `v` starts at the same 16-byte phase as the matching row of x.
bool same_phase(const rn_view* x, const rn_view* v) {
  const int es = elem_size(x->dtype);
  const uintptr_t xa = reinterpret_cast<uintptr_t>(x->data);
  const uintptr_t va = reinterpret_cast<uintptr_t>(v->data);
  if ((va - xa) % 16) return false;
  if (strides_aligned(x) && strides_aligned(v)) return true;
  if (two_level(x) != two_level(v)) return false;
  if (!two_level(x)) return x->rows <= 1 || ((v->row_stride - x->row_stride) * es) % 16 == 0;
  return x->inner_rows == v->inner_rows &&
         ((v->row_stride - x->row_stride) * es) % 16 == 0 &&
         ((v->outer_stride - x->outer_stride) * es) % 16 == 0;
}

// Widest rows of the lane-group family: a warp of 32 lanes of at most 8
// chunks (binary32 1024 columns, bf16 2048).
int64_t warp_family_max_dim(int dtype) { return dtype == RN_F32 ? 1024 : 2048; }

int pow2_ceil(int64_t v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Widest rows the register kernels hold; wider RMSNorm / LayerNorm rows stream.
int64_t register_max_dim(int dtype) { return dtype == RN_F32 ? RN_MAX_DIM_F32 : RN_MAX_DIM_BF16; }

struct SegPlan {
  int family;        // 0 warp, 1 block, 2 streaming block (rows wider than registers hold)
  int lanes;         // family 0: lanes per row; family 1: threads per block
  int chunks;        // capacity of 16-byte chunks per thread
  int vector_y;      // y rows share x's 16-byte phase
  int phase_period;  // distinct 16-byte phases among the rows of x
  int exact;         // every x and y row 16-byte aligned, dim % V == 0
  int64_t nfull_max; // full 16-byte chunks of a row: at most / at least
  int64_t nfull_min;
};

// The lane count / block size is a function of (dtype, dim) and, for lane
// groups, of whether every row of x starts on a 16-byte boundary with
// dim % V == 0; so the summation tree of a row never depends on anything
// else about the call. Rows that are not so aligned have up to 2 (V - 1)
// edge elements, one per thread, so their lane groups hold at least that
// many lanes (blocks always do).
SegPlan plan_segment(const rn_view* x, const rn_view* y, const void* w, const void* b) {
  const int es = elem_size(x->dtype);
  const int V = 16 / es;
  const int64_t D = x->dim;
  const uintptr_t xa = reinterpret_cast<uintptr_t>(x->data);
  const bool rows_aligned = (xa % 16 == 0) && (D % V == 0) && strides_aligned(x);
  const int64_t nfull = D / V;  // full chunks of a row, at most (any phase)
  SegPlan p{};
  const int per_thread = rn::kTargetChunksPerThread;
  if (D > register_max_dim(x->dtype)) {
    p.family = 2;
    p.lanes = rn::kStreamBlockThreads;
    p.chunks = (int)ceil_div(nfull, p.lanes);
  } else if (D <= warp_family_max_dim(x->dtype)) {
    p.family = 0;
    int g = pow2_ceil(ceil_div(ceil_div(D, V), per_thread));
    if (!rows_aligned && g < pow2_ceil(2 * (V - 1))) g = pow2_ceil(2 * (V - 1));
    p.lanes = g > 32 ? 32 : g;
    p.chunks = (int)ceil_div(nfull, p.lanes);
    if (p.chunks < 1) p.chunks = 1;
  } else {
    p.family = 1;
    // the fewest threads (a power of two, 128..1024) that hold a row in at
    // most kCtaMaxChunks chunks each: the block reductions and the per-row
    // setup are paid once per row per thread, so more work per thread is
    // cheaper
    int nt = pow2_ceil(ceil_div(nfull, rn::kCtaMaxChunks));
    p.lanes = nt < 128 ? 128 : (nt > 1024 ? 1024 : nt);
    p.chunks = (int)ceil_div(nfull, p.lanes);
    if (p.chunks < rn::kCtaMinChunks) p.chunks = rn::kCtaMinChunks;
  }
  const uintptr_t ya = reinterpret_cast<uintptr_t>(y->data);
  p.vector_y = same_phase(x, y);
  p.phase_period = 1;
  if (x->rows > 1 && !two_level(x)) {
    int64_t step = (x->row_stride * es) % 16;  // row-to-row phase advance, bytes
    int period = 1;
    for (int64_t acc = step; acc % 16 != 0; acc += step) ++period;
    p.phase_period = period;
  }
  p.exact = rows_aligned && ya % 16 == 0 &&
            strides_aligned(y) &&
            reinterpret_cast<uintptr_t>(w) % 16 == 0 && reinterpret_cast<uintptr_t>(b) % 16 == 0;
  p.nfull_max = nfull;
  p.nfull_min = rows_aligned ? nfull : (nfull > 0 ? nfull - 1 : 0);
  return p;
}

// The slots of a thread that every row of segment p fills when each thread
// has `chunks` slots: all of them (rows divide evenly; EXACT only), all but
// the last, or no guarantee.
int slot_class(const SegPlan& p, int chunks) {
  if (p.exact && p.nfull_max == (int64_t)p.lanes * chunks && chunks <= rn::kFullMaxChunks)
    return rn::kSlotsFull;
  // block-family kernels with more than kFullMaxChunks slots spill when
  // specialized and measured faster testing every slot
  if (p.family == 1 && chunks > rn::kFullMaxChunks) return rn::kSlotsTested;
  if ((int64_t)(chunks - 1) * p.lanes <= p.nfull_min) return rn::kSlotsTail;
  return rn::kSlotsTested;
}

const void* kernel_for(int dtype, int op, const SegPlan& p, int slots) {
  const bool ex = p.exact != 0;
  if (p.family == 2) return rn::stream_kernel(dtype == RN_F32, op, ex, p.lanes);
  if (p.family == 0)
    return dtype == RN_F32 ? rn::warp_kernel_f32(op, ex, slots, p.chunks)
                           : rn::warp_kernel_bf16(op, ex, slots, p.chunks);
  return dtype == RN_F32 ? rn::cta_kernel_f32(op, ex, slots, p.lanes, p.chunks)
                         : rn::cta_kernel_bf16(op, ex, slots, p.lanes, p.chunks);
}

struct DeviceInfo {
  int sms = 0;
  int smem_per_sm = 0;
  int smem_per_block = 0;
};

struct OccKey {
  const void* fn;
  int smem;
  bool operator==(const OccKey& o) const { return fn == o.fn && smem == o.smem; }
};
struct OccKeyHash {
  size_t operator()(const OccKey& k) const {
    return std::hash<const void*>()(k.fn) ^ (std::hash<int>()(k.smem) << 1);
  }
};

std::mutex g_mu;
DeviceInfo g_dev[64];
std::unordered_map<OccKey, int, OccKeyHash> g_occ[64];  // resident blocks per SM
std::unordered_map<const void*, int> g_smem_attr[64];   // kernels given the opt-in limit

int device_sms(int dev, int* sms) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (dev < 0 || dev >= 64) return fail(RN_ERR_CUDA, "device ordinal %d out of range", dev);
  if (!g_dev[dev].sms) {
    DeviceInfo d;
    cudaError_t e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (e == cudaSuccess)
      e = cudaDeviceGetAttribute(&d.smem_per_block, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return fail(RN_ERR_CUDA, "device query: %s", cudaGetErrorString(e));
    g_dev[dev] = d;
  }
  *sms = g_dev[dev].sms;
  return RN_OK;
}

DeviceInfo device_info(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  return g_dev[dev];
}

// Resident blocks per SM of `fn` at `smem` bytes of dynamic shared memory.
// The first query of a kernel on a device also lifts its dynamic shared
// memory limit to the device's opt-in maximum (the default is 48 KB).
int blocks_per_sm(int dev, const void* fn, int threads, int smem, int* out) {
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_occ[dev].find(OccKey{fn, smem});
  if (it != g_occ[dev].end()) {
    *out = it->second;
    return RN_OK;
  }
  cudaError_t e;
  if (!g_smem_attr[dev].count(fn)) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, fn);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               g_dev[dev].smem_per_block - (int)fa.sharedSizeBytes);
    if (e != cudaSuccess)
      return fail(RN_ERR_CUDA, "shared memory attribute: %s", cudaGetErrorString(e));
    g_smem_attr[dev][fn] = g_dev[dev].smem_per_block - (int)fa.sharedSizeBytes;
  }
  if (smem > g_smem_attr[dev][fn])
    return fail(RN_ERR_UNSUPPORTED, "%d B of shared memory above the limit %d B", smem,
                g_smem_attr[dev][fn]);
  int n = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem);
  if (e != cudaSuccess) return fail(RN_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
  if (n < 1) return fail(RN_ERR_UNSUPPORTED, "kernel does not fit on an SM (%d B shared)", smem);
  g_occ[dev][OccKey{fn, smem}] = n;
  *out = n;
  return RN_OK;
}

struct Launch {
  const void* fn;
  int smem;
  int prefetch;     // register kernels: rows ahead prefetched through shared memory
  int ring;         // 1: rows_ring_kernel, 2: rows_cta_ring_kernel (RingParams)
  rn_launch_info info;
  // ring kernels only
  int stages, stage_bytes, tile_rows[2], contiguous[2], table_bytes, affine_word;
  int stage_word;   // kOpRmsRope: staging rows after the slots and the cache
};

// Ring tiles: R rows of a lane-group segment per stage, about this many
// bytes (at least one round of the warp's lane groups); S stages per warp.
#ifndef RN_RING_TILE_BYTES
#define RN_RING_TILE_BYTES 2048
#endif
constexpr int kRingTileBytes = RN_RING_TILE_BYTES;
#ifndef RN_RING_STAGES
#define RN_RING_STAGES 4
#endif
constexpr int kRingStages = RN_RING_STAGES;
// LayerNorm rows of a whole warp go two to a tile when two fit in
// rn::kRingPairTileBytes (ring_ln_pair normalizes them together), with this
// many stages.
// Measured on B200 (bf16, 65536 rows, cold / back to back, us): D = 768
// 40.9 / 37.0 -> 37.0 / 38.5, D = 1000 55.4 / 53.3 -> 48.0 / 50.2, D = 1024
// 51.2 / 49.3 -> 49.2 / 50.0; two stages ran faster cold still (768: 36.9)
// but slower back to back (1000: 51.7), four slower back to back at 768
// (39.6). RMSNorm rows measured mixed in pairs (1024: 41.0 -> 44.9 cold,
// 51.6 -> 50.3 back to back) and stay one to a tile.
constexpr int kRingPairStages = 3;
// RoPE tiles (table row staged): whole lane-group rounds of one token, up
// to this many bytes of rows. Measured on B200 (bf16 dual head norm + RoPE,
// 8192 tokens of 32 + 8 heads of 128, cold / back to back, us): tiles of 8 q
// rows 45.9 / 41.0, 16 rows 43.0 / 37.6, 32 rows 43.0 / 40.3.
#ifndef RN_RING_ROPE_TILE_BYTES
#define RN_RING_ROPE_TILE_BYTES 4096
#endif
constexpr int kRingRopeTileBytes = RN_RING_ROPE_TILE_BYTES;

int round_up(int64_t v, int64_t m) { return (int)((v + m - 1) / m * m); }

// Whether the planner uses the per-warp bulk-copy rings by default for these
// segments (they must qualify, see plan_ring). Measured on B200 against the
// register lane-group kernels with their per-thread prefetch (bf16, 65536
// rows, cold / back to back, us):
//   rows whose lane groups fill a warp: LayerNorm 768 45.1 / 45.1 -> 36.9 /
//     38.4, 1000 61.5 / 62.7 -> 47.1 / 49.8, 1024 52.1 / 51.8 -> 49.1 / 50.0,
//     RMSNorm 1024 44.9 / 51.6 -> 41.0 / 50.6;
//   the dual head norm + RoPE (q [8192, 32, 128], k [8192, 8, 128]) with
//     the token's table row staged with each tile: split-half planes 43.0 /
//     41.1 -> 36.9 / 35.2, interleaved planes 52.2 / 49.1 -> 38.9 / 37.0;
//     with the table read from global memory per row the rings ran slower
//     (47.1 -> 53.2 cold), so that stays on the register kernels unless the
//     rings are forced (plan_ring checks the staging);
//   but the plain dual head norm (same shapes, 4 lanes per row) 26.7 / 31.2
//     -> 30.9 / 31.5, bf16 LayerNorm 512 (16 lanes per row) 31.8 -> 34.7
//     and binary32 LayerNorm 1024 88.1 -> 94.1 ran slower, and stay on the
//     register kernels.
bool ring_preferred(int dtype, int op, const SegPlan* plans, int nseg, const rn_rope* rope) {
  if (dtype != RN_BF16) return false;
  if (op == rn::kOpRmsRopeLocal) return nseg == 2 && rope;
  if (op != rn::kOpRms && op != rn::kOpLn) return false;
  for (int i = 0; i < nseg; ++i)
    if (plans[i].lanes != 32) return false;
  return true;
}

// Plans a ring launch for RMSNorm / LayerNorm segments of the lane-group
// family in EXACT layouts: by default where ring_preferred says so, everywhere
// it qualifies with rn_set_path_override(2), never with 1 or 3. Returns
// false (the register-kernel plan stays in charge) otherwise.
bool plan_ring(int dtype, int op, const SegPlan* plans, const rn_view* const* xs, int nseg,
               int chunks, int slots, int dev, int sms, const rn_rope* rope, Launch* out) {
  const int path = g_path_override.load(std::memory_order_relaxed);
  if (path == 1 || path == 3) return false;
  if (op != rn::kOpRms && op != rn::kOpLn && op != rn::kOpRmsRopeLocal) return false;
  if (op == rn::kOpLn && nseg != 1) return false;  // one weight / bias area per block
  for (int i = 0; i < nseg; ++i)
    if (plans[i].family != 0 || !plans[i].exact) return false;
  if (path == 0 && !ring_preferred(dtype, op, plans, nseg, rope)) return false;
  const void* fn = dtype == RN_F32 ? rn::ring_kernel_f32(op, slots, chunks)
                                   : rn::ring_kernel_bf16(op, slots, chunks);
  if (!fn) return false;
  Launch l{};
  l.ring = 1;
  const int es = elem_size(dtype);
  int64_t stage_bytes = 16;
  int64_t tiles_max = 1;
  bool paired = false;
  for (int i = 0; i < nseg; ++i) {
    const int64_t row_bytes = xs[i]->dim * es;
    const int64_t per = 32 / plans[i].lanes;  // rows a warp takes at once
    int64_t rounds = kRingTileBytes / (per * row_bytes);
    if (rounds < 1) rounds = 1;
    if (op == rn::kOpLn && per == 1 && rounds < 2 && rn::ring_pairs_fit(chunks)) {
      rounds = 2;
      paired = true;
    }
    if (op == rn::kOpRmsRopeLocal && rope && rope->table && nseg == 2) {
      // tiles of whole lane-group rounds inside one token, as large as fit
      // kRingRopeTileBytes: the table row staged with the tile serves every
      // row a lane takes from it
      const int64_t heads = i == 0 ? rope->heads_q : rope->heads_k;
      int64_t best = 0;
      for (int64_t rd = 1; per * rd * row_bytes <= kRingRopeTileBytes; ++rd)
        if (heads % (per * rd) == 0) best = rd;
      if (best) rounds = best;
    }
    const int64_t tr = per * rounds;
    l.tile_rows[i] = (int)tr;
    l.contiguous[i] = !two_level(xs[i]) && (xs[i]->rows <= 1 || xs[i]->row_stride == xs[i]->dim);
    const int64_t tiles = ceil_div(xs[i]->rows, tr);
    if (tiles > tiles_max) tiles_max = tiles;
    if (tr * row_bytes > stage_bytes) stage_bytes = tr * row_bytes;
  }
  // RoPE rows: stage each tile's token's table row beside its rows when
  // every tile lies in one token (tile rows divide both head counts) and the
  // table rows start on the 16-byte grid
  l.table_bytes = 0;
  if (op == rn::kOpRmsRopeLocal && rope && rope->table && nseg == 2) {
    const int64_t tb = (int64_t)rope->dims * 4;
    const bool one_token = rope->heads_q % l.tile_rows[0] == 0 &&
                           rope->heads_k % l.tile_rows[1] == 0;
    if (one_token && tb % 16 == 0 && reinterpret_cast<uintptr_t>(rope->table) % 16 == 0) {
      l.table_bytes = (int)tb;
      int64_t sb = 16;
      for (int i = 0; i < nseg; ++i) {
        const int64_t b = (int64_t)l.tile_rows[i] * xs[i]->dim * es + tb;
        if (b > sb) sb = b;
      }
      stage_bytes = sb;
    }
  }
  if (path == 0 && op == rn::kOpRmsRopeLocal && l.table_bytes == 0) return false;
  l.stage_bytes = round_up(stage_bytes, 16);
  const DeviceInfo di = device_info(dev);
  // LayerNorm rings keep the block's binary32 weight and bias after the
  // barriers (ring_affine_bytes)
  const int affine = op == rn::kOpLn ? rn::ring_affine_bytes((int)xs[0]->dim) : 0;
  int stages = paired ? kRingPairStages : kRingStages;
  // as many stages as keep kRingBlocksPerSm blocks on an SM (1 KB of each
  // block's shared memory is the system's)
  auto smem_of = [&](int k) { return rn::ring_smem_bytes(k, l.stage_bytes) + affine; };
  while (stages > 2 && (smem_of(stages) > di.smem_per_block - 1024 ||
                        rn::kRingBlocksPerSm * (smem_of(stages) + 1024) > di.smem_per_sm))
    --stages;
  if (smem_of(stages) > di.smem_per_block - 1024) return false;
  l.stages = stages;
  l.fn = fn;
  l.smem = smem_of(stages);
  l.affine_word = affine ? rn::ring_smem_bytes(stages, l.stage_bytes) / 16 : -1;
  int bps = 0;
  if (blocks_per_sm(dev, fn, rn::kRingWarps * 32, l.smem, &bps)) return false;
  int64_t grid = (int64_t)sms * bps;
  const int64_t needed = ceil_div(tiles_max, rn::kRingWarps);
  if (needed < grid) grid = needed;
  if (const int go = g_grid_override.load(std::memory_order_relaxed)) grid = go;
  rn_launch_info& in = l.info;
  in.family = 0;
  in.threads_per_row = plans[0].lanes;
  in.chunks_per_thread = chunks;
  in.smem_bytes = l.smem;
  in.block_threads = rn::kRingWarps * 32;
  in.grid_blocks = (int32_t)grid;
  in.blocks_per_sm = bps;
  in.vector_y = plans[0].vector_y;
  in.phase_period = plans[0].phase_period;
  in.exact = slots == rn::kSlotsFull ? 2 : 1;
  in.staged = 1;
  in.stages = l.stages;
  in.stage_bytes = l.stage_bytes;
  *out = l;
  return true;
}

// Whether the planner uses the block rings by default for this block-family
// segment (it must qualify, see plan_cta_ring): blocks of 512 or more
// threads, which run two or fewer rows per SM at a time. Measured on B200
// (bf16 LayerNorm, 65536 rows, cold): D = 16384 (512 threads) 760.6 ->
// 722.9 us; at D = 8192 (256 threads) the register kernel with per-thread
// prefetch stayed ahead (352.5 against 374.8 us), and at 4097 (128 threads)
// too (204.9 against 222.2 us).
// (Measured again after the rings' register trim: D = 16384 768.9 -> 698.2 us,
// the same before and after a full bench run.) RMSNorm rows of blocks of 512
// threads ran faster on the register kernel with its prefetch (bf16, cold:
// D = 16384, 32768 rows, 356.2 -> 348.3 us; D = 12288, 16384 rows, 129.5 ->
// 123.0 us), so only LayerNorm takes the block rings by default.
bool cta_ring_preferred(const SegPlan& p, int op) { return op == rn::kOpLn && p.lanes >= 512; }

// Plans a block-ring launch for one RMSNorm / LayerNorm segment of the block
// family (any layout): by default where cta_ring_preferred says so,
// everywhere with rn_set_path_override(2), never with 1 or 3. Returns false
// (the register-kernel plan stays in charge) otherwise.
bool plan_cta_ring(int dtype, int op, const SegPlan* plans, const rn_view* const* xs, int nseg,
                   int slots, int dev, int sms, Launch* out) {
  const int path = g_path_override.load(std::memory_order_relaxed);
  if (path == 1 || path == 3 || nseg != 1) return false;
  if (op != rn::kOpRms && op != rn::kOpLn) return false;
  const SegPlan& p = plans[0];
  if (p.family != 1) return false;
  if (path == 0 && !cta_ring_preferred(p, op)) return false;
  const bool ex = p.exact != 0;
  const void* fn = dtype == RN_F32 ? rn::cta_ring_kernel_f32(op, ex, slots, p.lanes, p.chunks)
                                   : rn::cta_ring_kernel_bf16(op, ex, slots, p.lanes, p.chunks);
  if (!fn) return false;
  Launch l{};
  l.ring = 2;
  l.stages = rn::cta_ring_stages(p.lanes);
  l.stage_bytes = round_up(p.nfull_max * 16 > 16 ? p.nfull_max * 16 : 16, 16);
  const int cache = ex ? 0 : rn::affine_cache_smem_bytes(op, p.lanes, p.chunks);
  l.smem = l.stages * l.stage_bytes + cache;
  if (l.smem > device_info(dev).smem_per_block - 1024) return false;
  l.fn = fn;
  int bps = 0;
  if (blocks_per_sm(dev, fn, p.lanes, l.smem, &bps)) return false;
  int64_t grid = (int64_t)sms * bps;
  if (grid >= p.phase_period) grid -= grid % p.phase_period;
  if (xs[0]->rows < grid) grid = xs[0]->rows > 0 ? xs[0]->rows : 1;
  if (const int go = g_grid_override.load(std::memory_order_relaxed)) grid = go;
  rn_launch_info& in = l.info;
  in.family = 1;
  in.threads_per_row = p.lanes;
  in.chunks_per_thread = p.chunks;
  in.smem_bytes = l.smem;
  in.block_threads = p.lanes;
  in.grid_blocks = (int32_t)grid;
  in.blocks_per_sm = bps;
  in.vector_y = p.vector_y;
  in.phase_period = p.phase_period;
  in.exact = ex ? (slots == rn::kSlotsFull ? 2 : 1) : 0;
  in.staged = 1;
  in.stages = l.stages;
  in.stage_bytes = l.stage_bytes;
  *out = l;
  return true;
}

// Plans the launch for one or two segments that share one kernel: the
// per-warp bulk-copy rings where they apply and are chosen, else the register
// kernels.
int plan_launch(int dtype, int op, const SegPlan* plans, const rn_view* const* xs,
                const void* const* ws, const void* const* bs, int nseg, Launch* out,
                const rn_rope* rope = nullptr) {
  int64_t rows[2] = {xs[0]->rows, nseg > 1 ? xs[1]->rows : 0};
  SegPlan merged = plans[0];
  for (int i = 1; i < nseg; ++i) {
    if (plans[i].chunks > merged.chunks) merged.chunks = plans[i].chunks;
    merged.exact = merged.exact && plans[i].exact;
  }
  // every segment runs with the merged slot count
  int slots = rn::kSlotsFull;
  for (int i = 0; i < nseg; ++i) {
    const int c = slot_class(plans[i], merged.chunks);
    if (c < slots) slots = c;
  }
  if (!merged.exact && slots == rn::kSlotsFull) slots = rn::kSlotsTail;
  const void* fn = kernel_for(dtype, op, merged, slots);
  if (!fn) return fail(RN_ERR_UNSUPPORTED, "no compiled kernel for this shape");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(RN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  int sms = 0, bps = 0;
  int st = device_sms(dev, &sms);
  if (st) return st;
  if (plan_ring(dtype, op, plans, xs, nseg, merged.chunks, slots, dev, sms, rope, out))
    return RN_OK;
  if (plan_cta_ring(dtype, op, plans, xs, nseg, slots, dev, sms, out)) return RN_OK;
  const int threads = merged.family == 0 ? rn::kWarpBlock : merged.lanes;
  // the streaming kernels keep no weight cache and prefetch nothing
  const bool stream = merged.family == 2;
  const int cache = (merged.exact || stream)
                        ? 0
                        : rn::affine_cache_smem_bytes(op, threads, merged.chunks);
  const int stages =
      merged.family == 0 ? rn::kWarpPrefetchStages : rn::cta_prefetch_stages(threads, op);
  const int pf_bytes = rn::prefetch_slots_smem_bytes(threads, merged.chunks, stages) *
                       (rn::op_has_second(op) ? 2 : 1);
  // Prefetch of the rows ahead where it measured faster on B200 (bf16, 65536
  // rows, cold): lane groups; blocks of 256 or more threads (few blocks per
  // SM, so few rows in flight); blocks of 128 threads on rows off the
  // 16-byte grid (LayerNorm 4097: 203.6 -> 200.0 us with two stages, 186.4
  // us with one) and on LayerNorm rows
  // of at most 3 chunks per thread (D = 2048: 114.8 -> 110.7 us, 3072: 143.4
  // -> 137.2 us). Aligned rows in blocks of 128 threads otherwise keep 8 rows
  // per SM in flight and ran slower with it (LayerNorm 4096: 174.1 -> 177.0
  // us; RMSNorm 3072: 125.0 -> 135.3 us). Only when the slots fit beside the
  // weight cache (with a margin for the kernel's static shared memory).
  const int path = g_path_override.load(std::memory_order_relaxed);
  const bool want_prefetch =
      path == 3 ||
      (path == 0 && (merged.family == 0 || merged.lanes >= 256 || !merged.exact ||
                     (op == rn::kOpLn && merged.chunks <= 3)));
  const int prefetch =
      !stream && want_prefetch && cache + pf_bytes <= device_info(dev).smem_per_block - 1024
          ? 1
          : 0;
  int smem = cache + (prefetch ? pf_bytes : 0);
  out->stage_word = smem / 16;
  if (op == rn::kOpRmsRope) {
    // one binary32 staging row per lane group of the block
    int64_t stage = 0;
    for (int i = 0; i < nseg; ++i) {
      const int64_t b = (int64_t)(rn::kWarpBlock / plans[i].lanes) * xs[i]->dim * 4;
      if (b > stage) stage = b;
    }
    smem += (int)stage;
  }
  st = blocks_per_sm(dev, fn, threads, smem, &bps);
  if (st) return st;
  int64_t needed = 1;
  for (int i = 0; i < nseg; ++i) {
    int64_t n;
    if (merged.family == 0) {
      const int64_t groups_per_block = (rn::kWarpBlock / 32) * (32 / plans[i].lanes);
      n = ceil_div(rows[i], groups_per_block);
    } else {
      n = rows[i];
    }
    if (n > needed) needed = n;
  }
  int64_t grid = (int64_t)sms * bps;
  if (merged.family == 1 && grid >= plans[0].phase_period) {
    // Every block then sees rows of a single 16-byte phase, so it loads its
    // weight/bias registers once.
    grid -= grid % plans[0].phase_period;
  }
  if (needed < grid) grid = needed;
  if (const int go = g_grid_override.load(std::memory_order_relaxed)) grid = go;
  out->fn = fn;
  out->smem = smem;
  out->prefetch = prefetch;
  out->ring = 0;
  rn_launch_info& in = out->info;
  in.family = merged.family;
  in.threads_per_row = plans[0].lanes;
  in.chunks_per_thread = merged.chunks;
  in.smem_bytes = smem;
  in.block_threads = threads;
  in.grid_blocks = (int32_t)grid;
  in.blocks_per_sm = bps;
  in.vector_y = plans[0].vector_y;
  in.phase_period = plans[0].phase_period;
  in.exact = merged.exact ? (slots == rn::kSlotsFull ? 2 : 1) : 0;
  return RN_OK;
}

rn::Segment make_segment(const rn_view* x, const rn_view* y, const void* w, const void* b,
                         const SegPlan& p) {
  rn::Segment s{};
  s.x = x->data;
  s.y = y->data;
  s.w = w;
  s.b = b;
  s.rows = x->rows;
  s.x_stride = x->rows > 1 ? x->row_stride : x->dim;
  s.y_stride = y->rows > 1 ? y->row_stride : y->dim;
  s.x_inner = two_level(x) ? (int)x->inner_rows : 0;
  s.x_outer = x->outer_stride;
  s.y_inner = two_level(y) ? (int)y->inner_rows : 0;
  s.y_outer = y->outer_stride;
  s.dim = (int)x->dim;
  s.lanes = p.lanes;
  s.vector_y = p.vector_y;
  s.x2 = nullptr;
  s.h = nullptr;
  return s;
}

int launch(const Launch& l, const rn::Params& params, void* stream) {
  cudaError_t e;
  if (l.ring) {
    rn::RingParams rp{};
    for (int i = 0; i < 2; ++i) {
      rp.seg[i] = params.seg[i];
      rp.tile_rows[i] = i < params.nseg ? l.tile_rows[i] : 1;
      rp.contiguous[i] = l.contiguous[i];
    }
    rp.nseg = params.nseg;
    rp.eps = params.eps;
    rp.stages = l.stages;
    rp.stage_bytes = l.stage_bytes;
    const bool wait_test = g_ring_wait_test.load(std::memory_order_relaxed) != 0;
    rp.wait_ns = wait_test ? 1000000ull : rn::kRingWaitLimitNs;
    rp.drain_ns = wait_test ? 2000000ull : rn::kRingDrainLimitNs;
    rp.tx_extra = wait_test ? 16 : 0;
    rp.table_bytes = l.table_bytes;
    rp.affine_word = l.affine_word;
    void* args[] = {&rp};
    e = cudaLaunchKernel(l.fn, dim3((unsigned)l.info.grid_blocks),
                         dim3((unsigned)l.info.block_threads), args, (size_t)l.smem,
                         static_cast<cudaStream_t>(stream));
  } else {
    rn::Params pr = params;
    pr.prefetch = l.prefetch;
    pr.stage_word = l.stage_word;
    void* args[] = {&pr};
    e = cudaLaunchKernel(l.fn, dim3((unsigned)l.info.grid_blocks),
                         dim3((unsigned)l.info.block_threads), args, (size_t)l.smem,
                         static_cast<cudaStream_t>(stream));
  }
  if (e != cudaSuccess) return fail(RN_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(e));
  return RN_OK;
}

// Shared validation of a single-tensor op (RMSNorm / LayerNorm).
int validate_single(const rn_view* x, const void* w, const void* b, float eps,
                    const rn_view* y) {
  int st;
  if ((st = check_view(x, "x"))) return st;
  if ((st = check_view(y, "y"))) return st;
  if ((st = check_pair(x, y, "x", "y"))) return st;
  if ((st = check_eps(eps))) return st;
  if ((st = check_vector(w, x->dtype, "weight"))) return st;
  if ((st = check_vector(b, x->dtype, "bias"))) return st;
  const void* vecs[2] = {w, b};
  const int64_t dims[2] = {x->dim, x->dim};
  return check_output(y, x, nullptr, 0, vecs, dims, 2, "y");
}

// Streaming rows: LayerNorm reads each row three times, the last two from
// L2, so while several rows per SM fit there (rows of at most
// kStreamPairMaxRowBytes; at 38 registers 3 blocks of 512 threads run per
// SM, 444 rows in flight, 85 MB of the 126 MB L2 at the limit) it runs
// blocks of 512 threads, one row's passes overlapping the others'. Measured on B200: bf16 D = 65536 497 -> 412 us, binary32
// D = 32768 457 -> 404 us, bf16 D = 40001 1161 -> 993 us; at bf16
// D = 262144 (512 KB rows, which several per SM overflow L2) 642 -> 662 us.
// RMSNorm (two passes) ran slower with two blocks (381 -> 403 us at bf16
// D = 65536) and keeps one block of 1024.
SegPlan stream_plan(int op, const rn_view* x, SegPlan p) {
  const int64_t row_bytes = x->dim * elem_size(x->dtype);
  if (op == rn::kOpLn && row_bytes <= rn::kStreamPairMaxRowBytes) {
    p.lanes = rn::kStreamPairThreads;
    p.chunks = (int)ceil_div(x->dim / (16 / elem_size(x->dtype)), p.lanes);
  }
  return p;
}

int run_single(int op, const rn_view* x, const void* w, const void* b, float eps,
               const rn_view* y, void* stream, rn_launch_info* plan_only) {
  int st = validate_single(x, w, b, eps, y);
  if (st) return st;
  if (x->rows == 0 && !plan_only) return RN_OK;
  SegPlan p = plan_segment(x, y, w, b);
  if (p.family == 2) p = stream_plan(op, x, p);
  Launch l{};
  const rn_view* xs[1] = {x};
  const void* ws[1] = {w};
  const void* bs[1] = {b};
  if ((st = plan_launch(x->dtype, op, &p, xs, ws, bs, 1, &l))) return st;
  if (plan_only) {
    *plan_only = l.info;
    return RN_OK;
  }
  rn::Params params{};
  params.seg[0] = make_segment(x, y, w, b, p);
  params.nseg = 1;
  params.eps = eps;
  return launch(l, params, stream);
}

int run_dual(const rn_view* q, const rn_view* k, const void* wq, const void* wk, float eps,
             const rn_view* yq, const rn_view* yk, void* stream, rn_launch_info* plan_only) {
  int st;
  if ((st = check_view(q, "q"))) return st;
  if ((st = check_view(k, "k"))) return st;
  if ((st = check_view(yq, "yq"))) return st;
  if ((st = check_view(yk, "yk"))) return st;
  if (q->dtype != k->dtype) return fail(RN_ERR_DTYPE, "q and k differ in dtype");
  if ((st = check_pair(q, yq, "q", "yq"))) return st;
  if ((st = check_pair(k, yk, "k", "yk"))) return st;
  if (!wq || !wk) return fail(RN_ERR_NULL, "dual head norm: wq and wk are required");
  if ((st = check_eps(eps))) return st;
  if ((st = check_vector(wq, q->dtype, "wq"))) return st;
  if ((st = check_vector(wk, q->dtype, "wk"))) return st;
  if (q->dim > RN_MAX_HEAD_DIM || k->dim > RN_MAX_HEAD_DIM)
    return fail(RN_ERR_UNSUPPORTED, "dual head norm: head dims %lld, %lld above %d",
                (long long)q->dim, (long long)k->dim, RN_MAX_HEAD_DIM);
  const void* vecs[2] = {wq, wk};
  const int64_t dims[2] = {q->dim, k->dim};
  const rn_view* not_yq[2] = {k, yk};
  const rn_view* not_yk[1] = {q};
  if ((st = check_output(yq, q, not_yq, 2, vecs, dims, 2, "yq"))) return st;
  if ((st = check_output(yk, k, not_yk, 1, vecs, dims, 2, "yk"))) return st;
  if (q->rows == 0 && k->rows == 0 && !plan_only) return RN_OK;
  const SegPlan plans[2] = {plan_segment(q, yq, wq, nullptr), plan_segment(k, yk, wk, nullptr)};
  const rn_view* xs[2] = {q, k};
  const void* ws[2] = {wq, wk};
  const void* bs[2] = {nullptr, nullptr};
  Launch l{};
  if ((st = plan_launch(q->dtype, rn::kOpRms, plans, xs, ws, bs, 2, &l))) return st;
  if (plan_only) {
    *plan_only = l.info;
    return RN_OK;
  }
  rn::Params params{};
  params.seg[0] = make_segment(q, yq, wq, nullptr, plans[0]);
  params.seg[1] = make_segment(k, yk, wk, nullptr, plans[1]);
  params.nseg = 2;
  params.eps = eps;
  return launch(l, params, stream);
}

// Residual add + RMSNorm (op kOpAddRms: x2 = residual, h = stored sum) and
// gated RMSNorm (kOpGatedRms: x2 = gate, h unused).
int run_second(int op, const rn_view* x, const rn_view* x2, const void* w, float eps,
               const rn_view* y, const rn_view* h, void* stream, rn_launch_info* plan_only) {
  const bool add = op == rn::kOpAddRms;
  const char* x2n = add ? "residual" : "z";
  int st;
  if ((st = check_view(x, "x"))) return st;
  if ((st = check_view(x2, x2n))) return st;
  if ((st = check_view(y, "y"))) return st;
  if (add && (st = check_view(h, "h"))) return st;
  if ((st = check_pair(x, x2, "x", x2n))) return st;
  if ((st = check_pair(x, y, "x", "y"))) return st;
  if (add && (st = check_pair(x, h, "x", "h"))) return st;
  if ((st = check_eps(eps))) return st;
  if ((st = check_vector(w, x->dtype, "weight"))) return st;
  if (x->dim > register_max_dim(x->dtype))
    return fail(RN_ERR_UNSUPPORTED, "%s: dim %lld above %lld (fused ops hold rows in registers)",
                add ? "add_rms_norm" : "gated_rms_norm", (long long)x->dim,
                (long long)register_max_dim(x->dtype));
  if (!same_phase(x, x2))
    return fail(RN_ERR_ALIGN, "%s rows must share x's 16-byte alignment", x2n);
  if (add && !same_phase(x, h))
    return fail(RN_ERR_ALIGN, "h rows must share x's 16-byte alignment");
  const void* vecs[1] = {w};
  const int64_t dims[1] = {x->dim};
  // y may be x itself; it must not touch the second input, h or the weight
  const rn_view* not_y[2] = {x2, h};
  if ((st = check_output(y, x, not_y, add ? 2 : 1, vecs, dims, 1, "y"))) return st;
  if (add) {
    // h may be x or the residual exactly (an in-place residual stream)
    const Span sh = span_of(h);
    if (views_overlap(h, x) && !same_view(h, x))
      return fail(RN_ERR_OVERLAP, "h partially overlaps x");
    if (views_overlap(h, x2) && !same_view(h, x2))
      return fail(RN_ERR_OVERLAP, "h partially overlaps the residual");
    if (w && intersects(sh, span_of_vector(w, x->dim, x->dtype)))
      return fail(RN_ERR_OVERLAP, "h overlaps the weight");
  }
  if (x->rows == 0 && !plan_only) return RN_OK;
  const SegPlan p = plan_segment(x, y, w, nullptr);
  Launch l{};
  const rn_view* xs[1] = {x};
  const void* ws[1] = {w};
  const void* bs[1] = {nullptr};
  if ((st = plan_launch(x->dtype, op, &p, xs, ws, bs, 1, &l))) return st;
  if (plan_only) {
    *plan_only = l.info;
    return RN_OK;
  }
  rn::Params params{};
  params.seg[0] = make_segment(x, y, w, nullptr, p);
  params.seg[0].x2 = x2->data;
  params.seg[0].x2_stride = x2->rows > 1 ? x2->row_stride : x2->dim;
  params.seg[0].x2_inner = two_level(x2) ? (int)x2->inner_rows : 0;
  params.seg[0].x2_outer = x2->outer_stride;
  if (add) {
    params.seg[0].h = h->data;
    params.seg[0].h_stride = h->rows > 1 ? h->row_stride : h->dim;
    params.seg[0].h_inner = two_level(h) ? (int)h->inner_rows : 0;
    params.seg[0].h_outer = h->outer_stride;
  }
  params.nseg = 1;
  params.eps = eps;
  return launch(l, params, stream);
}

// Dual q/k head RMSNorm followed by RoPE, one launch over both row spaces.
int run_dual_rope(const rn_view* q, const rn_view* k, const void* wq, const void* wk, float eps,
                  const rn_rope* rope, const rn_view* yq, const rn_view* yk, void* stream) {
  int st;
  if (!rope) return fail(RN_ERR_NULL, "rope is NULL");
  if ((st = check_view(q, "q"))) return st;
  if ((st = check_view(k, "k"))) return st;
  if ((st = check_view(yq, "yq"))) return st;
  if ((st = check_view(yk, "yk"))) return st;
  if (q->dtype != k->dtype) return fail(RN_ERR_DTYPE, "q and k differ in dtype");
  if ((st = check_pair(q, yq, "q", "yq"))) return st;
  if ((st = check_pair(k, yk, "k", "yk"))) return st;
  if (!wq || !wk) return fail(RN_ERR_NULL, "dual head norm: wq and wk are required");
  if ((st = check_eps(eps))) return st;
  if ((st = check_vector(wq, q->dtype, "wq"))) return st;
  if ((st = check_vector(wk, q->dtype, "wk"))) return st;
  if (q->dim > RN_MAX_HEAD_DIM || k->dim > RN_MAX_HEAD_DIM)
    return fail(RN_ERR_UNSUPPORTED, "dual head norm: head dims %lld, %lld above %d",
                (long long)q->dim, (long long)k->dim, RN_MAX_HEAD_DIM);
  if (rope->heads_q < 1 || rope->heads_k < 1)
    return fail(RN_ERR_SHAPE, "rope: head counts must be >= 1");
  if (q->rows % rope->heads_q || k->rows % rope->heads_k)
    return fail(RN_ERR_SHAPE, "rope: rows are not whole tokens of heads");
  const int64_t tokens = q->rows / rope->heads_q;
  if (k->rows / rope->heads_k != tokens)
    return fail(RN_ERR_SHAPE, "rope: q has %lld tokens, k has %lld", (long long)tokens,
                (long long)(k->rows / rope->heads_k));
  if (rope->dims < 0 || rope->dims % 2 || rope->dims > q->dim || rope->dims > k->dim)
    return fail(RN_ERR_SHAPE, "rope: dims %d must be even and <= both head dims",
                (int)rope->dims);
  if (rope->offset < 0 || rope->n_pos < 0 || (tokens > 0 && rope->offset + tokens > rope->n_pos))
    return fail(RN_ERR_SHAPE, "rope: positions [%lld, %lld) outside the table's %lld",
                (long long)rope->offset, (long long)(rope->offset + tokens),
                (long long)rope->n_pos);
  if (rope->dims > 0 && tokens > 0 && !rope->table) return fail(RN_ERR_NULL, "rope: table is NULL");
  if (reinterpret_cast<uintptr_t>(rope->table) % 4)
    return fail(RN_ERR_ALIGN, "rope: table not aligned to 4 bytes");
  // the table (binary32, n_pos x dims) is checked as a vector of the outputs' type
  const void* vecs[3] = {wq, wk, rope->table};
  const int64_t dims[3] = {q->dim, k->dim, rope->n_pos * rope->dims * 4 / elem_size(q->dtype)};
  const rn_view* not_yq[2] = {k, yk};
  const rn_view* not_yk[1] = {q};
  if ((st = check_output(yq, q, not_yq, 2, vecs, dims, 3, "yq"))) return st;
  if ((st = check_output(yk, k, not_yk, 1, vecs, dims, 3, "yk"))) return st;
  if (q->rows == 0 && k->rows == 0) return RN_OK;
  const SegPlan plans[2] = {plan_segment(q, yq, wq, nullptr), plan_segment(k, yk, wk, nullptr)};
  const rn_view* xs[2] = {q, k};
  const void* ws[2] = {wq, wk};
  const void* bs[2] = {nullptr, nullptr};
  // in-thread planes when every plane's partner is the same thread's: on
  // 16-byte aligned rows whose rotated width is a multiple of 2 V, either
  // interleaved planes, or full split-half rotary whose chunks divide evenly
  // over an even slot count (slot p's partner is slot p + slots / 2)
  const int V = 16 / elem_size(q->dtype);
  const int slots = plans[0].chunks > plans[1].chunks ? plans[0].chunks : plans[1].chunks;
  bool local = rope->dims > 0 && rope->dims % (2 * V) == 0;
  for (int i = 0; i < 2; ++i) {
    local = local && plans[i].exact;
    if (!rope->traditional)
      local = local && slots % 2 == 0 && rope->dims / 2 == plans[i].lanes * (slots / 2) * V;
  }
  Launch l{};
  if ((st = plan_launch(q->dtype, local ? rn::kOpRmsRopeLocal : rn::kOpRmsRope, plans, xs, ws,
                        bs, 2, &l, rope)))
    return st;
  rn::Params params{};
  params.seg[0] = make_segment(q, yq, wq, nullptr, plans[0]);
  params.seg[1] = make_segment(k, yk, wk, nullptr, plans[1]);
  const int heads[2] = {(int)rope->heads_q, (int)rope->heads_k};
  for (int i = 0; i < 2; ++i) {
    params.seg[i].rope_table = rope->table;
    params.seg[i].rope_offset = rope->offset;
    params.seg[i].rope_heads = heads[i];
    params.seg[i].rope_dims = rope->dims;
    params.seg[i].rope_trad = rope->traditional ? 1 : 0;
  }
  params.nseg = 2;
  params.eps = eps;
  return launch(l, params, stream);
}

}  // namespace

extern "C" {

RN_API int rn_rms_norm(const rn_view* x, const void* weight, float eps, const rn_view* y,
                       void* stream) {
  return run_single(rn::kOpRms, x, weight, nullptr, eps, y, stream, nullptr);
}

RN_API int rn_layer_norm(const rn_view* x, const void* weight, const void* bias, float eps,
                         const rn_view* y, void* stream) {
  return run_single(rn::kOpLn, x, weight, bias, eps, y, stream, nullptr);
}

RN_API int rn_add_rms_norm(const rn_view* x, const rn_view* residual, const void* weight,
                           float eps, const rn_view* y, const rn_view* h, void* stream) {
  return run_second(rn::kOpAddRms, x, residual, weight, eps, y, h, stream, nullptr);
}

RN_API int rn_gated_rms_norm(const rn_view* x, const rn_view* z, const void* weight, float eps,
                             const rn_view* y, void* stream) {
  return run_second(rn::kOpGatedRms, x, z, weight, eps, y, nullptr, stream, nullptr);
}

RN_API int rn_dual_head_rms_norm_rope(const rn_view* q, const rn_view* k, const void* wq,
                                      const void* wk, float eps, const rn_rope* rope,
                                      const rn_view* yq, const rn_view* yk, void* stream) {
  return run_dual_rope(q, k, wq, wk, eps, rope, yq, yk, stream);
}

RN_API int rn_rope_table(int32_t dims, float base, float scale, const float* inv_freq,
                         int64_t n_pos, float* table) {
  if (dims < 0 || dims % 2) return fail(RN_ERR_SHAPE, "rope table: dims %d must be even", dims);
  if (n_pos < 0) return fail(RN_ERR_SHAPE, "rope table: n_pos < 0");
  if (n_pos > 0 && dims > 0 && !table) return fail(RN_ERR_NULL, "rope table: table is NULL");
  if (!inv_freq && !(base > 0.0f && std::isfinite(base)))
    return fail(RN_ERR_EPS, "rope table: base must be finite and > 0");
  if (!std::isfinite(scale)) return fail(RN_ERR_EPS, "rope table: scale must be finite");
  const int half = dims / 2;
  for (int i = 0; i < half; ++i) {
    const double f = inv_freq ? (double)inv_freq[i]
                              : std::pow((double)base, -2.0 * (double)i / (double)dims);
    for (int64_t p = 0; p < n_pos; ++p) {
      const double theta = (double)p * (double)scale * f;
      table[p * dims + i] = (float)std::cos(theta);
      table[p * dims + half + i] = (float)std::sin(theta);
    }
  }
  return RN_OK;
}

RN_API int rn_dual_head_rms_norm(const rn_view* q, const rn_view* k, const void* wq,
                                 const void* wk, float eps, const rn_view* yq,
                                 const rn_view* yk, void* stream) {
  return run_dual(q, k, wq, wk, eps, yq, yk, stream, nullptr);
}

RN_API const char* rn_status_string(int status) {
  switch (status) {
    case RN_OK: return "ok";
    case RN_ERR_NULL: return "a required pointer is NULL";
    case RN_ERR_SHAPE: return "invalid or mismatched shape";
    case RN_ERR_DTYPE: return "unknown or mixed element types";
    case RN_ERR_EPS: return "eps must be finite and non-negative";
    case RN_ERR_ALIGN: return "pointer not aligned to its element size";
    case RN_ERR_OVERLAP: return "an output overlaps an input or another output";
    case RN_ERR_UNSUPPORTED: return "dimension not supported";
    case RN_ERR_CUDA: return "CUDA runtime error";
    default: return "unknown status";
  }
}

RN_API const char* rn_last_error(void) { return g_last_error; }

RN_API int rn_abi_version(void) { return RN_ABI_VERSION; }

RN_API int rn_plan(int op, const rn_view* x, const rn_view* y, const rn_view* x2,
                   const rn_view* y2, const void* weight, const void* bias,
                   rn_launch_info* info) {
  if (!info) return fail(RN_ERR_NULL, "info is NULL");
  if (op == RN_OP_DUAL) return run_dual(x, x2, weight, bias, 1e-6f, y, y2, nullptr, info);
  if (op == RN_OP_RMS) return run_single(rn::kOpRms, x, weight, nullptr, 1e-6f, y, nullptr, info);
  if (op == RN_OP_LN) return run_single(rn::kOpLn, x, weight, bias, 1e-6f, y, nullptr, info);
  if (op == RN_OP_ADD_RMS)
    return run_second(rn::kOpAddRms, x, x2, weight, 1e-6f, y, y2, nullptr, info);
  if (op == RN_OP_GATED_RMS)
    return run_second(rn::kOpGatedRms, x, x2, weight, 1e-6f, y, nullptr, nullptr, info);
  return fail(RN_ERR_UNSUPPORTED, "unknown op %d", op);
}

RN_API int rn_set_grid_override(int blocks) {
  if (blocks < 0) return fail(RN_ERR_SHAPE, "grid override must be >= 0");
  g_grid_override.store(blocks, std::memory_order_relaxed);
  return RN_OK;
}

RN_API int rn_set_path_override(int path) {
  if (path < 0 || path > 3) return fail(RN_ERR_SHAPE, "path override must be 0, 1, 2 or 3");
  g_path_override.store(path, std::memory_order_relaxed);
  return RN_OK;
}

RN_API int rn_set_ring_wait_test(int on) {
  if (on != 0 && on != 1) return fail(RN_ERR_SHAPE, "ring wait test must be 0 or 1");
  g_ring_wait_test.store(on, std::memory_order_relaxed);
  return RN_OK;
}

RN_API int rn_device_error_count(unsigned int* count, int reset) {
  if (!count) return fail(RN_ERR_NULL, "count is NULL");
  unsigned int a = 0, b = 0;
  unsigned int c = 0, d = 0;
  int e = rn::ring_timeouts_f32(&a, reset != 0);
  if (e == 0) e = rn::ring_timeouts_bf16(&b, reset != 0);
  if (e == 0) e = rn::cta_ring_timeouts_f32(&c, reset != 0);
  if (e == 0) e = rn::cta_ring_timeouts_bf16(&d, reset != 0);
  if (e != 0)
    return fail(RN_ERR_CUDA, "device error counter: %s", cudaGetErrorString((cudaError_t)e));
  *count = a + b + c + d;
  return RN_OK;
}

}  // extern "C"
