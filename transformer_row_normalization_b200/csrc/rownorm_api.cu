// C ABI of librownorm.so: argument validation, launch planning and dispatch.
// The operations and conventions are documented in include/rownorm.h.
#include <cuda_runtime.h>

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

namespace {

thread_local char g_last_error[512] = "";
int g_grid_override = 0;

int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return status;
}

int elem_size(int dtype) { return dtype == RN_F32 ? 4 : 2; }

// rows == 0 views are valid (they enqueue nothing); the checks below still
// run so that malformed descriptors are reported consistently.
int check_view(const rn_view* v, const char* name) {
  if (!v) return fail(RN_ERR_NULL, "%s: view pointer is NULL", name);
  if (v->dtype != RN_F32 && v->dtype != RN_BF16)
    return fail(RN_ERR_DTYPE, "%s: unknown dtype %d", name, (int)v->dtype);
  if (v->rows < 0) return fail(RN_ERR_SHAPE, "%s: rows %lld < 0", name, (long long)v->rows);
  if (v->dim < 1) return fail(RN_ERR_SHAPE, "%s: dim %lld < 1", name, (long long)v->dim);
  if (v->rows > 1 && v->row_stride < v->dim)
    return fail(RN_ERR_SHAPE, "%s: row_stride %lld < dim %lld", name,
                (long long)v->row_stride, (long long)v->dim);
  const int es = elem_size(v->dtype);
  if (v->rows > 1) {
    const int64_t limit = (INT64_MAX / es - v->dim) / (v->rows - 1);
    if (v->row_stride > limit) return fail(RN_ERR_SHAPE, "%s: extent overflows", name);
  }
  if (v->rows > 0 && !v->data) return fail(RN_ERR_NULL, "%s: data is NULL", name);
  if (reinterpret_cast<uintptr_t>(v->data) % es)
    return fail(RN_ERR_ALIGN, "%s: data not aligned to its %d-byte element", name, es);
  const int64_t max_dim = v->dtype == RN_F32 ? RN_MAX_DIM_F32 : RN_MAX_DIM_BF16;
  if (v->dim > max_dim)
    return fail(RN_ERR_UNSUPPORTED, "%s: dim %lld above the supported maximum %lld", name,
                (long long)v->dim, (long long)max_dim);
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
  const int64_t n = (v->rows - 1) * v->row_stride + v->dim;
  return {lo, lo + static_cast<uintptr_t>(n) * elem_size(v->dtype)};
}

Span span_of_vector(const void* p, int64_t dim, int dtype) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return {lo, p ? lo + static_cast<uintptr_t>(dim) * elem_size(dtype) : lo};
}

bool intersects(Span a, Span b) { return a.lo < b.hi && b.lo < a.hi && a.lo != a.hi && b.lo != b.hi; }

bool same_view(const rn_view* a, const rn_view* b) {
  return a->data == b->data && (a->rows <= 1 || a->row_stride == b->row_stride);
}

// An output may be its own input exactly, and must not touch anything else.
int check_output(const rn_view* y, const rn_view* x_own, const rn_view* const* others,
                 int n_others, const void* const* vecs, const int64_t* vec_dims,
                 int n_vecs, const char* name) {
  const Span sy = span_of(y);
  if (intersects(sy, span_of(x_own)) && !same_view(y, x_own))
    return fail(RN_ERR_OVERLAP, "%s partially overlaps its input", name);
  for (int i = 0; i < n_others; ++i)
    if (intersects(sy, span_of(others[i])))
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

constexpr int kWarpFamilyMaxDim = 1024;

int pow2_ceil(int64_t v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct SegPlan {
  int family;        // 0 warp, 1 block
  int lanes;         // family 0: lanes per row; family 1: threads per block
  int chunks;        // capacity of 16-byte chunks per thread
  int vector_y;      // y rows share x's 16-byte phase
  int phase_period;  // distinct 16-byte phases among the rows of x
  int exact;         // every x and y row 16-byte aligned, dim % V == 0
};

// The lane count / block size is a function of (dtype, dim) only, so the
// summation tree of a row never depends on the call; `chunks` (register
// capacity) may grow for rows that are not 16-byte aligned, which only adds
// empty slots.
SegPlan plan_segment(const rn_view* x, const rn_view* y, const void* w, const void* b) {
  const int es = elem_size(x->dtype);
  const int V = 16 / es;
  const int64_t D = x->dim;
  const uintptr_t xa = reinterpret_cast<uintptr_t>(x->data);
  const bool rows_aligned = (xa % 16 == 0) && (D % V == 0) &&
                            (x->rows <= 1 || (x->row_stride * es) % 16 == 0);
  const int64_t nch = rows_aligned ? D / V : (D + 2 * V - 2) / V;
  SegPlan p{};
  const int per_thread = rn::kTargetChunksPerThread;
  if (D <= kWarpFamilyMaxDim) {
    p.family = 0;
    int g = pow2_ceil(ceil_div(ceil_div(D, V), per_thread));
    p.lanes = g > 32 ? 32 : g;
    p.chunks = (int)ceil_div(nch, p.lanes);
  } else {
    p.family = 1;
    int nt = pow2_ceil(ceil_div(ceil_div(D, V), per_thread));
    p.lanes = nt < 128 ? 128 : (nt > 1024 ? 1024 : nt);
    p.chunks = (int)ceil_div(nch, p.lanes);
    if (p.chunks < rn::kCtaMinChunks) p.chunks = rn::kCtaMinChunks;
  }
  const uintptr_t ya = reinterpret_cast<uintptr_t>(y->data);
  p.vector_y = ((ya - xa) % 16 == 0) &&
               (x->rows <= 1 || (((y->row_stride - x->row_stride) * es) % 16 == 0));
  p.phase_period = 1;
  if (x->rows > 1) {
    int64_t step = (x->row_stride * es) % 16;  // row-to-row phase advance, bytes
    int period = 1;
    for (int64_t acc = step; acc % 16 != 0; acc += step) ++period;
    p.phase_period = period;
  }
  p.exact = rows_aligned && ya % 16 == 0 &&
            (y->rows <= 1 || (y->row_stride * es) % 16 == 0);
  (void)w;
  (void)b;
  return p;
}

const void* kernel_for(int dtype, int op, const SegPlan& p) {
  const bool ex = p.exact != 0;
  if (p.family == 0)
    return dtype == RN_F32 ? rn::warp_kernel_f32(op, ex, p.chunks)
                           : rn::warp_kernel_bf16(op, ex, p.chunks);
  return dtype == RN_F32 ? rn::cta_kernel_f32(op, ex, p.lanes, p.chunks)
                         : rn::cta_kernel_bf16(op, ex, p.lanes, p.chunks);
}

struct DeviceInfo {
  int sms = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[64];
std::unordered_map<const void*, int> g_occ[64];

int device_sms(int dev, int* sms) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (dev < 0 || dev >= 64) return fail(RN_ERR_CUDA, "device ordinal %d out of range", dev);
  if (!g_dev[dev].sms) {
    cudaError_t e = cudaDeviceGetAttribute(&g_dev[dev].sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(RN_ERR_CUDA, "SM count query: %s", cudaGetErrorString(e));
  }
  *sms = g_dev[dev].sms;
  return RN_OK;
}

// Also raises the kernel's dynamic shared memory limit the first time a
// configuration needs more than the default 48 KB.
int blocks_per_sm(int dev, const void* fn, int threads, int smem, int* out) {
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_occ[dev].find(fn);
  if (it != g_occ[dev].end()) {
    *out = it->second;
    return RN_OK;
  }
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess)
    return fail(RN_ERR_CUDA, "shared memory attribute: %s", cudaGetErrorString(e));
  int n = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem);
  if (e != cudaSuccess) return fail(RN_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
  if (n < 1) n = 1;
  g_occ[dev][fn] = n;
  *out = n;
  return RN_OK;
}

struct Launch {
  const void* fn;
  int smem;
  rn_launch_info info;
};

// Plans the launch for one or two segments that share one kernel.
int plan_launch(int dtype, int op, const SegPlan* plans, const int64_t* rows, int nseg,
                Launch* out) {
  SegPlan merged = plans[0];
  for (int i = 1; i < nseg; ++i) {
    if (plans[i].chunks > merged.chunks) merged.chunks = plans[i].chunks;
    merged.exact = merged.exact && plans[i].exact;
  }
  const void* fn = kernel_for(dtype, op, merged);
  if (!fn) return fail(RN_ERR_UNSUPPORTED, "no compiled kernel for this shape");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(RN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  int sms = 0, bps = 0;
  int st = device_sms(dev, &sms);
  if (st) return st;
  const int threads = merged.family == 0 ? rn::kWarpBlock : merged.lanes;
  const int smem = rn::affine_smem_bytes(op, threads, merged.chunks);
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
  if (g_grid_override > 0) grid = g_grid_override;
  out->fn = fn;
  out->smem = smem;
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
  in.exact = merged.exact;
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
  s.dim = (int)x->dim;
  s.lanes = p.lanes;
  s.vector_y = p.vector_y;
  return s;
}

int launch(const Launch& l, const rn::Params& params, void* stream) {
  void* args[] = {const_cast<rn::Params*>(&params)};
  cudaError_t e = cudaLaunchKernel(l.fn, dim3((unsigned)l.info.grid_blocks),
                                   dim3((unsigned)l.info.block_threads), args, (size_t)l.smem,
                                   static_cast<cudaStream_t>(stream));
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

int run_single(int op, const rn_view* x, const void* w, const void* b, float eps,
               const rn_view* y, void* stream, rn_launch_info* plan_only) {
  int st = validate_single(x, w, b, eps, y);
  if (st) return st;
  if (x->rows == 0 && !plan_only) return RN_OK;
  const SegPlan p = plan_segment(x, y, w, b);
  Launch l{};
  const int64_t rows = x->rows > 0 ? x->rows : 1;
  if ((st = plan_launch(x->dtype, op, &p, &rows, 1, &l))) return st;
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
  const int64_t rows[2] = {q->rows, k->rows};
  Launch l{};
  if ((st = plan_launch(q->dtype, rn::kOpRms, plans, rows, 2, &l))) return st;
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
  return fail(RN_ERR_UNSUPPORTED, "unknown op %d", op);
}

RN_API int rn_set_grid_override(int blocks) {
  if (blocks < 0) return fail(RN_ERR_SHAPE, "grid override must be >= 0");
  g_grid_override = blocks;
  return RN_OK;
}

}  // extern "C"
