// Fused last-axis row normalization kernels for sm_100a.
//
// What is computed (per row of D elements, binary32 arithmetic):
//   RMSNorm   ("Emily.Fast", rms_norm/3):
//               ss   = sum_i x_i^2
//               rstd = rsqrt(ss / D + eps)
//               y_j  = (x_j * rstd) * w_j
//   LayerNorm ("Emily.Fast", layer_norm/4; population variance):
//               K    = x_0                       (shift: a constant row gives
//               d_i  = x_i - K                    exactly zero deviations)
//               mean = (sum_i d_i) / D
//               var  = (sum_i (d_i - mean)^2) / D
//               rstd = rsqrt(var + eps)
//               y_j  = ((d_j - mean) * rstd) * w_j + b_j   (one fused multiply-add)
//   The page calls its LayerNorm statistic "Welford-style"; the two passes
//   above run over a row already held in registers, so they cost no extra
//   HBM traffic and give the same population mean and variance.
//
// Data movement. A row is read from HBM exactly once, into registers, as
// 16-byte chunks aligned to the 16-byte address grid: chunk k of a row whose
// first element sits `phase` elements past a 16-byte boundary covers columns
// [k*V - phase, k*V - phase + V), V = 16 / sizeof(element). Chunks lying
// wholly inside the row move with one 16-byte load / store; the (at most two)
// partial chunks at the row ends move element by element, so no byte outside
// the caller's views is touched.
//
// Weight and bias. A thread always owns the same chunk slots of every row it
// handles, and rows are strided over threads so that (for the block family
// when the grid is a multiple of the phase period, and always for the lane
// group family) all rows a thread sees share one 16-byte phase. So each
// thread copies the weight/bias columns of its chunks once, realigned to its
// x chunks, into its own slots of shared memory, and recopies them only if a
// row arrives with a different phase.
//
// Summation order (fixed; it depends only on D, the element type and the
// row's 16-byte phase): each thread accumulates its chunks in increasing
// chunk order and, inside a chunk, in increasing column order; then an xor
// butterfly across the lanes that share the row (offsets G/2 .. 1); in the
// block-per-row family the per-warp sums are then added by every thread in
// warp order 0 .. NW-1. Butterfly partners add the same two values, so all
// lanes end with bit-identical totals.
//
// Two families:
//   rows_warp_kernel  a group of G lanes (G = 1..32, a power of two) of one
//                     warp owns a row; G is chosen so each lane holds about
//                     four 16-byte chunks. Used for D <= 1024.
//   rows_cta_kernel   one block of NT threads owns a row. Used for D > 1024.
// Both are persistent: the grid is sized to the SM count times resident
// blocks per SM, and rows are strided statically over the lane groups /
// blocks (no atomics, no work queue, no inter-block communication, no waits
// other than __syncthreads).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace rn {

enum : int { kOpRms = 0, kOpLn = 1 };

// One row space (a tensor viewed as [rows, dim]); strides in elements.
struct Segment {
  const void* x;
  void* y;
  const void* w;   // nullptr: all ones
  const void* b;   // nullptr: all zeros (LayerNorm only)
  long long rows;
  long long x_stride;
  long long y_stride;
  int dim;
  int lanes;       // rows_warp_kernel: lanes per row (power of two <= 32)
  int vector_y;    // 1: every y row has its x row's 16-byte phase
  int pad_;
};

struct Params {
  Segment seg[2];
  int nseg;
  float eps;
};

// ---------------------------------------------------------------------------
// element types

template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int V = 4;
  static constexpr uint32_t kOneBits = 0x3f800000u;
  static __device__ __forceinline__ float get(const float* p) { return *p; }
  static __device__ __forceinline__ uint32_t get_bits(const float* p) {
    return __float_as_uint(*p);
  }
  static __device__ __forceinline__ void put(float* p, float v) { *p = v; }
  static __device__ __forceinline__ void unpack(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
  static __device__ __forceinline__ uint4 pack(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                      __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
  // 4 element bit patterns -> one chunk
  static __device__ __forceinline__ uint4 assemble(const uint32_t (&e)[4]) {
    return make_uint4(e[0], e[1], e[2], e[3]);
  }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int V = 8;
  static constexpr uint32_t kOneBits = 0x3f80u;
  static __device__ __forceinline__ float get(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
  }
  static __device__ __forceinline__ uint32_t get_bits(const __nv_bfloat16* p) {
    return *reinterpret_cast<const unsigned short*>(p);
  }
  static __device__ __forceinline__ void put(__nv_bfloat16* p, float v) {
    *p = __float2bfloat16_rn(v);
  }
  static __device__ __forceinline__ float2 pair(uint32_t w) {
    __nv_bfloat162 h;
    *reinterpret_cast<uint32_t*>(&h) = w;
    return __bfloat1622float2(h);
  }
  static __device__ __forceinline__ uint32_t pack_pair(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ void unpack(const uint4& u, float (&f)[8]) {
    float2 t;
    t = pair(u.x); f[0] = t.x; f[1] = t.y;
    t = pair(u.y); f[2] = t.x; f[3] = t.y;
    t = pair(u.z); f[4] = t.x; f[5] = t.y;
    t = pair(u.w); f[6] = t.x; f[7] = t.y;
  }
  static __device__ __forceinline__ uint4 pack(const float (&f)[8]) {
    return make_uint4(pack_pair(f[0], f[1]), pack_pair(f[2], f[3]),
                      pack_pair(f[4], f[5]), pack_pair(f[6], f[7]));
  }
  static __device__ __forceinline__ uint4 assemble(const uint32_t (&e)[8]) {
    return make_uint4(e[0] | (e[1] << 16), e[2] | (e[3] << 16), e[4] | (e[5] << 16),
                      e[6] | (e[7] << 16));
  }
};

// ---------------------------------------------------------------------------
// memory access (16-byte chunks)

__device__ __forceinline__ uint4 load_stream(const void* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void store_stream(void* p, const uint4& v) {
  __stcs(reinterpret_cast<uint4*>(p), v);
}
__device__ __forceinline__ uint4 load_cached(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// Geometry of one row.
template <typename T>
struct Row {
  const T* x_al;   // x row start minus phase: 16-byte aligned
  T* y_row;        // y row start
  int phase;       // elements between the 16-byte boundary and the row start
  int nch;         // chunks touched by the row
  int tail_full;   // 1: the last chunk ends exactly at the row end
};

// EXACT: the caller guarantees every x and y row starts on a 16-byte
// boundary and D is a multiple of V, so every chunk is full and the phase is
// 0 (the planner checks this on the host).
template <typename T, bool EXACT>
__device__ __forceinline__ Row<T> row_geometry(const Segment& s, long long r) {
  constexpr int V = Elem<T>::V;
  Row<T> g;
  const T* xr = static_cast<const T*>(s.x) + r * s.x_stride;
  g.phase = EXACT ? 0 : (int)((reinterpret_cast<uintptr_t>(xr) & 15u) / sizeof(T));
  g.x_al = xr - g.phase;
  g.y_row = static_cast<T*>(s.y) + r * s.y_stride;
  g.nch = EXACT ? s.dim / V : (g.phase + s.dim + V - 1) / V;
  g.tail_full = EXACT ? 1 : (((g.phase + s.dim) % V) == 0);
  return g;
}

template <typename T, bool EXACT>
__device__ __forceinline__ bool chunk_full(const Row<T>& g, int k) {
  if constexpr (EXACT) return k < g.nch;
  return k < g.nch && (k > 0 || g.phase == 0) && (k < g.nch - 1 || g.tail_full);
}

// Load chunk k of a row into binary32 registers; columns outside [0, D)
// (and chunks past the row) read as 0 and are never dereferenced.
template <typename T, bool EXACT>
__device__ __forceinline__ void load_chunk(const Row<T>& g, int D, int k,
                                           float (&f)[Elem<T>::V]) {
  constexpr int V = Elem<T>::V;
  if (chunk_full<T, EXACT>(g, k)) {
    Elem<T>::unpack(load_stream(g.x_al + (long long)k * V), f);
  } else if constexpr (EXACT) {
#pragma unroll
    for (int e = 0; e < V; ++e) f[e] = 0.f;
  } else {
#pragma unroll
    for (int e = 0; e < V; ++e) {
      const int c = k * V + e - g.phase;
      f[e] = ((unsigned)c < (unsigned)D) ? Elem<T>::get(g.x_al + k * V + e) : 0.f;
    }
  }
}

// Weight and bias bit patterns for the chunk slots a thread owns, aligned to
// the columns of its x chunks in one row phase, cached in shared memory at
// [slot][thread] (each thread reads and writes only its own entries, so no
// barrier is involved; consecutive threads touch consecutive 16-byte words,
// so accesses are bank-conflict free). A NULL weight reads as ones, a NULL
// bias as zeros.
template <typename T, int NSLOT, bool BIAS>
struct Affine {
  uint4* w;        // [NSLOT][blockDim.x]
  uint4* b;        // [NSLOT][blockDim.x] (BIAS only)
  int phase;
};

template <int NSLOT, bool BIAS>
__device__ __forceinline__ constexpr int affine_smem_bytes_per_thread() {
  return NSLOT * 16 * (BIAS ? 2 : 1);
}

template <typename T, int NSLOT, bool BIAS>
__device__ __forceinline__ Affine<T, NSLOT, BIAS> affine_in_smem(unsigned char* smem) {
  Affine<T, NSLOT, BIAS> a;
  a.w = reinterpret_cast<uint4*>(smem);
  a.b = a.w + NSLOT * blockDim.x;
  a.phase = -1;
  return a;
}

template <typename T, int NSLOT, bool BIAS>
__device__ __forceinline__ void load_affine(const Segment& s, int phase, int k0, int step,
                                            Affine<T, NSLOT, BIAS>& a) {
  constexpr int V = Elem<T>::V;
  const T* w = static_cast<const T*>(s.w);
  const T* b = static_cast<const T*>(s.b);
  const int D = s.dim;
  const int me = threadIdx.x;
  const int nthr = blockDim.x;
#pragma unroll
  for (int p = 0; p < NSLOT; ++p) {
    const int c0 = (k0 + step * p) * V - phase;
    // columns c0 .. c0+V-1 inside [0, D) starting on a 16-byte boundary of
    // the vector: one aligned load; otherwise element by element
    const bool inside = c0 >= 0 && c0 + V <= D;
    uint4 wv;
    if (w && inside && (reinterpret_cast<uintptr_t>(w + c0) & 15u) == 0) {
      wv = load_cached(w + c0);
    } else {
      uint32_t e[V];
#pragma unroll
      for (int i = 0; i < V; ++i) {
        const int c = c0 + i;
        e[i] = (w && (unsigned)c < (unsigned)D) ? Elem<T>::get_bits(w + c) : Elem<T>::kOneBits;
      }
      wv = Elem<T>::assemble(e);
    }
    a.w[p * nthr + me] = wv;
    if constexpr (BIAS) {
      uint4 bv;
      if (b && inside && (reinterpret_cast<uintptr_t>(b + c0) & 15u) == 0) {
        bv = load_cached(b + c0);
      } else {
        uint32_t e[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
          const int c = c0 + i;
          e[i] = (b && (unsigned)c < (unsigned)D) ? Elem<T>::get_bits(b + c) : 0u;
        }
        bv = Elem<T>::assemble(e);
      }
      a.b[p * nthr + me] = bv;
    }
  }
  a.phase = phase;
}

// ---------------------------------------------------------------------------
// per-thread partial sums (fixed order: slot, then column)

template <typename T, int NSLOT>
__device__ __forceinline__ float sum_squares(const float (&v)[NSLOT][Elem<T>::V]) {
  constexpr int V = Elem<T>::V;
  float acc = 0.f;
#pragma unroll
  for (int p = 0; p < NSLOT; ++p)
#pragma unroll
    for (int e = 0; e < V; ++e) acc = __fmaf_rn(v[p][e], v[p][e], acc);
  return acc;
}

// LayerNorm pass 1: replaces x by d = x - K (zero outside the row) and
// returns the thread's sum of d.
template <typename T, bool EXACT, int NSLOT>
__device__ __forceinline__ float shift_and_sum(float (&v)[NSLOT][Elem<T>::V],
                                               const Row<T>& g, int D, int k0,
                                               int step, float K) {
  constexpr int V = Elem<T>::V;
  float acc = 0.f;
#pragma unroll
  for (int p = 0; p < NSLOT; ++p) {
    const int k = k0 + step * p;
    if (chunk_full<T, EXACT>(g, k)) {
#pragma unroll
      for (int e = 0; e < V; ++e) {
        v[p][e] = __fsub_rn(v[p][e], K);
        acc = __fadd_rn(acc, v[p][e]);
      }
    } else {
#pragma unroll
      for (int e = 0; e < V; ++e) {
        const int c = k * V + e - g.phase;
        v[p][e] = ((unsigned)c < (unsigned)D) ? __fsub_rn(v[p][e], K) : 0.f;
        acc = __fadd_rn(acc, v[p][e]);
      }
    }
  }
  return acc;
}

// LayerNorm pass 2: the thread's sum of (d - mean)^2 over the row's columns.
template <typename T, bool EXACT, int NSLOT>
__device__ __forceinline__ float sum_dev_squares(const float (&v)[NSLOT][Elem<T>::V],
                                                 const Row<T>& g, int D, int k0,
                                                 int step, float mean) {
  constexpr int V = Elem<T>::V;
  float acc = 0.f;
#pragma unroll
  for (int p = 0; p < NSLOT; ++p) {
    const int k = k0 + step * p;
    if (chunk_full<T, EXACT>(g, k)) {
#pragma unroll
      for (int e = 0; e < V; ++e) {
        const float t = __fsub_rn(v[p][e], mean);
        acc = __fmaf_rn(t, t, acc);
      }
    } else {
#pragma unroll
      for (int e = 0; e < V; ++e) {
        const int c = k * V + e - g.phase;
        const float t = ((unsigned)c < (unsigned)D) ? __fsub_rn(v[p][e], mean) : 0.f;
        acc = __fmaf_rn(t, t, acc);
      }
    }
  }
  return acc;
}

// Normalize the thread's chunks of one row, apply weight (and bias) and store.
template <typename T, int OP, bool EXACT, int NSLOT, bool BIAS>
__device__ __forceinline__ void normalize_store(const Segment& s, const Row<T>& g,
                                                const float (&v)[NSLOT][Elem<T>::V],
                                                const Affine<T, NSLOT, BIAS>& a, int k0,
                                                int step, float rstd, float mean) {
  constexpr int V = Elem<T>::V;
  const int D = s.dim;
#pragma unroll
  for (int p = 0; p < NSLOT; ++p) {
    const int k = k0 + step * p;
    if (k >= g.nch) continue;
    float wf[V], o[V];
    Elem<T>::unpack(a.w[p * blockDim.x + threadIdx.x], wf);
    if constexpr (OP == kOpRms) {
#pragma unroll
      for (int e = 0; e < V; ++e) o[e] = __fmul_rn(__fmul_rn(v[p][e], rstd), wf[e]);
    } else {
      float bf[V];
      if constexpr (BIAS) {
        Elem<T>::unpack(a.b[p * blockDim.x + threadIdx.x], bf);
      } else {
#pragma unroll
        for (int e = 0; e < V; ++e) bf[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < V; ++e)
        o[e] = __fmaf_rn(__fmul_rn(__fsub_rn(v[p][e], mean), rstd), wf[e], bf[e]);
    }
    if (EXACT || (s.vector_y && chunk_full<T, EXACT>(g, k))) {
      store_stream(g.y_row - g.phase + (long long)k * V, Elem<T>::pack(o));
    } else {
#pragma unroll
      for (int e = 0; e < V; ++e) {
        const int c = k * V + e - g.phase;
        if ((unsigned)c < (unsigned)D) Elem<T>::put(g.y_row + c, o[e]);
      }
    }
  }
}

__device__ __forceinline__ Segment pick_segment(const Params& p, int i) {
  return i == 0 ? p.seg[0] : p.seg[1];
}

// ---------------------------------------------------------------------------
// Family 0: a group of G lanes of one warp per row.

constexpr int kWarpBlock = 256;
// Register budgets: at least this many threads resident per SM (lane-group
// family: 768, i.e. up to 85 registers; block family: 1024, 64 registers).
constexpr int kMinThreadsPerSmWarp = 768;
constexpr int kMinThreadsPerSm = 1024;

template <typename T, int OP, bool EXACT, int VPL>
__global__ void __launch_bounds__(kWarpBlock, kMinThreadsPerSmWarp / kWarpBlock)
rows_warp_kernel(const Params p) {
  constexpr int V = Elem<T>::V;
  constexpr bool BIAS = OP == kOpLn;
  extern __shared__ __align__(16) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const long long warp = (long long)blockIdx.x * (kWarpBlock / 32) + (threadIdx.x >> 5);
  const long long nwarps = (long long)gridDim.x * (kWarpBlock / 32);
#pragma unroll 1
  for (int si = 0; si < p.nseg; ++si) {
    const Segment s = pick_segment(p, si);
    const int G = s.lanes;
    const int per_warp = 32 / G;
    const int gl = lane & (G - 1);
    const int gi = lane / G;
    const unsigned mask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << (gi * G));
    const long long ngroups = nwarps * per_warp;
    const int D = s.dim;
    const float d_f = (float)D;
    Affine<T, VPL, BIAS> a = affine_in_smem<T, VPL, BIAS>(smem);
#pragma unroll 1
    for (long long r = warp * per_warp + gi; r < s.rows; r += ngroups) {
      float v[VPL][V];
      const Row<T> g = row_geometry<T, EXACT>(s, r);
      float K = 0.f;
#pragma unroll
      for (int q = 0; q < VPL; ++q) load_chunk<T, EXACT>(g, D, gl + G * q, v[q]);
      if (OP == kOpLn) K = Elem<T>::get(static_cast<const T*>(s.x) + r * s.x_stride);
      if (g.phase != a.phase) load_affine<T, VPL, BIAS>(s, g.phase, gl, G, a);
      float rstd, mean = 0.f;
      if (OP == kOpRms) {
        float ss = sum_squares<T, VPL>(v);
        for (int off = G >> 1; off > 0; off >>= 1)
          ss = __fadd_rn(ss, __shfl_xor_sync(mask, ss, off));
        rstd = rsqrtf(__fadd_rn(__fdiv_rn(ss, d_f), p.eps));
      } else {
        float s1 = shift_and_sum<T, EXACT, VPL>(v, g, D, gl, G, K);
        for (int off = G >> 1; off > 0; off >>= 1)
          s1 = __fadd_rn(s1, __shfl_xor_sync(mask, s1, off));
        mean = __fdiv_rn(s1, d_f);
        float s2 = sum_dev_squares<T, EXACT, VPL>(v, g, D, gl, G, mean);
        for (int off = G >> 1; off > 0; off >>= 1)
          s2 = __fadd_rn(s2, __shfl_xor_sync(mask, s2, off));
        rstd = rsqrtf(__fadd_rn(__fdiv_rn(s2, d_f), p.eps));
      }
      normalize_store<T, OP, EXACT, VPL, BIAS>(s, g, v, a, gl, G, rstd, mean);
    }
  }
}

// ---------------------------------------------------------------------------
// Family 1: one block of NT threads per row.

template <int NT>
__device__ __forceinline__ float block_sum(float x, float* red) {
  constexpr int NW = NT / 32;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x = __fadd_rn(x, __shfl_xor_sync(0xffffffffu, x, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
  __syncthreads();
  float t = red[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) t = __fadd_rn(t, red[w]);
  return t;
}

template <typename T, int OP, bool EXACT, int NT, int VPT>
__global__ void __launch_bounds__(NT, kMinThreadsPerSm / NT)
rows_cta_kernel(const Params p) {
  constexpr int V = Elem<T>::V;
  constexpr int NW = NT / 32;
  constexpr bool BIAS = OP == kOpLn;
  // Two alternating slots: a slot is rewritten only after every thread has
  // passed the barrier of the reduction in between, i.e. finished reading it.
  __shared__ float red[2][NW];
  extern __shared__ __align__(16) unsigned char smem[];
  int slot = 0;
  const int tid = threadIdx.x;
#pragma unroll 1
  for (int si = 0; si < p.nseg; ++si) {
    const Segment s = pick_segment(p, si);
    const int D = s.dim;
    const float d_f = (float)D;
    Affine<T, VPT, BIAS> a = affine_in_smem<T, VPT, BIAS>(smem);
#pragma unroll 1
    for (long long r = blockIdx.x; r < s.rows; r += gridDim.x) {
      float v[VPT][V];
      const Row<T> g = row_geometry<T, EXACT>(s, r);
      float K = 0.f;
#pragma unroll
      for (int q = 0; q < VPT; ++q) load_chunk<T, EXACT>(g, D, tid + NT * q, v[q]);
      if (OP == kOpLn) K = Elem<T>::get(static_cast<const T*>(s.x) + r * s.x_stride);
      if (g.phase != a.phase) load_affine<T, VPT, BIAS>(s, g.phase, tid, NT, a);
      float rstd, mean = 0.f;
      if (OP == kOpRms) {
        const float ss = block_sum<NT>(sum_squares<T, VPT>(v), red[slot]);
        slot ^= 1;
        rstd = rsqrtf(__fadd_rn(__fdiv_rn(ss, d_f), p.eps));
      } else {
        const float s1 = block_sum<NT>(shift_and_sum<T, EXACT, VPT>(v, g, D, tid, NT, K), red[slot]);
        slot ^= 1;
        mean = __fdiv_rn(s1, d_f);
        const float s2 = block_sum<NT>(sum_dev_squares<T, EXACT, VPT>(v, g, D, tid, NT, mean), red[slot]);
        slot ^= 1;
        rstd = rsqrtf(__fadd_rn(__fdiv_rn(s2, d_f), p.eps));
      }
      normalize_store<T, OP, EXACT, VPT, BIAS>(s, g, v, a, tid, NT, rstd, mean);
    }
  }
}

}  // namespace rn
