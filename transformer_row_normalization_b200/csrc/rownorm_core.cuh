// Per-row arithmetic shared by every row-normalization kernel (sm_100a).
//
// What is computed (per row of D elements, binary32 arithmetic):
//   RMSNorm   ("Emily.Fast", rms_norm/3):
//               ss   = sum_i x_i^2
//               rstd = rsqrt(ss * (1/D) + eps)
//               y_j  = (x_j * rstd) * w_j
//   LayerNorm ("Emily.Fast", layer_norm/4; population variance):
//               K    = x_0                       (shift: a constant row gives
//               d_i  = x_i - K                    exactly zero deviations)
//               mean = (sum_i d_i) * (1/D)
//               var  = (sum_i (d_i - mean)^2) * (1/D)
//               rstd = rsqrt(var + eps)
//               y_j  = ((d_j - mean) * rstd) * w_j + b_j   (one fused multiply-add)
//   The page calls its LayerNorm statistic "Welford-style"; the two passes
//   here run over a row already on chip, so they cost no extra HBM traffic
//   and give the same population mean and variance.
//   Residual add + RMSNorm and gated RMSNorm ("norm_fusion.rs", module doc
//   comment: the elementwise fusions kept composed until a kernel pins the
//   summation order, which this one does):
//               h_j  = round_T(x_j + r_j)        (stored; the row statistics
//               y_j  = (h_j * rstd) * w_j          use the stored values)
//               y_j  = ((x_j * rstd) * w_j) * silu(z_j),
//               silu(t) = t / (1 + exp(-t))       (binary32, __expf called)
//   Dual q/k head RMSNorm + RoPE ("Emily.Fast", rope/3, rope_with_freqs/4):
//               o_j  = (x_j * rstd) * w_j          (binary32, not rounded)
//               plane (a, b), angle theta at the row's position:
//               y_a  = o_a * cos - o_b * sin,  y_b = o_b * cos + o_a * sin
//               (each as fma(o_own, cos, -/+ (o_partner * sin)); columns
//               from rope_dims on: y = o)
//
// Row layout. A row is moved as 16-byte chunks on the 16-byte address grid:
// the columns between the first and the last 16-byte boundary inside the row
// form its full chunks, each moved with one 16-byte access; the at most
// 2 (V - 1) columns before the first and after the last boundary (V = 16 /
// element size) are its edge elements, moved one by one, so no byte outside
// the caller's views is touched. A thread owns the full chunks k0,
// k0 + step, k0 + 2*step, ... of every row it works on (slots) and at most
// one edge element.
//
// Arithmetic. Elements are processed as pairs (columns 2j, 2j+1 of a chunk)
// with the packed binary32 instructions of sm_100 (add/sub/mul/fma .f32x2);
// each lane of a packed instruction rounds exactly like its scalar form.
// (1/D) is the binary32 reciprocal of D, rounded to nearest.
//
// Summation order (fixed; it depends only on D, the element type, the
// threads per row and the row's 16-byte phase):
//   1. each thread keeps four partial sums: binary32 pairs (columns 2j,
//      2j + 1 of a chunk) go to one of two packed accumulators by the parity
//      of j, each added in slot order then pair order; the two accumulators
//      are added, then the two lanes of the result (the even and the odd
//      columns), plus the term of its edge element if it owns one;
//   2. an xor butterfly over the G lanes sharing the row (offsets G/2 .. 1);
//   3. for rows owned by a whole block of NW warps, the per-warp sums are
//      combined by the same xor butterfly over lanes 0 .. NW-1 (warp w's sum
//      at lane w) in every warp, then broadcast from lane 0, so every thread
//      ends with the same bits.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace rn {

enum : int {
  kOpRms = 0,
  kOpLn = 1,
  kOpAddRms = 2,
  kOpGatedRms = 3,
  kOpRmsRope = 4,       // RMSNorm + RoPE, plane partners through shared memory
  kOpRmsRopeLocal = 5,  // RMSNorm + RoPE, every plane's partner in the same thread
};
__host__ __device__ constexpr bool op_is_rope(int op) {
  return op == kOpRmsRope || op == kOpRmsRopeLocal;
}

// A second input row space read beside x: the residual (kOpAddRms) or the
// gate (kOpGatedRms).
__host__ __device__ constexpr bool op_has_second(int op) {
  return op == kOpAddRms || op == kOpGatedRms;
}

// Which of a thread's NSLOT chunk slots the planner guarantees present in
// every row of a launch:
//   kSlotsTested  none: each slot is tested against the row's chunk count;
//   kSlotsTail    all but the last (tested): slot counts are ceil(chunks /
//                 threads) and a row's chunk count varies by at most one
//                 between 16-byte phases;
//   kSlotsFull    all: the row's chunks divide evenly over its threads
//                 (EXACT layouts only), so no slot is ever tested.
enum : int { kSlotsTested = 0, kSlotsTail = 1, kSlotsFull = 2 };

template <int SLOTS, int NSLOT>
__device__ __forceinline__ bool slot_present(int p, int f, int nfull) {
  if constexpr (SLOTS == kSlotsFull) return true;
  if (SLOTS == kSlotsTail && p < NSLOT - 1) return true;
  return f < nfull;
}

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
  int lanes;       // threads per row in the lane-group kernels (power of two <= 32)
  int vector_y;    // 1: every y row has its x row's 16-byte phase
  int pad_;
  // second input and stored sum (kOpAddRms: residual r and h = x + r;
  // kOpGatedRms: gate z); every row shares its x row's 16-byte phase
  const void* x2;
  void* h;
  long long x2_stride;
  long long h_stride;
  // RoPE after the norm (kOpRmsRope): row r is token r / rope_heads at
  // position rope_offset + token; rope_table[pos][i] = cos theta_i and
  // rope_table[pos][rope_dims / 2 + i] = sin theta_i (binary32)
  const float* rope_table;
  long long rope_offset;
  int rope_heads;
  int rope_dims;
  int rope_trad;   // 1: planes (2i, 2i + 1); 0: planes (i, i + rope_dims / 2)
  // rows in blocks (head rows of a packed buffer): for a tensor with inner
  // count n > 0, row r starts at (r / n) * outer + (r % n) * stride; n = 0:
  // at r * stride
  int x_inner;
  int y_inner;
  int x2_inner;
  int h_inner;
  int blocks_pad_;
  long long x_outer;
  long long y_outer;
  long long x2_outer;
  long long h_outer;
};

// Element offset of row r of a tensor with row stride `stride` and block
// layout (inner, outer) as in Segment (32-bit division while r fits).
__device__ __forceinline__ long long row_off(long long r, long long stride, int inner,
                                             long long outer) {
  if (inner <= 0) return r * stride;
  const long long t = r < 0x7fffffffLL ? (long long)((unsigned)r / (unsigned)inner) : r / inner;
  return t * outer + (r - t * inner) * stride;
}

// ---------------------------------------------------------------------------
// packed binary32 pairs
//
// A pair lives in one 64-bit register (low half = the element at the even
// column), so the packed instructions take their operands without any
// register shuffling.

using F2 = float2;

__device__ __forceinline__ F2 make2(float lo, float hi) { return make_float2(lo, hi); }
__device__ __forceinline__ F2 make2_bits(uint32_t lo, uint32_t hi) {
  return make_float2(__uint_as_float(lo), __uint_as_float(hi));
}
__device__ __forceinline__ void split2(F2 a, float& lo, float& hi) {
  lo = a.x;
  hi = a.y;
}
__device__ __forceinline__ F2 zero2() { return make_float2(0.f, 0.f); }
__device__ __forceinline__ F2 splat(float v) { return make_float2(v, v); }
__device__ __forceinline__ F2 add2(F2 a, F2 b) { return __fadd2_rn(a, b); }
// a - b is a + (-b): negation is exact and the sum rounds as the difference.
__device__ __forceinline__ F2 sub2(F2 a, F2 b) { return __fadd2_rn(a, make_float2(-b.x, -b.y)); }
__device__ __forceinline__ F2 mul2(F2 a, F2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ F2 fma2(F2 a, F2 b, F2 c) { return __ffma2_rn(a, b, c); }
// lo + hi, rounded once.
__device__ __forceinline__ float hsum2(F2 a) {
  float lo, hi;
  split2(a, lo, hi);
  return __fadd_rn(lo, hi);
}

// silu(t) = t / (1 + exp(-t)) in binary32, with CUDA's fast exponential and
// divide intrinsics (__expf, __fdividef; documented error 2 + 1.2 |t| ulps
// for the exponential, 2 ulps for the divide). At the gate magnitudes of a
// model (|t| < ~20) that is ~1e-6 relative: below half a bfloat16 ulp of the
// output, and inside the binary32 bound the tests derive for this op. A
// gate below -88 gives exp = inf and silu = -0.
__device__ __forceinline__ float silu(float t) {
  return __fdividef(t, __fadd_rn(1.f, __expf(-t)));
}
__device__ __forceinline__ F2 silu2(F2 t) { return make2(silu(t.x), silu(t.y)); }

// ---------------------------------------------------------------------------
// element types: a 16-byte chunk <-> P = V/2 binary32 pairs

template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int V = 4;
  static constexpr int P = 2;
  static constexpr uint32_t kOneBits = 0x3f800000u;
  static __device__ __forceinline__ float get(const float* p) { return *p; }
  static __device__ __forceinline__ uint32_t get_bits(const float* p) {
    return __float_as_uint(*p);
  }
  static __device__ __forceinline__ void put(float* p, float v) { *p = v; }
  // the element in the low bytes of a little-endian 32-bit word
  static __device__ __forceinline__ float low(uint32_t w) { return __uint_as_float(w); }
  // v as stored: binary32 already is
  static __device__ __forceinline__ float stored(float v) { return v; }
  static __device__ __forceinline__ void unpack(const uint4& u, F2 (&f)[2]) {
    f[0] = make2_bits(u.x, u.y);
    f[1] = make2_bits(u.z, u.w);
  }
  static __device__ __forceinline__ uint4 pack(const F2 (&f)[2]) {
    return make_uint4(__float_as_uint(f[0].x), __float_as_uint(f[0].y), __float_as_uint(f[1].x),
                      __float_as_uint(f[1].y));
  }
  static __device__ __forceinline__ uint4 assemble(const uint32_t (&e)[4]) {
    return make_uint4(e[0], e[1], e[2], e[3]);
  }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int V = 8;
  static constexpr int P = 4;
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
  // the element in the low bytes of a little-endian 32-bit word, widened
  static __device__ __forceinline__ float low(uint32_t w) { return __uint_as_float(w << 16); }
  // v rounded to bfloat16 (nearest, ties to even), widened back exactly
  static __device__ __forceinline__ float stored(float v) {
    return __bfloat162float(__float2bfloat16_rn(v));
  }
  // bfloat16 is the upper half of a binary32 pattern: widening is exact bit
  // placement (low element: shift up; high element: clear the low half).
  static __device__ __forceinline__ F2 pair(uint32_t w) {
    return make2_bits(w << 16, w & 0xffff0000u);
  }
  static __device__ __forceinline__ uint32_t pack_pair(F2 v) {
    float lo, hi;
    split2(v, lo, hi);
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ void unpack(const uint4& u, F2 (&f)[4]) {
    f[0] = pair(u.x);
    f[1] = pair(u.y);
    f[2] = pair(u.z);
    f[3] = pair(u.w);
  }
  static __device__ __forceinline__ uint4 pack(const F2 (&f)[4]) {
    return make_uint4(pack_pair(f[0]), pack_pair(f[1]), pack_pair(f[2]), pack_pair(f[3]));
  }
  static __device__ __forceinline__ uint4 assemble(const uint32_t (&e)[8]) {
    return make_uint4(e[0] | (e[1] << 16), e[2] | (e[3] << 16), e[4] | (e[5] << 16),
                      e[6] | (e[7] << 16));
  }
};

// ---------------------------------------------------------------------------
// memory access

// The block's dynamic shared memory (prefetch slots, weight/bias cache,
// staged tiles), addressed by 16-byte word offsets so that the compiler uses
// 32-bit shared-window addresses rather than generic pointers.
extern __shared__ __align__(128) uint4 dyn_smem[];

__device__ __forceinline__ uint4 load_stream(const void* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void store_stream(void* p, const uint4& v) {
  __stcs(reinterpret_cast<uint4*>(p), v);
}
__device__ __forceinline__ uint4 load_cached(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Per-thread asynchronous 16-byte copy global -> shared (L2 only, not L1),
// grouped with commit/wait; a thread waits only for its own copies.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem_dst)), "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Geometry of one row. Its D columns split into three runs: `head` edge
// elements before the first 16-byte boundary inside the row, `nfull` full
// 16-byte chunks starting there (x_full), and the tail edge elements after
// the last such boundary; nedge = head + tail <= 2 (V - 1).
//
// Ownership: of the `step` threads that share a row, thread k0 owns the full
// chunks f = k0, k0 + step, k0 + 2 step, ... (its slots) and, when
// k0 < nedge, edge element k0 (the head elements first, then the tail). The
// planner gives rows that can have edge elements at least 2 (V - 1) threads,
// so every edge element has an owner and all threads run the same
// straight-line code on whole chunks.
template <typename T>
struct Row {
  const T* x_row;   // x row start
  const T* x_full;  // first full chunk (16-byte aligned)
  T* y_row;         // y row start
  int phase;        // elements between the 16-byte boundary and the row start
  int head;         // edge elements before the first full chunk
  int nfull;        // full chunks
  int nedge;        // edge elements
};

// EXACT: the planner guarantees that every x and y row starts on a 16-byte
// boundary, D is a multiple of V, and the weight and bias (where present)
// start on 16-byte boundaries; so the phase is 0 and there are no edges.
template <typename T, bool EXACT>
__device__ __forceinline__ Row<T> row_geometry(const Segment& s, long long r) {
  constexpr int V = Elem<T>::V;
  Row<T> g;
  g.x_row = static_cast<const T*>(s.x) + row_off(r, s.x_stride, s.x_inner, s.x_outer);
  g.y_row = static_cast<T*>(s.y) + row_off(r, s.y_stride, s.y_inner, s.y_outer);
  if constexpr (EXACT) {
    g.phase = 0;
    g.head = 0;
    g.nfull = s.dim / V;
    g.nedge = 0;
  } else {
    g.phase = (int)((reinterpret_cast<uintptr_t>(g.x_row) & 15u) / sizeof(T));
    g.head = g.phase ? min(V - g.phase, s.dim) : 0;
    g.nfull = (s.dim - g.head) / V;
    g.nedge = s.dim - g.nfull * V;
  }
  g.x_full = g.x_row + g.head;
  return g;
}

// Column of edge element e < nedge.
template <typename T>
__device__ __forceinline__ int edge_column(const Row<T>& g, int D, int e) {
  return e < g.head ? e : D - g.nedge + e;
}

// The edge element of thread k0 (0 when it owns none), read on its own so
// that no byte outside the row is touched.
template <typename T, bool EXACT>
__device__ __forceinline__ float load_edge(const Row<T>& g, int D, int k0) {
  if constexpr (EXACT) return 0.f;
  return k0 < g.nedge ? Elem<T>::get(g.x_row + edge_column(g, D, k0)) : 0.f;
}

// ---------------------------------------------------------------------------
// per-thread partial sums over the slots and the edge element of one row
//
// Each is (sum over the even positions) + (sum over the odd positions) of
// the thread's slots, then, for a thread that owns an edge element, that
// element's term added (a square by one fused multiply-add).

// Two packed accumulators per pass: pair j of every chunk goes to
// acc[j & 1], so the dependent chains are half as long; the thread's partial
// is (acc[0] + acc[1]), then its two lanes added.
__device__ __forceinline__ float hsum_acc(const F2 (&acc)[2]) { return hsum2(add2(acc[0], acc[1])); }

// RMSNorm: sum of squares (absent slots hold zeros, which add nothing).
template <typename T, bool EXACT, int NSLOT>
__device__ __forceinline__ float sum_squares(const F2 (&v)[NSLOT][Elem<T>::P], float xe,
                                             bool has_edge) {
  constexpr int P = Elem<T>::P;
  F2 acc[2] = {zero2(), zero2()};
#pragma unroll
  for (int p = 0; p < NSLOT; ++p)
#pragma unroll
    for (int j = 0; j < P; ++j) acc[j & 1] = fma2(v[p][j], v[p][j], acc[j & 1]);
  float s = hsum_acc(acc);
  if (!EXACT && has_edge) s = __fmaf_rn(xe, xe, s);
  return s;
}

// LayerNorm pass 1: replaces x by d = x - K (slots and edge element) and
// returns the thread's sum of d.
template <typename T, bool EXACT, int SLOTS, int NSLOT>
__device__ __forceinline__ float shift_and_sum(F2 (&v)[NSLOT][Elem<T>::P], float& xe,
                                               const Row<T>& g, int k0, int step, float K,
                                               bool has_edge) {
  constexpr int P = Elem<T>::P;
  const F2 K2 = splat(K);
  F2 acc[2] = {zero2(), zero2()};
#pragma unroll
  for (int p = 0; p < NSLOT; ++p) {
    if (slot_present<SLOTS, NSLOT>(p, k0 + step * p, g.nfull)) {
#pragma unroll
      for (int j = 0; j < P; ++j) {
        v[p][j] = sub2(v[p][j], K2);
        acc[j & 1] = add2(acc[j & 1], v[p][j]);
      }
    }
  }
  float s = hsum_acc(acc);
  if (!EXACT && has_edge) {
    xe = __fsub_rn(xe, K);
    s = __fadd_rn(s, xe);
  }
  return s;
}

// LayerNorm pass 2: replaces d by the centred c = d - mean (slots and edge
// element; the normalization uses c as it is) and returns the thread's sum
// of c^2.
template <typename T, bool EXACT, int SLOTS, int NSLOT>
__device__ __forceinline__ float sum_dev_squares(F2 (&v)[NSLOT][Elem<T>::P], float& xe,
                                                 const Row<T>& g, int k0, int step, float mean,
                                                 bool has_edge) {
  constexpr int P = Elem<T>::P;
  const F2 M2 = splat(mean);
  F2 acc[2] = {zero2(), zero2()};
#pragma unroll
  for (int p = 0; p < NSLOT; ++p) {
    if (slot_present<SLOTS, NSLOT>(p, k0 + step * p, g.nfull)) {
#pragma unroll
      for (int j = 0; j < P; ++j) {
        v[p][j] = sub2(v[p][j], M2);
        acc[j & 1] = fma2(v[p][j], v[p][j], acc[j & 1]);
      }
    }
  }
  float s = hsum_acc(acc);
  if (!EXACT && has_edge) {
    xe = __fsub_rn(xe, mean);
    s = __fmaf_rn(xe, xe, s);
  }
  return s;
}

// ---------------------------------------------------------------------------
// reductions across the threads of a row

// xor butterfly over the G lanes of `mask` (G a power of two <= 32): offsets
// G/2, ..., 1, unrolled (G is uniform across the warp).
__device__ __forceinline__ float group_sum(float x, int G, unsigned mask) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    if (off < G) x = __fadd_rn(x, __shfl_xor_sync(mask, x, off));
  return x;
}

// Sum over a block of NT threads: warp butterflies, then the per-warp sums
// (warp w at lane w) through the same NW-lane butterfly in every warp and a
// broadcast from lane 0. `red` holds NT/32 floats; the caller alternates two
// such buffers so that a buffer is rewritten only after a barrier that
// follows every read of it.
template <int NT>
__device__ __forceinline__ float block_sum(float x, float* red) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x = __fadd_rn(x, __shfl_xor_sync(0xffffffffu, x, off));
  if constexpr (NW == 1) {
    return x;
  } else {
    if (lane == 0) red[threadIdx.x >> 5] = x;
    __syncthreads();
    float t = lane < NW ? red[lane] : 0.f;
#pragma unroll
    for (int off = NW >> 1; off > 0; off >>= 1)
      t = __fadd_rn(t, __shfl_xor_sync(0xffffffffu, t, off));
    return __shfl_sync(0xffffffffu, t, 0);
  }
}

// ---------------------------------------------------------------------------
// weight and bias

// EXACT rows: the weight/bias columns of chunk f are one aligned 16-byte
// chunk of each vector (L1-resident after the first row). EXACT rows have
// no edge elements. AFF: the weight (and bias) are known to be present, so
// no per-chunk test of a NULL vector remains in the row loop.
template <typename T, bool BIAS, bool AFF>
struct AffineDirect {
  const T* w;
  const T* b;
  __device__ __forceinline__ void get(int /*p*/, int f, F2 (&wf)[Elem<T>::P],
                                      F2 (&bf)[Elem<T>::P]) const {
    constexpr int V = Elem<T>::V;
    constexpr int P = Elem<T>::P;
    if (AFF || w) {
      Elem<T>::unpack(load_cached(w + f * V), wf);
    } else {
#pragma unroll
      for (int j = 0; j < P; ++j) wf[j] = splat(1.f);
    }
    if constexpr (BIAS) {
      if (AFF || b) {
        Elem<T>::unpack(load_cached(b + f * V), bf);
      } else {
#pragma unroll
        for (int j = 0; j < P; ++j) bf[j] = zero2();
      }
    }
  }
  __device__ __forceinline__ void edge(float& w_, float& b_) const {
    w_ = 1.f;
    b_ = 0.f;
  }
};

// Any layout: the weight/bias columns of each of the thread's slots,
// realigned to the row phase, in the thread's own shared memory entries
// [slot][thread] (no other thread touches them, so no barrier; consecutive
// threads use consecutive 16-byte words, so no bank conflicts), and those of
// its edge element in registers. Refilled when a row with another phase
// arrives (the split of a row into edge elements and chunks depends only on
// D and the phase). NULL weight = ones, NULL bias = zeros.
template <typename T, int NSLOT, bool BIAS>
struct AffineCache {
  int base;  // first 16-byte word: weight [NSLOT][blockDim.x], then bias (BIAS)
  float we, be;
  int phase;

  __device__ __forceinline__ void init(int word_offset) {
    base = word_offset;
    we = 1.f;
    be = 0.f;
    phase = -1;
  }
  __device__ __forceinline__ uint4& wslot(int p) const {
    return dyn_smem[base + p * blockDim.x + threadIdx.x];
  }
  __device__ __forceinline__ uint4& bslot(int p) const {
    return dyn_smem[base + (NSLOT + p) * blockDim.x + threadIdx.x];
  }

  __device__ __forceinline__ void fill(const Segment& s, const Row<T>& g, int k0, int step) {
    constexpr int V = Elem<T>::V;
    const T* wv = static_cast<const T*>(s.w);
    const T* bv = static_cast<const T*>(s.b);
    const int D = s.dim;
#pragma unroll 1
    for (int p = 0; p < NSLOT; ++p) {
      const int c0 = g.head + (k0 + step * p) * V;
      uint32_t e[V];
#pragma unroll
      for (int i = 0; i < V; ++i) {
        const int c = c0 + i;
        e[i] = (wv && (unsigned)c < (unsigned)D) ? Elem<T>::get_bits(wv + c) : Elem<T>::kOneBits;
      }
      wslot(p) = Elem<T>::assemble(e);
      if constexpr (BIAS) {
#pragma unroll
        for (int i = 0; i < V; ++i) {
          const int c = c0 + i;
          e[i] = (bv && (unsigned)c < (unsigned)D) ? Elem<T>::get_bits(bv + c) : 0u;
        }
        bslot(p) = Elem<T>::assemble(e);
      }
    }
    if (k0 < g.nedge) {
      const int c = edge_column(g, D, k0);
      we = wv ? Elem<T>::get(wv + c) : 1.f;
      be = (BIAS && bv) ? Elem<T>::get(bv + c) : 0.f;
    }
    phase = g.phase;
  }

  __device__ __forceinline__ void get(int p, int /*f*/, F2 (&wf)[Elem<T>::P],
                                      F2 (&bf)[Elem<T>::P]) const {
    Elem<T>::unpack(wslot(p), wf);
    if constexpr (BIAS) Elem<T>::unpack(bslot(p), bf);
  }
  __device__ __forceinline__ void edge(float& w_, float& b_) const {
    w_ = we;
    b_ = be;
  }
};

template <int NSLOT, bool BIAS>
constexpr int affine_cache_bytes(int threads) {
  return threads * NSLOT * 16 * (BIAS ? 2 : 1);
}

// No gate (every op but kOpGatedRms).
struct NoGate {
  template <int P>
  __device__ __forceinline__ void get(int, int, F2 (&)[P]) const {}
  __device__ __forceinline__ float edge() const { return 0.f; }
};

// Normalize the thread's chunks and edge element of one row, apply weight
// (and bias, or the gate's silu), store.
template <typename T, int OP, bool EXACT, int SLOTS, int NSLOT, typename Src,
          typename Gate = NoGate>
__device__ __forceinline__ void normalize_store(const Segment& s, const Row<T>& g,
                                                const F2 (&v)[NSLOT][Elem<T>::P], float xe,
                                                const Src& src, int k0, int step, float rstd,
                                                float mean, bool has_edge,
                                                const Gate& gate = Gate()) {
  constexpr int V = Elem<T>::V;
  constexpr int P = Elem<T>::P;
  const F2 R2 = splat(rstd);
  (void)mean;  // LayerNorm rows arrive centred (row_stats)
#pragma unroll
  for (int p = 0; p < NSLOT; ++p) {
    const int f = k0 + step * p;
    if (!slot_present<SLOTS, NSLOT>(p, f, g.nfull)) continue;
    F2 wf[P], bf[P], o[P];
    src.get(p, f, wf, bf);
#pragma unroll
    for (int j = 0; j < P; ++j) {
      if constexpr (OP == kOpLn)  // v holds the centred c = d - mean
        o[j] = fma2(mul2(v[p][j], R2), wf[j], bf[j]);
      else
        o[j] = mul2(mul2(v[p][j], R2), wf[j]);
    }
    if constexpr (OP == kOpGatedRms) {
      F2 zf[P];
      gate.template get<P>(p, f, zf);
#pragma unroll
      for (int j = 0; j < P; ++j) o[j] = mul2(o[j], silu2(zf[j]));
    }
    T* yc = g.y_row + g.head + (long long)f * V;
    if (EXACT || s.vector_y) {
      store_stream(yc, Elem<T>::pack(o));
    } else {
#pragma unroll
      for (int j = 0; j < P; ++j) {
        float lo, hi;
        split2(o[j], lo, hi);
        Elem<T>::put(yc + 2 * j, lo);
        Elem<T>::put(yc + 2 * j + 1, hi);
      }
    }
  }
  if (!EXACT && has_edge) {
    float we, be;
    src.edge(we, be);
    float o = OP == kOpLn ? __fmaf_rn(__fmul_rn(xe, rstd), we, be)  // xe centred
                          : __fmul_rn(__fmul_rn(xe, rstd), we);
    if constexpr (OP == kOpGatedRms) o = __fmul_rn(o, silu(gate.edge()));
    Elem<T>::put(g.y_row + edge_column(g, s.dim, k0), o);
  }
}

// RoPE after the RMSNorm (kOpRmsRope, lane-group rows). Each thread forms
// the normalized, weighted values o of its columns (binary32). A column's
// plane partner is usually another thread's, so the values go to the lane
// group's staging row in shared memory (`stage`, dim floats) and, after a
// sync of the group's lanes (`mask`), each thread reads its partners back,
// rotates, stores, and syncs again before the staging row is rewritten.
// Aligned rows (EXACT, dims a multiple of 2 V) take whole chunks at a time:
// a chunk lies in one half of the rotated columns, so its partners and its
// cos / sin are contiguous 16-byte vectors; interleaved planes need no
// staging at all (both values of a plane are one pair of the thread's), nor
// does full split-half rotary whose chunks divide evenly over the threads
// (a chunk's partner chunk is then the same thread's). Every path computes
// the same operations, so the bits do not depend on the path.
template <int N>
__device__ __forceinline__ void load_floats(const float* p, float (&d)[N]) {
#pragma unroll
  for (int i = 0; i < N; i += 4) {
    const float4 t = *reinterpret_cast<const float4*>(p + i);
    d[i] = t.x;
    d[i + 1] = t.y;
    d[i + 2] = t.z;
    d[i + 3] = t.w;
  }
}

template <int N>
__device__ __forceinline__ void ldg_floats(const float* p, float (&d)[N]) {
#pragma unroll
  for (int i = 0; i < N; i += 4) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(p + i));
    d[i] = t.x;
    d[i + 1] = t.y;
    d[i + 2] = t.z;
    d[i + 3] = t.w;
  }
}

template <typename T>
__device__ __forceinline__ void store_chunk(const Segment& s, T* yc, const F2 (&o)[Elem<T>::P],
                                            bool vector) {
  constexpr int P = Elem<T>::P;
  if (vector) {
    store_stream(yc, Elem<T>::pack(o));
  } else {
#pragma unroll
    for (int j = 0; j < P; ++j) {
      Elem<T>::put(yc + 2 * j, o[j].x);
      Elem<T>::put(yc + 2 * j + 1, o[j].y);
    }
  }
}

// Split-half planes of one chunk pair held by the thread: a (columns c0 ..
// c0 + V - 1 of the first half) and b (its partner chunk, `half` columns
// on), rotated by their columns' cos / sin and stored: packed pairs of
// planes, y_a = fma(a, cos, -(b sin)), y_b = fma(b, cos, a sin).
template <typename T>
__device__ __forceinline__ void rotate_split_store(const Segment& s, T* yc, int half,
                                                   const F2 (&a)[Elem<T>::P],
                                                   const F2 (&b)[Elem<T>::P],
                                                   const float (&cs)[Elem<T>::V],
                                                   const float (&sn)[Elem<T>::V], bool vstore) {
  constexpr int P = Elem<T>::P;
  F2 ya[P], yb[P];
#pragma unroll
  for (int j = 0; j < P; ++j) {
    const F2 c = make2(cs[2 * j], cs[2 * j + 1]), sn2 = make2(sn[2 * j], sn[2 * j + 1]);
    const F2 bs = mul2(b[j], sn2), as = mul2(a[j], sn2);
    ya[j] = fma2(a[j], c, make2(-bs.x, -bs.y));
    yb[j] = fma2(b[j], c, as);
  }
  store_chunk<T>(s, yc, ya, vstore);
  store_chunk<T>(s, yc + half, yb, vstore);
}

// rotate_split_store with the negated sines given (nsn = -sn): b (-s) is
// -(b s) exactly (rounding to nearest is symmetric), so the bits are the
// same, without a sign flip per element.
template <typename T>
__device__ __forceinline__ void rotate_split_store_ns(const Segment& s, T* yc, int half,
                                                      const F2 (&a)[Elem<T>::P],
                                                      const F2 (&b)[Elem<T>::P],
                                                      const float (&cs)[Elem<T>::V],
                                                      const float (&sn)[Elem<T>::V],
                                                      const float (&nsn)[Elem<T>::V],
                                                      bool vstore) {
  constexpr int P = Elem<T>::P;
  F2 ya[P], yb[P];
#pragma unroll
  for (int j = 0; j < P; ++j) {
    const F2 c = make2(cs[2 * j], cs[2 * j + 1]);
    const F2 sn2 = make2(sn[2 * j], sn[2 * j + 1]), nsn2 = make2(nsn[2 * j], nsn[2 * j + 1]);
    ya[j] = fma2(a[j], c, mul2(b[j], nsn2));
    yb[j] = fma2(b[j], c, mul2(a[j], sn2));
  }
  store_chunk<T>(s, yc, ya, vstore);
  store_chunk<T>(s, yc + half, yb, vstore);
}

// The split-half in-thread RoPE path of normalize_rope_store (full rotary,
// every slot present, EXACT rows) with the thread's cos / sin already in
// registers: cs[p] / sn[p] for its first-half slot p, nsn[p] = -sn[p]. For
// several rows of one token whose angles the caller loaded once; the
// operations are those of normalize_rope_store, so the bits are too.
template <typename T, int NSLOT, typename Src>
__device__ __forceinline__ void normalize_rope_split_pre(
    const Segment& s, const Row<T>& g, F2 (&v)[NSLOT][Elem<T>::P], const Src& src, int k0,
    int step, float rstd, const float (&cs)[NSLOT / 2][Elem<T>::V],
    const float (&sn)[NSLOT / 2][Elem<T>::V], const float (&nsn)[NSLOT / 2][Elem<T>::V]) {
  static_assert(NSLOT % 2 == 0, "chunk pairs");
  constexpr int V = Elem<T>::V;
  constexpr int P = Elem<T>::P;
  const int half = s.rope_dims >> 1;
  const F2 R2 = splat(rstd);
#pragma unroll
  for (int p = 0; p < NSLOT; ++p) {
    F2 wf[P], bf[P];
    src.get(p, k0 + step * p, wf, bf);
#pragma unroll
    for (int j = 0; j < P; ++j) v[p][j] = mul2(mul2(v[p][j], R2), wf[j]);
  }
#pragma unroll
  for (int p = 0; p < NSLOT / 2; ++p)
    rotate_split_store_ns<T>(s, g.y_row + (k0 + step * p) * V, half, v[p], v[p + NSLOT / 2],
                             cs[p], sn[p], nsn[p], true);
}

// The row's cos / sin come from the table in global memory, or (TAB_SHARED,
// in-thread planes only) from `tab_shared`: a copy of the row's table row
// that the caller staged in shared memory.
template <bool TAB_SHARED, int N>
__device__ __forceinline__ void table_floats(const float* p, float (&d)[N]) {
  if constexpr (TAB_SHARED)
    load_floats<N>(p, d);
  else
    ldg_floats<N>(p, d);
}

template <typename T, bool LOCAL, bool EXACT, int SLOTS, int NSLOT, typename Src,
          bool TAB_SHARED = false>
__device__ __forceinline__ void normalize_rope_store(const Segment& s, const Row<T>& g,
                                                     F2 (&v)[NSLOT][Elem<T>::P], float xe,
                                                     const Src& src, int k0, int step,
                                                     float rstd, bool has_edge, long long r,
                                                     float* stage, unsigned mask,
                                                     const float* tab_shared = nullptr) {
  static_assert(!TAB_SHARED || LOCAL, "a staged table row serves in-thread planes");
  constexpr int V = Elem<T>::V;
  constexpr int P = Elem<T>::P;
  const int dims = s.rope_dims;
  const int half = dims >> 1;
  const bool trad = s.rope_trad != 0;
  // whole-chunk rotation: every chunk lies in one half (or past dims), and
  // every vector access below is 16-byte aligned
  const bool vec = EXACT && dims % (2 * V) == 0;
  static_assert(!LOCAL || EXACT, "in-thread planes need 16-byte aligned rows");
  const bool vstore = EXACT || s.vector_y;
  const F2 R2 = splat(rstd);
  // token = r / heads (32-bit division: head rows never reach 2^31)
  const long long token = r < 0x7fffffffLL ? (long long)((unsigned)r / (unsigned)s.rope_heads)
                                           : r / s.rope_heads;
  const float* tab = TAB_SHARED ? tab_shared : s.rope_table + (s.rope_offset + token) * dims;
  if constexpr (LOCAL && NSLOT % 2 == 0) {
    if (!trad) {
      // full split-half rotary whose chunks divide evenly: slot p < NSLOT/2
      // holds chunk f of the first half, slot p + NSLOT/2 its partner chunk
      // f + half / V (same planes, same cos / sin); all slots are present
      // (dims / V = step * NSLOT full chunks), nothing is staged
#pragma unroll
      for (int p = 0; p < NSLOT; ++p) {
        F2 wf[P], bf[P];
        src.get(p, k0 + step * p, wf, bf);
#pragma unroll
        for (int j = 0; j < P; ++j) v[p][j] = mul2(mul2(v[p][j], R2), wf[j]);
      }
#pragma unroll
      for (int p = 0; p < NSLOT / 2; ++p) {
        const int c0 = (k0 + step * p) * V;
        float cs[V], sn[V];
        table_floats<TAB_SHARED, V>(tab + c0, cs);
        table_floats<TAB_SHARED, V>(tab + half + c0, sn);
        rotate_split_store<T>(s, g.y_row + c0, half, v[p], v[p + NSLOT / 2], cs, sn, vstore);
      }
      return;
    }
  }
  if constexpr (LOCAL) {
    // planes (c0 + 2j, c0 + 2j + 1) are pairs of this thread's own chunk:
    // rotate as the chunk is normalized, nothing staged
#pragma unroll
    for (int p = 0; p < NSLOT; ++p) {
      const int f = k0 + step * p;
      if (!slot_present<SLOTS, NSLOT>(p, f, g.nfull)) continue;
      F2 wf[P], bf[P], o[P];
      src.get(p, f, wf, bf);
      const int c0 = f * V;
#pragma unroll
      for (int j = 0; j < P; ++j) o[j] = mul2(mul2(v[p][j], R2), wf[j]);
      if (c0 < dims) {
        float cs[P], sn[P];
        if constexpr (P % 4 == 0) {
          table_floats<TAB_SHARED, P>(tab + (c0 >> 1), cs);
          table_floats<TAB_SHARED, P>(tab + half + (c0 >> 1), sn);
        } else {
#pragma unroll
          for (int j = 0; j < P; ++j) {
            cs[j] = TAB_SHARED ? tab[(c0 >> 1) + j] : __ldg(tab + (c0 >> 1) + j);
            sn[j] = TAB_SHARED ? tab[half + (c0 >> 1) + j] : __ldg(tab + half + (c0 >> 1) + j);
          }
        }
#pragma unroll
        for (int j = 0; j < P; ++j) {
          // plane (a, b) = o[j]: (a cos - b sin, b cos + a sin) as one packed
          // multiply of the swapped pair and one packed fused multiply-add
          const F2 t = mul2(make2(o[j].y, o[j].x), splat(sn[j]));
          o[j] = fma2(o[j], splat(cs[j]), make2(-t.x, t.y));
        }
      }
      store_chunk<T>(s, g.y_row + c0, o, vstore);
    }
    return;
  }
#pragma unroll
  for (int p = 0; p < NSLOT; ++p) {
    const int f = k0 + step * p;
    if (!slot_present<SLOTS, NSLOT>(p, f, g.nfull)) continue;
    F2 wf[P], bf[P];
    src.get(p, f, wf, bf);
    float* dst = stage + g.head + f * V;
#pragma unroll
    for (int j = 0; j < P; ++j) {
      const F2 o = mul2(mul2(v[p][j], R2), wf[j]);
      if constexpr (EXACT) {
        *reinterpret_cast<float2*>(dst + 2 * j) = o;
      } else {
        dst[2 * j] = o.x;
        dst[2 * j + 1] = o.y;
      }
    }
  }
  if (!EXACT && has_edge) {
    float we, be;
    src.edge(we, be);
    stage[edge_column(g, s.dim, k0)] = __fmul_rn(__fmul_rn(xe, rstd), we);
  }
  __syncwarp(mask);
  // column c rotated with its plane partner, both read from the staging row
  auto rotate = [&](int c) -> float {
    const float o = stage[c];
    if (c >= dims) return o;
    int i, partner;
    bool first;
    if (trad) {
      i = c >> 1;
      partner = c ^ 1;
      first = (c & 1) == 0;
    } else {
      first = c < half;
      i = first ? c : c - half;
      partner = first ? c + half : c - half;
    }
    const float t = __fmul_rn(stage[partner], __ldg(tab + half + i));
    return __fmaf_rn(o, __ldg(tab + i), first ? -t : t);
  };
  // one chunk at a time: its own, partner and cos / sin vectors are 32
  // floats in flight, kept out of the next chunk's registers
#pragma unroll 1
  for (int p = 0; p < NSLOT; ++p) {
    const int f = k0 + step * p;
    if (!slot_present<SLOTS, NSLOT>(p, f, g.nfull)) continue;
    const int c0 = g.head + f * V;
    F2 o[P];
    if (vec && c0 < dims) {
      // split-half, whole chunk: its partners are the chunk half a
      // rotated width away
      const bool first = c0 < half;
      const int i0 = first ? c0 : c0 - half;
      float own[V], pt[V], cs[V], sn[V];
      load_floats<V>(stage + c0, own);
      load_floats<V>(stage + (first ? c0 + half : c0 - half), pt);
      ldg_floats<V>(tab + i0, cs);
      ldg_floats<V>(tab + half + i0, sn);
#pragma unroll
      for (int j = 0; j < V; j += 2) {
        const float t0 = __fmul_rn(pt[j], sn[j]);
        const float t1 = __fmul_rn(pt[j + 1], sn[j + 1]);
        o[j / 2] = make2(__fmaf_rn(own[j], cs[j], first ? -t0 : t0),
                         __fmaf_rn(own[j + 1], cs[j + 1], first ? -t1 : t1));
      }
    } else {
#pragma unroll
      for (int j = 0; j < P; ++j) o[j] = make2(rotate(c0 + 2 * j), rotate(c0 + 2 * j + 1));
    }
    store_chunk<T>(s, g.y_row + c0, o, vstore);
  }
  if (!EXACT && has_edge) {
    const int c = edge_column(g, s.dim, k0);
    Elem<T>::put(g.y_row + c, rotate(c));
  }
  __syncwarp(mask);
}

// Means are sums times 1/D rounded to binary32 (one multiply instead of a
// divide per row; exact for power-of-two D, within 2 ulps otherwise).
__device__ __forceinline__ float inv_dim(int D) { return __frcp_rn((float)D); }

// rstd (and mean) of one row from the thread's slots and edge element, with
// `reduce` summing a per-thread partial over the threads of the row. For
// LayerNorm the slots and edge element leave centred (x - K - mean).
// inv_d is inv_dim(D), computed once per row space by the caller.
template <typename T, int OP, bool EXACT, int SLOTS, int NSLOT, typename Reduce>
__device__ __forceinline__ void row_stats(F2 (&v)[NSLOT][Elem<T>::P], float& xe,
                                          const Row<T>& g, float inv_d, int k0, int step, float K,
                                          float eps, bool has_edge, Reduce reduce, float& rstd,
                                          float& mean) {
  if (OP != kOpLn) {
    const float ss = reduce(sum_squares<T, EXACT, NSLOT>(v, xe, has_edge));
    mean = 0.f;
    rstd = rsqrtf(__fadd_rn(__fmul_rn(ss, inv_d), eps));
  } else {
    const float s1 = reduce(shift_and_sum<T, EXACT, SLOTS, NSLOT>(v, xe, g, k0, step, K, has_edge));
    mean = __fmul_rn(s1, inv_d);
    const float s2 =
        reduce(sum_dev_squares<T, EXACT, SLOTS, NSLOT>(v, xe, g, k0, step, mean, has_edge));
    rstd = rsqrtf(__fadd_rn(__fmul_rn(s2, inv_d), eps));
  }
}

}  // namespace rn
