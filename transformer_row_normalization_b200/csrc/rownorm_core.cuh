// Per-row arithmetic shared by every row-normalization kernel (sm_100a).
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
//   here run over a row already on chip, so they cost no extra HBM traffic
//   and give the same population mean and variance.
//
// Row layout. A row is moved as 16-byte chunks on the 16-byte address grid:
// chunk k of a row whose first element sits `phase` elements past a 16-byte
// boundary covers columns [k*V - phase, k*V - phase + V), V = 16 / element
// size. Chunks wholly inside the row move with one 16-byte access; the (at
// most two) partial chunks at the row ends move element by element, so no
// byte outside the caller's views is touched. A thread owns chunks
// k0, k0 + step, k0 + 2*step, ... of every row it works on (slots).
//
// Arithmetic. Elements are processed as pairs (columns 2j, 2j+1 of a chunk)
// with the packed binary32 instructions of sm_100 (add/sub/mul/fma .f32x2);
// each lane of a packed instruction rounds exactly like its scalar form.
//
// Summation order (fixed; it depends only on D, the element type, the
// threads per row and the row's 16-byte phase):
//   1. each thread keeps two partial sums, one over the elements at even
//      positions of its chunks and one over the odd positions, each added in
//      slot order then position order; its partial is even + odd;
//   2. an xor butterfly over the G lanes sharing the row (offsets G/2 .. 1);
//   3. for rows owned by a whole block of NW warps, the per-warp sums are
//      combined by the same xor butterfly over lanes 0 .. NW-1 (warp w's sum
//      at lane w) in every warp, then broadcast from lane 0, so every thread
//      ends with the same bits.
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
  int lanes;       // threads per row in the lane-group kernels (power of two <= 32)
  int vector_y;    // 1: every y row has its x row's 16-byte phase
  int pad_;
};

// ---------------------------------------------------------------------------
// packed binary32 pairs

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " add.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " sub.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " mul.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " mov.b64 rc, {%6, %7};\n fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 splat(float v) { return make_float2(v, v); }

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
  static __device__ __forceinline__ void unpack(const uint4& u, float2 (&f)[2]) {
    f[0] = make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
    f[1] = make_float2(__uint_as_float(u.z), __uint_as_float(u.w));
  }
  static __device__ __forceinline__ uint4 pack(const float2 (&f)[2]) {
    return make_uint4(__float_as_uint(f[0].x), __float_as_uint(f[0].y),
                      __float_as_uint(f[1].x), __float_as_uint(f[1].y));
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
  static __device__ __forceinline__ float2 pair(uint32_t w) {
    __nv_bfloat162 h;
    *reinterpret_cast<uint32_t*>(&h) = w;
    return __bfloat1622float2(h);
  }
  static __device__ __forceinline__ uint32_t pack_pair(float2 v) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ void unpack(const uint4& u, float2 (&f)[4]) {
    f[0] = pair(u.x);
    f[1] = pair(u.y);
    f[2] = pair(u.z);
    f[3] = pair(u.w);
  }
  static __device__ __forceinline__ uint4 pack(const float2 (&f)[4]) {
    return make_uint4(pack_pair(f[0]), pack_pair(f[1]), pack_pair(f[2]), pack_pair(f[3]));
  }
  static __device__ __forceinline__ uint4 assemble(const uint32_t (&e)[8]) {
    return make_uint4(e[0] | (e[1] << 16), e[2] | (e[3] << 16), e[4] | (e[5] << 16),
                      e[6] | (e[7] << 16));
  }
};

// ---------------------------------------------------------------------------
// memory access

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

// EXACT: the planner guarantees that every x and y row starts on a 16-byte
// boundary, D is a multiple of V, and the weight and bias (where present)
// start on 16-byte boundaries; so the phase is 0 and every chunk is full.
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

// Chunk k of a row from global memory; columns outside [0, D) (and chunks
// past the row) read as 0 and are never dereferenced.
template <typename T, bool EXACT>
__device__ __forceinline__ void load_chunk(const Row<T>& g, int D, int k,
                                           float2 (&f)[Elem<T>::P]) {
  constexpr int V = Elem<T>::V;
  constexpr int P = Elem<T>::P;
  if (chunk_full<T, EXACT>(g, k)) {
    Elem<T>::unpack(load_stream(g.x_al + (long long)k * V), f);
  } else if constexpr (EXACT) {
#pragma unroll
    for (int j = 0; j < P; ++j) f[j] = make_float2(0.f, 0.f);
  } else {
#pragma unroll
    for (int j = 0; j < P; ++j) {
      const int c = k * V + 2 * j - g.phase;
      f[j].x = ((unsigned)c < (unsigned)D) ? Elem<T>::get(g.x_al + k * V + 2 * j) : 0.f;
      f[j].y = ((unsigned)(c + 1) < (unsigned)D) ? Elem<T>::get(g.x_al + k * V + 2 * j + 1)
                                                 : 0.f;
    }
  }
}

// ---------------------------------------------------------------------------
// per-thread partial sums over the slots of one row

// RMSNorm: sum of squares (absent columns hold zeros, which add nothing).
template <typename T, int NSLOT>
__device__ __forceinline__ float sum_squares(const float2 (&v)[NSLOT][Elem<T>::P]) {
  constexpr int P = Elem<T>::P;
  float2 acc = make_float2(0.f, 0.f);
#pragma unroll
  for (int p = 0; p < NSLOT; ++p)
#pragma unroll
    for (int j = 0; j < P; ++j) acc = fma2(v[p][j], v[p][j], acc);
  return __fadd_rn(acc.x, acc.y);
}

// LayerNorm pass 1: replaces x by d = x - K (zero outside the row) and
// returns the thread's sum of d.
template <typename T, bool EXACT, int NSLOT>
__device__ __forceinline__ float shift_and_sum(float2 (&v)[NSLOT][Elem<T>::P], const Row<T>& g,
                                               int D, int k0, int step, float K) {
  constexpr int V = Elem<T>::V;
  constexpr int P = Elem<T>::P;
  const float2 K2 = splat(K);
  float2 acc = make_float2(0.f, 0.f);
#pragma unroll
  for (int p = 0; p < NSLOT; ++p) {
    const int k = k0 + step * p;
    if (chunk_full<T, EXACT>(g, k)) {
#pragma unroll
      for (int j = 0; j < P; ++j) {
        v[p][j] = sub2(v[p][j], K2);
        acc = add2(acc, v[p][j]);
      }
    } else if constexpr (!EXACT) {
#pragma unroll
      for (int j = 0; j < P; ++j) {
        const int c = k * V + 2 * j - g.phase;
        const float2 d = sub2(v[p][j], K2);
        v[p][j].x = ((unsigned)c < (unsigned)D) ? d.x : 0.f;
        v[p][j].y = ((unsigned)(c + 1) < (unsigned)D) ? d.y : 0.f;
        acc = add2(acc, v[p][j]);
      }
    }
  }
  return __fadd_rn(acc.x, acc.y);
}

// LayerNorm pass 2: the thread's sum of (d - mean)^2 over the row's columns.
template <typename T, bool EXACT, int NSLOT>
__device__ __forceinline__ float sum_dev_squares(const float2 (&v)[NSLOT][Elem<T>::P],
                                                 const Row<T>& g, int D, int k0, int step,
                                                 float mean) {
  constexpr int V = Elem<T>::V;
  constexpr int P = Elem<T>::P;
  const float2 M2 = splat(mean);
  float2 acc = make_float2(0.f, 0.f);
#pragma unroll
  for (int p = 0; p < NSLOT; ++p) {
    const int k = k0 + step * p;
    if (chunk_full<T, EXACT>(g, k)) {
#pragma unroll
      for (int j = 0; j < P; ++j) {
        const float2 t = sub2(v[p][j], M2);
        acc = fma2(t, t, acc);
      }
    } else if constexpr (!EXACT) {
#pragma unroll
      for (int j = 0; j < P; ++j) {
        const int c = k * V + 2 * j - g.phase;
        float2 t = sub2(v[p][j], M2);
        t.x = ((unsigned)c < (unsigned)D) ? t.x : 0.f;
        t.y = ((unsigned)(c + 1) < (unsigned)D) ? t.y : 0.f;
        acc = fma2(t, t, acc);
      }
    }
  }
  return __fadd_rn(acc.x, acc.y);
}

// ---------------------------------------------------------------------------
// reductions across the threads of a row

// xor butterfly over the G lanes of `mask` (G a power of two <= 32).
__device__ __forceinline__ float group_sum(float x, int G, unsigned mask) {
  for (int off = G >> 1; off > 0; off >>= 1) x = __fadd_rn(x, __shfl_xor_sync(mask, x, off));
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

// EXACT rows: the weight/bias columns of chunk k are one aligned 16-byte
// chunk of each vector (L1-resident after the first row).
template <typename T, bool BIAS>
struct AffineDirect {
  const T* w;
  const T* b;
  __device__ __forceinline__ void get(int /*p*/, int k, float2 (&wf)[Elem<T>::P],
                                      float2 (&bf)[Elem<T>::P]) const {
    constexpr int V = Elem<T>::V;
    constexpr int P = Elem<T>::P;
    if (w) {
      Elem<T>::unpack(load_cached(w + k * V), wf);
    } else {
#pragma unroll
      for (int j = 0; j < P; ++j) wf[j] = make_float2(1.f, 1.f);
    }
    if constexpr (BIAS) {
      if (b) {
        Elem<T>::unpack(load_cached(b + k * V), bf);
      } else {
#pragma unroll
        for (int j = 0; j < P; ++j) bf[j] = make_float2(0.f, 0.f);
      }
    }
  }
};

// Any layout: the weight/bias columns of each of the thread's slots,
// realigned to the row phase, in the thread's own shared memory entries
// [slot][thread] (no other thread touches them, so no barrier; consecutive
// threads use consecutive 16-byte words, so no bank conflicts). Refilled
// when a row with another phase arrives. NULL weight = ones, NULL bias =
// zeros.
template <typename T, int NSLOT, bool BIAS>
struct AffineCache {
  uint4* w;  // [NSLOT][blockDim.x]
  uint4* b;  // [NSLOT][blockDim.x] (BIAS)
  int phase;

  __device__ __forceinline__ void init(unsigned char* smem) {
    w = reinterpret_cast<uint4*>(smem);
    b = w + NSLOT * blockDim.x;
    phase = -1;
  }

  __device__ __forceinline__ void fill(const Segment& s, int row_phase, int k0, int step) {
    constexpr int V = Elem<T>::V;
    const T* wv = static_cast<const T*>(s.w);
    const T* bv = static_cast<const T*>(s.b);
    const int D = s.dim;
#pragma unroll 1
    for (int p = 0; p < NSLOT; ++p) {
      const int c0 = (k0 + step * p) * V - row_phase;
      uint32_t e[V];
#pragma unroll
      for (int i = 0; i < V; ++i) {
        const int c = c0 + i;
        e[i] = (wv && (unsigned)c < (unsigned)D) ? Elem<T>::get_bits(wv + c) : Elem<T>::kOneBits;
      }
      w[p * blockDim.x + threadIdx.x] = Elem<T>::assemble(e);
      if constexpr (BIAS) {
#pragma unroll
        for (int i = 0; i < V; ++i) {
          const int c = c0 + i;
          e[i] = (bv && (unsigned)c < (unsigned)D) ? Elem<T>::get_bits(bv + c) : 0u;
        }
        b[p * blockDim.x + threadIdx.x] = Elem<T>::assemble(e);
      }
    }
    phase = row_phase;
  }

  __device__ __forceinline__ void get(int p, int /*k*/, float2 (&wf)[Elem<T>::P],
                                      float2 (&bf)[Elem<T>::P]) const {
    Elem<T>::unpack(w[p * blockDim.x + threadIdx.x], wf);
    if constexpr (BIAS) Elem<T>::unpack(b[p * blockDim.x + threadIdx.x], bf);
  }
};

template <int NSLOT, bool BIAS>
constexpr int affine_cache_bytes(int threads) {
  return threads * NSLOT * 16 * (BIAS ? 2 : 1);
}

// Normalize the thread's chunks of one row, apply weight (and bias), store.
template <typename T, int OP, bool EXACT, int NSLOT, typename Src>
__device__ __forceinline__ void normalize_store(const Segment& s, const Row<T>& g,
                                                const float2 (&v)[NSLOT][Elem<T>::P],
                                                const Src& src, int k0, int step, float rstd,
                                                float mean) {
  constexpr int V = Elem<T>::V;
  constexpr int P = Elem<T>::P;
  const int D = s.dim;
  const float2 R2 = splat(rstd);
  const float2 M2 = splat(mean);
#pragma unroll
  for (int p = 0; p < NSLOT; ++p) {
    const int k = k0 + step * p;
    if (k >= g.nch) continue;
    float2 wf[P], bf[P], o[P];
    src.get(p, k, wf, bf);
#pragma unroll
    for (int j = 0; j < P; ++j) {
      if constexpr (OP == kOpRms)
        o[j] = mul2(mul2(v[p][j], R2), wf[j]);
      else
        o[j] = fma2(mul2(sub2(v[p][j], M2), R2), wf[j], bf[j]);
    }
    if (EXACT || (s.vector_y && chunk_full<T, EXACT>(g, k))) {
      store_stream(g.y_row - g.phase + (long long)k * V, Elem<T>::pack(o));
    } else {
#pragma unroll
      for (int j = 0; j < P; ++j) {
        const int c = k * V + 2 * j - g.phase;
        if ((unsigned)c < (unsigned)D) Elem<T>::put(g.y_row + c, o[j].x);
        if ((unsigned)(c + 1) < (unsigned)D) Elem<T>::put(g.y_row + c + 1, o[j].y);
      }
    }
  }
}

// rstd (and mean) of one row from the thread's slots, with `reduce` summing
// a per-thread partial over the threads of the row.
template <typename T, int OP, bool EXACT, int NSLOT, typename Reduce>
__device__ __forceinline__ void row_stats(float2 (&v)[NSLOT][Elem<T>::P], const Row<T>& g,
                                          int D, int k0, int step, float K, float eps,
                                          Reduce reduce, float& rstd, float& mean) {
  const float d_f = (float)D;
  if (OP == kOpRms) {
    const float ss = reduce(sum_squares<T, NSLOT>(v));
    mean = 0.f;
    rstd = rsqrtf(__fadd_rn(__fdiv_rn(ss, d_f), eps));
  } else {
    const float s1 = reduce(shift_and_sum<T, EXACT, NSLOT>(v, g, D, k0, step, K));
    mean = __fdiv_rn(s1, d_f);
    const float s2 = reduce(sum_dev_squares<T, EXACT, NSLOT>(v, g, D, k0, step, mean));
    rstd = rsqrtf(__fadd_rn(__fdiv_rn(s2, d_f), eps));
  }
}

}  // namespace rn
