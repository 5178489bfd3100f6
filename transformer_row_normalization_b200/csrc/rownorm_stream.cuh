// Streaming row normalization for rows too wide to hold in registers
// (sm_100a).
//
// One block of NT threads per row (1024, or 512 for several rows per SM),
// rows strided statically over a persistent grid. The row is read once per
// pass: RMSNorm makes two passes (sum of squares, then normalize and store),
// LayerNorm three (sum of d = x - K with K = x_0, then sum of (d - mean)^2,
// then normalize and store): the same shifted two-pass statistics as the
// register kernels, so a constant row still gives exactly the bias. (One
// pass of per-chunk (count, mean, squared deviations) merged by Chan et
// al.'s formula, then the store pass, gave the same results within
// tolerance but ran slower on B200: bf16 LayerNorm 8192 x 65536 416 -> 477
// us; each chunk's merge waits on the last, with a division.) Passes
// after the first find the row in L2 while the rows in flight (one or a few
// per SM) fit there.
//
// Ownership and summation order (fixed; they depend only on D, the element
// type and the row's 16-byte phase): thread t owns the full chunks t,
// t + NT, ... and edge element t (rownorm_core.cuh's row split);
// each pass sums the thread's chunks into even / odd binary32 pair
// partials in chunk order, adds the edge element's term, and combines the
// threads with block_sum. The arithmetic of each element is that of the
// register kernels.
#pragma once

#include "rownorm_core.cuh"
#include "rownorm_kernels.cuh"

namespace rn {

// chunks a thread loads before it uses the first of them (loads in flight)
constexpr int kStreamUnroll = 4;

// Cached 16-byte load (the row is read again by the next pass).
__device__ __forceinline__ uint4 load_keep(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// Where a vector's columns stand relative to the 16-byte grid at the row's
// chunks: kVecAligned (each chunk's columns are one aligned 16-byte word),
// an offset O in 1..V-1 elements past a boundary, or kVecElementwise
// (weight and bias at different offsets: element-by-element loads).
constexpr int kVecAligned = 0;
constexpr int kVecElementwise = -1;

// The V elements at p = pa + O (pa 16-byte aligned, 0 < O < V): the two
// aligned words at pa shifted down by O elements. Funnel shifts over the
// little-endian 32-bit lanes of the pair; both words must lie inside the
// vector (the caller checks).
template <typename T, int O>
__device__ __forceinline__ uint4 load_shifted(const T* pa) {
  constexpr int V = Elem<T>::V;
  constexpr int kBytes = O * (int)sizeof(T);
  static_assert(O > 0 && O < V, "offset within one 16-byte word");
  const uint4 lo = load_cached(pa);
  const uint4 hi = load_cached(pa + V);
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  uint32_t r[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if constexpr (kBytes % 4 == 0)
      r[j] = w[kBytes / 4 + j];
    else
      r[j] = __funnelshift_r(w[kBytes / 4 + j], w[kBytes / 4 + j + 1], 8 * (kBytes % 4));
  }
  return make_uint4(r[0], r[1], r[2], r[3]);
}

// Chunk f's columns of vector v (NULL: `none` everywhere) under offset
// class O.
template <typename T, int O>
__device__ __forceinline__ void stream_vector(const T* v, const Row<T>& g, int D, int f,
                                              float none, F2 (&vf)[Elem<T>::P]) {
  constexpr int V = Elem<T>::V;
  constexpr int P = Elem<T>::P;
  if (!v) {
#pragma unroll
    for (int j = 0; j < P; ++j) vf[j] = splat(none);
    return;
  }
  const int c0 = g.head + f * V;
  if constexpr (O == kVecAligned) {
    Elem<T>::unpack(load_cached(v + c0), vf);
    return;
  } else {
    if constexpr (O != kVecElementwise) {
      // both aligned words inside the vector: all chunks but at most the
      // first and the last
      if (c0 - O >= 0 && c0 - O + 2 * V <= D) {
        Elem<T>::unpack(load_shifted<T, O>(v + (c0 - O)), vf);
        return;
      }
    }
#pragma unroll
    for (int j = 0; j < P; ++j)
      vf[j] = make2(Elem<T>::get(v + c0 + 2 * j), Elem<T>::get(v + c0 + 2 * j + 1));
  }
}

// One pass over the thread's chunks of row g: `chunk(v)` folds each chunk's
// pairs into the accumulator (chunk order), kStreamUnroll loads in flight.
template <typename T, int NT, typename Fold>
__device__ __forceinline__ void stream_pass(const Row<T>& g, int tid, Fold fold) {
  constexpr int V = Elem<T>::V;
  constexpr int P = Elem<T>::P;
  int f = tid;
  constexpr int kStep = kStreamUnroll * NT;
  for (; f + (kStreamUnroll - 1) * NT < g.nfull; f += kStep) {
    uint4 u[kStreamUnroll];
#pragma unroll
    for (int q = 0; q < kStreamUnroll; ++q)
      u[q] = load_keep(g.x_full + (long long)(f + q * NT) * V);
#pragma unroll
    for (int q = 0; q < kStreamUnroll; ++q) {
      F2 v[P];
      Elem<T>::unpack(u[q], v);
      fold(v);
    }
  }
#pragma unroll 1
  for (; f < g.nfull; f += NT) {
    F2 v[P];
    Elem<T>::unpack(load_keep(g.x_full + (long long)f * V), v);
    fold(v);
  }
}

// The last pass over row g: normalize, weight (and bias) under vector
// offset class O, store the thread's full chunks.
template <typename T, int OP, bool EXACT, int NT, int O>
__device__ __forceinline__ void stream_store(const Segment& s, const Row<T>& g, int tid, F2 R2,
                                             F2 M2, F2 K2) {
  constexpr int V = Elem<T>::V;
  constexpr int P = Elem<T>::P;
  const T* w = static_cast<const T*>(s.w);
  const T* b = static_cast<const T*>(s.b);
#pragma unroll 1
  for (int f = tid; f < g.nfull; f += NT) {
    F2 v[P], wf[P], bf[P], o[P];
    Elem<T>::unpack(load_stream(g.x_full + (long long)f * V), v);
    stream_vector<T, O>(w, g, s.dim, f, 1.f, wf);
    if constexpr (OP == kOpLn) stream_vector<T, O>(b, g, s.dim, f, 0.f, bf);
#pragma unroll
    for (int j = 0; j < P; ++j) {
      if constexpr (OP == kOpLn)
        o[j] = fma2(mul2(sub2(sub2(v[j], K2), M2), R2), wf[j], bf[j]);
      else
        o[j] = mul2(mul2(v[j], R2), wf[j]);
    }
    T* yc = g.y_row + g.head + (long long)f * V;
    if (EXACT || s.vector_y) {
      store_stream(yc, Elem<T>::pack(o));
    } else {
#pragma unroll
      for (int j = 0; j < P; ++j) {
        Elem<T>::put(yc + 2 * j, o[j].x);
        Elem<T>::put(yc + 2 * j + 1, o[j].y);
      }
    }
  }
}

// stream_store under the runtime offset class `cls` (rows off the grid).
template <typename T, int OP, int NT, int O = 1>
__device__ __forceinline__ void stream_store_offset(int cls, const Segment& s, const Row<T>& g,
                                                    int tid, F2 R2, F2 M2, F2 K2) {
  if constexpr (O < Elem<T>::V) {
    if (cls == O) {
      stream_store<T, OP, false, NT, O>(s, g, tid, R2, M2, K2);
    } else {
      stream_store_offset<T, OP, NT, O + 1>(cls, s, g, tid, R2, M2, K2);
    }
  } else if (cls == kVecAligned) {
    stream_store<T, OP, false, NT, kVecAligned>(s, g, tid, R2, M2, K2);
  } else {
    stream_store<T, OP, false, NT, kVecElementwise>(s, g, tid, R2, M2, K2);
  }
}

template <typename T, int OP, bool EXACT, int NT>
__global__ void __launch_bounds__(NT, 1024 / NT) rows_stream_kernel(const Params p) {
  static_assert(OP == kOpRms || OP == kOpLn, "streaming covers RMSNorm and LayerNorm");
  constexpr int P = Elem<T>::P;
  constexpr bool BIAS = OP == kOpLn;
  __shared__ float red[2][NT / 32];
  int slot = 0;
  auto reduce = [&](float t) {
    const float r = block_sum<NT>(t, red[slot]);
    slot ^= 1;
    return r;
  };
  const Segment& s = p.seg[0];
  const int tid = threadIdx.x;
  const int D = s.dim;
  const float inv_d = __frcp_rn((float)D);
#pragma unroll 1
  for (long long r = blockIdx.x; r < s.rows; r += gridDim.x) {
    const Row<T> g = row_geometry<T, EXACT>(s, r);
    const bool has_edge = !EXACT && tid < g.nedge;
    float xe = load_edge<T, EXACT>(g, D, tid);
    // LayerNorm shift K = x_0, read once before any pass: with y == x the
    // store pass overwrites column 0, so the row must not be read from
    // global memory again once the final reduction is done.
    const float K = OP == kOpLn ? Elem<T>::get(g.x_row) : 0.f;
    const F2 K2 = splat(K);
    float rstd, mean = 0.f;
    if constexpr (OP == kOpRms) {
      F2 acc = zero2();
      stream_pass<T, NT>(g, tid, [&](F2 (&v)[P]) {
#pragma unroll
        for (int j = 0; j < P; ++j) acc = fma2(v[j], v[j], acc);
      });
      float part = hsum2(acc);
      if (has_edge) part = __fmaf_rn(xe, xe, part);
      rstd = rsqrtf(__fadd_rn(__fmul_rn(reduce(part), inv_d), p.eps));
    } else {
      F2 acc = zero2();
      stream_pass<T, NT>(g, tid, [&](F2 (&v)[P]) {
#pragma unroll
        for (int j = 0; j < P; ++j) acc = add2(acc, sub2(v[j], K2));
      });
      float part = hsum2(acc);
      if (has_edge) {
        xe = __fsub_rn(xe, K);
        part = __fadd_rn(part, xe);
      }
      mean = __fmul_rn(reduce(part), inv_d);
      const F2 M2 = splat(mean);
      acc = zero2();
      stream_pass<T, NT>(g, tid, [&](F2 (&v)[P]) {
#pragma unroll
        for (int j = 0; j < P; ++j) {
          const F2 t = sub2(sub2(v[j], K2), M2);
          acc = fma2(t, t, acc);
        }
      });
      part = hsum2(acc);
      if (has_edge) {
        const float t = __fsub_rn(xe, mean);
        part = __fmaf_rn(t, t, part);
      }
      rstd = rsqrtf(__fadd_rn(__fmul_rn(reduce(part), inv_d), p.eps));
    }
    // last pass: normalize, weight (and bias), store
    const F2 R2 = splat(rstd);
    const F2 M2 = splat(mean);
    if constexpr (EXACT) {
      stream_store<T, OP, true, NT, kVecAligned>(s, g, tid, R2, M2, K2);
    } else {
      // elements from the 16-byte boundary to the columns of the row's
      // first chunk, per present vector; different offsets go element-wise
      auto offset = [&](const void* v) {
        return v ? (int)((reinterpret_cast<uintptr_t>(static_cast<const T*>(v) + g.head) % 16) /
                         sizeof(T))
                 : -2;
      };
      const int ow = offset(s.w);
      const int ob = BIAS ? offset(s.b) : -2;
      const int cls = ow == -2 ? (ob == -2 ? kVecAligned : ob)
                               : (ob == -2 || ob == ow ? ow : kVecElementwise);
      stream_store_offset<T, OP, NT>(cls, s, g, tid, R2, M2, K2);
    }
    if (has_edge) {
      const int c = edge_column(g, D, tid);
      const T* w = static_cast<const T*>(s.w);
      const T* b = static_cast<const T*>(s.b);
      const float we = w ? Elem<T>::get(w + c) : 1.f;
      float o;
      if constexpr (OP == kOpLn) {
        const float be = b ? Elem<T>::get(b + c) : 0.f;
        o = __fmaf_rn(__fmul_rn(__fsub_rn(xe, mean), rstd), we, be);
      } else {
        o = __fmul_rn(__fmul_rn(xe, rstd), we);
      }
      Elem<T>::put(g.y_row + c, o);
    }
  }
}

}  // namespace rn
