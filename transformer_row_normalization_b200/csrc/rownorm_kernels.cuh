// Register-resident row normalization kernels (sm_100a).
//
// Each row is read from HBM once into registers (as binary32 pairs), reduced
// and written back; the per-row arithmetic, layout and summation order are
// those of rownorm_core.cuh. Two families:
//   rows_warp_kernel  a group of G lanes (a power of two <= 32) of one warp
//                     owns a row; G is chosen so each lane holds about four
//                     16-byte chunks. Used for D <= 1024.
//   rows_cta_kernel   one block of NT threads owns a row. Used for D > 1024.
// Both are persistent: the grid is sized to the SM count times resident
// blocks per SM, and rows are strided statically over the lane groups /
// blocks (no atomics, no work queue, no inter-block communication, no waits
// other than __syncthreads). Static striding also means a lane group or
// block sees rows of one 16-byte phase (lane groups always; blocks when the
// grid is a multiple of the phase period), so the realigned weight/bias
// cache of non-aligned layouts is filled once.
//
// The bulk-copy staged kernels (rownorm_staged.cuh) run the same per-row
// code on rows streamed through shared memory; the planner prefers them for
// large row counts, and the two give identical bits.
#pragma once

#include "rownorm_core.cuh"

namespace rn {

struct Params {
  Segment seg[2];
  int nseg;
  float eps;
};

__device__ __forceinline__ Segment pick_segment(const Segment (&seg)[2], int i) {
  return i == 0 ? seg[0] : seg[1];
}

constexpr int kWarpBlock = 256;
// Register budgets: at least this many threads resident per SM (lane-group
// family 768, i.e. up to 85 registers; block family 1024, 64 registers).
constexpr int kMinThreadsPerSmWarp = 768;
constexpr int kMinThreadsPerSm = 1024;

template <typename T, int OP, bool EXACT, int VPL>
__global__ void __launch_bounds__(kWarpBlock, kMinThreadsPerSmWarp / kWarpBlock)
rows_warp_kernel(const Params p) {
  constexpr int P = Elem<T>::P;
  constexpr bool BIAS = OP == kOpLn;
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const long long warp = (long long)blockIdx.x * (kWarpBlock / 32) + (threadIdx.x >> 5);
  const long long nwarps = (long long)gridDim.x * (kWarpBlock / 32);
#pragma unroll 1
  for (int si = 0; si < p.nseg; ++si) {
    const Segment s = pick_segment(p.seg, si);
    const int G = s.lanes;
    const int per_warp = 32 / G;
    const int gl = lane & (G - 1);
    const int gi = lane / G;
    const unsigned mask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << (gi * G));
    const long long ngroups = nwarps * per_warp;
    const int D = s.dim;
    AffineCache<T, VPL, BIAS> cache;
    if constexpr (!EXACT) cache.init(smem);
    const AffineDirect<T, BIAS> direct{static_cast<const T*>(s.w), static_cast<const T*>(s.b)};
    auto reduce = [&](float t) { return group_sum(t, G, mask); };
#pragma unroll 1
    for (long long r = warp * per_warp + gi; r < s.rows; r += ngroups) {
      float2 v[VPL][P];
      const Row<T> g = row_geometry<T, EXACT>(s, r);
#pragma unroll
      for (int q = 0; q < VPL; ++q) load_chunk<T, EXACT>(g, D, gl + G * q, v[q]);
      const float K =
          OP == kOpLn ? Elem<T>::get(static_cast<const T*>(s.x) + r * s.x_stride) : 0.f;
      float rstd, mean;
      row_stats<T, OP, EXACT, VPL>(v, g, D, gl, G, K, p.eps, reduce, rstd, mean);
      if constexpr (EXACT) {
        normalize_store<T, OP, EXACT, VPL>(s, g, v, direct, gl, G, rstd, mean);
      } else {
        if (g.phase != cache.phase) cache.fill(s, g.phase, gl, G);
        normalize_store<T, OP, EXACT, VPL>(s, g, v, cache, gl, G, rstd, mean);
      }
    }
  }
}

template <typename T, int OP, bool EXACT, int NT, int VPT>
__global__ void __launch_bounds__(NT, kMinThreadsPerSm / NT)
rows_cta_kernel(const Params p) {
  constexpr int P = Elem<T>::P;
  constexpr bool BIAS = OP == kOpLn;
  // Two alternating reduction buffers: a buffer is rewritten only after every
  // thread has passed the barrier of the reduction in between.
  __shared__ float red[2][NT / 32];
  extern __shared__ __align__(128) unsigned char smem[];
  int slot = 0;
  const int tid = threadIdx.x;
  auto reduce = [&](float t) {
    const float r = block_sum<NT>(t, red[slot]);
    slot ^= 1;
    return r;
  };
#pragma unroll 1
  for (int si = 0; si < p.nseg; ++si) {
    const Segment s = pick_segment(p.seg, si);
    const int D = s.dim;
    AffineCache<T, VPT, BIAS> cache;
    if constexpr (!EXACT) cache.init(smem);
    const AffineDirect<T, BIAS> direct{static_cast<const T*>(s.w), static_cast<const T*>(s.b)};
#pragma unroll 1
    for (long long r = blockIdx.x; r < s.rows; r += gridDim.x) {
      float2 v[VPT][P];
      const Row<T> g = row_geometry<T, EXACT>(s, r);
#pragma unroll
      for (int q = 0; q < VPT; ++q) load_chunk<T, EXACT>(g, D, tid + NT * q, v[q]);
      const float K =
          OP == kOpLn ? Elem<T>::get(static_cast<const T*>(s.x) + r * s.x_stride) : 0.f;
      float rstd, mean;
      row_stats<T, OP, EXACT, VPT>(v, g, D, tid, NT, K, p.eps, reduce, rstd, mean);
      if constexpr (EXACT) {
        normalize_store<T, OP, EXACT, VPT>(s, g, v, direct, tid, NT, rstd, mean);
      } else {
        if (g.phase != cache.phase) cache.fill(s, g.phase, tid, NT);
        normalize_store<T, OP, EXACT, VPT>(s, g, v, cache, tid, NT, rstd, mean);
      }
    }
  }
}

}  // namespace rn
