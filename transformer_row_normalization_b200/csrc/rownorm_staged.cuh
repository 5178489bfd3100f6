// Bulk-copy staged row normalization (sm_100a).
//
// The register kernels (rownorm_kernels.cuh) issue a row's loads only after
// the previous row has been reduced and stored, so an SM has little more
// than its current rows in flight. Here one thread per block keeps S stages
// of upcoming rows streaming from HBM into shared memory with the bulk-copy
// engine (cp.async.bulk, completion counted on an mbarrier), while all
// threads work on earlier stages. A stage is refilled only after the block
// barrier that follows everyone's reads of it, so up to S tiles (tens of KB
// per block) are in flight at all times.
//
// Each thread moves its chunks of a row from the stage into registers once
// and then runs exactly the register kernels' per-row code (rownorm_core.cuh):
// the same threads per row (lane groups of G for D <= 1024, a block of NT
// for wider rows), chunk-to-thread mapping, summation order, shift K = x_0
// and operation order. Which kernel the planner picks never changes a bit.
//
// Tiles. NARROW (lane groups; EXACT layouts only): a tile is TR consecutive
// rows, moved as one bulk copy when they are adjacent in memory, otherwise
// one copy per row. WIDE (one block per row): a tile is one row; its full
// 16-byte chunks move as one bulk copy and its edge elements are read one by
// one from global memory by their owners.
//
// Waits are bounded: a thread waiting for a stage gives up after
// kWaitLimitNs, the block leaves its loop together (the decision is taken
// with __syncthreads_or), the issuing thread then waits, again bounded, for
// its copies still in flight, and the device error counter is raised
// (read on the host with rn_device_error_count()).
#pragma once

#include "rownorm_kernels.cuh"

namespace rn {

// Timed-out waits. Each translation unit that instantiates these kernels has
// its own copy (internal linkage) and a host accessor beside its table.
static __device__ unsigned int g_wait_timeouts;

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s
constexpr int kMaxStagesDevice = 8;

struct StagedParams {
  Segment seg[2];
  int nseg;
  float eps;
  int stages;          // S <= kMaxStagesDevice
  int stage_bytes;     // bytes per stage (multiple of 128)
  int tile_rows[2];    // rows per tile, per segment (WIDE: 1)
  int contiguous[2];   // 1: a tile's rows are adjacent in memory
  long long tiles[2];  // tiles per segment
  int cache_offset;    // byte offset of the weight/bias cache in shared memory
};

__device__ __forceinline__ unsigned long long global_timer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait for the phase of `bar` with the given parity to complete.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// Global -> shared bulk copy of `bytes` (16-byte aligned addresses, a
// multiple of 16 bytes), completion counted on `bar`. No multicast.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Tiles of segment `si` owned by this block: blockIdx.x, blockIdx.x + grid, ...
__device__ __forceinline__ long long my_tiles(const StagedParams& p, int si) {
  return p.tiles[si] > blockIdx.x ? (p.tiles[si] - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
}

// The i-th tile of this block's sequence (segment 0's tiles, then segment 1's).
__device__ __forceinline__ void locate_tile(long long mine0, long long i, int& si,
                                            long long& tile) {
  si = i < mine0 ? 0 : 1;
  tile = blockIdx.x + (i - (si ? mine0 : 0)) * (long long)gridDim.x;
}

template <typename T, bool WIDE>
__device__ __forceinline__ void issue_tile(const StagedParams& p, long long mine0, long long i,
                                           unsigned char* dst, uint64_t* bar) {
  constexpr int V = Elem<T>::V;
  int si;
  long long tile;
  locate_tile(mine0, i, si, tile);
  const Segment& s = p.seg[si];
  if constexpr (WIDE) {
    const Row<T> g = row_geometry<T, false>(s, tile);
    const uint32_t bytes = (uint32_t)g.nfull * 16u;
    mbar_expect_tx(bar, bytes);
    if (bytes) bulk_load(dst, g.x_full, bytes, bar);
  } else {
    const long long r0 = tile * p.tile_rows[si];
    long long nr = s.rows - r0;
    if (nr > p.tile_rows[si]) nr = p.tile_rows[si];
    const uint32_t row_bytes = (uint32_t)s.dim * sizeof(T);
    const T* x0 = static_cast<const T*>(s.x) + r0 * s.x_stride;
    mbar_expect_tx(bar, (uint32_t)nr * row_bytes);
    if (p.contiguous[si]) {
      bulk_load(dst, x0, (uint32_t)nr * row_bytes, bar);
    } else {
      for (long long r = 0; r < nr; ++r)
        bulk_load(dst + r * row_bytes, x0 + r * s.x_stride, row_bytes, bar);
    }
  }
}

template <typename T, int OP, bool WIDE, bool EXACT, int NT, int VPT>
__global__ void __launch_bounds__(NT, (NT >= 1024 ? 1 : 1024 / NT))
rows_staged_kernel(const StagedParams p) {
  constexpr int P = Elem<T>::P;
  constexpr bool BIAS = OP == kOpLn;
  static_assert(WIDE || EXACT, "lane-group rows are staged only for 16-byte aligned layouts");
  static_assert(!WIDE || NT >= 2 * (Elem<T>::V - 1), "every edge element needs its own thread");
  unsigned char* const smem = reinterpret_cast<unsigned char*>(dyn_smem);
  __shared__ __align__(8) uint64_t full[kMaxStagesDevice];
  __shared__ float red[2][NT / 32];
  const int tid = threadIdx.x;
  const int S = p.stages;
  const long long mine0 = my_tiles(p, 0);
  const long long n = mine0 + (p.nseg > 1 ? my_tiles(p, 1) : 0);

  if (tid == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  long long issued = 0;  // meaningful in thread 0 only
  if (tid == 0) {
    for (; issued < n && issued < S; ++issued)
      issue_tile<T, WIDE>(p, mine0, issued, smem + (issued % S) * (long long)p.stage_bytes,
                          &full[issued % S]);
  }

  int slot = 0;
  auto block_reduce = [&](float t) {
    const float r = block_sum<NT>(t, red[slot]);
    slot ^= 1;
    return r;
  };
  int cur_seg = -1;
  AffineCache<T, VPT, BIAS> cache;
  if constexpr (!EXACT) cache.init(p.cache_offset / 16);
  bool aborted = false;
#pragma unroll 1
  for (long long i = 0; i < n; ++i) {
    const int st = (int)(i % S);
    const bool ok = mbar_wait(&full[st], (uint32_t)((i / S) & 1));
    // Uniform exit on a timed-out wait; this barrier also proves that every
    // thread has finished with tile i-1, so its stage can be refilled.
    if (__syncthreads_or(!ok)) {
      aborted = true;
      break;
    }
    if (tid == 0 && i >= 1 && issued < n) {
      fence_async_shared();
      const int rs = (int)((i - 1) % S);
      issue_tile<T, WIDE>(p, mine0, issued, smem + rs * (long long)p.stage_bytes, &full[rs]);
      ++issued;
    }
    int si;
    long long tile;
    locate_tile(mine0, i, si, tile);
    const Segment s = pick_segment(p.seg, si);
    const unsigned char* stage = smem + st * (long long)p.stage_bytes;
    const AffineDirect<T, BIAS, false> direct{static_cast<const T*>(s.w), static_cast<const T*>(s.b)};
    if constexpr (!EXACT) {
      if (si != cur_seg) cache.phase = -1;
    }
    cur_seg = si;
    if constexpr (WIDE) {
      const int D = s.dim;
      const Row<T> g = row_geometry<T, EXACT>(s, tile);
      F2 v[VPT][P];
#pragma unroll
      for (int q = 0; q < VPT; ++q) {
        const int f = tid + NT * q;
        if (f < g.nfull) {
          Elem<T>::unpack(*reinterpret_cast<const uint4*>(stage + 16 * f), v[q]);
        } else {
#pragma unroll
          for (int j = 0; j < P; ++j) v[q][j] = zero2();
        }
      }
      float K = 0.f;
      if (OP == kOpLn)
        K = (g.head || !g.nfull) ? Elem<T>::get(g.x_row)
                                 : Elem<T>::get(reinterpret_cast<const T*>(stage));
      const bool has_edge = !EXACT && tid < g.nedge;
      float xe = load_edge<T, EXACT>(g, D, tid);
      float rstd, mean;
      row_stats<T, OP, EXACT, kSlotsTested, VPT>(v, xe, g, D, tid, NT, K, p.eps, has_edge, block_reduce,
                                          rstd, mean);
      if constexpr (EXACT) {
        normalize_store<T, OP, EXACT, kSlotsTested, VPT>(s, g, v, xe, direct, tid, NT, rstd, mean,
                                                  has_edge);
      } else {
        if (g.phase != cache.phase) cache.fill(s, g, tid, NT);
        normalize_store<T, OP, EXACT, kSlotsTested, VPT>(s, g, v, xe, cache, tid, NT, rstd, mean,
                                                  has_edge);
      }
    } else {
      const int G = s.lanes;
      const int lane = tid & 31;
      const int gl = lane & (G - 1);
      const int gi = lane / G;
      const unsigned mask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << (gi * G));
      auto group_reduce = [&](float t) { return group_sum(t, G, mask); };
      const int groups = NT / G;
      const int group = (tid >> 5) * (32 / G) + gi;
      const long long r0 = tile * p.tile_rows[si];
      long long nr = s.rows - r0;
      if (nr > p.tile_rows[si]) nr = p.tile_rows[si];
      const int D = s.dim;
      const int row_bytes = D * (int)sizeof(T);
#pragma unroll 1
      for (int rr = group; rr < nr; rr += groups) {
        const Row<T> g = row_geometry<T, true>(s, r0 + rr);
        const unsigned char* row = stage + rr * row_bytes;
        F2 v[VPT][P];
#pragma unroll
        for (int q = 0; q < VPT; ++q) {
          const int f = gl + G * q;
          if (f < g.nfull) {
            Elem<T>::unpack(*reinterpret_cast<const uint4*>(row + 16 * f), v[q]);
          } else {
#pragma unroll
            for (int j = 0; j < P; ++j) v[q][j] = zero2();
          }
        }
        const float K = OP == kOpLn ? Elem<T>::get(reinterpret_cast<const T*>(row)) : 0.f;
        float xe = 0.f, rstd, mean;
        row_stats<T, OP, true, kSlotsTested, VPT>(v, xe, g, D, gl, G, K, p.eps, false, group_reduce, rstd,
                                    mean);
        normalize_store<T, OP, true, kSlotsTested, VPT>(s, g, v, xe, direct, gl, G, rstd, mean, false);
      }
    }
  }
  if (aborted && tid == 0) {
    atomicAdd(&g_wait_timeouts, 1u);
    // wait (bounded) for this block's copies still in flight
    for (long long j = issued - S < 0 ? 0 : issued - S; j < issued; ++j)
      mbar_wait(&full[j % S], (uint32_t)((j / S) & 1));
  }
}

}  // namespace rn
