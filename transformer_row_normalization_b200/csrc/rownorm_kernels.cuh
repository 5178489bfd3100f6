// Register-resident row normalization kernels (sm_100a).
//
// Each row is read from HBM once and normalized from registers (as binary32
// pairs); the per-row arithmetic, layout and summation order are those of
// rownorm_core.cuh. Two families:
//   rows_warp_kernel  a group of G lanes (a power of two <= 32) of one warp
//                     owns a row; G is chosen so each lane holds about four
//                     16-byte chunks (whole warps of up to 8 chunks per lane
//                     for the widest rows). Used for D <= 1024 (binary32) or
//                     2048 (bf16).
//   rows_cta_kernel   one block of NT threads owns a row. Used above that.
// Both are persistent: the grid is sized to the SM count times resident
// blocks per SM, and rows are strided statically over the lane groups /
// blocks (no atomics, no work queue, no inter-block communication, no waits
// other than __syncthreads). Static striding also means a lane group or
// block sees rows of one 16-byte phase (lane groups always; blocks when the
// grid is a multiple of the phase period), so the realigned weight/bias
// cache of non-aligned layouts is filled once.
//
// Prefetch. While a thread normalizes row r, its share of the rows ahead
// (r + stride, up to NST rows) is already on its way: each thread copies
// its own full chunks of those rows into its own shared memory slots with
// cp.async and waits only for its own copies (cp.async.wait_group), so the
// HBM latency of a row hides behind earlier rows' arithmetic without any
// barrier. The shift K of each row ahead (LayerNorm) and the thread's edge
// element of it are loaded into registers when its copies are issued.
//
// The bulk-copy ring kernels (rownorm_ring.cuh) run the same per-row code;
// which kernel the planner picks never changes a bit.
#pragma once

#include "rownorm_core.cuh"

namespace rn {

struct Params {
  Segment seg[2];
  int nseg;
  float eps;
  int prefetch;  // 1: rows ahead prefetched through shared memory; 0: direct loads
  int stage_word;  // kOpRmsRope: first 16-byte word of the lane groups' staging rows
};

constexpr int kWarpBlock = 256;
// Block-family register budget: at least 1024 threads resident per SM (64
// registers).
constexpr int kMinThreadsPerSm = 1024;

// Lane-group register budget, as blocks of kWarpBlock threads resident per
// SM: 3 (up to 80 registers, 24 warps) or 2 (up to 128, 16 warps). Measured
// on B200 over bf16 and binary32 rows of 64 to 1024 columns, LayerNorm ran
// 7-22 % faster with more warps except where its values spill at 80
// registers (bf16 rows of 4 chunks per lane with a partial last chunk;
// binary32 rows of 6 or more chunks per lane: 2-8 % faster with 128, 1.6x at
// D = 1001), and every RMSNorm ran as fast or faster with 128.
// bf16 rows of 5 to 8 chunks per lane (1025 to 2048 columns) hold up to 64
// values and take 128.
template <typename T, int OP, int SLOTS, int VPL>
__host__ __device__ constexpr int warp_blocks_per_sm() {
  if (OP != kOpLn) return 2;
  if (Elem<T>::V == 8) return VPL >= 5 || (VPL == 4 && SLOTS != kSlotsFull) ? 2 : 3;
  return VPL >= 6 ? 2 : 3;
}

// Per-thread prefetch slots: [stages][NSLOT][blockDim.x] 16-byte words
// from 16-byte word `base` of the dynamic shared memory (a second bank
// follows the first for ops with a second input). When the slots do not fit
// in shared memory next to the weight cache (the planner decides), `on` is
// 0: nothing is copied ahead and rows are loaded straight from global memory
// when they are taken.
template <typename T, int NSLOT>
struct Prefetch {
  int on;
  int base;
  __device__ __forceinline__ uint4* slot(int stage, int p) const {
    return &dyn_smem[base + (stage * NSLOT + p) * blockDim.x + threadIdx.x];
  }
  // Start the copies of the thread's full chunks of a row (first full chunk
  // at `full`) into `stage`.
  template <int SLOTS>
  __device__ __forceinline__ void issue(const T* full, int nfull, int k0, int step,
                                        int stage) const {
    constexpr int V = Elem<T>::V;
    if (!on) return;
#pragma unroll
    for (int p = 0; p < NSLOT; ++p) {
      const int f = k0 + step * p;
      if (slot_present<SLOTS, NSLOT>(p, f, nfull))
        cp_async16(slot(stage, p), full + (long long)f * V);
    }
  }
  // Slot p of the row in `stage` (copy complete), or straight from global
  // memory when nothing was copied ahead.
  __device__ __forceinline__ uint4 chunk(const T* full, int f, int stage, int p) const {
    constexpr int V = Elem<T>::V;
    return on ? *slot(stage, p) : load_stream(full + (long long)f * V);
  }
  // The thread's slots of a row; absent ones zero. (The test of `on` stays
  // outside the slot loop: one uniform branch per row.)
  template <int SLOTS>
  __device__ __forceinline__ void take(const T* full, int nfull, int k0, int step, int stage,
                                       F2 (&v)[NSLOT][Elem<T>::P]) const {
    constexpr int V = Elem<T>::V;
    constexpr int P = Elem<T>::P;
    if (on) {
#pragma unroll
      for (int p = 0; p < NSLOT; ++p) {
        if (slot_present<SLOTS, NSLOT>(p, k0 + step * p, nfull)) {
          Elem<T>::unpack(*slot(stage, p), v[p]);
        } else {
#pragma unroll
          for (int j = 0; j < P; ++j) v[p][j] = zero2();
        }
      }
    } else {
#pragma unroll
      for (int p = 0; p < NSLOT; ++p) {
        const int f = k0 + step * p;
        if (slot_present<SLOTS, NSLOT>(p, f, nfull)) {
          Elem<T>::unpack(load_stream(full + (long long)f * V), v[p]);
        } else {
#pragma unroll
          for (int j = 0; j < P; ++j) v[p][j] = zero2();
        }
      }
    }
  }
};

// Prefetch stages per thread: rows in flight while one is normalized from
// registers. Measured on B200 (back-to-back bf16 LayerNorm, D = 768 to
// 16384): lane groups keep two (a third moved them by no more than noise).
// Blocks keep one: one row in flight in half the shared memory leaves L1
// room for the weight and bias and more blocks per SM (LayerNorm 16384: 777
// -> 746 us, 8192: 357 -> 349 us against two stages, a third stage cost
// 10-14 %; blocks of 128 threads on LayerNorm 4097, which prefetch: 200.7 ->
// 186.4 us, 8 blocks per SM instead of 6; RMSNorm and LayerNorm 4096, which
// do not prefetch, unchanged). The gated op reads its gate from the stage
// until the row is stored, so it refills late and keeps two stages: one row
// in flight while it normalizes.
constexpr int kWarpPrefetchStages = 2;
__host__ __device__ constexpr int cta_prefetch_stages(int threads, int op) {
  (void)threads;
  return op != kOpGatedRms ? 1 : 2;
}

// 16-byte words of prefetch slots of one bank.
template <int NSLOT, int NST>
__host__ __device__ constexpr int prefetch_smem_words(int threads) {
  return NST * NSLOT * threads;
}

template <typename T>
__device__ __forceinline__ const T* x2_row_of(const Segment& s, long long r) {
  return static_cast<const T*>(s.x2) + row_off(r, s.x2_stride, s.x2_inner, s.x2_outer);
}

// The edge element of thread k0 in a row of a second row space that shares
// x's 16-byte phase (0 when it owns none).
template <typename T, bool EXACT>
__device__ __forceinline__ float load_edge_at(const T* row, const Row<T>& g, int D, int k0) {
  if constexpr (EXACT) return 0.f;
  return k0 < g.nedge ? Elem<T>::get(row + edge_column(g, D, k0)) : 0.f;
}

// The gate's chunks for the store (kOpGatedRms): from the second prefetch
// bank, or global memory, and its edge element.
template <typename T, int NSLOT>
struct GateSrc {
  const Prefetch<T, NSLOT>* pf;
  const T* full;
  int stage;
  float ze;
  template <int P>
  __device__ __forceinline__ void get(int p, int f, F2 (&zf)[P]) const {
    Elem<T>::unpack(pf->chunk(full, f, stage, p), zf);
  }
  __device__ __forceinline__ float edge() const { return ze; }
};

// The rows r0, r0 + stride, ... of one segment, owned by one thread group (a
// lane group, or a block) in which this thread is k0 of `step`. Each row's
// chunks (and those of the second input) are prefetched NST rows ahead into
// the thread's own slots, stage i % NST holding row i. A row's stage is
// refilled with the row NST ahead as soon as the thread has read the stage
// into registers, so NST rows are in flight while the row is normalized (for
// the gated op, whose gate is read from its stage while the row is stored,
// once the row is stored). The shift K and the thread's edge elements of the
// rows ahead wait in register queues. `src` supplies weight and bias.
template <typename T, int OP, bool EXACT, int SLOTS, int NSLOT, int NST, typename Src,
          typename Reduce>
__device__ __forceinline__ void segment_rows(const Segment& seg, const Prefetch<T, NSLOT>& pf,
                                             const Prefetch<T, NSLOT>& pf2, long long r0,
                                             long long stride, int k0, int step, float eps,
                                             Reduce reduce, Src& src, float* stage,
                                             unsigned mask) {
  static_assert(NST >= 1, "at least one row ahead");
  const Segment& s = seg;
  constexpr int V = Elem<T>::V;
  constexpr int P = Elem<T>::P;
  constexpr bool SECOND = op_has_second(OP);
  constexpr bool LATE_REFILL = OP == kOpGatedRms;
  const int D = s.dim;
  const float inv_d = inv_dim(D);
  float Kq[NST], Eq[NST], E2q[NST];
  // queue the loads of row ra into stage `stage`, its scalars at queue entry j
  auto ahead = [&](long long ra, int stage, int j) {
    const Row<T> ga = row_geometry<T, EXACT>(s, ra);
    pf.template issue<SLOTS>(ga.x_full, ga.nfull, k0, step, stage);
    if (OP == kOpLn) Kq[j] = Elem<T>::get(ga.x_row);
    Eq[j] = load_edge<T, EXACT>(ga, D, k0);
    if constexpr (SECOND) {
      const T* row2 = x2_row_of<T>(s, ra);
      pf2.template issue<SLOTS>(row2 + ga.head, ga.nfull, k0, step, stage);
      E2q[j] = load_edge_at<T, EXACT>(row2, ga, D, k0);
    }
  };
  // stage `st` is free again: start row r + NST there (an empty group past
  // the end keeps one group per row)
  auto refill = [&](long long r, int st) {
    const long long ra = r + NST * stride;
    if (ra < s.rows) ahead(ra, st, NST - 1);
    cp_async_commit();
  };
#pragma unroll
  for (int j = 0; j < NST; ++j) {
    const long long rj = r0 + j * stride;
    Kq[j] = 0.f;
    Eq[j] = 0.f;
    E2q[j] = 0.f;
    if (rj < s.rows) ahead(rj, j, j);
    cp_async_commit();
  }
  int st = 0;  // stage of row r
#pragma unroll 1
  for (long long r = r0; r < s.rows; r += stride) {
    const float K = Kq[0];
    float xe = Eq[0];
    const float x2e = E2q[0];
#pragma unroll
    for (int j = 0; j + 1 < NST; ++j) {
      Kq[j] = Kq[j + 1];
      Eq[j] = Eq[j + 1];
      E2q[j] = E2q[j + 1];
    }
    cp_async_wait<NST - 1>();  // row r has landed
    const Row<T> g = row_geometry<T, EXACT>(s, r);
    const bool has_edge = !EXACT && k0 < g.nedge;
    F2 v[NSLOT][P];
    if constexpr (OP == kOpAddRms) {
      // h = x + r rounded to T: stored, and what the row statistics see
      const T* full2 = x2_row_of<T>(s, r) + g.head;
      T* hrow = static_cast<T*>(s.h) + row_off(r, s.h_stride, s.h_inner, s.h_outer);
#pragma unroll
      for (int p = 0; p < NSLOT; ++p) {
        const int f = k0 + step * p;
        if (slot_present<SLOTS, NSLOT>(p, f, g.nfull)) {
          F2 a[P], b[P];
          Elem<T>::unpack(pf.chunk(g.x_full, f, st, p), a);
          Elem<T>::unpack(pf2.chunk(full2, f, st, p), b);
#pragma unroll
          for (int j = 0; j < P; ++j) a[j] = add2(a[j], b[j]);
          const uint4 hv = Elem<T>::pack(a);
          store_stream(hrow + g.head + (long long)f * V, hv);
          Elem<T>::unpack(hv, v[p]);
        } else {
#pragma unroll
          for (int j = 0; j < P; ++j) v[p][j] = zero2();
        }
      }
      if constexpr (!LATE_REFILL) refill(r, st);
      if (has_edge) {
        xe = Elem<T>::stored(__fadd_rn(xe, x2e));
        Elem<T>::put(hrow + edge_column(g, D, k0), xe);
      }
    } else {
      pf.template take<SLOTS>(g.x_full, g.nfull, k0, step, st, v);
      if constexpr (!LATE_REFILL) refill(r, st);
    }
    float rstd, mean;
    row_stats<T, OP, EXACT, SLOTS, NSLOT>(v, xe, g, inv_d, k0, step, K, eps, has_edge, reduce,
                                          rstd, mean);
    if constexpr (!EXACT) {
      if (g.phase != src.phase) src.fill(s, g, k0, step);
    }
    if constexpr (OP == kOpGatedRms) {
      const GateSrc<T, NSLOT> gate{&pf2, x2_row_of<T>(s, r) + g.head, st, x2e};
      normalize_store<T, OP, EXACT, SLOTS, NSLOT>(s, g, v, xe, src, k0, step, rstd, mean,
                                                  has_edge, gate);
    } else if constexpr (op_is_rope(OP)) {
      normalize_rope_store<T, OP == kOpRmsRopeLocal, EXACT, SLOTS, NSLOT>(
          s, g, v, xe, src, k0, step, rstd, has_edge, r, stage, mask);
    } else {
      normalize_store<T, OP, EXACT, SLOTS, NSLOT>(s, g, v, xe, src, k0, step, rstd, mean,
                                                  has_edge);
    }
    if constexpr (LATE_REFILL) refill(r, st);
    st = st == NST - 1 ? 0 : st + 1;
  }
  cp_async_wait<0>();
}

// One segment with the weight/bias source its layout calls for: for EXACT
// layouts straight from the vectors (a loop without NULL tests when every
// vector the op uses is present), otherwise the realigned per-thread cache
// at 16-byte word `cache_word` of the dynamic shared memory.
template <typename T, int OP, bool EXACT, int SLOTS, int NSLOT, int NST, typename Reduce>
__device__ __forceinline__ void run_segment(const Segment& s, const Prefetch<T, NSLOT>& pf,
                                            const Prefetch<T, NSLOT>& pf2, long long r0,
                                            long long stride, int k0, int step, float eps,
                                            Reduce reduce, int cache_word, float* stage,
                                            unsigned mask) {
  constexpr bool BIAS = OP == kOpLn;
  static_assert(EXACT || SLOTS != kSlotsFull, "only EXACT rows divide evenly");
  const T* w = static_cast<const T*>(s.w);
  const T* b = static_cast<const T*>(s.b);
  if constexpr (EXACT) {
    if (w && (!BIAS || b)) {
      AffineDirect<T, BIAS, true> src{w, b};
      segment_rows<T, OP, true, SLOTS, NSLOT, NST>(
          s, pf, pf2, r0, stride, k0, step, eps, reduce, src, stage, mask);
    } else {
      AffineDirect<T, BIAS, false> src{w, b};
      segment_rows<T, OP, true, SLOTS, NSLOT, NST>(
          s, pf, pf2, r0, stride, k0, step, eps, reduce, src, stage, mask);
    }
  } else {
    AffineCache<T, NSLOT, BIAS> src;
    src.init(cache_word);
    segment_rows<T, OP, false, SLOTS, NSLOT, NST>(
        s, pf, pf2, r0, stride, k0, step, eps, reduce, src, stage, mask);
  }
}

// One row space of the lane-group kernel.
template <typename T, int OP, bool EXACT, int SLOTS, int VPL>
__device__ __forceinline__ void warp_segment(const Params& p, const Segment& s,
                                             const Prefetch<T, VPL>& pf,
                                             const Prefetch<T, VPL>& pf2, int lane,
                                             long long warp, long long nwarps, int cache_word) {
  const int G = s.lanes;
  const int per_warp = 32 / G;
  const int gl = lane & (G - 1);
  const int gi = lane / G;
  const unsigned mask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << (gi * G));
  auto reduce = [&](float t) { return group_sum(t, G, mask); };
  float* stage = nullptr;
  if constexpr (OP == kOpRmsRope)  // the in-thread variant stages nothing
    stage = reinterpret_cast<float*>(dyn_smem + p.stage_word) +
            ((threadIdx.x >> 5) * per_warp + gi) * s.dim;
  run_segment<T, OP, EXACT, SLOTS, VPL, kWarpPrefetchStages>(
      s, pf, pf2, warp * per_warp + gi, nwarps * per_warp, gl, G, p.eps, reduce, cache_word,
      stage, mask);
}

template <typename T, int OP, bool EXACT, int SLOTS, int VPL>
__global__ void __launch_bounds__(kWarpBlock, (warp_blocks_per_sm<T, OP, SLOTS, VPL>()))
rows_warp_kernel(const Params p) {
  constexpr int BANK = prefetch_smem_words<VPL, kWarpPrefetchStages>(kWarpBlock);
  const Prefetch<T, VPL> pf{p.prefetch, 0};
  const Prefetch<T, VPL> pf2{p.prefetch, BANK};
  const int lane = threadIdx.x & 31;
  const long long warp = (long long)blockIdx.x * (kWarpBlock / 32) + (threadIdx.x >> 5);
  const long long nwarps = (long long)gridDim.x * (kWarpBlock / 32);
  const int cache_word = p.prefetch ? BANK * (op_has_second(OP) ? 2 : 1) : 0;
  // each row space by a reference fixed at compile time (p.seg[0], p.seg[1]),
  // so that its fields stay kernel-parameter operands rather than registers
  warp_segment<T, OP, EXACT, SLOTS, VPL>(p, p.seg[0], pf, pf2, lane, warp, nwarps, cache_word);
  if (p.nseg > 1)
    warp_segment<T, OP, EXACT, SLOTS, VPL>(p, p.seg[1], pf, pf2, lane, warp, nwarps, cache_word);
}

template <typename T, int OP, bool EXACT, int SLOTS, int NT, int VPT>
__global__ void __launch_bounds__(NT, kMinThreadsPerSm / NT)
rows_cta_kernel(const Params p) {
  static_assert(NT >= 2 * (Elem<T>::V - 1), "every edge element needs its own thread");
  static_assert(!op_is_rope(OP), "RoPE rows are head rows: lane groups only");
  // Two alternating reduction buffers: a buffer is rewritten only after every
  // thread has passed the barrier of the reduction in between.
  __shared__ float red[2][NT / 32];
  constexpr int BANK = prefetch_smem_words<VPT, cta_prefetch_stages(NT, OP)>(NT);
  const Prefetch<T, VPT> pf{p.prefetch, 0};
  const Prefetch<T, VPT> pf2{p.prefetch, BANK};
  int slot = 0;
  auto reduce = [&](float t) {
    const float r = block_sum<NT>(t, red[slot]);
    slot ^= 1;
    return r;
  };
  const int cache_word = p.prefetch ? BANK * (op_has_second(OP) ? 2 : 1) : 0;
  if constexpr (EXACT) {
    // the row space by a compile-time reference to the kernel parameters, as
    // the lane-group and ring kernels take it (LayerNorm 65536 x 8192: 345.0
    // -> 338.9 us on B200)
    run_segment<T, OP, EXACT, SLOTS, VPT, cta_prefetch_stages(NT, OP)>(
        p.seg[0], pf, pf2, blockIdx.x, gridDim.x, threadIdx.x, NT, p.eps, reduce, cache_word,
        nullptr, 0u);
    if (p.nseg > 1)
      run_segment<T, OP, EXACT, SLOTS, VPT, cta_prefetch_stages(NT, OP)>(
          p.seg[1], pf, pf2, blockIdx.x, gridDim.x, threadIdx.x, NT, p.eps, reduce, cache_word,
          nullptr, 0u);
  } else {
    // rows off the 16-byte grid take a copy picked at run time: with the
    // compile-time reference the off-grid LayerNorm kernel spilled 12 bytes
    // in its row loop at 64 registers (LayerNorm 65536 x 4097: 303 against
    // 204 us), and ran 332 us at 80 registers (the copy: 199 us at 64 or 80)
#pragma unroll 1
    for (int si = 0; si < p.nseg; ++si) {
      const Segment s = si == 0 ? p.seg[0] : p.seg[1];
      run_segment<T, OP, EXACT, SLOTS, VPT, cta_prefetch_stages(NT, OP)>(
          s, pf, pf2, blockIdx.x, gridDim.x, threadIdx.x, NT, p.eps, reduce, cache_word, nullptr,
          0u);
    }
  }
}

}  // namespace rn
