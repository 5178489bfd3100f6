// Per-warp bulk-copy row rings (sm_100a), for rows whose lane groups fit in
// one warp (dim <= 1024 binary32, 2048 bf16) in 16-byte aligned layouts:
// RMSNorm, LayerNorm, and the q/k head RMSNorm + RoPE whose plane partners
// are the same thread's (with each tile's token's cos / sin row staged
// beside the tile's rows).
//
// Every warp of a block runs its own pipeline, with no block barrier: a ring
// of S stages in shared memory, each holding one tile of R consecutive rows
// of the warp's static share of the row space (tiles w, w + W, w + 2W, ...
// for warp w of W). The warp fills a stage with the bulk-copy engine
// (cp.async.bulk global -> shared, completion counted in bytes on the
// stage's mbarrier, announced by lane 0): one copy for a tile whose rows are
// adjacent in memory, else one copy per row, lane i copying row i. The warp
// waits for the stage, its lane groups
// normalize the tile's rows from shared memory and store them to global
// memory, and lane 0 refills the stage with the tile S ahead. So S tiles of
// every warp are in flight while it computes, independently of its register
// budget, and a tile costs one copy instruction instead of one per 16-byte
// chunk and lane.
//
// The per-row arithmetic is that of the register kernels (rownorm_core.cuh):
// the same lanes per row, chunk-to-lane mapping, shift K = x_0, summation
// order and operation order. Which kernel the planner picks never changes a
// bit.
//
// Waits are bounded. A warp whose stage wait gives up after kRingWaitLimitNs
// stops issuing, then waits for every copy it still has in flight (bounded
// by kRingDrainLimitNs; the copies read valid memory and always complete),
// records the timeout in the device counter (rn_device_error_count) and
// returns. No warp leaves with a copy into its shared memory outstanding.
// The wait test (rn_set_ring_wait_test) makes every stage announce 16 bytes
// more than its copies bring, so that no stage completes: every first wait
// runs out after a millisecond and the timeout path runs, with all copies
// landed and nothing faulted.
#pragma once

#include <type_traits>

#include "rownorm_kernels.cuh"

namespace rn {

// Timed-out stage waits. Each translation unit that instantiates the ring
// kernels has its own counter (internal linkage) and a host accessor beside
// its table.
static __device__ unsigned int g_ring_timeouts;

constexpr int kRingWarps = 4;        // warps (independent rings) per block
constexpr int kRingMaxStages = 8;    // barrier slots reserved per warp
constexpr unsigned long long kRingWaitLimitNs = 2000000000ull;    // 2 s
constexpr unsigned long long kRingDrainLimitNs = 30000000000ull;  // 30 s

struct RingParams {
  Segment seg[2];
  int nseg;
  float eps;
  int stages;          // S, 2 .. kRingMaxStages
  int stage_bytes;     // bytes of one stage (the widest tile), a multiple of 16
  int tile_rows[2];    // R per segment: a multiple of the rows a warp takes at once
  int contiguous[2];   // 1: a tile's rows are adjacent in memory (one copy)
  unsigned long long wait_ns;   // stage wait limit (normally kRingWaitLimitNs)
  unsigned long long drain_ns;  // limit of the wait for copies in flight after a timeout
  int tx_extra;        // bytes announced beyond the copies' (0; > 0 only under the
                       // wait test, so that no stage completes and every wait runs out)
  int table_bytes;     // RoPE rows: bytes of the token's table row staged after a
                       // tile's rows (every tile lies in one token); 0: not staged
  int affine_word;     // LayerNorm rows: 16-byte word of the block's binary32 copy of
                       // the weight and bias (ring_affine_bytes), after the barriers
};

// Shared memory of a block: the warps' rings, then their barrier slots (and,
// for LayerNorm rows, the block's binary32 weight and bias: ring_affine_bytes).
__host__ __device__ constexpr int ring_smem_bytes(int stages, int stage_bytes) {
  return kRingWarps * stages * stage_bytes + kRingWarps * kRingMaxStages * 8;
}
// The binary32 weight and bias of a LayerNorm row space of `dim` columns.
__host__ __device__ constexpr int ring_affine_bytes(int dim) { return dim * 4 * 2; }

__device__ __forceinline__ unsigned long long global_timer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Makes the initialized barriers visible to the bulk-copy (async) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Orders this thread's earlier shared-memory reads before bulk copies it
// issues next into the same bytes.
__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// The one arrival of a stage's phase, announcing the bytes its copies bring.
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

// Wait for the phase of `bar` with the given parity to complete; false after
// `limit_ns` without completion.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer() - t0 > limit_ns) return false;
  }
  return true;
}

// Global -> shared bulk copy of `bytes` (both addresses 16-byte aligned, a
// multiple of 16 bytes), completion counted on `bar`. Into this CTA's shared memory only.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Weight and bias of a LayerNorm row space as binary32 in shared memory,
// written once per block (ring_affine_fill) and read as 16-byte vectors at
// each use: [vector (w, b)][quarter of a chunk][chunk] float4s, so that the
// lanes' reads of one quarter of their chunks are contiguous. The values are
// those of the element type's words (widened exactly; NULL weight = ones,
// NULL bias = zeros), so the bits of the results are those of AffineDirect.
template <typename T>
struct AffineSmemF32 {
  static constexpr int Q = Elem<T>::V / 4;  // float4s per chunk and vector
  const float4* area;
  int nchunks;
  __device__ __forceinline__ void get(int /*p*/, int f, F2 (&wf)[Elem<T>::P],
                                      F2 (&bf)[Elem<T>::P]) const {
#pragma unroll
    for (int h = 0; h < Q; ++h) {
      const float4 a = area[h * nchunks + f];
      const float4 b = area[(Q + h) * nchunks + f];
      wf[2 * h] = make_float2(a.x, a.y);
      wf[2 * h + 1] = make_float2(a.z, a.w);
      bf[2 * h] = make_float2(b.x, b.y);
      bf[2 * h + 1] = make_float2(b.z, b.w);
    }
  }
  __device__ __forceinline__ void edge(float& w_, float& b_) const {
    w_ = 1.f;
    b_ = 0.f;
  }
};

// Every thread of the block: write segment s's weight and bias into the
// area at 16-byte word `word` (then the caller syncs the block).
template <typename T>
__device__ __forceinline__ void ring_affine_fill(const Segment& s, int word) {
  constexpr int V = Elem<T>::V;
  constexpr int P = Elem<T>::P;
  constexpr int Q = V / 4;
  float4* area = reinterpret_cast<float4*>(dyn_smem + word);
  const int n = s.dim / V;
  const T* w = static_cast<const T*>(s.w);
  const T* b = static_cast<const T*>(s.b);
  for (int f = threadIdx.x; f < n; f += blockDim.x) {
    F2 wf[P], bf[P];
    if (w) {
      Elem<T>::unpack(load_cached(w + (long long)f * V), wf);
    } else {
#pragma unroll
      for (int j = 0; j < P; ++j) wf[j] = splat(1.f);
    }
    if (b) {
      Elem<T>::unpack(load_cached(b + (long long)f * V), bf);
    } else {
#pragma unroll
      for (int j = 0; j < P; ++j) bf[j] = zero2();
    }
#pragma unroll
    for (int h = 0; h < Q; ++h) {
      area[h * n + f] = make_float4(wf[2 * h].x, wf[2 * h].y, wf[2 * h + 1].x, wf[2 * h + 1].y);
      area[(Q + h) * n + f] =
          make_float4(bf[2 * h].x, bf[2 * h].y, bf[2 * h + 1].x, bf[2 * h + 1].y);
    }
  }
}

// Weight and bias of a lane's chunk slots: the packed 16-byte words of the
// first NREG slots held in registers (loaded once per row space: in an
// aligned layout a lane owns the same chunks of every row), the others read
// from L1 at each use; unpacked at each use. NULL weight = ones, NULL bias =
// zeros, as AffineDirect; the values, and so the bits, are the same.
template <typename T, bool BIAS, int NSLOT, int NREG>
struct AffineRegs {
  static_assert(NREG >= 1 && NREG <= NSLOT, "slots in registers");
  uint4 w[NREG];
  uint4 b[BIAS ? NREG : 1];
  const T* wv;
  const T* bv;
  int k0, step;
  __device__ __forceinline__ void load(const Segment& s, int k0_, int step_) {
    constexpr int V = Elem<T>::V;
    wv = static_cast<const T*>(s.w);
    bv = static_cast<const T*>(s.b);
    k0 = k0_;
    step = step_;
    const uint32_t one = Elem<T>::kOneBits | (sizeof(T) == 2 ? Elem<T>::kOneBits << 16 : 0u);
    const int nfull = s.dim / V;
#pragma unroll
    for (int p = 0; p < NREG; ++p) {
      const int f = k0 + step * p;
      const bool in = f < nfull;
      w[p] = (wv && in) ? load_cached(wv + f * V) : make_uint4(one, one, one, one);
      if constexpr (BIAS) b[p] = (bv && in) ? load_cached(bv + f * V) : make_uint4(0, 0, 0, 0);
    }
  }
  __device__ __forceinline__ void get(int p, int f, F2 (&wf)[Elem<T>::P],
                                      F2 (&bf)[Elem<T>::P]) const {
    constexpr int V = Elem<T>::V;
    constexpr int P = Elem<T>::P;
    if (p < NREG) {
      Elem<T>::unpack(w[p < NREG ? p : 0], wf);
      if constexpr (BIAS) Elem<T>::unpack(b[p < NREG ? p : 0], bf);
      return;
    }
    if (wv) {
      Elem<T>::unpack(load_cached(wv + f * V), wf);
    } else {
#pragma unroll
      for (int j = 0; j < P; ++j) wf[j] = splat(1.f);
    }
    if constexpr (BIAS) {
      if (bv) {
        Elem<T>::unpack(load_cached(bv + f * V), bf);
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

// The warp starts the copies of tile `tile` of row space s (R rows per tile)
// into `dst`, counted on `bar`: lane 0 announces the bytes, then one copy for
// adjacent rows, else lane i copies row i (rows i + 32, ... too). Rows sit
// `pitch` 16-byte words apart in the stage: their own size. (Padding rows of
// under 8 lanes against shared-memory bank conflicts, which then takes a
// copy per row, measured slower on B200: dual head norm prefill 30.7 ->
// 33.5 us.)
template <typename T>
__device__ __forceinline__ void ring_issue(const Segment& s, long long tile, int R,
                                           bool contiguous, int pitch, int tx_extra,
                                           int table_bytes, uint4* dst, uint64_t* bar) {
  const int lane = threadIdx.x & 31;
  const long long r0 = tile * R;
  const int nr = (int)(s.rows - r0 < R ? s.rows - r0 : R);
  const uint32_t row_bytes = (uint32_t)s.dim * (uint32_t)sizeof(T);
  const T* x = static_cast<const T*>(s.x);
  if (lane == 0) {
    mbar_expect_tx(bar, (uint32_t)nr * row_bytes + (uint32_t)table_bytes + (uint32_t)tx_extra);
    if (table_bytes) {
      // the tile's token's cos / sin row, after the tile's R row slots
      const long long token = r0 < 0x7fffffffLL ? (long long)((unsigned)r0 / (unsigned)s.rope_heads)
                                                : r0 / s.rope_heads;
      bulk_load(dst + R * pitch, s.rope_table + (s.rope_offset + token) * s.rope_dims,
                (uint32_t)table_bytes, bar);
    }
  }
  if (contiguous) {
    if (lane == 0)
      bulk_load(dst, x + row_off(r0, s.x_stride, s.x_inner, s.x_outer),
                (uint32_t)nr * row_bytes, bar);
  } else {
    __syncwarp();  // the bytes are announced before any of these copies starts
    for (int rr = lane; rr < nr; rr += 32)
      bulk_load(dst + rr * pitch, x + row_off(r0 + rr, s.x_stride, s.x_inner, s.x_outer),
                row_bytes, bar);
  }
}

// LayerNorm rows of a whole warp go two to a ring tile when two rows fit in
// kRingPairTileBytes (the planner decides; ring_ln_pair normalizes them
// together). Lanes of more chunks never pair, and their kernels carry no
// pair code (it would only add to their register pressure).
constexpr int kRingPairTileBytes = 4096;
__host__ __device__ constexpr bool ring_pairs_fit(int vpl) {
  return 2 * 32 * 16 * vpl <= kRingPairTileBytes;
}

// The xor butterfly of two rows' partial sums at once over the whole warp:
// each step adds the partner lane's pair with one packed add, which rounds
// each half as the scalar add of the one-row butterfly does.
__device__ __forceinline__ F2 warp_sum_pair(F2 t) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    F2 u;
    u.x = __shfl_xor_sync(0xffffffffu, t.x, off);
    u.y = __shfl_xor_sync(0xffffffffu, t.y, off);
    t = add2(t, u);
  }
  return t;
}

// Two whole-warp LayerNorm rows of a stage at once: rows r and r + 1, at
// 16-byte words `row` and `row + pitch`. Each row takes the operations of
// one row, in the same order (row_stats, normalize_store), so its bits are
// those of the one-row path; the two rows' independent chains interleave,
// their butterflies share each step's add, and each weight / bias value is
// read once for both rows.
template <typename T, int SLOTS, int VPL, typename Src>
__device__ __forceinline__ void ring_ln_pair(const Segment& s, int row, int pitch, long long r,
                                             float eps, float inv_d, int gl, const Src& src) {
  constexpr int P = Elem<T>::P;
  constexpr int V = Elem<T>::V;
  const Row<T> ga = row_geometry<T, true>(s, r);
  const Row<T> gb = row_geometry<T, true>(s, r + 1);
  F2 va[VPL][P], vb[VPL][P];
#pragma unroll
  for (int q = 0; q < VPL; ++q) {
    if (slot_present<SLOTS, VPL>(q, gl + 32 * q, ga.nfull)) {
      Elem<T>::unpack(dyn_smem[row + gl + 32 * q], va[q]);
      Elem<T>::unpack(dyn_smem[row + pitch + gl + 32 * q], vb[q]);
    } else {
#pragma unroll
      for (int j = 0; j < P; ++j) va[q][j] = vb[q][j] = zero2();
    }
  }
  // each row's first element, from the first 4 bytes of its first chunk
  const uint32_t* words = reinterpret_cast<const uint32_t*>(dyn_smem);
  const float Ka = Elem<T>::low(words[4 * row]);
  const float Kb = Elem<T>::low(words[4 * (row + pitch)]);
  float xe = 0.f;  // no edge elements in these layouts
  F2 s1 = make_float2(shift_and_sum<T, true, SLOTS, VPL>(va, xe, ga, gl, 32, Ka, false),
                      shift_and_sum<T, true, SLOTS, VPL>(vb, xe, gb, gl, 32, Kb, false));
  s1 = warp_sum_pair(s1);
  const float ma = __fmul_rn(s1.x, inv_d), mb = __fmul_rn(s1.y, inv_d);
  F2 s2 = make_float2(sum_dev_squares<T, true, SLOTS, VPL>(va, xe, ga, gl, 32, ma, false),
                      sum_dev_squares<T, true, SLOTS, VPL>(vb, xe, gb, gl, 32, mb, false));
  s2 = warp_sum_pair(s2);
  const F2 Ra = splat(rsqrtf(__fadd_rn(__fmul_rn(s2.x, inv_d), eps)));
  const F2 Rb = splat(rsqrtf(__fadd_rn(__fmul_rn(s2.y, inv_d), eps)));
#pragma unroll
  for (int q = 0; q < VPL; ++q) {
    const int f = gl + 32 * q;
    if (!slot_present<SLOTS, VPL>(q, f, ga.nfull)) continue;
    F2 wf[P], bf[P], oa[P], ob[P];
    src.get(q, f, wf, bf);
#pragma unroll
    for (int j = 0; j < P; ++j) {  // the rows are centred
      oa[j] = fma2(mul2(va[q][j], Ra), wf[j], bf[j]);
      ob[j] = fma2(mul2(vb[q][j], Rb), wf[j], bf[j]);
    }
    store_stream(ga.y_row + (long long)f * V, Elem<T>::pack(oa));
    store_stream(gb.y_row + (long long)f * V, Elem<T>::pack(ob));
  }
}

// The rows of one staged tile (rows r0 .. r0 + nr - 1), normalized by the
// warp's lane groups: lane group gi takes rows gi, gi + 32/G, ... GC = 32
// compiles the whole-warp case (one row at a time, a fixed butterfly); GC =
// 0 takes G from the row space. Both add in the same order.
// The stage starts at 16-byte word `stage_word` of the dynamic shared memory
// (indexed from the shared array itself, so that the loads use 32-bit
// shared-window addresses).
template <typename T, int OP, int SLOTS, int VPL, int GC, typename Src>
__device__ __forceinline__ void ring_tile_rows(const Segment& s, int stage_word, int pitch,
                                               long long r0, int nr, float eps, float inv_d,
                                               int gl, int gi, unsigned mask, const Src& src,
                                               int table_word) {
  constexpr int P = Elem<T>::P;
  const int G = GC ? GC : s.lanes;
  auto reduce = [&](float t) {
    if constexpr (GC == 32) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        t = __fadd_rn(t, __shfl_xor_sync(0xffffffffu, t, off));
      return t;
    } else {
      return group_sum(t, G, mask);
    }
  };
  int rr = gi;
  if constexpr (OP == kOpRmsRopeLocal && VPL % 2 == 0) {
    if (table_word >= 0 && !s.rope_trad) {
      // full split-half rotary, the tile's token's table row staged beside
      // its rows: the lane's cos / sin, the same for every row it takes
      // here, are read once per tile
      constexpr int V = Elem<T>::V;
      const float* tab = reinterpret_cast<const float*>(dyn_smem + table_word);
      const int half = s.rope_dims >> 1;
      float cs[VPL / 2][V], sn[VPL / 2][V], nsn[VPL / 2][V];
#pragma unroll
      for (int q = 0; q < VPL / 2; ++q) {
        load_floats<V>(tab + (gl + G * q) * V, cs[q]);
        load_floats<V>(tab + half + (gl + G * q) * V, sn[q]);
#pragma unroll
        for (int k = 0; k < V; ++k) nsn[q][k] = -sn[q][k];
      }
#pragma unroll 1
      for (; rr < nr; rr += 32 / G) {
        const Row<T> g = row_geometry<T, true>(s, r0 + rr);
        const int row = stage_word + rr * pitch;
        F2 v[VPL][P];
#pragma unroll
        for (int q = 0; q < VPL; ++q) Elem<T>::unpack(dyn_smem[row + gl + G * q], v[q]);
        float xe = 0.f, rstd, mean;
        row_stats<T, OP, true, SLOTS, VPL>(v, xe, g, inv_d, gl, G, 0.f, eps, false, reduce, rstd,
                                           mean);
        normalize_rope_split_pre<T, VPL>(s, g, v, src, gl, G, rstd, cs, sn, nsn);
      }
      return;
    }
  }
  if constexpr (GC == 32 && OP == kOpLn && ring_pairs_fit(VPL)) {
#pragma unroll 1
    for (; rr + 1 < nr; rr += 2)
      ring_ln_pair<T, SLOTS, VPL>(s, stage_word + rr * pitch, pitch, r0 + rr, eps, inv_d, gl, src);
  }
#pragma unroll 1
  for (; rr < nr; rr += 32 / G) {
    const Row<T> g = row_geometry<T, true>(s, r0 + rr);
    const int row = stage_word + rr * pitch;
    F2 v[VPL][P];
#pragma unroll
    for (int q = 0; q < VPL; ++q) {
      if (slot_present<SLOTS, VPL>(q, gl + G * q, g.nfull)) {
        Elem<T>::unpack(dyn_smem[row + gl + G * q], v[q]);
      } else {
#pragma unroll
        for (int j = 0; j < P; ++j) v[q][j] = zero2();
      }
    }
    // the row's first element, from the first 4 bytes of its first chunk
    const float K =
        OP == kOpLn ? Elem<T>::low(reinterpret_cast<const uint32_t*>(dyn_smem)[4 * row]) : 0.f;
    float xe = 0.f, rstd, mean;
    row_stats<T, OP, true, SLOTS, VPL>(v, xe, g, inv_d, gl, G, K, eps, false, reduce, rstd,
                                       mean);
    if constexpr (OP == kOpRmsRopeLocal) {
      if (table_word >= 0)
        normalize_rope_store<T, true, true, SLOTS, VPL, Src, true>(
            s, g, v, xe, src, gl, G, rstd, false, r0 + rr, nullptr, mask,
            reinterpret_cast<const float*>(dyn_smem + table_word));
      else
        normalize_rope_store<T, true, true, SLOTS, VPL>(s, g, v, xe, src, gl, G, rstd, false,
                                                        r0 + rr, nullptr, mask);
    } else {
      normalize_store<T, OP, true, SLOTS, VPL>(s, g, v, xe, src, gl, G, rstd, mean, false);
    }
  }
}

// Slots whose weight (and bias) words stay in registers (AffineRegs; the
// others are read from L1 at each use): as many as keep a lane's row values
// (VPL chunks as binary32) plus those words within 48 registers, so that the
// kernel fits the 128-register budget without spilling (ptxas, both element
// types); none for LayerNorm rows; up to 4 for RoPE rows.
template <typename T, int OP, int VPL>
__host__ __device__ constexpr int ring_weight_slots_in_regs() {
  // RoPE rows keep the weight words of up to 4 slots (ptxas: no spill with
  // the cos / sin of a tile also in registers). Measured on B200, bf16 dual
  // head norm + RoPE prefill, cold / back to back: weight from L1 and sign
  // flips per row 39.7 / 37.1 us; weight in registers 38.8 / 37.0; both the
  // weight in registers and the negated sines kept per tile 37.8 / 35.3 (the
  // negated sines alone: 40.9 / 38.5). A block-wide binary32 copy of the
  // weights in shared memory instead, as for LayerNorm rows, measured the
  // same (38.9 / 35.3).
  if (OP == kOpRmsRopeLocal) return VPL < 4 ? VPL : 4;
  // LayerNorm rows read the block's binary32 copy in shared memory
  // (AffineSmemF32): two rows' values in pairs (ring_ln_pair) leave no room
  // for the words (ptxas spilled), and the copy also saves their unpacking.
  // Measured on B200 (bf16, 65536 rows, cold / back to back, us), against
  // the words read from L1 and unpacked once per pair: D = 768 37.2 / 38.3 ->
  // 34.2 / 41.2, D = 1000 47.1 / 49.6 -> 43.0 / 51.9, D = 1024 49.5 / 51.1 ->
  // 43.2 / 52.0; over the whole bench step the same (444 M rows/s).
  if (OP == kOpLn) return 0;
#ifndef RN_RING_WB_BUDGET
#define RN_RING_WB_BUDGET 48
#endif
  const int room = (RN_RING_WB_BUDGET - VPL * Elem<T>::V) / (4 * (OP == kOpLn ? 2 : 1));
  return room < 0 ? 0 : (room > VPL ? VPL : room);
}

// Register budget: 4 blocks of kRingWarps warps per SM (16 warps, up to 128
// registers). The rows in flight sit in the rings, not in registers, so more
// warps buy nothing; measured on B200 (LayerNorm bf16 65536 x 768), a budget
// of 80 registers spilled and ran 10 % slower.
constexpr int kRingBlocksPerSm = 4;

// The state of one warp's ring between row spaces: the stage to use next,
// bit k of `parity` the phase parity with which stage k completes next (the
// stages run round robin across the row spaces).
struct RingState {
  int st;
  uint32_t parity;
  bool ok;
};

// One row space (segment SI, a compile-time index, so that its fields stay
// kernel-parameter operands rather than registers) through this warp's ring.
template <typename T, int OP, int SLOTS, int VPL, int SI>
__device__ __forceinline__ void ring_segment(const RingParams& p, RingState& rs, int ring_word,
                                             int stage_words, uint64_t* bars, long long w,
                                             long long W) {
  constexpr bool BIAS = OP == kOpLn;
  const Segment& s = p.seg[SI];
  const int lane = threadIdx.x & 31;
  const int S = p.stages;
  const int R = p.tile_rows[SI];
  const bool contiguous = p.contiguous[SI] != 0;
  const long long ntiles = (s.rows + R - 1) / R;
  const long long n = ntiles > w ? (ntiles - w + W - 1) / W : 0;  // this warp's tiles
  if (n == 0) return;
  const int G = s.lanes;
  const int gl = lane & (G - 1);
  const int gi = lane / G;
  const unsigned mask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << (gi * G));
  const float inv_d = inv_dim(s.dim);
  constexpr int NREG = ring_weight_slots_in_regs<T, OP, VPL>();
  using Regs = AffineRegs<T, BIAS, VPL, NREG ? NREG : 1>;
  using Direct = AffineDirect<T, BIAS, false>;
  // LayerNorm: the block's binary32 copy in shared memory (one row space)
  using Smem = AffineSmemF32<T>;
  std::conditional_t<BIAS, Smem, std::conditional_t<(NREG > 0), Regs, Direct>> src;
  if constexpr (BIAS)
    src = Smem{reinterpret_cast<const float4*>(dyn_smem + p.affine_word), s.dim / Elem<T>::V};
  else if constexpr (NREG > 0)
    src.load(s, gl, G);
  else
    src = Direct{static_cast<const T*>(s.w), static_cast<const T*>(s.b)};
  int st = rs.st;
  uint32_t parity = rs.parity;
  const int pitch = s.dim * (int)sizeof(T) / 16;  // a row's 16-byte words
  // every stage is free here: the previous row space's tiles are consumed
  {
    int k = st;
    for (long long i = 0; i < n && i < S; ++i) {
      ring_issue<T>(s, w + i * W, R, contiguous, pitch, p.tx_extra, p.table_bytes,
                    dyn_smem + ring_word + k * stage_words, &bars[k]);
      k = k + 1 == S ? 0 : k + 1;
    }
  }
  __syncwarp();
  long long i = 0;
  bool ok = true;
#pragma unroll 1
  for (; i < n; ++i) {
    ok = mbar_wait(&bars[st], (parity >> st) & 1u, p.wait_ns);
    if (__any_sync(0xffffffffu, !ok)) {
      ok = false;
      break;
    }
    parity ^= 1u << st;
    const long long r0 = (w + i * W) * R;
    const int nr = (int)(s.rows - r0 < R ? s.rows - r0 : R);
    const int stage_word = ring_word + st * stage_words;
    const int table_word = p.table_bytes ? stage_word + R * pitch : -1;
    // (head rows with RoPE keep one copy of the row code, with the lane
    // count read at run time: without the second, whole-warp copy the dual
    // head norm + RoPE prefill ran 43.0 -> 39.1 us cold, 37.6 -> 37.0 back to
    // back on B200, where ncu had counted 1.45 cycles per issue stalled on
    // instruction fetch)
    if (OP != kOpRmsRopeLocal && G == 32)
      ring_tile_rows<T, OP, SLOTS, VPL, 32>(s, stage_word, pitch, r0, nr, p.eps, inv_d, gl, gi,
                                            mask, src, table_word);
    else
      ring_tile_rows<T, OP, SLOTS, VPL, 0>(s, stage_word, pitch, r0, nr, p.eps, inv_d, gl, gi,
                                           mask, src, table_word);
    // every lane has read the stage: refill it with the tile S ahead
    __syncwarp();
    if (i + S < n) {
      fence_async_shared();
      ring_issue<T>(s, w + (i + S) * W, R, contiguous, pitch, p.tx_extra, p.table_bytes,
                    dyn_smem + ring_word + st * stage_words, &bars[st]);
    }
    st = st + 1 == S ? 0 : st + 1;
  }
  if (!ok && lane == 0) {
    // tiles i .. min(n, i + S) - 1 are issued and not yet consumed, in
    // stages st, st + 1, ... (mod S)
    int k = st;
    for (long long j = i; j < n && j < i + S; ++j) {
      mbar_wait(&bars[k], (parity >> k) & 1u, p.drain_ns);
      k = k + 1 == S ? 0 : k + 1;
    }
    atomicAdd(&g_ring_timeouts, 1u);
  }
  rs.st = st;
  rs.parity = parity;
  rs.ok = ok;
}

template <typename T, int OP, int SLOTS, int VPL>
__global__ void __launch_bounds__(kRingWarps * 32, kRingBlocksPerSm)
rows_ring_kernel(const RingParams p) {
  static_assert(OP == kOpRms || OP == kOpLn || OP == kOpRmsRopeLocal,
                "rings carry RMSNorm and LayerNorm rows, and head rows rotated in-thread");
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int S = p.stages;
  const int stage_words = p.stage_bytes / 16;
  const int ring_word = warp * S * stage_words;  // this warp's stages, in 16-byte words
  uint64_t* const bars =
      reinterpret_cast<uint64_t*>(dyn_smem + kRingWarps * S * stage_words) + warp * kRingMaxStages;
  const long long w = (long long)blockIdx.x * kRingWarps + warp;
  const long long W = (long long)gridDim.x * kRingWarps;
  if (lane == 0) {
    for (int k = 0; k < S; ++k) mbar_init(&bars[k], 1);
    fence_mbar_init();
  }
  if constexpr (OP == kOpLn) {
    // LayerNorm rings carry one row space (the planner's rule)
    ring_affine_fill<T>(p.seg[0], p.affine_word);
    __syncthreads();
  }
  __syncwarp();
  RingState rs{0, 0u, true};
  ring_segment<T, OP, SLOTS, VPL, 0>(p, rs, ring_word, stage_words, bars, w, W);
  if (p.nseg > 1 && rs.ok)
    ring_segment<T, OP, SLOTS, VPL, 1>(p, rs, ring_word, stage_words, bars, w, W);
}

}  // namespace rn

namespace rn {

// ---------------------------------------------------------------------------
// Block rings: rows wider than one warp's lane groups hold (the block
// family, one block of NT threads per row). Thread 0 fills a ring of NST
// stages, each holding the full 16-byte chunks of one row (one bulk copy:
// they are contiguous and 16-byte aligned whatever the row's phase); every
// thread waits for the stage of its current row, reads its chunks from it,
// and the row is reduced and stored as in rows_cta_kernel (same threads per
// row, chunk ownership, edge elements, shift, summation and operation
// order: the same bits). The stage of row i is refilled with row i + NST at
// the start of row i + 1, when every thread has passed row i's reduction
// barriers and so has read it; NST - 1 rows are in flight while one is
// normalized. Each thread's edge element and the shift K of the rows ahead
// are loaded into register queues when their copies are issued.

template <typename T, bool EXACT>
__device__ __forceinline__ void cta_ring_issue(const Segment& s, long long r, uint4* dst,
                                               uint64_t* bar, int tx_extra) {
  const Row<T> g = row_geometry<T, EXACT>(s, r);
  const uint32_t bytes = (uint32_t)g.nfull * 16u;
  mbar_expect_tx(bar, bytes + (uint32_t)tx_extra);
  if (bytes) bulk_load(dst, g.x_full, bytes, bar);
}

template <typename T, int OP, bool EXACT, int SLOTS, int NT, int VPT, int NST, typename Src>
__device__ __forceinline__ void cta_ring_rows(const RingParams& p, const Segment& seg,
                                              uint64_t* bars, Src& src,
                                              float (*red)[NT / 32], bool& ok) {
  constexpr int P = Elem<T>::P;
  const Segment& s = seg;
  const int tid = threadIdx.x;
  const int D = s.dim;
  const float inv_d = inv_dim(D);
  const long long stride = gridDim.x;
  const long long r0 = blockIdx.x;
  int slot = 0;
  auto reduce = [&](float t) {
    const float v = block_sum<NT>(t, red[slot]);
    slot ^= 1;
    return v;
  };
  float Kq[NST], Eq[NST];
  // thread 0 starts the copies; every thread queues its scalars of the row
  auto ahead = [&](long long ra, int st, int j) {
    const Row<T> ga = row_geometry<T, EXACT>(s, ra);
    if (tid == 0)
      cta_ring_issue<T, EXACT>(s, ra, dyn_smem + st * (p.stage_bytes / 16), &bars[st], p.tx_extra);
    Kq[j] = OP == kOpLn ? Elem<T>::get(ga.x_row) : 0.f;
    Eq[j] = load_edge<T, EXACT>(ga, D, tid);
  };
#pragma unroll
  for (int j = 0; j < NST; ++j) {
    Kq[j] = 0.f;
    Eq[j] = 0.f;
    const long long rj = r0 + j * stride;
    if (rj < s.rows) ahead(rj, j, j);
  }
  long long i = 0;
  int st = 0;           // stage of row i: i % NST
  uint32_t parity = 0;  // phase parity of row i: (i / NST) & 1
#pragma unroll 1
  for (long long r = r0; r < s.rows; r += stride, ++i) {
    if (i > 0) {
      // every thread has passed row i - 1's reduction barriers: its stage
      // is free for row i - 1 + NST (refilling it already after row i - 1's
      // first reduction, half a row earlier, measured slower on B200: bf16
      // LayerNorm 65536 x 16384 698 -> 762 us)
      const long long ra = r + (NST - 1) * stride;
      const int rs = st == 0 ? NST - 1 : st - 1;
      if (tid == 0) fence_async_shared();
      if (ra < s.rows) ahead(ra, rs, NST - 1);
    }
    const float K = Kq[0];
    float xe = Eq[0];
#pragma unroll
    for (int j = 0; j + 1 < NST; ++j) {
      Kq[j] = Kq[j + 1];
      Eq[j] = Eq[j + 1];
    }
    const bool done = mbar_wait(&bars[st], parity, p.wait_ns);
    if (__syncthreads_or(!done)) {
      ok = false;
      if (tid == 0) {
        // rows i .. i + NST - 1 are issued and not yet consumed; row j sits
        // in stage (st + j - i) mod NST, one phase later once it wraps
        for (int j = 0; j < NST && r + j * stride < s.rows; ++j) {
          const int k = st + j;
          mbar_wait(&bars[k < NST ? k : k - NST], k < NST ? parity : parity ^ 1u, p.drain_ns);
        }
        atomicAdd(&g_ring_timeouts, 1u);
      }
      return;
    }
    const Row<T> g = row_geometry<T, EXACT>(s, r);
    const bool has_edge = !EXACT && tid < g.nedge;
    const int stage = st * (p.stage_bytes / 16);  // 16-byte words
    F2 v[VPT][P];
#pragma unroll
    for (int q = 0; q < VPT; ++q) {
      if (slot_present<SLOTS, VPT>(q, tid + NT * q, g.nfull)) {
        Elem<T>::unpack(dyn_smem[stage + tid + NT * q], v[q]);
      } else {
#pragma unroll
        for (int j = 0; j < P; ++j) v[q][j] = zero2();
      }
    }
    float rstd, mean;
    row_stats<T, OP, EXACT, SLOTS, VPT>(v, xe, g, inv_d, tid, NT, K, p.eps, has_edge, reduce,
                                        rstd, mean);
    if constexpr (!EXACT) {
      if (g.phase != src.phase) src.fill(s, g, tid, NT);
    }
    normalize_store<T, OP, EXACT, SLOTS, VPT>(s, g, v, xe, src, tid, NT, rstd, mean, has_edge);
    if (++st == NST) {
      st = 0;
      parity ^= 1u;
    }
  }
}

// Rows in flight per block ring: NST - 1 while one is normalized.
// Stages of a block ring. Measured on B200 (bf16 LayerNorm 65536 x 16384,
// 512 threads, cold): two stages 699 us, three 774 us (and blocks of 1024
// threads at two chunks each 1191 us; blocks of 256 threads at eight chunks
// each, 128 registers, 776 us (ptxas spilled 68 bytes); one block of 512
// threads per SM, with 128 registers holding the weight and bias, 3 or 4
// stages: 965-975 us, its two reduction barriers per row no longer
// overlapped by a second block).
__host__ __device__ constexpr int cta_ring_stages(int threads) { return threads >= 512 ? 2 : 3; }

// Register budget: the rows ahead wait in the ring, not in registers, so
// blocks of up to 256 threads take 80 registers (768 threads per SM) rather
// than spill at 64; wider blocks keep 1024 threads per SM.
__host__ __device__ constexpr int cta_ring_min_blocks(int threads) {
  return threads >= 512 ? kMinThreadsPerSm / threads : 768 / threads;
}

template <typename T, int OP, bool EXACT, int SLOTS, int NT, int VPT>
__global__ void __launch_bounds__(NT, cta_ring_min_blocks(NT))
rows_cta_ring_kernel(const RingParams p) {
  static_assert(OP == kOpRms || OP == kOpLn, "block rings carry RMSNorm and LayerNorm rows");
  static_assert(NT >= 2 * (Elem<T>::V - 1), "every edge element needs its own thread");
  constexpr int NST = cta_ring_stages(NT);
  constexpr bool BIAS = OP == kOpLn;
  __shared__ float red[2][NT / 32];
  __shared__ __align__(8) uint64_t bars[NST];
  if (threadIdx.x == 0) {
    for (int st = 0; st < NST; ++st) mbar_init(&bars[st], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const Segment& s = p.seg[0];
  bool ok = true;
  const T* w = static_cast<const T*>(s.w);
  const T* b = static_cast<const T*>(s.b);
  if constexpr (EXACT) {
    if (w && (!BIAS || b)) {
      AffineDirect<T, BIAS, true> src{w, b};
      cta_ring_rows<T, OP, true, SLOTS, NT, VPT, NST>(p, s, bars, src, red, ok);
    } else {
      AffineDirect<T, BIAS, false> src{w, b};
      cta_ring_rows<T, OP, true, SLOTS, NT, VPT, NST>(p, s, bars, src, red, ok);
    }
  } else {
    AffineCache<T, VPT, BIAS> src;
    src.init(NST * p.stage_bytes / 16);
    cta_ring_rows<T, OP, false, SLOTS, NT, VPT, NST>(p, s, bars, src, red, ok);
  }
}

}  // namespace rn
