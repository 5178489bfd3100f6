// Internal: the table of compiled kernel configurations shared by the host
// API and the per-element-type instantiation files.
#pragma once

namespace rn {

constexpr int kCtaMinChunks = 1;             // chunks per thread, block family
constexpr int kCtaMaxChunks = 5;
constexpr int kTargetChunksPerThread = 4;    // 64 bytes of loads in flight per thread
// Most chunks per thread of a kSlotsFull kernel, and of a block-family
// kSlotsTail kernel: at 5 those instantiations spill under the 64-register
// budget and measured slower on B200 than the loop that tests every slot.
constexpr int kFullMaxChunks = 4;

// Shared memory of the realigned weight/bias cache (layouts that are not
// EXACT): each thread's chunk slots of the weight (and bias).
constexpr int affine_cache_smem_bytes(int op, int threads, int chunks) {
  return threads * chunks * 16 * (op == 1 ? 2 : 1);
}
// Shared memory of the register kernels' prefetch slots (`stages` stages of
// each thread's chunk slots).
constexpr int prefetch_slots_smem_bytes(int threads, int chunks, int stages) {
  return stages * chunks * threads * 16;
}

// slots: kSlotsTested / kSlotsTail / kSlotsFull (0 / 1 / 2)
constexpr int warp_key(int op, bool exact, int slots, int chunks) {
  return ((op * 2 + (exact ? 1 : 0)) * 3 + slots) * 16 + chunks;
}
constexpr int cta_key(int op, bool exact, int slots, int threads, int chunks) {
  return (((op * 2 + (exact ? 1 : 0)) * 3 + slots) * 2048 + threads) * 8 + chunks;
}

constexpr int ring_key(int op, int slots, int chunks) { return (op * 3 + slots) * 16 + chunks; }

// Kernel entry for (op, exact, chunks per lane) in the warp family; nullptr
// if that configuration is not compiled. op: 0 RMSNorm, 1 LayerNorm. exact:
// every row of x and y starts 16-byte aligned, dim is a multiple of the
// 16-byte vector width, and the weight and bias start 16-byte aligned.
const void* warp_kernel_f32(int op, bool exact, int slots, int chunks);
const void* warp_kernel_bf16(int op, bool exact, int slots, int chunks);
// Kernel entry for (op, exact, threads per block, chunks per thread) in the
// block family; nullptr if not compiled.
const void* cta_kernel_f32(int op, bool exact, int slots, int threads, int chunks);
const void* cta_kernel_bf16(int op, bool exact, int slots, int threads, int chunks);
// Streaming kernels (rows wider than the register kernels hold): RMSNorm
// and LayerNorm, any layout.
const void* stream_kernel(int dtype_f32, int op, bool exact, int threads);
// Threads per row of the streaming kernels: 1024 (one block per SM), or 512
// for LayerNorm rows up to kStreamPairMaxRowBytes (several blocks per SM).
constexpr int kStreamBlockThreads = 1024;
constexpr int kStreamPairThreads = 512;
constexpr long long kStreamPairMaxRowBytes = 192 * 1024;

// Per-warp bulk-copy ring kernels (lane-group rows, 16-byte aligned
// layouts) for (op, slot policy, chunks per lane); op 0 RMSNorm, 1
// LayerNorm, 5 RMSNorm + RoPE with in-thread planes; nullptr if not compiled.
const void* ring_kernel_f32(int op, int slots, int chunks);
const void* ring_kernel_bf16(int op, int slots, int chunks);
// Block bulk-copy ring kernels (the block family's rows, any layout) for
// (op, exact, slot policy, threads per block, chunks per thread), keyed like
// the register block kernels; op 0 RMSNorm, 1 LayerNorm; nullptr if not
// compiled.
const void* cta_ring_kernel_f32(int op, bool exact, int slots, int threads, int chunks);
const void* cta_ring_kernel_bf16(int op, bool exact, int slots, int threads, int chunks);
// Timed-out stage waits recorded by the ring kernels of each table
// (optionally resetting the counter); returns a cudaError_t value.
int ring_timeouts_f32(unsigned int* count, bool reset);
int ring_timeouts_bf16(unsigned int* count, bool reset);
int cta_ring_timeouts_f32(unsigned int* count, bool reset);
int cta_ring_timeouts_bf16(unsigned int* count, bool reset);

}  // namespace rn
