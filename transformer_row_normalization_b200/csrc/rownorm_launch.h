// Internal: the table of compiled kernel configurations shared by the host
// API and the per-element-type instantiation files.
#pragma once

namespace rn {

constexpr int kWarpFamilyMaxChunksF32 = 9;   // dim <= 1024, any 16-byte phase
constexpr int kWarpFamilyMaxChunksBf16 = 5;
constexpr int kCtaMinChunks = 2;             // chunks per thread, block family
constexpr int kCtaMaxChunks = 5;
constexpr int kTargetChunksPerThread = 4;    // 64 bytes of loads in flight per thread

// Shared memory holding each thread's weight (and bias) chunk slots.
constexpr int affine_smem_bytes(int op, int threads, int chunks) {
  return threads * chunks * 16 * (op == 1 ? 2 : 1);
}

constexpr int warp_key(int op, bool exact, int chunks) {
  return (op * 2 + (exact ? 1 : 0)) * 16 + chunks;
}
constexpr int cta_key(int op, bool exact, int threads, int chunks) {
  return ((op * 2 + (exact ? 1 : 0)) * 2048 + threads) * 8 + chunks;
}

// Kernel entry for (op, exact, chunks per lane) in the warp family; nullptr
// if that configuration is not compiled. op: 0 RMSNorm, 1 LayerNorm. exact:
// every row of x and y starts 16-byte aligned and dim is a multiple of the
// 16-byte vector width.
const void* warp_kernel_f32(int op, bool exact, int chunks);
const void* warp_kernel_bf16(int op, bool exact, int chunks);
// Kernel entry for (op, exact, threads per block, chunks per thread) in the
// block family; nullptr if not compiled.
const void* cta_kernel_f32(int op, bool exact, int threads, int chunks);
const void* cta_kernel_bf16(int op, bool exact, int threads, int chunks);

}  // namespace rn
