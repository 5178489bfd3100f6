// The streaming kernels (rows wider than the register kernels hold) for both
// element types, and the table the host planner selects them from.
#include "rownorm_launch.h"
#include "rownorm_stream.cuh"

namespace rn {

template <typename T, int NT>
const void* stream_kernel_for(int op, bool exact) {
  if (op == kOpRms)
    return exact ? reinterpret_cast<const void*>(&rows_stream_kernel<T, kOpRms, true, NT>)
                 : reinterpret_cast<const void*>(&rows_stream_kernel<T, kOpRms, false, NT>);
  if (op == kOpLn)
    return exact ? reinterpret_cast<const void*>(&rows_stream_kernel<T, kOpLn, true, NT>)
                 : reinterpret_cast<const void*>(&rows_stream_kernel<T, kOpLn, false, NT>);
  return nullptr;
}

template <typename T>
const void* stream_kernel_for(int op, bool exact, int threads) {
  if (threads == kStreamPairThreads) return stream_kernel_for<T, kStreamPairThreads>(op, exact);
  if (threads == kStreamBlockThreads) return stream_kernel_for<T, kStreamBlockThreads>(op, exact);
  return nullptr;
}

const void* stream_kernel(int dtype_f32, int op, bool exact, int threads) {
  return dtype_f32 ? stream_kernel_for<float>(op, exact, threads)
                   : stream_kernel_for<__nv_bfloat16>(op, exact, threads);
}

}  // namespace rn
