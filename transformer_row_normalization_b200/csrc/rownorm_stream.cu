// The streaming kernels (rows wider than the register kernels hold) for both
// element types, and the table the host planner selects them from.
#include "rownorm_launch.h"
#include "rownorm_stream.cuh"

namespace rn {

template <typename T>
const void* stream_kernel_for(int op, bool exact) {
  if (op == kOpRms)
    return exact ? reinterpret_cast<const void*>(&rows_stream_kernel<T, kOpRms, true>)
                 : reinterpret_cast<const void*>(&rows_stream_kernel<T, kOpRms, false>);
  if (op == kOpLn)
    return exact ? reinterpret_cast<const void*>(&rows_stream_kernel<T, kOpLn, true>)
                 : reinterpret_cast<const void*>(&rows_stream_kernel<T, kOpLn, false>);
  return nullptr;
}

const void* stream_kernel(int dtype_f32, int op, bool exact) {
  return dtype_f32 ? stream_kernel_for<float>(op, exact)
                   : stream_kernel_for<__nv_bfloat16>(op, exact);
}

}  // namespace rn
