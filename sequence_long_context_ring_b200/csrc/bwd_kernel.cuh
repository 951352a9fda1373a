// bwd_kernel.cuh — backward of ring attention for sm_100a (recompute from the stored LSE).
#pragma once
#include <cstddef>
#include "sm100.cuh"

namespace cpattn {

// Extra workspace the backward kernels need beyond the dQ accumulator and D.
inline size_t bwd_workspace_extra(int, int, int, int, int) { return 0; }

}  // namespace cpattn
