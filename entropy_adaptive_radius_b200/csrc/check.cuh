// Index checks of the checked build (compiled with -DTRA_CHECK, built beside
// the library as libtra_check.so).  Sanitizer tools are not available on every
// machine this library runs on, so the kernels can check themselves: each
// index a kernel derives from the tile-major layout or from data it read (a
// decoded token position, a key block's frame, a footprint row) is compared
// with the extent of what it indexes before the access.  An index outside
// records kErrIndex in the device error word (tra_get_device_error reports
// TRA_ERR_BAD_INPUT with code 12) and the access is skipped.  Without
// TRA_CHECK every check is `true` and compiles away.
#pragma once
#include "ptx.cuh"

namespace tra {

__device__ __forceinline__ bool in_bounds(long long i, long long n, int* err) {
#ifdef TRA_CHECK
  if (i >= 0 && i < n) return true;
  if (err != nullptr) atomicCAS(err, 0, kErrIndex);
  return false;
#else
  (void)i;
  (void)n;
  (void)err;
  return true;
#endif
}

}  // namespace tra
