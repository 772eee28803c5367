// Bounds-checking build (-DUSP_BOUNDS_CHECK): every global offset a copy or
// store kernel computes is checked against the extent of the buffer it
// addresses. An offset outside [0, extent) records `site` in the translation
// unit's device error word and the access is skipped. Without the flag the
// check is `true` and costs nothing. usp_device_status reports a recorded site
// as USP_ERR_BOUNDS.
#pragma once

#include <cstdint>

namespace usp {

#ifdef USP_BOUNDS_CHECK
constexpr bool kBoundsCheck = true;
#else
constexpr bool kBoundsCheck = false;
#endif

// True when [off, off + len) lies inside [0, ext); otherwise records `site`.
__device__ __forceinline__ bool in_bounds(int64_t off, int64_t len, int64_t ext, uint32_t site, uint32_t* word) {
  if constexpr (!kBoundsCheck) {
    return true;
  } else {
    if (off >= 0 && len >= 0 && off + len <= ext) return true;
    atomicCAS(word, 0u, site);
    return false;
  }
}

}  // namespace usp
