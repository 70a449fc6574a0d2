// The device-side error word shared by every kernel of the library.
#pragma once

namespace fa2 {

// 0 = OK.  A kernel that gives up a bounded wait, or meets an input it must
// not trust (see seq_view), records a site code here and winds down instead
// of spinning or touching memory outside its tensors.  The library is a
// single translation unit, so the definition lives in this header.
__device__ int g_fa2_device_status = 0;

// Site code: cu_seqlens of a variable-length call was not a non-decreasing
// list of offsets in [0, total] with every length <= max_seqlen.
constexpr int SITE_BAD_SEQLENS = 0xF10;

}  // namespace fa2
