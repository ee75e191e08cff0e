// State shared by every kernel of the library.
#pragma once
#include <cstdint>

namespace attn {

// Device-side error word: 0, or (site << 8) | kind for the first bounded wait that ran out. Read and cleared
// through attn_get_device_error / attn_clear_device_error.
__device__ uint32_t g_device_error;

}  // namespace attn
