// The text of the last CUDA error this library met on the calling thread (returned by attn_last_cuda_error),
// shared by every translation unit of the library.
#pragma once
#include <cstddef>

namespace attn {
constexpr std::size_t kErrorTextBytes = 256;
extern thread_local char g_cuda_error[kErrorTextBytes];
}  // namespace attn
