// State shared by the library's translation units: the text of the last CUDA error met on the calling thread
// (returned by attn_last_cuda_error), and access to the prologue unit's device error word.
#pragma once
#include <cstddef>
#include <cstdint>

namespace attn {
constexpr std::size_t kErrorTextBytes = 256;
extern thread_local char g_cuda_error[kErrorTextBytes];

// The prologue's translation unit keeps its own device error word; these read and clear it (a cudaError_t
// value: 0 on success). attn_get_device_error / attn_clear_device_error combine it with the attention kernels'.
int rope_error_word(std::uint32_t* word);
int rope_error_clear();
}  // namespace attn
