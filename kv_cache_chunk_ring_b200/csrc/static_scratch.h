// Library-owned staging array used by chunk_attention_fwd_static_scratch():
// rotated queries, then rotated current keys (each half at most 18 MiB).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace kvcr {

constexpr size_t kStaticScratchBytes = 36u << 20;

// Device address of the array on the current device (looked up once per device).
cudaError_t static_scratch_address(void** ptr);

}  // namespace kvcr
