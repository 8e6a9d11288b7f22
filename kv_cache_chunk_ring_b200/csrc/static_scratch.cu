// Library-owned staging memory for chunk_attention_fwd_static_scratch().
//
// Some callers cannot allocate device memory when they call into the
// library: hosts whose memory pool owns every allocation and hands out exactly
// the cache buffer and nothing more, and real-time loops that must not take
// the implicit device synchronisation of cudaMalloc/cudaFree.  For them the
// rotated queries and current-chunk keys of one chunk are staged in this fixed
// file-scope array instead of a caller buffer.
//
// The array is kStaticScratchBytes (36 MiB) and lives on every GPU on which
// this module is loaded, until the process exits.  All calls on a device share
// it and it keeps the last call's contents; nothing in it has to start at
// zero because every call overwrites the part it reads.  Calls whose GPU work
// overlaps (several streams, or several host threads) race on it.
#include <mutex>

#include "static_scratch.h"

namespace kvcr {

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

cudaError_t static_scratch_address(void** ptr) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> g(mu);
  if (addr[dev] == nullptr) {
    // Host code may not use g_static_scratch as an address: ask the runtime for
    // the device address of the array on the current device (done once per device).
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  return cudaSuccess;
}

}  // namespace kvcr
