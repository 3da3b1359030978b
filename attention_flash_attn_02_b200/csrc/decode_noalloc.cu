// decode_noalloc.cu -- paged decode for callers that cannot allocate device
// memory at the call site.
//
// Some callers have no way to obtain device memory when they run attention:
// a plugin or enqueue hook of another inference runtime that owns all device
// memory and forbids allocation while it executes, or a service that must not
// grow its device footprint after start-up (a cudaMalloc there would also
// synchronise the device and stall every other stream).  For them this file
// provides attn_decode_paged_noalloc: the same decode as attn_decode_paged,
// but its scratch (the split partials) lives in a fixed array that is part of
// the library image, so the call itself allocates nothing.
//
// Costs of that choice, stated plainly:
//   * the array (kScratchBytes) is device memory of the library's image.  The
//     CUDA runtime loads this file's code and data onto a GPU when it is
//     first needed there -- with lazy module loading (the default), at the
//     first call of this entry point on that device, whose address look-up
//     needs the array.  That first call per device therefore allocates the
//     array and may synchronise: make it once at start-up, with the device
//     current, outside any context that forbids allocation or
//     synchronisation and before any stream capture (a call with B == 0 does
//     only this set-up).  Every later call on that device allocates nothing,
//     and the array stays until the process exits;
//   * all calls share the one array and it keeps the last call's contents;
//     two calls that overlap on the GPU (different streams without ordering
//     between them) race on it and give wrong results;
//   * sizes whose scratch would exceed the array are rejected;
//   * the array's address is cached per device for the life of the process:
//     after cudaDeviceReset the cached address is stale, and this entry point
//     (like the rest of the library, which caches per-device state the same
//     way) must not be called again in that process.
// Nothing in the array has to start at zero: each call writes every partial
// it later reads before reading it.
#include <cstdio>
#include <mutex>

#include "../../include/attn.h"
#include "internal.h"

namespace attn {
namespace {

constexpr size_t kScratchBytes = ATTN_DECODE_NOALLOC_SCRATCH_BYTES;

// The scratch itself: a file-scope device array of fixed size.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;
thread_local char g_noalloc_msg[256] = "";

// Device address of the array on the current device.  Host code cannot use
// the symbol `g_decode_scratch` itself as a device pointer (on the host it
// names a stand-in object), so the address is looked up once per device,
// with that device current, and cached.
int scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail_cuda("decode (no-alloc): cudaGetDevice", err);
  if (dev < 0 || dev >= kMaxDevices) return fail_cuda("decode (no-alloc): device index", cudaErrorInvalidDevice);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    err = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (err != cudaSuccess || ptr == nullptr) return fail_cuda("decode (no-alloc): cudaGetSymbolAddress", err);
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return ATTN_OK;
}

}  // namespace
}  // namespace attn

using namespace attn;

ATTN_API int attn_decode_paged_noalloc(const void* q, const void* k_pages, const void* v_pages,
                                       const int* block_table, const int* seq_lens, void* o, float* lse, int B,
                                       int Hq, int Hkv, int D, int page_size, int num_pages, int max_pages_per_seq,
                                       float scale, attn_stream_t stream) {
  // The same argument checks as attn_decode_paged, in the same order, so the
  // two return the same status for the same arguments.
  int st = validate_decode(q, k_pages, v_pages, block_table, seq_lens, o, lse, B, Hq, Hkv, 1, D, D, page_size,
                           num_pages, max_pages_per_seq, scale);
  if (st != ATTN_OK) return st;
  // Set-up (first call per device, B == 0 included): the array's address.
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != ATTN_OK || B == 0) return st;
  const size_t need = attn_decode_workspace_bytes(B, Hq, max_pages_per_seq > 0 ? max_pages_per_seq : 1, D);
  if (need > kScratchBytes) {
    // Too large for the fixed array: refuse before launching anything.
    snprintf(g_noalloc_msg, sizeof(g_noalloc_msg),
             "attn_decode_paged_noalloc: these sizes need %zu bytes of scratch, the built-in array holds %zu",
             need, kScratchBytes);
    return fail_invalid(g_noalloc_msg);
  }
  return attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, o, lse, B, Hq, Hkv, D, page_size,
                           num_pages, max_pages_per_seq, scale, scratch, kScratchBytes, stream);
}
