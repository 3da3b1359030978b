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
//   * every GPU that loads the library holds the array (kScratchBytes) until
//     the process exits, whether or not the entry point is used;
//   * all calls share the one array and it keeps the last call's contents;
//     two calls that overlap on the GPU (different streams without ordering
//     between them) race on it and give wrong results;
//   * sizes whose scratch would exceed the array are rejected.
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
  if (B < 0 || Hq <= 0 || D <= 0 || max_pages_per_seq < 0) return ATTN_ERR_INVALID;
  if (B == 0) return ATTN_OK;
  const size_t need = attn_decode_workspace_bytes(B, Hq, max_pages_per_seq > 0 ? max_pages_per_seq : 1, D);
  if (need > kScratchBytes) {
    // Too large for the fixed array: refuse before touching the GPU.
    snprintf(g_noalloc_msg, sizeof(g_noalloc_msg),
             "attn_decode_paged_noalloc: these sizes need %zu bytes of scratch, the built-in array holds %zu",
             need, kScratchBytes);
    fail_cuda(g_noalloc_msg, cudaErrorInvalidValue);
    return ATTN_ERR_INVALID;
  }
  void* scratch = nullptr;
  const int st = scratch_for_current_device(&scratch);
  if (st != ATTN_OK) return st;
  return attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, o, lse, B, Hq, Hkv, D, page_size,
                           num_pages, max_pages_per_seq, scale, scratch, kScratchBytes, stream);
}
