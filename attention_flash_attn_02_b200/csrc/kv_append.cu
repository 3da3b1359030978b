// kv_append.cu -- write the K/V of each sequence's newest tokens into their
// slots of the paged pools (the KV cache of the PagedAttention section of
// the page "LLM 中的 Attention 实现及优化", zeeklog.com: fixed-size pages of
// a shared pool, found through a per-sequence block table).
//
// Token t of sequence b (of L_new new ones) sits at position
// seq_lens[b] - L_new + t, i.e. page block_table[b][pos / 16], slot pos % 16.
// One thread copies 16 bytes (8 bf16 features) of K and of V; consecutive
// threads take consecutive features, so both sides are coalesced.  This is a
// pure copy bound by HBM bandwidth.  Page ids are checked before any write:
// an id outside [0, num_pages) is skipped and reported as ATTN_ERR_BOUNDS.
#include <cuda_bf16.h>
#include <cstdint>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace attn {
namespace {

constexpr int kPageTokens = 16;

struct AppendParams {
  const uint4* k_new;  // [B, Hkv, L_new, D] bf16
  const uint4* v_new;
  uint4* k_pages;      // [num_pages, 16, Hkv, D] bf16
  uint4* v_pages;
  const int* block_table;
  const int* seq_lens;
  int B, Hkv, L_new, chunks;  // chunks: 16-byte pieces per row (D / 8)
  int num_pages, max_pages;
  int* status;
};

__global__ void __launch_bounds__(256) kv_append_kernel(const AppendParams p) {
  const long long total = (long long)p.B * p.L_new * p.Hkv * p.chunks;
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < total; i += (long long)gridDim.x * 256) {
    const int c = (int)(i % p.chunks);
    long long r = i / p.chunks;
    const int kvh = (int)(r % p.Hkv);
    r /= p.Hkv;
    const int t = (int)(r % p.L_new);
    const int b = (int)(r / p.L_new);
    int n = p.seq_lens[b];
    const int cap = p.max_pages * kPageTokens;
    n = n > cap ? cap : n;
    const int pos = n - p.L_new + t;
    if (pos < 0) continue;
    const int page = p.block_table[(size_t)b * p.max_pages + pos / kPageTokens];
    if (page < 0 || page >= p.num_pages) {
      atomicExch(p.status, kErrBounds);
      continue;
    }
    const size_t src = (((size_t)b * p.Hkv + kvh) * p.L_new + t) * p.chunks + c;
    const size_t dst = (((size_t)page * kPageTokens + pos % kPageTokens) * p.Hkv + kvh) * p.chunks + c;
    p.k_pages[dst] = p.k_new[src];
    p.v_pages[dst] = p.v_new[src];
  }
}

}  // namespace

int launch_kv_append(const void* k_new, const void* v_new, void* k_pages, void* v_pages, const int* block_table,
                     const int* seq_lens, int B, int Hkv, int L_new, int D, int num_pages, int max_pages,
                     cudaStream_t stream) {
  AppendParams p{};
  p.k_new = static_cast<const uint4*>(k_new);
  p.v_new = static_cast<const uint4*>(v_new);
  p.k_pages = static_cast<uint4*>(k_pages);
  p.v_pages = static_cast<uint4*>(v_pages);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.B = B;
  p.Hkv = Hkv;
  p.L_new = L_new;
  p.chunks = D / 8;
  p.num_pages = num_pages;
  p.max_pages = max_pages;
  p.status = device_status_word();
  if (!p.status) return fail_cuda("kv append: status word", cudaGetLastError());
  const long long total = (long long)B * L_new * Hkv * p.chunks;
  long long blocks = (total + 255) / 256;
  const long long cap = 8ll * sm_count();
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  kv_append_kernel<<<(unsigned)blocks, 256, 0, stream>>>(p);
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? 0 : fail_cuda("kv append: launch", err);
}

}  // namespace attn
