// internal.h -- declarations shared by the library's translation units (not
// part of the public ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace attn {

struct PrefillArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int B, Hq, Hkv, Lq, Lk, D;
  float scale;
  int causal, window;
  bool fp8;
  float q_descale, k_descale, v_descale;
  // Paged K/V (chunked prefill over a paged cache): k, v are the page pools
  // [num_pages, 16, Hkv, D]; Lk is unused (each sequence has seq_lens[b]).
  bool paged;
  const int* block_table;
  const int* seq_lens;
  int num_pages, max_pages;
  bool e5m2 = false;  // fp8 inputs in e5m2 (else e4m3)
};

// Attention with query/key width Dqk and value width Dv (64..256 each).
struct WideArgs {
  const void* q;  // [B, Hq, Lq, Dqk] bf16
  const void* k;  // [B, Hkv, Lk, Dqk]
  const void* v;  // [B, Hkv, Lk, Dv]
  void* o;        // [B, Hq, Lq, Dv]
  float* lse;
  int B, Hq, Hkv, Lq, Lk, Dqk, Dv;
  float scale;
  int causal, window;
};
int launch_prefill_wide(const WideArgs& a, cudaStream_t stream);

struct DecodeArgs {
  const void* q;
  const void* k_pages;
  const void* v_pages;
  const int* block_table;
  const int* seq_lens;
  void* o;
  float* lse;
  int B, Hq, Hkv, D, page_size, num_pages, max_pages;
  float scale;
  void* workspace;
  size_t workspace_bytes;
  int q_len;  // new tokens per sequence (queries), the last q_len cached ones
  int Dv = 0;  // value width (0: D); D is the query/key width
};

// Device status word of the current device (nullptr on failure).
int* device_status_word();
// Current debug flags / wait limit (set by attn_set_debug).
int debug_flags();
unsigned long long wait_timeout_ns();
// Number of SMs of the current device (cached).
int sm_count();

// Records a host-side failure for attn_last_error_message(); returns -3.
int fail_cuda(const char* where, cudaError_t err);
// Records an argument refusal for attn_last_error_message(); returns -1.
int fail_invalid(const char* msg);
// Checks of the decode arguments, workspace excepted (attn_api.cu).
int validate_decode(const void* q, const void* k_pages, const void* v_pages, const int* block_table,
                    const int* seq_lens, const void* o, const float* lse, int B, int Hq, int Hkv, int q_len, int D,
                    int Dv, int page_size, int num_pages, int max_pages_per_seq, float scale);

// Launchers: return a status code of include/attn.h.
int launch_prefill(const PrefillArgs& a, cudaStream_t stream);

struct BackwardArgs {
  const void* q;     // [B, Hq, Lq, D] bf16
  const void* k;     // [B, Hkv, Lk, D]
  const void* v;
  const void* o;     // forward output [B, Hq, Lq, D]
  const void* dout;  // dO
  const float* lse;  // forward LSE [B, Hq, Lq] (natural log)
  void* dq;          // [B, Hq, Lq, D] bf16
  void* dk;          // [B, Hkv, Lk, D]
  void* dv;
  int B, Hq, Hkv, Lq, Lk, D;
  float scale;
  int causal, window;
  void* workspace;   // backward_workspace_bytes(...)
};
int launch_backward(const BackwardArgs& a, cudaStream_t stream);
// dQ accumulator [B*Hq*Lq][D] fp32, then LSE (log2) and Dvec [B*Hq*Lq] fp32.
inline size_t backward_workspace_bytes(int B, int Hq, int Lq, int D) {
  return (size_t)B * Hq * Lq * (size_t)(D + 2) * 4;
}
// New tokens' K/V into their slots of the page pools (KV append).
int launch_kv_append(const void* k_new, const void* v_new, void* k_pages, void* v_pages, const int* block_table,
                     const int* seq_lens, int B, int Hkv, int L_new, int D, int num_pages, int max_pages,
                     cudaStream_t stream);
int launch_decode(const DecodeArgs& a, cudaStream_t stream);

// Decode work partition.  Every CTA streams a contiguous share of all cached
// pages of the batch, at least kDecodeMinChunk pages, so a sequence of P pages
// is cut into at most ceil(P / kDecodeMinChunk) + 1 segments; each segment
// leaves one partial (D floats + its log-sum-exp) per query head.
#ifndef ATTN_DECODE_MIN_CHUNK
#define ATTN_DECODE_MIN_CHUNK 32
#endif
constexpr int kDecodeMinChunk = ATTN_DECODE_MIN_CHUNK;  // pages (512 tokens)
inline int decode_max_segments(int max_pages) {
  return (max_pages + kDecodeMinChunk - 1) / kDecodeMinChunk + 1;
}
// Workspace: partial outputs [B*Hq][S][D] f32 and their log2-sum-exp
// [B*Hq][S] f32, S = segments (D: the value width).
inline size_t decode_workspace_bytes(int B, int Hq, int max_pages, int D) {
  const size_t rows = (size_t)B * Hq, segs = (size_t)decode_max_segments(max_pages);
  return rows * segs * (size_t)(D + 1) * 4;
}

}  // namespace attn
