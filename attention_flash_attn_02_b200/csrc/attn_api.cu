// attn_api.cu -- the C ABI of include/attn.h: argument validation (before any
// CUDA call), the per-device status word, debug switches, and dispatch to the
// kernel launchers.
#include <atomic>
#include <cstdio>
#include <cstdint>
#include <mutex>

#include "../../include/attn.h"
#include "internal.h"

namespace attn {

// One status word per device, written by kernels (never trapped on).
__device__ int g_status;

namespace {
constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {nullptr};
int g_sms[kMaxDevices] = {0};
std::mutex g_mu;
std::atomic<int> g_debug_flags{0};
std::atomic<unsigned long long> g_timeout_ns{2000000000ull};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

int* device_status_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (g_status_ptr[dev]) return g_status_ptr[dev];
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_status_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(ptr);
  }
  return g_status_ptr[dev];
}

namespace {
thread_local char g_msg[256] = "";
}

int fail_cuda(const char* where, cudaError_t err) {
  snprintf(g_msg, sizeof(g_msg), "%s: %s", where, cudaGetErrorString(err));
  return ATTN_ERR_CUDA;
}

int fail_invalid(const char* msg) {
  snprintf(g_msg, sizeof(g_msg), "%s", msg);
  return ATTN_ERR_INVALID;
}

int debug_flags() { return g_debug_flags.load(); }
unsigned long long wait_timeout_ns() { return g_timeout_ns.load(); }

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (!g_sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

}  // namespace attn

using namespace attn;

namespace {

int validate_prefill(const void* q, const void* k, const void* v, void* o, const float* lse, int B, int Hq,
                     int Hkv, int Lq, int Lk, int D, float scale, int causal, int window) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Lq < 0 || Lk < 0 || D <= 0) return ATTN_ERR_INVALID;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID;
  if (window > 0 && !causal) return ATTN_ERR_INVALID;
  if (!(scale == scale) || scale <= 0.f) return ATTN_ERR_INVALID;  // NaN or non-positive
  const long long nq = (long long)B * Hq * Lq;
  const long long nk = (long long)B * Hkv * Lk;
  if (nq > 0 && (!q || !o || !aligned16(q) || !aligned16(o))) return ATTN_ERR_INVALID;
  if (nq > 0 && lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_INVALID;
  if (nk > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return ATTN_ERR_INVALID;
  if (B > 65535 || (long long)B * Hq > (1ll << 31) - 1 || Lq > (1 << 30) || Lk > (1 << 30))
    return ATTN_ERR_INVALID;
  return ATTN_OK;
}

}  // namespace

ATTN_API int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                      int Lq, int Lk, int D, float scale, int causal, int window, attn_stream_t stream) {
  int st = validate_prefill(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, D, scale, causal, window);
  if (st != ATTN_OK) return st;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * Hq * Lq == 0) return ATTN_OK;
  PrefillArgs a{q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, D, scale, causal, window > 0 ? window : 0, false, 1.f, 1.f, 1.f};
  return launch_prefill(a, static_cast<cudaStream_t>(stream));
}

ATTN_API int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                          int Hkv, int Lq, int Lk, int D, float scale, int causal, int window, float q_descale,
                          float k_descale, float v_descale, attn_stream_t stream) {
  int st = validate_prefill(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, D, scale, causal, window);
  if (st != ATTN_OK) return st;
  if (!(q_descale > 0.f) || !(k_descale > 0.f) || !(v_descale > 0.f)) return ATTN_ERR_INVALID;
  if (D != 128) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * Hq * Lq == 0) return ATTN_OK;
  PrefillArgs a{q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, D, scale, causal, window > 0 ? window : 0, true,
                q_descale, k_descale, v_descale};
  return launch_prefill(a, static_cast<cudaStream_t>(stream));
}

ATTN_API int attn_fwd_e5m2(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                           int Hkv, int Lq, int Lk, int D, float scale, int causal, int window, float q_descale,
                           float k_descale, float v_descale, attn_stream_t stream) {
  int st = validate_prefill(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, D, scale, causal, window);
  if (st != ATTN_OK) return st;
  if (!(q_descale > 0.f) || !(k_descale > 0.f) || !(v_descale > 0.f)) return ATTN_ERR_INVALID;
  if (D != 128) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * Hq * Lq == 0) return ATTN_OK;
  PrefillArgs a{q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, D, scale, causal, window > 0 ? window : 0, true,
                q_descale, k_descale, v_descale};
  a.e5m2 = true;
  return launch_prefill(a, static_cast<cudaStream_t>(stream));
}

ATTN_API int attn_fwd_mla(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                          int Hkv, int Lq, int Lk, int D_qk, int D_v, float scale, int causal, int window,
                          attn_stream_t stream) {
  if (D_v <= 0) return ATTN_ERR_INVALID;
  int st = validate_prefill(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, D_qk, scale, causal, window);
  if (st != ATTN_OK) return st;
  auto ok_dim = [](int d) { return d == 64 || d == 128 || d == 192 || d == 256; };
  if (!ok_dim(D_qk) || !ok_dim(D_v)) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * Hq * Lq == 0) return ATTN_OK;
  WideArgs a{q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, D_qk, D_v, scale, causal, window > 0 ? window : 0};
  return launch_prefill_wide(a, static_cast<cudaStream_t>(stream));
}

ATTN_API size_t attn_decode_workspace_bytes(int B, int Hq, int max_pages_per_seq, int D) {
  if (B <= 0 || Hq <= 0 || max_pages_per_seq <= 0 || D <= 0) return 0;
  return decode_workspace_bytes(B, Hq, max_pages_per_seq, D);
}

namespace attn {
// Every check of the decode arguments except the workspace: ATTN_OK to go on
// (B == 0 included: nothing to launch), else the status to return.
int validate_decode(const void* q, const void* k_pages, const void* v_pages, const int* block_table,
                    const int* seq_lens, const void* o, const float* lse, int B, int Hq, int Hkv, int q_len, int D,
                    int Dv, int page_size, int num_pages, int max_pages_per_seq, float scale) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Dv <= 0 || page_size <= 0 || num_pages < 0 ||
      max_pages_per_seq < 0 || q_len <= 0)
    return ATTN_ERR_INVALID;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID;
  if (!(scale == scale) || scale <= 0.f) return ATTN_ERR_INVALID;
  if (B == 0) return ATTN_OK;
  if (!q || !o || !seq_lens || !aligned16(q) || !aligned16(o)) return ATTN_ERR_INVALID;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_INVALID;
  if (max_pages_per_seq > 0 && (!block_table || (reinterpret_cast<uintptr_t>(block_table) & 3u)))
    return ATTN_ERR_INVALID;
  if (num_pages > 0 && (!k_pages || !v_pages || !aligned16(k_pages) || !aligned16(v_pages)))
    return ATTN_ERR_INVALID;
  auto ok_dim = [](int d) { return d == 64 || d == 128 || d == 192 || d == 256; };
  if (!ok_dim(D) || !ok_dim(Dv) || page_size != 16 || (Hq / Hkv) * q_len > 128) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}
}  // namespace attn

namespace {
int decode_checked(const void* q, const void* k_pages, const void* v_pages, const int* block_table,
                   const int* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int q_len, int D, int Dv,
                   int page_size, int num_pages, int max_pages_per_seq, float scale, void* workspace,
                   size_t workspace_bytes, attn_stream_t stream) {
  const int st = validate_decode(q, k_pages, v_pages, block_table, seq_lens, o, lse, B, Hq, Hkv, q_len, D, Dv,
                                 page_size, num_pages, max_pages_per_seq, scale);
  if (st != ATTN_OK || B == 0) return st;
  const int mp = max_pages_per_seq > 0 ? max_pages_per_seq : 1;
  const size_t need = attn_decode_workspace_bytes(B, Hq * q_len, mp, Dv);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return ATTN_ERR_INVALID;
  DecodeArgs a{q, k_pages, v_pages, block_table, seq_lens, o, lse, B, Hq, Hkv, D, page_size, num_pages,
               max_pages_per_seq, scale, workspace, workspace_bytes, q_len, Dv};
  return launch_decode(a, static_cast<cudaStream_t>(stream));
}
}  // namespace

ATTN_API int attn_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int* block_table,
                               const int* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int D,
                               int page_size, int num_pages, int max_pages_per_seq, float scale, void* workspace,
                               size_t workspace_bytes, attn_stream_t stream) {
  return decode_checked(q, k_pages, v_pages, block_table, seq_lens, o, lse, B, Hq, Hkv, 1, D, D, page_size,
                        num_pages, max_pages_per_seq, scale, workspace, workspace_bytes, stream);
}

ATTN_API int attn_decode_paged_multi(const void* q, const void* k_pages, const void* v_pages,
                                     const int* block_table, const int* seq_lens, void* o, float* lse, int B,
                                     int Hq, int Hkv, int q_len, int D, int page_size, int num_pages,
                                     int max_pages_per_seq, float scale, void* workspace, size_t workspace_bytes,
                                     attn_stream_t stream) {
  return decode_checked(q, k_pages, v_pages, block_table, seq_lens, o, lse, B, Hq, Hkv, q_len, D, D, page_size,
                        num_pages, max_pages_per_seq, scale, workspace, workspace_bytes, stream);
}

ATTN_API int attn_decode_paged_mla(const void* q, const void* k_pages, const void* v_pages, const int* block_table,
                                   const int* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int q_len,
                                   int D_qk, int D_v, int page_size, int num_pages, int max_pages_per_seq,
                                   float scale, void* workspace, size_t workspace_bytes, attn_stream_t stream) {
  return decode_checked(q, k_pages, v_pages, block_table, seq_lens, o, lse, B, Hq, Hkv, q_len, D_qk, D_v, page_size,
                        num_pages, max_pages_per_seq, scale, workspace, workspace_bytes, stream);
}

ATTN_API int attn_prefill_paged(const void* q, const void* k_pages, const void* v_pages, const int* block_table,
                                const int* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int Lq, int D,
                                int page_size, int num_pages, int max_pages_per_seq, float scale, int window,
                                attn_stream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || D <= 0 || page_size <= 0 || num_pages <= 0 ||
      max_pages_per_seq <= 0)
    return ATTN_ERR_INVALID;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID;
  if (!(scale == scale) || scale <= 0.f) return ATTN_ERR_INVALID;
  if (B == 0) return ATTN_OK;
  if (!q || !o || !k_pages || !v_pages || !block_table || !seq_lens) return ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(o) || !aligned16(k_pages) || !aligned16(v_pages)) return ATTN_ERR_INVALID;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return ATTN_ERR_INVALID;
  if ((D != 64 && D != 128) || page_size != 16) return ATTN_ERR_UNSUPPORTED;
  PrefillArgs a{q, k_pages, v_pages, o, lse, B, Hq, Hkv, Lq, 0, D, scale, 1, window > 0 ? window : 0, false,
                1.f, 1.f, 1.f, true, block_table, seq_lens, num_pages, max_pages_per_seq};
  return launch_prefill(a, static_cast<cudaStream_t>(stream));
}

ATTN_API int attn_kv_append(const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                            const int* block_table, const int* seq_lens, int B, int Hkv, int L_new, int D,
                            int page_size, int num_pages, int max_pages_per_seq, attn_stream_t stream) {
  if (B < 0 || Hkv <= 0 || L_new < 0 || D <= 0 || page_size <= 0 || num_pages < 0 || max_pages_per_seq < 0)
    return ATTN_ERR_INVALID;
  if (B == 0 || L_new == 0) return ATTN_OK;
  if (num_pages == 0 || max_pages_per_seq == 0) return ATTN_ERR_INVALID;  // nowhere to write
  if (!k_new || !v_new || !k_pages || !v_pages || !block_table || !seq_lens) return ATTN_ERR_INVALID;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pages) || !aligned16(v_pages)) return ATTN_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return ATTN_ERR_INVALID;
  if (D % 8 != 0 || page_size != 16) return ATTN_ERR_UNSUPPORTED;
  return launch_kv_append(k_new, v_new, k_pages, v_pages, block_table, seq_lens, B, Hkv, L_new, D, num_pages,
                          max_pages_per_seq, static_cast<cudaStream_t>(stream));
}

ATTN_API size_t attn_bwd_workspace_bytes(int B, int Hq, int Lq, int D) {
  if (B <= 0 || Hq <= 0 || Lq <= 0 || D <= 0) return 0;
  return backward_workspace_bytes(B, Hq, Lq, D);
}

ATTN_API int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                      const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Lq, int Lk, int D,
                      float scale, int causal, int window, void* workspace, size_t workspace_bytes,
                      attn_stream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Lq < 0 || Lk < 0 || D <= 0) return ATTN_ERR_INVALID;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID;
  if (!(scale == scale) || scale <= 0.f) return ATTN_ERR_INVALID;
  if (window > 0 && !causal) return ATTN_ERR_INVALID;
  if (B == 0 || Lq == 0) return ATTN_OK;
  const void* ptrs[] = {q, o, dout, dq, workspace};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return ATTN_ERR_INVALID;
  if (!lse || (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_INVALID;
  if (Lk > 0 && (!k || !v || !dk || !dv || !aligned16(k) || !aligned16(v) || !aligned16(dk) || !aligned16(dv)))
    return ATTN_ERR_INVALID;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (workspace_bytes < attn_bwd_workspace_bytes(B, Hq, Lq, D)) return ATTN_ERR_INVALID;
  BackwardArgs a{q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Lq, Lk, D, scale, causal ? 1 : 0,
                 window > 0 ? window : 0, workspace};
  return launch_backward(a, static_cast<cudaStream_t>(stream));
}

ATTN_API int attn_last_device_error(attn_stream_t stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  int* p = device_status_word();
  if (!p) return ATTN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return v;
}

ATTN_API const char* attn_status_str(int status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID: return "ATTN_ERR_INVALID";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    case ATTN_ERR_BOUNDS: return "ATTN_ERR_BOUNDS";
    default: return "ATTN_UNKNOWN_STATUS";
  }
}

ATTN_API int attn_set_debug(int flags, unsigned long long wait_timeout_ns) {
  const int prev = g_debug_flags.exchange(flags);
  g_timeout_ns.store(wait_timeout_ns ? wait_timeout_ns : 2000000000ull);
  return prev;
}

ATTN_API int attn_version(void) { return 1; }

ATTN_API const char* attn_last_error_message(void) { return g_msg; }
