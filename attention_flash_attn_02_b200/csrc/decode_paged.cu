// decode_paged.cu -- single-token attention against a paged KV cache
// (PagedAttention section of the page "LLM 中的 Attention 实现及优化",
// zeeklog.com: K/V kept in fixed-size pages of a shared pool, found through a
// per-sequence block table), for B200 (sm_100a).
//
// Two launches:
//   decode_split_kernel   grid (splits, B * Hkv).  Each CTA takes one K/V head
//       of one sequence and a run of kPagesPerSplit pages (512 tokens), gathers
//       the pages with 16-byte cp.async into swizzled shared memory (3-stage
//       ring), and computes, for all Hq/Hkv query heads of the group at once,
//       S = q K^T and O += P V on the tensor cores (mma.sync m16n8k16 bf16 ->
//       fp32) with the online-softmax recurrence.  It writes one partial
//       (normalised o, log2-sum-exp) per query head and split.
//   decode_combine_kernel one warp per (sequence, query head) merges the
//       partials: M = max_s lse_s, O = sum_s 2^(lse_s - M) o_s / sum_s
//       2^(lse_s - M), LSE = (M + log2 sum) ln 2.  This is the rescaling step of
//       the online softmax (page "003-注意力机制详解...", §二) applied once
//       across splits.
// All query heads of a K/V group share every gathered page (MQA/GQA: the
// tqpw.cn article §2.1/§3.1), which is what makes the tensor cores necessary:
// with 32 heads per K/V head, a SIMT dot product would be compute-bound.
#include <cuda_bf16.h>
#include <cstdint>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace attn {
namespace {

constexpr int kD = 128;
constexpr int kPage = 16;
constexpr int kThreads = 256;            // 8 warps
constexpr int kChunk = 64;               // tokens per pipeline stage
constexpr int kStages = 3;
constexpr int kRowBytes = kD * 2;        // 256
constexpr int kTileBytes = kChunk * kRowBytes;  // 16 KB (K or V of one stage)
constexpr int kQBytes = 32 * kRowBytes;          // 32 query rows (8 KB)
constexpr int kSmemBytes = kQBytes + kStages * 2 * kTileBytes + 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;

struct SplitParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_pages;
  const __nv_bfloat16* v_pages;
  const int* block_table;
  const int* seq_lens;
  float* ws_o;    // [B * Hq][max_splits][kD] normalised partial outputs
  float* ws_lse;  // [B * Hq][max_splits] log2-sum-exp of each partial
  int B, Hq, Hkv, group, num_pages, max_pages, max_splits;
  float scale_log2;
  int bounds_check;
  int* status;
};

__device__ __forceinline__ int seq_len_of(const SplitParams& p, int b) {
  int n = p.seq_lens[b];
  const int cap = p.max_pages * kPage;
  return n < 0 ? 0 : (n > cap ? cap : n);
}

// Byte offset of 16-byte chunk `c` of row `r` in a swizzled [rows][256 B] tile.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)(r * kRowBytes + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // 0: zero-fill, nothing read
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D = A * B + D, m16n8k16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kThreads, 2) decode_split_kernel(const SplitParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int split = blockIdx.x;
  const int bk = blockIdx.y;
  const int b = bk / p.Hkv, kvh = bk % p.Hkv;
  const int len = seq_len_of(p, b);
  const int npages = (len + kPage - 1) / kPage;
  const int pg0 = split * kDecodePagesPerSplit;
  if (pg0 >= npages) return;
  const int pg1 = min(pg0 + kDecodePagesPerSplit, npages);
  const int tok0 = pg0 * kPage;
  const int tok1 = min(pg1 * kPage, len);
  const int ntok = tok1 - tok0;
  const int nchunks = (ntok + kChunk - 1) / kChunk;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t s_q = smem_u32(smem);
  const uint32_t s_kv = s_q + kQBytes;
  int* s_pages = reinterpret_cast<int*>(smem + kQBytes + kStages * 2 * kTileBytes);

  // Page ids of this split (bounds-checked on request).
  if (tid < kDecodePagesPerSplit) {
    int id = 0;
    if (pg0 + tid < pg1) {
      id = p.block_table[(size_t)b * p.max_pages + pg0 + tid];
      if (p.bounds_check && (id < 0 || id >= p.num_pages)) {
        atomicExch(p.status, kErrBounds);
        id = -1;
      }
    }
    s_pages[tid] = id;
  }
  // Query rows of the group (rows >= group are zero).
  {
    const int row = tid >> 3;  // 32 rows x 16 chunks = 512 pieces, 2 per thread
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = (tid & 7) + 8 * i;
      const bool valid = row < p.group;
      const __nv_bfloat16* src = p.q + ((size_t)b * p.Hq + kvh * p.group + (valid ? row : 0)) * kD + c * 8;
      cp_async16(s_q + swz(row, c), src, valid);
    }
  }
  __syncthreads();  // s_pages visible

  auto load_chunk = [&](int ch, int stage) {
    const uint32_t dk = s_kv + stage * 2 * kTileBytes;
    const uint32_t dv = dk + kTileBytes;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int piece = tid + i * kThreads;  // 64 rows x 16 chunks
      const int row = piece >> 4, c = piece & 15;
      const int tok = ch * kChunk + row;      // token offset within the split
      const int pid = s_pages[tok >> 4];
      const bool valid = tok < ntok && pid >= 0;
      const size_t off = valid ? ((((size_t)pid * kPage + (tok & 15)) * p.Hkv + kvh) * kD + c * 8) : 0;
      cp_async16(dk + swz(row, c), p.k_pages + off, valid);
      cp_async16(dv + swz(row, c), p.v_pages + off, valid);
    }
  };
#pragma unroll
  for (int st = 0; st < kStages - 1; ++st) {
    if (st < nchunks) load_chunk(st, st);
    cp_async_commit();  // group 0 also carries the query rows
  }

  const int mt = warp & 1;   // 16-row query tile
  const int sub = warp >> 1; // 16-token slice of each chunk
  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  // per-lane partial row sums: exact fp32 (for the LSE) and of the rounded P
  // the tensor cores multiply (normalises o)
  float l_part[2] = {0.f, 0.f}, r_part[2] = {0.f, 0.f};
  const float sl2 = p.scale_log2;

  const int mi = lane >> 3, rr = lane & 7;
  uint32_t qa[kD / 16][4];  // A fragments of this warp's 16 query rows, loaded once
  for (int ch = 0; ch < nchunks; ++ch) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (ch == 0) {
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk)
        ldsm_x4(s_q + swz(mt * 16 + (mi & 1) * 8 + rr, kk * 2 + (mi >> 1)), qa[kk][0], qa[kk][1], qa[kk][2],
                qa[kk][3]);
    }
    if (ch + kStages - 1 < nchunks) load_chunk(ch + kStages - 1, (ch + kStages - 1) % kStages);
    cp_async_commit();
    const uint32_t sk = s_kv + (ch % kStages) * 2 * kTileBytes;
    const uint32_t sv = sk + kTileBytes;

    // S = q K^T for 16 query rows x 16 tokens
    float s[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sk + swz(sub * 16 + (mi >> 1) * 8 + rr, kk * 2 + (mi & 1)), b0, b1, b2, b3);
      mma_bf16(s[0], qa[kk], b0, b1);
      mma_bf16(s[1], qa[kk], b2, b3);
    }
    // mask tokens past the end of this split
    const int base_tok = ch * kChunk + sub * 16 + (lane & 3) * 2;
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = base_tok + n * 8 + (e & 1);
        s[n][e] = tok < ntok ? s[n][e] * sl2 : -INFINITY;
      }
    // online softmax for rows r (e = 0,1) and r + 8 (e = 2,3)
    float alpha[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float mx = fmaxf(fmaxf(s[0][2 * h], s[0][2 * h + 1]), fmaxf(s[1][2 * h], s[1][2 * h + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      alpha[h] = 1.f;
      if (mx > m_run[h] + kRescaleThreshold) {
        alpha[h] = ex2_approx(m_run[h] - mx);
        m_run[h] = mx;
      }
      l_part[h] *= alpha[h];
      r_part[h] *= alpha[h];
    }
    if (alpha[0] != 1.f || alpha[1] != 1.f) {
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        o[n][0] *= alpha[0];
        o[n][1] *= alpha[0];
        o[n][2] *= alpha[1];
        o[n][3] *= alpha[1];
      }
    }
    uint32_t pa[4];
    {
      const float nm0 = m_run[0] == -INFINITY ? 0.f : -m_run[0];
      const float nm1 = m_run[1] == -INFINITY ? 0.f : -m_run[1];
      float pv[2][4];
#pragma unroll
      for (int n = 0; n < 2; ++n) {
        pv[n][0] = ex2_approx(s[n][0] + nm0);
        pv[n][1] = ex2_approx(s[n][1] + nm0);
        pv[n][2] = ex2_approx(s[n][2] + nm1);
        pv[n][3] = ex2_approx(s[n][3] + nm1);
        l_part[0] += pv[n][0] + pv[n][1];
        l_part[1] += pv[n][2] + pv[n][3];
      }
      pa[0] = pack_bf16x2(pv[0][0], pv[0][1]);
      pa[1] = pack_bf16x2(pv[0][2], pv[0][3]);
      pa[2] = pack_bf16x2(pv[1][0], pv[1][1]);
      pa[3] = pack_bf16x2(pv[1][2], pv[1][3]);
      // row sums of the same rounded P the tensor cores multiply
      r_part[0] += sum_bf16x2(pa[0]) + sum_bf16x2(pa[2]);
      r_part[1] += sum_bf16x2(pa[1]) + sum_bf16x2(pa[3]);
    }
    // O += P V over 16 tokens x 128 features
#pragma unroll
    for (int n = 0; n < 16; n += 2) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(sv + swz(sub * 16 + (mi & 1) * 8 + rr, n + (mi >> 1)), b0, b1, b2, b3);
      mma_bf16(o[n], pa, b0, b1);
      mma_bf16(o[n + 1], pa, b2, b3);
    }
  }
  cp_async_wait<0>();
  __syncthreads();  // stages are free: reuse them for the merge

  // Merge the 4 token slices of each query tile through shared memory.
  constexpr int kOS = kD + 4;  // padded row stride of the merge buffer (bank spread)
  float* s_o = reinterpret_cast<float*>(smem + kQBytes);        // [8 warps][16 rows][kOS]
  float* s_ml = s_o + 8 * 16 * kOS;                             // [8 warps][16 rows][3]
  {
    const int r0 = lane >> 2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float l = l_part[h], lr = r_part[h];
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      lr += __shfl_xor_sync(0xffffffffu, lr, 1);
      lr += __shfl_xor_sync(0xffffffffu, lr, 2);
      if ((lane & 3) == 0) {
        s_ml[(warp * 16 + r0 + 8 * h) * 3 + 0] = m_run[h];
        s_ml[(warp * 16 + r0 + 8 * h) * 3 + 1] = l;
        s_ml[(warp * 16 + r0 + 8 * h) * 3 + 2] = lr;
      }
    }
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      const int col = n * 8 + (lane & 3) * 2;
      *reinterpret_cast<float2*>(&s_o[(warp * 16 + r0) * kOS + col]) = make_float2(o[n][0], o[n][1]);
      *reinterpret_cast<float2*>(&s_o[(warp * 16 + r0 + 8) * kOS + col]) = make_float2(o[n][2], o[n][3]);
    }
  }
  __syncthreads();
  // 32 rows x 128 features; each thread owns one row and 16 features.
  {
    const int row = tid >> 3;       // query row within the group tile (0..31)
    const int c0 = (tid & 7) * 16;  // first feature
    if (row < p.group) {
      const int mtile = row >> 4, r = row & 15;
      float M = -INFINITY;
#pragma unroll
      for (int sb = 0; sb < 4; ++sb) M = fmaxf(M, s_ml[((sb * 2 + mtile) * 16 + r) * 3]);
      float w[4], L = 0.f, LR = 0.f;
#pragma unroll
      for (int sb = 0; sb < 4; ++sb) {
        const float m = s_ml[((sb * 2 + mtile) * 16 + r) * 3];
        w[sb] = (m == -INFINITY) ? 0.f : ex2_approx(m - M);
        L += w[sb] * s_ml[((sb * 2 + mtile) * 16 + r) * 3 + 1];
        LR += w[sb] * s_ml[((sb * 2 + mtile) * 16 + r) * 3 + 2];
      }
      const float inv = LR > 0.f ? 1.f / LR : 0.f;
      const int h = kvh * p.group + row;
      const size_t rec = ((size_t)b * p.Hq + h) * p.max_splits + split;
      float* dst = p.ws_o + rec * kD;
#pragma unroll
      for (int c = 0; c < 16; c += 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int sb = 0; sb < 4; ++sb) {
          const float4 v = *reinterpret_cast<const float4*>(&s_o[((sb * 2 + mtile) * 16 + r) * kOS + c0 + c]);
          acc.x += w[sb] * v.x;
          acc.y += w[sb] * v.y;
          acc.z += w[sb] * v.z;
          acc.w += w[sb] * v.w;
        }
        *reinterpret_cast<float4*>(dst + c0 + c) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      }
      if (c0 == 0) p.ws_lse[rec] = (L > 0.f) ? M + __log2f(L) : -INFINITY;
    }
  }
}

struct CombineParams {
  const float* ws_o;
  const float* ws_lse;
  const int* seq_lens;
  __nv_bfloat16* o;
  float* lse;
  int B, Hq, max_pages, max_splits;
};

__global__ void __launch_bounds__(256) decode_combine_kernel(const CombineParams p) {
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= p.B * p.Hq) return;
  const int b = gw / p.Hq;
  int len = p.seq_lens[b];
  const int cap = p.max_pages * kPage;
  len = len < 0 ? 0 : (len > cap ? cap : len);
  const int nsplit = ((len + kPage - 1) / kPage + kDecodePagesPerSplit - 1) / kDecodePagesPerSplit;
  const float* base_o = p.ws_o + (size_t)gw * p.max_splits * kD;
  const float* base_l = p.ws_lse + (size_t)gw * p.max_splits;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float M = -INFINITY, L = 0.f;
  // splits in groups of 32: lane s owns split s of the group
  for (int s0 = 0; s0 < nsplit; s0 += 32) {
    const int n = min(32, nsplit - s0);
    const float l2 = lane < n ? base_l[s0 + lane] : -INFINITY;
    float gm = l2;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
    const float Mn = fmaxf(M, gm);
    if (Mn == -INFINITY) continue;
    const float scale_old = (M == -INFINITY) ? 0.f : ex2_approx(M - Mn);
    acc.x *= scale_old;
    acc.y *= scale_old;
    acc.z *= scale_old;
    acc.w *= scale_old;
    L *= scale_old;
    M = Mn;
    const float w = (l2 == -INFINITY) ? 0.f : ex2_approx(l2 - M);
    float ws = w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, o);
    L += ws;
    int s = 0;
    for (; s + 4 <= n; s += 4) {  // four independent loads in flight
      float4 v[4];
      float wv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        v[u] = *reinterpret_cast<const float4*>(base_o + (size_t)(s0 + s + u) * kD + lane * 4);
        wv[u] = __shfl_sync(0xffffffffu, w, s + u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc.x += wv[u] * v[u].x;
        acc.y += wv[u] * v[u].y;
        acc.z += wv[u] * v[u].z;
        acc.w += wv[u] * v[u].w;
      }
    }
    for (; s < n; ++s) {
      const float4 v = *reinterpret_cast<const float4*>(base_o + (size_t)(s0 + s) * kD + lane * 4);
      const float wv = __shfl_sync(0xffffffffu, w, s);
      acc.x += wv * v.x;
      acc.y += wv * v.y;
      acc.z += wv * v.z;
      acc.w += wv * v.w;
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint2 packed;
  packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  *reinterpret_cast<uint2*>(p.o + (size_t)gw * kD + lane * 4) = packed;
  if (lane == 0 && p.lse) p.lse[gw] = (L > 0.f) ? (M + __log2f(L)) * kLn2 : -INFINITY;
}

}  // namespace

int launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (a.D != kD || a.page_size != kPage) return -2;
  const int group = a.Hq / a.Hkv;
  if (group > 32) return -2;
  const int max_splits = decode_max_splits(a.max_pages);
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail_cuda("cudaGetDevice", err);
  if (dev < 64 && !attr_set[dev]) {
    err = cudaFuncSetAttribute(decode_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return fail_cuda("decode: cudaFuncSetAttribute", err);
    attr_set[dev] = true;
  }
  SplitParams sp{};
  sp.q = static_cast<const __nv_bfloat16*>(a.q);
  sp.k_pages = static_cast<const __nv_bfloat16*>(a.k_pages);
  sp.v_pages = static_cast<const __nv_bfloat16*>(a.v_pages);
  sp.block_table = a.block_table;
  sp.seq_lens = a.seq_lens;
  sp.ws_o = static_cast<float*>(a.workspace);
  sp.ws_lse = sp.ws_o + (size_t)a.B * a.Hq * max_splits * kD;
  sp.B = a.B;
  sp.Hq = a.Hq;
  sp.Hkv = a.Hkv;
  sp.group = group;
  sp.num_pages = a.num_pages;
  sp.max_pages = a.max_pages;
  sp.max_splits = max_splits;
  sp.scale_log2 = a.scale * kLog2e;
  sp.bounds_check = (debug_flags() & 1) ? 1 : 0;
  sp.status = device_status_word();
  if (!sp.status) return fail_cuda("decode: status word", cudaGetLastError());
  dim3 grid(max_splits, a.B * a.Hkv);
  decode_split_kernel<<<grid, kThreads, kSmemBytes, stream>>>(sp);
  err = cudaGetLastError();
  if (err != cudaSuccess) return fail_cuda("decode: split launch", err);
  CombineParams cp{};
  cp.ws_o = sp.ws_o;
  cp.ws_lse = sp.ws_lse;
  cp.seq_lens = a.seq_lens;
  cp.o = static_cast<__nv_bfloat16*>(a.o);
  cp.lse = a.lse;
  cp.B = a.B;
  cp.Hq = a.Hq;
  cp.max_pages = a.max_pages;
  cp.max_splits = max_splits;
  const int nw = a.B * a.Hq;
  decode_combine_kernel<<<(nw + 7) / 8, 256, 0, stream>>>(cp);
  err = cudaGetLastError();
  return err == cudaSuccess ? 0 : fail_cuda("decode: combine launch", err);
}

}  // namespace attn
