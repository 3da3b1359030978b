// decode_paged.cu -- single-token attention against a paged KV cache
// (PagedAttention section of the page "LLM 中的 Attention 实现及优化",
// zeeklog.com: K/V kept in fixed-size pages of a shared pool, found through a
// per-sequence block table), for B200 (sm_100a).
//
// Two launches:
//   decode_split_kernel   G = 3 CTAs per SM.  All cached pages of the batch,
//       sequence after sequence (and K/V head after K/V head), form one list
//       of T pages; CTA c streams the contiguous share [c T / G, (c+1) T / G)
//       of it (at least kDecodeMinChunk pages), so every CTA moves the same
//       number of bytes whatever the length mix.  Warp 2 is a TMA producer:
//       it loads the 32 query rows of each sequence segment it meets and
//       copies whole pages (K and V, 128-byte swizzled) straight from the pool
//       into a 6-stage ring tracked by mbarriers.  Warps 0 and 1 take query
//       rows [0, 16) and [16, 32) of the K/V group and compute S = q K^T and
//       O += P V on the tensor cores (mma.sync m16n8k16 bf16 -> fp32) with the
//       online-softmax recurrence; at the end of a segment they write one
//       partial (normalised o, log2-sum-exp) per query head.
//   decode_combine_kernel one warp per (sequence, query head) merges the
//       partials: M = max_s lse_s, O = sum_s 2^(lse_s - M) o_s / sum_s
//       2^(lse_s - M), LSE = (M + log2 sum) ln 2.  This is the rescaling step of
//       the online softmax (page "003-注意力机制详解...", §二) applied once
//       across segments.
// All query heads of a K/V group share every gathered page (MQA/GQA: the
// tqpw.cn article §2.1/§3.1), which is what makes the tensor cores necessary:
// with 32 heads per K/V head, a SIMT dot product would be compute-bound.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <cstdint>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace attn {
namespace {

constexpr int kD = 128;
constexpr int kPage = 16;
constexpr int kThreads = 96;                 // 2 consumer warps + 1 producer warp
#ifndef ATTN_DECODE_STAGES
#define ATTN_DECODE_STAGES 6
#define ATTN_DECODE_CTAS_PER_SM 3
#endif
constexpr int kStages = ATTN_DECODE_STAGES;
constexpr int kCtasPerSm = ATTN_DECODE_CTAS_PER_SM;
constexpr int kHalfBox = kPage * 128;        // 16 tokens x 64 features (bf16): 2 KB
constexpr int kPageBytes = 2 * kHalfBox;     // K (or V) of one page: 4 KB
constexpr int kStageBytes = 2 * kPageBytes;  // K and V of one page: 8 KB
constexpr int kQRows = 32;                   // query rows per K/V group tile
constexpr int kQBox = kQRows * 128;          // 32 rows x 64 features: 4 KB
constexpr int kQBytes = 2 * kQBox;           // 8 KB per query slot
constexpr int kRingOff = 2 * kQBytes;        // two query slots, then the ring
constexpr int kSmemBytes = 1024 + kRingOff + kStages * kStageBytes + 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;

struct SplitParams {
  const int* block_table;
  const int* seq_lens;
  float* ws_o;    // [B * Hq][S][kD] normalised partial outputs
  float* ws_lse;  // [B * Hq][S] log2-sum-exp of each partial
  int* ws_nseg;   // [B * Hkv] segments of each (sequence, K/V head)
  int B, Hq, Hkv, group, num_pages, max_pages, max_segs;
  float scale_log2;
  int bounds_check;
  int* status;
  unsigned long long timeout_ns;
  int stall;  // testing hook: the producer issues no loads, every wait runs out
};

struct DecSmem {
  uint64_t full[kStages], empty[kStages];
  uint64_t qfull[2], qempty[2];
  int valid[kStages];
  int abort_flag;
};
static_assert(sizeof(DecSmem) <= 256, "barrier block exceeds its reserve");
static_assert(kCtasPerSm * (kSmemBytes + 1024) <= 233472, "CTAs per SM do not fit in shared memory");

__device__ __forceinline__ int len_of(const int* seq_lens, int max_pages, int b) {
  const int n = seq_lens[b], cap = max_pages * kPage;
  return n < 0 ? 0 : (n > cap ? cap : n);
}
__device__ __forceinline__ int pages_of(const int* seq_lens, int max_pages, int b) {
  return (len_of(seq_lens, max_pages, b) + kPage - 1) / kPage;
}
// CTA that owns page x of the list when T pages are split over G CTAs.
__device__ __forceinline__ int owner(long long x, long long T, int G) {
  return (int)(((x + 1) * G - 1) / T);
}

// Walks the (sequence, K/V head) segments a CTA's page range [lo, hi) meets.
struct Segments {
  const SplitParams& p;
  long long hi;
  long long x;    // next page of the list
  long long pre;  // list index of the first page of the current (b, kvh)
  int b, kvh, P;  // current sequence, K/V head, its page count
  __device__ Segments(const SplitParams& p_, long long lo, long long hi_) : p(p_), hi(hi_), x(lo) {
    long long c = 0;
    b = 0;
    kvh = 0;
    P = 0;
    pre = 0;
    for (; b < p.B; ++b) {
      P = pages_of(p.seq_lens, p.max_pages, b);
      if (lo < c + (long long)p.Hkv * P) {
        kvh = (int)((lo - c) / P);
        pre = c + (long long)kvh * P;
        return;
      }
      c += (long long)p.Hkv * P;
    }
  }
  __device__ bool more() const { return x < hi; }
  // pages [pg_lo, pg_hi) of sequence b, K/V head kvh; then advances
  __device__ void take(int& sb, int& skvh, int& pg_lo, int& pg_hi, long long& spre, int& sP) {
    const long long end = pre + P < hi ? pre + P : hi;
    sb = b;
    skvh = kvh;
    spre = pre;
    sP = P;
    pg_lo = (int)(x - pre);
    pg_hi = (int)(end - pre);
    x = end;
    pre += P;
    if (++kvh == p.Hkv) {
      kvh = 0;
      do {
        ++b;
        P = b < p.B ? pages_of(p.seq_lens, p.max_pages, b) : 1;
      } while (b < p.B && P == 0);
    }
  }
};

// Byte offset of 16-byte chunk `c` (0..7) of row `r` in a 128-byte-swizzled
// TMA box (rows of 128 bytes, base 1024-aligned).
__device__ __forceinline__ uint32_t sw128(int r, int c) {
  return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
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

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const SplitParams p) {
  extern __shared__ uint8_t smem_raw[];
  // Total pages T of the batch and this CTA's share.
  long long T = 0;
  for (int b = 0; b < p.B; ++b) T += (long long)p.Hkv * pages_of(p.seq_lens, p.max_pages, b);
  long long G = T / kDecodeMinChunk;
  if (G > (long long)gridDim.x) G = gridDim.x;
  if (G < 1) G = 1;
  const int c = blockIdx.x;
  if (T == 0 || c >= G) return;
  const long long lo = c * T / G, hi = (c + 1) * T / G;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t s_q = base;                // 2 query slots of 8 KB
  const uint32_t s_ring = base + kRingOff;  // kStages x 8 KB
  DecSmem& sm = *reinterpret_cast<DecSmem*>(base_ptr + kRingOff + kStages * kStageBytes);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 2);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.qfull[s], 1);
      mbar_init(&sm.qempty[s], 2);
    }
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  const WaitGuard g{&sm.abort_flag, p.status, p.timeout_ns, true};
  const WaitGuard g_drain{&sm.abort_flag, p.status, p.timeout_ns, false};

  if (warp == 2) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    uint32_t n_st = 0, n_q = 0;
    bool ok = !p.stall;
    Segments seg(p, lo, hi);
    while (seg.more() && ok) {
      int b, kvh, pg_lo, pg_hi, P;
      long long pre;
      seg.take(b, kvh, pg_lo, pg_hi, pre, P);
      if (lane == 0) {  // query rows of this (sequence, K/V head)
        const uint32_t qs = n_q & 1;
        if (n_q >= 2) ok = mbar_wait(&sm.qempty[qs], ((n_q >> 1) - 1) & 1, g);
        if (ok) {
          mbar_arrive_expect_tx(&sm.qfull[qs], kQBytes);
          for (int h = 0; h < 2; ++h)
            tma_load_2d(s_q + qs * kQBytes + h * kQBox, &tm_q, &sm.qfull[qs], h * 64, b * p.Hq + kvh * p.group);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ++n_q;
      for (int k0 = pg_lo; k0 < pg_hi && ok; k0 += 32) {
        // 32 page ids at a time, one per lane
        int id = -1;
        if (k0 + lane < pg_hi) {
          id = p.block_table[(size_t)b * p.max_pages + k0 + lane];
          if (p.bounds_check && (id < 0 || id >= p.num_pages)) {
            atomicExch(p.status, kErrBounds);
            id = -1;
          }
        }
        const int kn = pg_hi - k0 < 32 ? pg_hi - k0 : 32;
        for (int k = 0; k < kn && ok; ++k) {
          const int pid = __shfl_sync(0xffffffffu, id, k);
          if (lane == 0) {
            const uint32_t st = n_st % kStages;
            if (n_st >= (uint32_t)kStages) ok = mbar_wait(&sm.empty[st], ((n_st / kStages) - 1) & 1, g);
            if (ok) {
              sm.valid[st] = pid >= 0;
              mbar_arrive_expect_tx(&sm.full[st], pid >= 0 ? kStageBytes : 0);
              if (pid >= 0) {
                const uint32_t dst = s_ring + st * kStageBytes;
                for (int h = 0; h < 2; ++h) {
                  tma_load_3d(dst + h * kHalfBox, &tm_k, &sm.full[st], h * 64, kvh, pid * kPage);
                  tma_load_3d(dst + kPageBytes + h * kHalfBox, &tm_v, &sm.full[st], h * 64, kvh, pid * kPage);
                }
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          ++n_st;
        }
      }
    }
    if (lane == 0) {
      // Drain: the last loads of every slot have landed before the CTA exits.
      for (uint32_t s = (n_st > (uint32_t)kStages ? n_st - kStages : 0); s < n_st; ++s)
        mbar_wait(&sm.full[s % kStages], (s / kStages) & 1, g_drain);
      for (uint32_t s = (n_q > 2u ? n_q - 2 : 0); s < n_q; ++s) mbar_wait(&sm.qfull[s & 1], (s >> 1) & 1, g_drain);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int mt = warp;  // query rows [16 mt, 16 mt + 16) of the group
  const int mi = lane >> 3, rr = lane & 7;
  const float sl2 = p.scale_log2;
  uint32_t n_st = 0, n_q = 0;
  bool ok = true;
  Segments seg(p, lo, hi);
  while (seg.more() && ok) {
    int b, kvh, pg_lo, pg_hi, P;
    long long pre;
    seg.take(b, kvh, pg_lo, pg_hi, pre, P);
    const int len = len_of(p.seq_lens, p.max_pages, b);
    const uint32_t qs = n_q & 1;
    ok = mbar_wait(&sm.qfull[qs], (n_q >> 1) & 1, g);
    if (!ok) break;
    ++n_q;
    uint32_t qa[kD / 16][4];
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk)
      ldsm_x4(s_q + qs * kQBytes + (kk >> 2) * kQBox + sw128(mt * 16 + (mi & 1) * 8 + rr, (kk & 3) * 2 + (mi >> 1)),
              qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.qempty[qs]);  // query fragments are in registers

    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};
    // per-lane partial row sums: exact fp32 (for the LSE) and of the rounded
    // P the tensor cores multiply (normalises o)
    float l_part[2] = {0.f, 0.f}, r_part[2] = {0.f, 0.f};

    for (int k = pg_lo; k < pg_hi; ++k) {
      const uint32_t st = n_st % kStages;
      ok = mbar_wait(&sm.full[st], (n_st / kStages) & 1, g);
      if (!ok) break;
      ++n_st;
      if (sm.valid[st]) {
        const uint32_t sk = s_ring + st * kStageBytes;
        const uint32_t sv = sk + kPageBytes;
        // S = q K^T for 16 query rows x 16 tokens; even and odd k-steps in
        // separate accumulators (two independent MMA chains)
        float s[2][4], s2[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) s[n][e] = s2[n][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(sk + (kk >> 2) * kHalfBox + sw128((mi >> 1) * 8 + rr, (kk & 3) * 2 + (mi & 1)), b0, b1, b2, b3);
          if (kk & 1) {
            mma_bf16(s2[0], qa[kk], b0, b1);
            mma_bf16(s2[1], qa[kk], b2, b3);
          } else {
            mma_bf16(s[0], qa[kk], b0, b1);
            mma_bf16(s[1], qa[kk], b2, b3);
          }
        }
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) s[n][e] += s2[n][e];
        // mask tokens past the end of the sequence
        const int base_tok = k * kPage + (lane & 3) * 2;
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tok = base_tok + n * 8 + (e & 1);
            s[n][e] = tok < len ? s[n][e] * sl2 : -INFINITY;
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
          r_part[0] += sum_bf16x2(pa[0]) + sum_bf16x2(pa[2]);
          r_part[1] += sum_bf16x2(pa[1]) + sum_bf16x2(pa[3]);
        }
        // O += P V over 16 tokens x 128 features
#pragma unroll
        for (int n = 0; n < 16; n += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sv + (n >> 3) * kHalfBox + sw128((mi & 1) * 8 + rr, (n & 7) + (mi >> 1)), b0, b1, b2, b3);
          mma_bf16(o[n], pa, b0, b1);
          mma_bf16(o[n + 1], pa, b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[st]);
    }
    if (!ok) break;
    // One partial per query row of this warp for this segment.
    const int sidx = c - owner(pre, T, (int)G);
    if (sidx < 0 || sidx >= p.max_segs) {  // cannot happen with chunks >= kDecodeMinChunk pages
      if (lane == 0) atomicExch(p.status, kErrBounds);
      continue;
    }
    const int r0 = lane >> 2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float l = l_part[h], lr = r_part[h];
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      lr += __shfl_xor_sync(0xffffffffu, lr, 1);
      lr += __shfl_xor_sync(0xffffffffu, lr, 2);
      const int row = mt * 16 + r0 + 8 * h;
      if (row < p.group) {
        const size_t rec = ((size_t)b * p.Hq + kvh * p.group + row) * p.max_segs + sidx;
        const float inv = lr > 0.f ? 1.f / lr : 0.f;
        float* dst = p.ws_o + rec * kD + (lane & 3) * 2;
#pragma unroll
        for (int n = 0; n < 16; ++n)
          *reinterpret_cast<float2*>(dst + n * 8) = make_float2(o[n][2 * h] * inv, o[n][2 * h + 1] * inv);
        if ((lane & 3) == 0) p.ws_lse[rec] = l > 0.f ? m_run[h] + __log2f(l) : -INFINITY;
      }
    }
    if (sidx == 0 && mt == 0 && lane == 0)
      p.ws_nseg[b * p.Hkv + kvh] = owner(pre + P - 1, T, (int)G) - owner(pre, T, (int)G) + 1;
  }
}

struct CombineParams {
  const float* ws_o;
  const float* ws_lse;
  const int* ws_nseg;
  const int* seq_lens;
  __nv_bfloat16* o;
  float* lse;
  int B, Hq, Hkv, group, max_pages, max_segs;
  int has_pool;  // 0: no page pool, every output is an empty attention
};

__global__ void __launch_bounds__(256) decode_combine_kernel(const CombineParams p) {
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= p.B * p.Hq) return;
  const int b = gw / p.Hq, h = gw % p.Hq;
  const int npg = p.has_pool ? pages_of(p.seq_lens, p.max_pages, b) : 0;
  int nseg = npg > 0 ? p.ws_nseg[b * p.Hkv + h / p.group] : 0;
  nseg = nseg < 0 ? 0 : (nseg > p.max_segs ? p.max_segs : nseg);
  const float* base_o = p.ws_o + (size_t)gw * p.max_segs * kD;
  const float* base_l = p.ws_lse + (size_t)gw * p.max_segs;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float M = -INFINITY, L = 0.f;
  // segments in groups of 32: lane s owns segment s of the group
  for (int s0 = 0; s0 < nseg; s0 += 32) {
    const int n = min(32, nseg - s0);
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

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// The pool [num_pages * 16 tokens, Hkv, D] bf16 as a 3-D tensor, box = one
// page of one K/V head, 64 features (128 bytes, 128-byte swizzle).
bool encode_pool(CUtensorMap* map, const void* pool, int num_pages, int Hkv) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)Hkv, (cuuint64_t)num_pages * kPage};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)Hkv * kD * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kPage};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pool), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// q [B * Hq rows, D] bf16, box = 32 rows x 64 features (128-byte swizzle).
bool encode_q(CUtensorMap* map, const void* q, int rows) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kQRows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (a.D != kD || a.page_size != kPage) return -2;
  const int group = a.Hq / a.Hkv;
  if (group > 32) return -2;
  const int max_pages = a.max_pages > 0 ? a.max_pages : 1;
  const int max_segs = decode_max_segments(max_pages);
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail_cuda("cudaGetDevice", err);
  if (dev < 64 && !attr_set[dev]) {
    err = cudaFuncSetAttribute(decode_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return fail_cuda("decode: cudaFuncSetAttribute", err);
    attr_set[dev] = true;
  }
  float* ws_o = static_cast<float*>(a.workspace);
  float* ws_lse = ws_o + (size_t)a.B * a.Hq * max_segs * kD;
  int* ws_nseg = reinterpret_cast<int*>(ws_lse + (size_t)a.B * a.Hq * max_segs);
  int* status = device_status_word();
  if (!status) return fail_cuda("decode: status word", cudaGetLastError());
  if (a.num_pages > 0 && a.max_pages > 0) {
    SplitParams sp{};
    sp.block_table = a.block_table;
    sp.seq_lens = a.seq_lens;
    sp.ws_o = ws_o;
    sp.ws_lse = ws_lse;
    sp.ws_nseg = ws_nseg;
    sp.B = a.B;
    sp.Hq = a.Hq;
    sp.Hkv = a.Hkv;
    sp.group = group;
    sp.num_pages = a.num_pages;
    sp.max_pages = a.max_pages;
    sp.max_segs = max_segs;
    sp.scale_log2 = a.scale * kLog2e;
    sp.bounds_check = (debug_flags() & 1) ? 1 : 0;
    sp.status = status;
    sp.timeout_ns = wait_timeout_ns();
    sp.stall = (debug_flags() & 2) ? 1 : 0;
    CUtensorMap tq, tk, tv;
    if (!encode_q(&tq, a.q, a.B * a.Hq) || !encode_pool(&tk, a.k_pages, a.num_pages, a.Hkv) ||
        !encode_pool(&tv, a.v_pages, a.num_pages, a.Hkv))
      return fail_cuda("decode: tensor map", cudaErrorInvalidValue);
    decode_split_kernel<<<kCtasPerSm * sm_count(), kThreads, kSmemBytes, stream>>>(tq, tk, tv, sp);
    err = cudaGetLastError();
    if (err != cudaSuccess) return fail_cuda("decode: split launch", err);
  }
  CombineParams cp{};
  cp.ws_o = ws_o;
  cp.ws_lse = ws_lse;
  cp.ws_nseg = ws_nseg;
  cp.seq_lens = a.seq_lens;
  cp.o = static_cast<__nv_bfloat16*>(a.o);
  cp.lse = a.lse;
  cp.B = a.B;
  cp.Hq = a.Hq;
  cp.Hkv = a.Hkv;
  cp.group = group;
  cp.max_pages = max_pages;
  cp.max_segs = max_segs;
  // Without a pool the split kernel did not run and wrote no segment counts:
  // the combine then treats every sequence as empty (O = 0, LSE = -inf).
  cp.has_pool = (a.num_pages > 0 && a.max_pages > 0) ? 1 : 0;
  const int nw = a.B * a.Hq;
  decode_combine_kernel<<<(nw + 7) / 8, 256, 0, stream>>>(cp);
  err = cudaGetLastError();
  return err == cudaSuccess ? 0 : fail_cuda("decode: combine launch", err);
}

}  // namespace attn
