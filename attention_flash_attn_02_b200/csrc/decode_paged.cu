// decode_paged.cu -- single-token attention against a paged KV cache
// (PagedAttention section of the page "LLM 中的 Attention 实现及优化",
// zeeklog.com: K/V kept in fixed-size pages of a shared pool, found through a
// per-sequence block table), for B200 (sm_100a).
//
// Two launches:
//   decode_split_kernel   2 CTAs per SM.  All cached pages of the batch,
//       sequence after sequence (and K/V head after K/V head), form one list
//       of T pages; CTA c streams the contiguous share [c T / G, (c+1) T / G)
//       of it (at least kDecodeMinChunk pages), so every CTA moves the same
//       number of bytes whatever the length mix.  Per CTA:
//         warp 4       TMA producer: the query rows of each (sequence, K/V
//                      head) segment it meets, and blocks of pages (K and V,
//                      128-byte swizzled) gathered straight from the pool into
//                      a ring; page ids come from the block table.
//         warp 5       allocates TMEM; one thread issues the tensor-core work
//                      of each block: S = Q K^T (tcgen05, M = 128 query rows
//                      of which the K/V group's heads are the first `group`,
//                      N = 16 per loaded page) into one of two TMEM S
//                      buffers, then O += P V (P read back from TMEM over S).
//         warps 0..3   softmax, one thread per query head (TMEM lane): online
//                      softmax over each block's scores, P written back to
//                      TMEM as bf16; at the end of a segment the normalised
//                      partial o and its log2-sum-exp go to the workspace.
//                      Only ceil(group / 32) of them have rows.
//   decode_combine_kernel one warp per (sequence, query head) merges the
//       partials: M = max_s lse_s, O = sum_s 2^(lse_s - M) o_s / sum_s
//       2^(lse_s - M), LSE = (M + log2 sum) ln 2 -- the rescaling step of the
//       online softmax (page "003-注意力机制详解...", §二) taken once across
//       segments.  It is launched as a programmatic dependent of the split
//       kernel and finds each pair's segments from seq_lens itself, so after
//       the split kernel ends it needs one round of loads.
// All query heads of a K/V group share every gathered page (MQA/GQA: the
// tqpw.cn article §2.1/§3.1): one MMA serves the whole group.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <cstdint>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace attn {
namespace {

constexpr int kPage = 16;
// Blocks of 4 pages (64 tokens) in a ring of up to 3 stages.  (Measured on
// B200 at D = 128 against 2-page blocks with two CTAs per SM and 8-page blocks
// with one: 4 pages was fastest.)  Features go in boxes of 64 (128 bytes,
// one row of the 128-byte swizzle): D_qk / 64 boxes of K and D_v / 64 of V.
constexpr int kBlkPages = 4;                    // pages per block
constexpr int kBlkTok = kBlkPages * kPage;      // 64 tokens per block
constexpr int kBox = kBlkTok * 128;             // a block's 64-feature box (bf16): 8 KB
constexpr int kPageBox = kPage * 128;           // one page's 64-feature box: 2 KB
constexpr int kMaxStages = 3;                   // ring stages (fewer when the query tile is large)
constexpr int kThreads = 192;                   // warps 0-3 softmax, 4 producer, 5 MMA
constexpr int kMaxGroup = 128;                  // query rows per K/V head tile: group * q_len
constexpr uint32_t kTmS0 = 0, kTmS1 = kBlkTok, kTmO = 2 * kBlkTok;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// The split kernel sees only rows of >= kShortKeys keys (shorter ones are the
// combine kernel's), where normalising o by the exact fp32 row sum is off by
// ~2^-9 / sqrt(n) of the weights' rounding: the sum of the rounded P, which
// costs three instructions per key pair, is kept only with ATTN_DEC_RSUM=1.
#ifndef ATTN_DEC_RSUM
#define ATTN_DEC_RSUM 0
#endif
constexpr int kSmemPerSm = 233472;  // shared memory of an SM, 1 KB of it reserved per CTA
// Sequences whose first query token sees fewer than kShortKeys cached tokens
// ("short") take no part in the split kernel's page partition: the combine
// kernel computes their rows directly in fp32 (exact softmax weights).  On a
// row of a few keys the tensor-core path's bf16 rounding of P alone moves O
// by up to ~2^-9 of the spread of its V values, which with the bf16 rounding
// of O can pass 1e-2; handling those rows elsewhere keeps the split kernel's
// hot loop free of any extra code (residual-product code there cost 0.5-4 us
// per call even when no segment used it).
constexpr int kShortKeys = 256;
__device__ __forceinline__ bool is_short(int len, int q_len) { return len - q_len + 1 < kShortKeys; }

// Per-width constants: query/key width DQK, value width DV (64..256).
template <int DQK, int DV>
struct DecCfg {
  static constexpr int KB = DQK / 64, VB = DV / 64;         // feature boxes of K and V
  static constexpr int STAGE = (KB + VB) * kBox;            // K boxes, then V boxes
  // TMEM: two S buffers of 64 columns and O of DV columns; 256 columns let
  // two CTAs share an SM, wider O takes all 512 (one CTA per SM).
  static constexpr uint32_t TMEM_COLS = kTmO + DV <= 256 ? 256u : 512u;
  static constexpr int TMEM_CTAS = 512 / (int)TMEM_COLS;    // CTAs an SM's TMEM holds
  static constexpr uint32_t IDESC_PV = make_idesc(1u, 128, DV, true);
  static_assert(DQK % 64 == 0 && DV % 64 == 0 && DQK <= 256 && DV <= 256, "widths 64..256 in steps of 64");
  static_assert(kTmO + DV <= TMEM_COLS, "TMEM budget");
};

struct SplitParams {
  const int* block_table;
  const int* seq_lens;
  float* ws_o;    // [B * Hq][S][D_v] normalised partial outputs
  float* ws_lse;  // [B * Hq][S] log2-sum-exp of each partial
  int B, Hq, Hkv, group, num_pages, max_pages, max_segs;
  int q_len;       // query tokens per sequence: the last q_len cached ones
  int rows;        // query rows per (sequence, K/V head): group * q_len
  int q_box;       // bytes of one 64-feature box of a query tile
  int q_slots;     // query tiles in flight (1 or 2)
  int stages;      // K/V ring stages (2 or 3)
  int sm_warps;    // softmax warps with rows: ceil(rows / 32)
  float scale_log2;
  int bounds_check;
  int* status;
  unsigned long long timeout_ns;
  int stall;  // testing hook: the producer issues no loads, every wait runs out
};

struct DecSmem {
  uint64_t kv_full[kMaxStages], kv_empty[kMaxStages];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done, o_full, o_empty, drain;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr int kBarBytes = 256;
static_assert(sizeof(DecSmem) <= kBarBytes, "barrier block exceeds its reserve");
// Shared memory: [query slot 0][query slot 1][ring][barriers], the base
// 1024-byte aligned.  Query slots (one or two, each DQK / 64 boxes) and ring
// stages are chosen per call (host side) so that as many CTAs share an SM as
// its TMEM holds (two at D_v <= 128): the deepest ring first, then the second
// query slot (it only hides the query load at a segment switch); where even
// the smallest layout does not fit twice, one CTA per SM.  A launch never
// asks for so little shared memory that more CTAs than the TMEM holds could
// share an SM (their allocation would wait).
template <int DQK, int DV>
__host__ __device__ constexpr int dec_smem_bytes(int q_box, int q_slots, int stages) {
  return q_slots * DecCfg<DQK, DV>::KB * q_box + stages * DecCfg<DQK, DV>::STAGE + kBarBytes;
}
constexpr bool fits(int bytes, int ctas) { return ctas * (bytes + 1024) <= kSmemPerSm; }
static_assert(fits(dec_smem_bytes<128, 128>(32 * 128, 2, kMaxStages), 2), "the MQA tile keeps the full layout");
static_assert(fits(dec_smem_bytes<128, 128>(kMaxGroup * 128, 1, 2), 2), "the largest tile still fits twice per SM");
static_assert(fits(dec_smem_bytes<256, 256>(kMaxGroup * 128, 1, 2), 1), "the widest tile fits once per SM");

// K/V pages are read once per call, so their TMA loads carry an L2
// evict-first policy: they then do not push out the small data that is read
// again (sequence lengths, the block table, the partials the combine reads).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void tma_load_3d_evict_first(uint32_t smem_dst, const CUtensorMap* map, uint64_t* bar,
                                                        int c0, int c1, int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}

__device__ __forceinline__ int len_of(const int* seq_lens, int max_pages, int b) {
  const int n = seq_lens[b], cap = max_pages * kPage;
  return n < 0 ? 0 : (n > cap ? cap : n);
}
// Pages of sequence b in the split kernel's partition (0 for a short one).
__device__ __forceinline__ int pages_of(const int* seq_lens, int max_pages, int q_len, int b) {
  const int n = len_of(seq_lens, max_pages, b);
  return is_short(n, q_len) ? 0 : (n + kPage - 1) / kPage;
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
  // Called by all 32 lanes of a warp: finds the sequence holding list page
  // `lo` with a warp-wide inclusive scan of the sequences' page counts, 32
  // sequences per step (lo < T, so some sequence holds it).
  __device__ Segments(const SplitParams& p_, long long lo, long long hi_, int lane)
      : p(p_), hi(hi_), x(lo), pre(0), b(0), kvh(0), P(0) {
    long long c = 0;
    for (int b0 = 0; b0 < p.B; b0 += 32) {
      const int bl = b0 + lane;
      const long long w = bl < p.B ? (long long)p.Hkv * pages_of(p.seq_lens, p.max_pages, p.q_len, bl) : 0;
      long long inc = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, c + inc > lo);
      if (hit) {
        const int L = __ffs(hit) - 1;  // first sequence whose pages reach past lo
        const long long excl = c + __shfl_sync(0xffffffffu, inc - w, L);
        b = b0 + L;
        P = pages_of(p.seq_lens, p.max_pages, p.q_len, b);
        kvh = (int)((lo - excl) / P);
        pre = excl + (long long)kvh * P;
        return;
      }
      c += __shfl_sync(0xffffffffu, inc, 31);
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
        P = b < p.B ? pages_of(p.seq_lens, p.max_pages, p.q_len, b) : 1;
      } while (b < p.B && P == 0);
    }
  }
};

// Number of CTAs of the split grid that own pages, for T pages in all.
__device__ __forceinline__ long long split_ctas(long long T, int grid) {
  long long G = T / kDecodeMinChunk;
  if (G > (long long)grid) G = grid;
  return G < 1 ? 1 : G;
}

struct CombineParams {
  const float* ws_o;
  const float* ws_lse;
  const int* seq_lens;
  __nv_bfloat16* o;
  float* lse;
  int B, Hq, Hkv, group, max_pages, max_segs;
  int q_len;       // query tokens per sequence
  int split_grid;  // CTAs launched for the split kernel
  int has_pool;    // 0: no page pool, every output is an empty attention
  // rows of short sequences, computed here: queries, pools, table
  const __nv_bfloat16* q;        // [B * Hq * q_len][D_qk]
  const __nv_bfloat16* k_pages;  // [num_pages * 16][Hkv][D_qk]
  const __nv_bfloat16* v_pages;  // [num_pages * 16][Hkv][D_v]
  const int* block_table;
  int num_pages;
  float scale_log2;
  int bounds_check;
  int* status;
};

// One warp per (sequence, query head).  Before waiting for the split kernel
// it works out, from seq_lens alone, which CTAs hold that pair's segments
// (the same partition the split kernel used); after the wait, lane s reads
// segment s's log2-sum-exp while every lane reads its 4 features of up to 8
// partials at once.
// F consecutive fp32 features from global memory (L2, bypassing L1), in
// 16-byte loads where F allows, else 8-byte ones.
template <int F>
__device__ __forceinline__ void ld_feats(const float* src, float (&v)[F]) {
  if constexpr (F % 4 == 0) {
#pragma unroll
    for (int i = 0; i < F / 4; ++i) {
      const float4 t = __ldcg(reinterpret_cast<const float4*>(src) + i);
      v[4 * i] = t.x;
      v[4 * i + 1] = t.y;
      v[4 * i + 2] = t.z;
      v[4 * i + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < F / 2; ++i) {
      const float2 t = __ldcg(reinterpret_cast<const float2*>(src) + i);
      v[2 * i] = t.x;
      v[2 * i + 1] = t.y;
    }
  }
}
// F bf16 features (F / 2 packed pairs) to global memory.
template <int F>
__device__ __forceinline__ void st_feats(__nv_bfloat16* dst, const uint32_t (&pk)[F / 2]) {
  if constexpr (F == 8) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  } else if constexpr (F == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
  } else {
#pragma unroll
    for (int i = 0; i < F / 2; ++i) reinterpret_cast<uint32_t*>(dst)[i] = pk[i];
  }
}

// Page id of token j of sequence b, or -1 if it lies outside the pool (such
// a page reads as zeros, as the TMA copies of the split kernel read it).
__device__ __forceinline__ int short_page(const CombineParams& p, int b, int j) {
  const int pg = p.block_table[(size_t)b * p.max_pages + j / kPage];
  if (pg < 0 || pg >= p.num_pages) {
    if (p.bounds_check) atomicExch(p.status, kErrBounds);
    return -1;
  }
  return pg;
}

// Row (b, h, token t) of a short sequence, by one warp in fp32, in one pass
// over the visible cached tokens: lane l holds query features l*FQ ..
// l*FQ+FQ-1 and value features l*FV .., each token's score is reduced across
// the warp, and the online-softmax recurrence (running max, rescaled sum and
// accumulator) runs on warp-uniform values.  Kept compact and out of line:
// it serves rare rows, and its code in the kernel should cost nothing else.
template <int DQK, int DV>
__device__ __noinline__ void short_row(const CombineParams& p, int gw, int b, int h, int t, int lane) {
  constexpr int FQ = DQK / 32, FV = DV / 32;
  const int len = len_of(p.seq_lens, p.max_pages, b);
  int vis = p.has_pool ? len - p.q_len + t + 1 : 0;  // tokens 0 .. vis - 1
  vis = vis < 0 ? 0 : (vis > len ? len : vis);
  const int kvh = h / p.group;
  float qv[FQ];
#pragma unroll
  for (int f = 0; f < FQ; f += 2) {
    const uint32_t w = *reinterpret_cast<const unsigned int*>(p.q + (size_t)gw * DQK + lane * FQ + f);
    qv[f] = __uint_as_float(w << 16) * p.scale_log2;
    qv[f + 1] = __uint_as_float(w & 0xFFFF0000u) * p.scale_log2;
  }
  float m = -INFINITY, l = 0.f, acc[FV];
#pragma unroll
  for (int f = 0; f < FV; ++f) acc[f] = 0.f;
#pragma unroll 1
  for (int j = 0; j < vis; ++j) {
    const int pg = short_page(p, b, j);  // the same for every lane
    const size_t tok = ((size_t)(pg < 0 ? 0 : pg) * kPage + j % kPage) * p.Hkv + kvh;
    float s = 0.f;
    if (pg >= 0) {
#pragma unroll
      for (int f = 0; f < FQ; f += 2) {
        const uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(p.k_pages + tok * DQK + lane * FQ + f));
        s = fmaf(__uint_as_float(w << 16), qv[f], s);
        s = fmaf(__uint_as_float(w & 0xFFFF0000u), qv[f + 1], s);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float m_new = fmaxf(m, s);
    const float c = ex2_approx(m - m_new);  // 0 for the first token
    const float e = ex2_approx(s - m_new);
    m = m_new;
    l = l * c + e;
#pragma unroll
    for (int f = 0; f < FV; f += 2) {
      float v0 = 0.f, v1 = 0.f;
      if (pg >= 0) {
        const uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(p.v_pages + tok * DV + lane * FV + f));
        v0 = __uint_as_float(w << 16);
        v1 = __uint_as_float(w & 0xFFFF0000u);
      }
      acc[f] = fmaf(e, v0, acc[f] * c);
      acc[f + 1] = fmaf(e, v1, acc[f + 1] * c);
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  uint32_t pk[FV / 2];
#pragma unroll
  for (int f = 0; f < FV / 2; ++f) pk[f] = pack_bf16x2(acc[2 * f] * inv, acc[2 * f + 1] * inv);
  st_feats<FV>(p.o + (size_t)gw * DV + lane * FV, pk);
  if (lane == 0 && p.lse) p.lse[gw] = (l > 0.f) ? (m + __log2f(l)) * kLn2 : -INFINITY;
}

template <int DQK, int DV>
__global__ void __launch_bounds__(256) decode_combine_kernel(const CombineParams p) {
  // The next decode's split kernel (a programmatic dependent) may launch and
  // set up while this grid runs; it waits for this grid before reading or
  // writing global memory.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);  // output row: (b, h, token)
  const int lane = threadIdx.x & 31;
  if (gw >= p.B * p.Hq * p.q_len) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    return;
  }
  const int b = gw / (p.Hq * p.q_len), h = (gw / p.q_len) % p.Hq, kvh = h / p.group;
  if (is_short(len_of(p.seq_lens, p.max_pages, b), p.q_len)) {
    // Reads only the call's inputs, which the kernels before this call's
    // split kernel had completed (that kernel waited for them before letting
    // this grid launch): no wait needed before the row is computed.
    short_row<DQK, DV>(p, gw, b, h, gw % p.q_len, lane);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    return;
  }
  int nseg = 0;
  if (p.has_pool) {
    // pages of sequences before b, and in all (seq_lens is an input of the
    // split kernel, complete before it started)
    long long before = 0, T = 0;
    for (int bb = lane; bb < p.B; bb += 32) {
      const long long w = pages_of(p.seq_lens, p.max_pages, p.q_len, bb);
      T += w;
      if (bb < b) before += w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      T += __shfl_xor_sync(0xffffffffu, T, o);
      before += __shfl_xor_sync(0xffffffffu, before, o);
    }
    T *= p.Hkv;
    const int P = pages_of(p.seq_lens, p.max_pages, p.q_len, b);
    if (P > 0 && T > 0) {
      const long long G = split_ctas(T, p.split_grid);
      const long long pre = before * p.Hkv + (long long)kvh * P;
      nseg = owner(pre + P - 1, T, (int)G) - owner(pre, T, (int)G) + 1;
      nseg = nseg > p.max_segs ? p.max_segs : nseg;
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the split kernel's partials are complete
  constexpr int F = DV / 32;  // features per lane
  const float* base_o = p.ws_o + (size_t)gw * p.max_segs * DV + lane * F;
  const float* base_l = p.ws_lse + (size_t)gw * p.max_segs;
  float acc[F];
#pragma unroll
  for (int f = 0; f < F; ++f) acc[f] = 0.f;
  float M = -INFINITY, L = 0.f;
  for (int s0 = 0; s0 < nseg; s0 += 32) {
    const int n = nseg - s0 < 32 ? nseg - s0 : 32;
    const float l2 = lane < n ? __ldcg(base_l + s0 + lane) : -INFINITY;
    float v[8][F];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (u < n) {
        ld_feats<F>(base_o + (size_t)(s0 + u) * DV, v[u]);
      } else {
#pragma unroll
        for (int f = 0; f < F; ++f) v[u][f] = 0.f;
      }
    }
    float gm = l2;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
    const float Mn = fmaxf(M, gm);
    if (Mn == -INFINITY) continue;
    const float scale_old = (M == -INFINITY) ? 0.f : ex2_approx(M - Mn);
#pragma unroll
    for (int f = 0; f < F; ++f) acc[f] *= scale_old;
    L *= scale_old;
    M = Mn;
    const float w = (l2 == -INFINITY) ? 0.f : ex2_approx(l2 - M);
    float ws = w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, o);
    L += ws;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float wv = __shfl_sync(0xffffffffu, w, u);
      if (u < n) {
#pragma unroll
        for (int f = 0; f < F; ++f) acc[f] += wv * v[u][f];
      }
    }
    for (int u = 8; u < n; ++u) {  // more than 8 segments in this group of 32
      float vv[F];
      ld_feats<F>(base_o + (size_t)(s0 + u) * DV, vv);
      const float wv = __shfl_sync(0xffffffffu, w, u);
#pragma unroll
      for (int f = 0; f < F; ++f) acc[f] += wv * vv[f];
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint32_t pk[F / 2];
#pragma unroll
  for (int f = 0; f < F / 2; ++f) pk[f] = pack_bf16x2(acc[2 * f] * inv, acc[2 * f + 1] * inv);
  st_feats<F>(p.o + (size_t)gw * DV + lane * F, pk);
  if (lane == 0 && p.lse) p.lse[gw] = (L > 0.f) ? (M + __log2f(L)) * kLn2 : -INFINITY;
}

template <int DQK, int DV>
__global__ void __launch_bounds__(kThreads, 2)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const SplitParams p) {
  using C = DecCfg<DQK, DV>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = smem_u32(smem_raw);
  // This grid is launched as a programmatic dependent of the kernel before it
  // in the stream, so that its launch, the set-up below (barriers, TMEM) and
  // the work partition overlap that kernel's tail.  The partition reads only
  // seq_lens and the block table, which that kernel does not write (the
  // contract in attn.h); everything else global -- pages, queries, the
  // workspace -- is touched only after griddepcontrol.wait.
  if (base & 1023u) {  // the layout below needs a 1024-byte aligned base
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (tid == 0) atomicExch(p.status, kErrBounds);
    return;
  }
  const uint32_t q_slot = (uint32_t)C::KB * p.q_box;
  const uint32_t nqs = (uint32_t)p.q_slots, nst = (uint32_t)p.stages;
  const uint32_t s_q = base;                       // query slots
  const uint32_t s_ring = base + nqs * q_slot;     // stages of C::STAGE bytes
  DecSmem& sm = *reinterpret_cast<DecSmem*>(smem_raw + nqs * q_slot + nst * C::STAGE);
  if (tid == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.q_empty[s], 1);
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], p.sm_warps);
    }
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.o_empty, p.sm_warps);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  const int sl0 = lane < p.B ? p.seq_lens[lane] : 0;
  const int sl1 = lane + 32 < p.B ? p.seq_lens[lane + 32] : 0;
  // Total pages T of the batch and this CTA's share.  Every warp sums the
  // page counts itself, lane l taking sequences l, l + 32, ... (independent
  // loads, then a shuffle reduction), so no warp waits for another.
  auto pages_from_len = [&](int n) {
    const int cap = p.max_pages * kPage;
    n = n < 0 ? 0 : (n > cap ? cap : n);
    return is_short(n, p.q_len) ? 0 : (n + kPage - 1) / kPage;
  };
  long long T = (long long)pages_from_len(sl0) + pages_from_len(sl1);
  for (int b = lane + 64; b < p.B; b += 32) T += pages_of(p.seq_lens, p.max_pages, p.q_len, b);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) T += __shfl_xor_sync(0xffffffffu, T, o);
  T *= p.Hkv;
  const long long G = split_ctas(T, gridDim.x);
  const int c = blockIdx.x;
  const bool idle = T == 0 || c >= G;
  const long long lo = idle ? 0 : c * T / G, hi = idle ? 0 : (c + 1) * T / G;
  if (warp == 4 && !idle) {
    // Request the first page ids of this CTA's share now, into L1 (the
    // producer reads them after the barrier below).
    const Segments s0(p, lo, hi, lane);
    const int pg = (int)(lo - s0.pre) + lane;
    if (pg < s0.P)
      asm volatile("prefetch.global.L1 [%0];" ::"l"(p.block_table + (size_t)s0.b * p.max_pages + pg));
  }
  // The kernel before this one has completed and its writes are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // The combine launch may start now: it waits for this grid's completion
  // (griddepcontrol.wait) before it reads any partial.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (idle) {  // no pages for this CTA
    if (warp == 5) tmem_dealloc(sm.tmem_base, C::TMEM_COLS);
    return;
  }
  const uint32_t tmem = sm.tmem_base;
  const WaitGuard g{&sm.abort_flag, p.status, p.timeout_ns, true};
  const WaitGuard g_drain{&sm.abort_flag, p.status, p.timeout_ns, false};
  // Teardown at the end of every role: all threads meet, then the owner warp
  // releases TMEM.
  auto finish = [&]() {
    tc_fence_before();
    asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
    if (warp == 5) {
      tc_fence_after();
      tmem_dealloc(tmem, C::TMEM_COLS);
    }
  };

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    uint32_t n_blk = 0, n_q = 0;
    bool ok = !p.stall;
    const uint64_t pol = l2_evict_first_policy();
    Segments seg(p, lo, hi, lane);
    while (seg.more() && ok) {
      int b, kvh, pg_lo, pg_hi, P;
      long long pre;
      seg.take(b, kvh, pg_lo, pg_hi, pre, P);
      if (lane == 0) {  // the K/V group's query rows
        const uint32_t qs = n_q % nqs;
        if (n_q >= nqs) ok = mbar_wait(&sm.q_empty[qs], ((n_q / nqs) - 1) & 1, g);
        if (ok) {
          mbar_arrive_expect_tx(&sm.q_full[qs], (uint32_t)C::KB * p.rows * 128u);
          for (int h = 0; h < C::KB; ++h)
            tma_load_2d(s_q + qs * q_slot + h * p.q_box, &tm_q, &sm.q_full[qs], h * 64,
                        (b * p.Hq + kvh * p.group) * p.q_len);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ++n_q;
      for (int k0 = pg_lo; k0 < pg_hi && ok; k0 += 32) {
        // 32 page ids at a time, one per lane (32 is a whole number of blocks)
        int id = 0;
        if (k0 + lane < pg_hi) {
          id = p.block_table[(size_t)b * p.max_pages + k0 + lane];
          if (p.bounds_check && (id < 0 || id >= p.num_pages)) {
            atomicExch(p.status, kErrBounds);
            id = p.num_pages;  // past the pool: the copy reads zeros
          }
        }
        const int kn = pg_hi - k0 < 32 ? pg_hi - k0 : 32;
        for (int kb = 0; kb < kn && ok; kb += kBlkPages) {
          const int nv = kn - kb < kBlkPages ? kn - kb : kBlkPages;
          int pid[kBlkPages];
#pragma unroll
          for (int i = 0; i < kBlkPages; ++i) pid[i] = __shfl_sync(0xffffffffu, id, (kb + i) & 31);
          if (lane == 0) {
            const uint32_t st = n_blk % nst;
            if (n_blk >= nst) ok = mbar_wait(&sm.kv_empty[st], ((n_blk / nst) - 1) & 1, g);
            if (ok) {
              mbar_arrive_expect_tx(&sm.kv_full[st], (uint32_t)nv * (C::KB + C::VB) * kPageBox);
              const uint32_t dst = s_ring + st * C::STAGE;
              for (int i = 0; i < nv; ++i) {
                const int tok = pid[i] * kPage;
                const uint32_t d = dst + i * kPageBox;
#pragma unroll
                for (int h = 0; h < C::KB; ++h)
                  tma_load_3d_evict_first(d + h * kBox, &tm_k, &sm.kv_full[st], h * 64, kvh, tok, pol);
#pragma unroll
                for (int h = 0; h < C::VB; ++h)
                  tma_load_3d_evict_first(d + (C::KB + h) * kBox, &tm_v, &sm.kv_full[st], h * 64, kvh, tok, pol);
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          ++n_blk;
        }
      }
    }
    if (lane == 0) {
      // Drain: the last loads of every slot have landed before the CTA exits.
      for (uint32_t s = (n_blk > nst ? n_blk - nst : 0); s < n_blk; ++s)
        mbar_wait(&sm.kv_full[s % nst], (s / nst) & 1, g_drain);
      for (uint32_t s = (n_q > nqs ? n_q - nqs : 0); s < n_q; ++s)
        mbar_wait(&sm.q_full[s % nqs], (s / nqs) & 1, g_drain);
    }
    finish();
  } else if (warp == 5) {
    // ----------------------------------------------------------- MMA issue
    Segments seg(p, lo, hi, lane);  // built by the whole warp (shuffles)
    if (lane == 0) {
      uint32_t n_blk = 0, n_q = 0, n_seg = 0;
      bool ok = true;
      auto tS = [&](uint32_t gb) { return tmem + ((gb & 1) ? kTmS1 : kTmS0); };
      // S = Q K^T for block gb (nv pages): both operands K-major; k-step kk
      // starts 32 bytes further into the 128-byte rows, every 64 features one
      // box further on.
      auto issue_s = [&](uint32_t gb, uint32_t q_addr, int nv) {
        const uint32_t stage = s_ring + (gb % nst) * C::STAGE;
        const uint64_t a0 = sw128_desc(q_addr, 16, 1024);
        const uint64_t b0 = sw128_desc(stage, 16, 1024);
        const uint32_t idesc = make_idesc(1u, 128, nv * kPage, false);
#pragma unroll
        for (int kk = 0; kk < DQK / 16; ++kk) {
          const uint32_t bk = kk * 32;
          const uint32_t offa = ((bk / 128) * p.q_box + (bk % 128)) >> 4;
          const uint32_t offb = ((bk / 128) * kBox + (bk % 128)) >> 4;
          mma_f16_ss(tS(gb), a0 + offa, b0 + offb, idesc, kk > 0);
        }
      };
      // O (+)= P V: P from TMEM over S (16 tokens = 8 columns per k-step), V
      // MN-major with its 64-feature boxes kBox apart.
      auto issue_pv = [&](uint32_t gb, int nv, bool acc) {
        const uint32_t stage = s_ring + (gb % nst) * C::STAGE;
        const uint64_t b0 = sw128_desc(stage + C::KB * kBox, kBox, 1024);
        for (int kk = 0; kk < nv; ++kk)
          mma_f16_ts(tmem + kTmO, tS(gb) + kk * 8, b0 + ((kk * kPageBox) >> 4), C::IDESC_PV,
                     (acc || kk > 0) ? 1u : 0u);
      };
      while (seg.more() && ok) {
        int b, kvh, pg_lo, pg_hi, P;
        long long pre;
        seg.take(b, kvh, pg_lo, pg_hi, pre, P);
        const int nb = (pg_hi - pg_lo + kBlkPages - 1) / kBlkPages;
        const uint32_t qs = n_q % nqs;
        ok = mbar_wait(&sm.q_full[qs], (n_q / nqs) & 1, g);
        if (!ok) break;
        ++n_q;
        const uint32_t q_addr = s_q + qs * q_slot;
        // S of block jj of the segment; the segment's last S is the last
        // reader of its query slot, which is then released.
        auto s_block = [&](int jj) {
          const uint32_t x = n_blk + jj;
          tc_fence_after();
          issue_s(x, q_addr, min(kBlkPages, pg_hi - (pg_lo + jj * kBlkPages)));
          tc_commit(&sm.s_full[x & 1]);
          if (jj == nb - 1) tc_commit(&sm.q_empty[qs]);
        };
        for (int j = 0; j < nb && ok; ++j) {
          const uint32_t gb = n_blk + j;
          if (j == 0) {
            ok = mbar_wait(&sm.kv_full[gb % nst], (gb / nst) & 1, g);
            if (!ok) break;
            s_block(0);
          }
          // The next block's scores go first, so that they are ready when this
          // block's softmax ends, but only if its K/V has already landed:
          // waiting for it here would hold back this block's P V and with it
          // the release of its stage, leaving the producer one load in flight.
          const bool has_next = j + 1 < nb;
          const uint32_t gn = gb + 1;
          const bool s_first = has_next && mbar_test(&sm.kv_full[gn % nst], (gn / nst) & 1);
          if (s_first) s_block(j + 1);
          ok = mbar_wait(&sm.p_full[gb & 1], (gb >> 1) & 1, g);
          if (!ok) break;
          if (j == 0 && n_seg > 0) {
            ok = mbar_wait(&sm.o_empty, (n_seg - 1) & 1, g);
            if (!ok) break;
          }
          tc_fence_after();
          issue_pv(gb, min(kBlkPages, pg_hi - (pg_lo + j * kBlkPages)), j > 0);
          tc_commit(&sm.kv_empty[gb % nst]);
          tc_commit(&sm.pv_done);
          if (has_next && !s_first) {
            ok = mbar_wait(&sm.kv_full[gn % nst], (gn / nst) & 1, g);
            if (!ok) break;
            s_block(j + 1);
          }
        }
        if (!ok) break;
        tc_commit(&sm.o_full);
        n_blk += nb;
        ++n_seg;
      }
      // Drain: all issued MMAs complete before TMEM is released.
      tc_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, g_drain);
    }
    __syncwarp();
    finish();
  } else if (warp < p.sm_warps) {
    // ------------------------------------------------------------ softmax
    // Row of the group's query tile = TMEM lane: query head r / q_len of the
    // K/V group, new token r % q_len, which sees the cached tokens up to and
    // including its own position len - q_len + r % q_len.
    const int r = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    uint32_t n_blk = 0, n_seg = 0;
    bool ok = true;
    Segments seg(p, lo, hi, lane);
    while (seg.more() && ok) {
      int b, kvh, pg_lo, pg_hi, P;
      long long pre;
      seg.take(b, kvh, pg_lo, pg_hi, pre, P);
      const int len = len_of(p.seq_lens, p.max_pages, b);
      const int nb = (pg_hi - pg_lo + kBlkPages - 1) / kBlkPages;
      // l_run: exact fp32 row sum (gives the LSE); l_rnd: sum of the rounded P
      // the MMA multiplies (normalises o so its weights sum to one).
      float m_run = -INFINITY, l_run = 0.f, l_rnd = 0.f;
      for (int j = 0; j < nb; ++j) {
        const uint32_t gb = n_blk + j;
        const uint32_t tS = tmem + ((gb & 1) ? kTmS1 : kTmS0) + lane_off;
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full[gb & 1], (gb >> 1) & 1, g));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[kBlkTok];
        tmem_ld64(tS, sr);
        const int pg0 = pg_lo + j * kBlkPages;
        const int nv = pg_hi - pg0 < kBlkPages ? pg_hi - pg0 : kBlkPages;
        const int tok0 = pg0 * kPage;
        const int valid = min(nv * kPage, len - tok0);  // tokens of this block that exist
        const int seen = min(valid, len - p.q_len + r % p.q_len + 1 - tok0);  // ... and this row sees
        if (seen < kBlkTok) {
#pragma unroll
          for (int i = 0; i < kBlkTok; ++i)
            if (i >= seen) sr[i] = 0xFF800000u;  // -inf
        }
        float pm[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pm[i] = fmaxf(__uint_as_float(sr[i]), __uint_as_float(sr[8 + i]));
#pragma unroll
        for (int i0 = 16; i0 < kBlkTok; i0 += 16)
#pragma unroll
          for (int i = 0; i < 8; ++i) pm[i] = max3(pm[i], __uint_as_float(sr[i0 + i]), __uint_as_float(sr[i0 + 8 + i]));
        const float mx = fmaxf(max3(pm[0], pm[1], pm[2]), max3(max3(pm[3], pm[4], pm[5]), pm[6], pm[7]));
        const float m_blk = mx * sl2;
        float alpha = 1.f;
        if (m_blk > m_run + kRescaleThreshold) {
          alpha = ex2_approx(m_run - m_blk);  // m_run = -inf -> 0
          m_run = m_blk;
        }
        l_run *= alpha;
        l_rnd *= alpha;
        // Rescale o when the running max moved; the previous block's P V must
        // have completed first.
        if (__any_sync(0xffffffffu, j > 0 && alpha != 1.f)) {
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done, (gb - 1) & 1, g));
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int c4 = 0; c4 < DV / 32; ++c4) {
            uint32_t raw[32];
            tmem_ld32(tmem + kTmO + lane_off + c4 * 32, raw);
#pragma unroll
            for (int i = 0; i < 32; ++i) raw[i] = __float_as_uint(__uint_as_float(raw[i]) * alpha);
            tmem_st32(tmem + kTmO + lane_off + c4 * 32, raw);
          }
        }
        const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
        const uint64_t sc2 = f2(sl2, sl2), nm2 = f2(neg_m, neg_m);
        uint64_t rs2[4] = {0, 0, 0, 0}, rr2[4] = {0, 0, 0, 0};
        uint32_t pk[kBlkTok / 2];
#pragma unroll
        for (int q2 = 0; q2 < kBlkTok / 2; ++q2) {
          const uint64_t x2 = fma2(f2(__uint_as_float(sr[2 * q2]), __uint_as_float(sr[2 * q2 + 1])), sc2, nm2);
          float p0, p1;
          if ((q2 & 7) >= 6) {  // 2 of every 8 pairs on the FMA pipe
            f2_split(exp2_poly2(x2), p0, p1);
          } else {
            float x0, x1;
            f2_split(x2, x0, x1);
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          rs2[q2 & 3] = add2(rs2[q2 & 3], f2(p0, p1));
          const uint32_t bb = pack_bf16x2(p0, p1);
          pk[q2] = bb;
          if (ATTN_DEC_RSUM)
            rr2[q2 & 3] = add2(rr2[q2 & 3], f2(__uint_as_float(bb << 16), __uint_as_float(bb & 0xFFFF0000u)));
        }
        {
          const uint64_t a = add2(add2(rs2[0], rs2[1]), add2(rs2[2], rs2[3]));
          const uint64_t bq = add2(add2(rr2[0], rr2[1]), add2(rr2[2], rr2[3]));
          float a0, a1, b0, b1;
          f2_split(a, a0, a1);
          f2_split(bq, b0, b1);
          l_run += a0 + a1;
          l_rnd += b0 + b1;
        }
        tmem_st32(tS, pk);
        if (warp == 0 && valid < nv * kPage) {
          // Tokens past the end of the sequence inside its last page: P is 0
          // there, but the cache slots may hold anything (0 * NaN = NaN), so
          // their V rows are cleared before the MMA reads them.
          const uint32_t vst = s_ring + (gb % nst) * C::STAGE + C::KB * kBox;
          const int nrow = nv * kPage - valid;  // rows valid .. nv*16-1 of the block
          for (int e = lane; e < nrow * C::VB * 8; e += 32) {
            const int row = valid + e / (8 * C::VB), h = (e / 8) % C::VB, ch = e & 7;
            const uint32_t a = vst + h * kBox + row * 128 + ch * 16;
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[gb & 1]);
      }
      if (!ok) break;
      // End of the segment.
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_full, n_seg & 1, g));
      if (!ok) break;
      tc_fence_after();
      // One partial per query head.
      const int sidx = c - owner(pre, T, (int)G);
      const bool in_range = sidx >= 0 && sidx < p.max_segs;  // always, with chunks >= kDecodeMinChunk
      if (lane == 0 && !in_range) atomicExch(p.status, kErrBounds);
      const bool write = r < p.rows && in_range;
      const size_t rec = (((size_t)b * p.Hq + kvh * p.group) * p.q_len + r) * p.max_segs + sidx;
      const float l_o = ATTN_DEC_RSUM ? l_rnd : l_run;  // normalises o
      const float inv = l_o > 0.f ? 1.f / l_o : 0.f;
#pragma unroll 1
      for (int c4 = 0; c4 < DV / 32; ++c4) {
        uint32_t raw[32];
        tmem_ld32(tmem + kTmO + lane_off + c4 * 32, raw);
        if (write) {
          float4* dst = reinterpret_cast<float4*>(p.ws_o + rec * DV + c4 * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(raw[4 * i]) * inv, __uint_as_float(raw[4 * i + 1]) * inv,
                                 __uint_as_float(raw[4 * i + 2]) * inv, __uint_as_float(raw[4 * i + 3]) * inv);
        }
      }
      if (write) p.ws_lse[rec] = l_run > 0.f ? m_run + __log2f(l_run) : -INFINITY;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.o_empty);
      n_blk += nb;
      ++n_seg;
    }
    finish();
  } else {
    finish();  // softmax warp without rows (group <= 32 * warp)
  }
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
bool encode_pool(CUtensorMap* map, const void* pool, int num_pages, int Hkv, int D) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)num_pages * kPage};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kPage};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pool), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// q [B * Hq rows, D] bf16, box = `box_rows` rows x 64 features (128-byte swizzle).
bool encode_q(CUtensorMap* map, const void* q, int rows, int box_rows, int D) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


template <int DQK, int DV>
int run_decode(const DecodeArgs& a, cudaStream_t stream) {
  using C = DecCfg<DQK, DV>;
  const int group = a.Hq / a.Hkv;
  const int q_len = a.q_len > 0 ? a.q_len : 1;
  const int rows = group * q_len;  // query rows per (sequence, K/V head) tile
  if (rows > kMaxGroup) return -2;
  const int max_pages = a.max_pages > 0 ? a.max_pages : 1;
  const int max_segs = decode_max_segments(max_pages);
  const int q_box = (rows + 7) / 8 * 8 * 128;
  // Layout: as many CTAs per SM as the TMEM holds if some layout fits that
  // many, deepest ring first, then a second query slot; else one per SM.
  int ctas = 1, q_slots = 1, stages = 2;
  bool chosen = false;
  for (int n = C::TMEM_CTAS; n >= 1 && !chosen; --n) {
    const int cand[4][2] = {{2, 3}, {1, 3}, {2, 2}, {1, 2}};  // (query slots, stages)
    for (int i = 0; i < 4 && !chosen; ++i) {
      if (fits(dec_smem_bytes<DQK, DV>(q_box, cand[i][0], cand[i][1]), n)) {
        ctas = n;
        q_slots = cand[i][0];
        stages = cand[i][1];
        chosen = true;
      }
    }
  }
  if (!chosen) return -2;  // not reached: every width fits once (static_assert)
  int smem = dec_smem_bytes<DQK, DV>(q_box, q_slots, stages);
  const int min_smem = kSmemPerSm / (ctas + 1) - 1024 + 16;  // no extra CTA may share the SM
  if (smem < min_smem) smem = min_smem;
  static int attr_smem[64] = {0};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail_cuda("cudaGetDevice", err);
  if (dev >= 64 || attr_smem[dev] < smem) {
    err = cudaFuncSetAttribute(decode_split_kernel<DQK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return fail_cuda("decode: cudaFuncSetAttribute", err);
    if (dev < 64) attr_smem[dev] = smem;
  }
  float* ws_o = static_cast<float*>(a.workspace);
  float* ws_lse = ws_o + (size_t)a.B * a.Hq * q_len * max_segs * DV;
  int* status = device_status_word();
  if (!status) return fail_cuda("decode: status word", cudaGetLastError());
  const int split_grid = ctas * sm_count();
  const bool has_pool = a.num_pages > 0 && a.max_pages > 0;
  if (has_pool) {
    SplitParams sp{};
    sp.block_table = a.block_table;
    sp.seq_lens = a.seq_lens;
    sp.ws_o = ws_o;
    sp.ws_lse = ws_lse;
    sp.B = a.B;
    sp.Hq = a.Hq;
    sp.Hkv = a.Hkv;
    sp.group = group;
    sp.num_pages = a.num_pages;
    sp.max_pages = a.max_pages;
    sp.max_segs = max_segs;
    sp.q_len = q_len;
    sp.rows = rows;
    sp.q_box = q_box;
    sp.q_slots = q_slots;
    sp.stages = stages;
    sp.sm_warps = (rows + 31) / 32;
    sp.scale_log2 = a.scale * kLog2e;
    sp.bounds_check = (debug_flags() & 1) ? 1 : 0;
    sp.status = status;
    sp.timeout_ns = wait_timeout_ns();
    sp.stall = (debug_flags() & 2) ? 1 : 0;
    CUtensorMap tq, tk, tv;
    if (!encode_q(&tq, a.q, a.B * a.Hq * q_len, rows, DQK) || !encode_pool(&tk, a.k_pages, a.num_pages, a.Hkv, DQK) ||
        !encode_pool(&tv, a.v_pages, a.num_pages, a.Hkv, DV))
      return fail_cuda("decode: tensor map", cudaErrorInvalidValue);
    cudaLaunchConfig_t scfg{};
    scfg.gridDim = dim3(split_grid);
    scfg.blockDim = dim3(kThreads);
    scfg.dynamicSmemBytes = smem;
    scfg.stream = stream;
    cudaLaunchAttribute sattr[1];
    sattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    sattr[0].val.programmaticStreamSerializationAllowed = 1;
    scfg.attrs = sattr;
    scfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&scfg, decode_split_kernel<DQK, DV>, tq, tk, tv, sp);
    if (err == cudaSuccess) err = cudaGetLastError();
    if (err != cudaSuccess) return fail_cuda("decode: split launch", err);
  }
  CombineParams cp{};
  cp.ws_o = ws_o;
  cp.ws_lse = ws_lse;
  cp.seq_lens = a.seq_lens;
  cp.o = static_cast<__nv_bfloat16*>(a.o);
  cp.lse = a.lse;
  cp.B = a.B;
  cp.Hq = a.Hq;
  cp.Hkv = a.Hkv;
  cp.group = group;
  cp.max_pages = max_pages;
  cp.max_segs = max_segs;
  cp.q_len = q_len;
  cp.split_grid = split_grid;
  // Without a pool the split kernel did not run: the combine then treats
  // every sequence as empty (O = 0, LSE = -inf).
  cp.has_pool = has_pool ? 1 : 0;
  cp.q = static_cast<const __nv_bfloat16*>(a.q);
  cp.k_pages = static_cast<const __nv_bfloat16*>(a.k_pages);
  cp.v_pages = static_cast<const __nv_bfloat16*>(a.v_pages);
  cp.block_table = a.block_table;
  cp.num_pages = a.num_pages;
  cp.scale_log2 = a.scale * kLog2e;
  cp.bounds_check = (debug_flags() & 1) ? 1 : 0;
  cp.status = status;
  const int nw = a.B * a.Hq * q_len;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((nw + 7) / 8);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, decode_combine_kernel<DQK, DV>, cp);
  if (err == cudaSuccess) err = cudaGetLastError();
  return err == cudaSuccess ? 0 : fail_cuda("decode: combine launch", err);
}

template <int DQK>
int run_decode_dv(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.Dv) {
    case 64: return run_decode<DQK, 64>(a, stream);
    case 128: return run_decode<DQK, 128>(a, stream);
    case 192: return run_decode<DQK, 192>(a, stream);
    case 256: return run_decode<DQK, 256>(a, stream);
    default: return -2;
  }
}

}  // namespace

int launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (a.page_size != kPage) return -2;
  switch (a.D) {
    case 64: return run_decode_dv<64>(a, stream);
    case 128: return run_decode_dv<128>(a, stream);
    case 192: return run_decode_dv<192>(a, stream);
    case 256: return run_decode_dv<256>(a, stream);
    default: return -2;
  }
}

}  // namespace attn
