// prefill_sm100.cu -- fused attention forward for B200 (sm_100a).
//
// Computes O = softmax(scale * Q K^T + mask) V and the per-row LSE with the
// online-softmax recurrence of the tiled FlashAttention loop (page
// "003-注意力机制详解：从基础Attention到DeepSeek的优化策略", §二): per K/V
// block, S = Q K^T, new running max, rescale of the accumulator and of the
// running sum, P = exp(S - max), acc += P V, sum += rowsum(P); at the end
// O = acc / sum.  Scores and the accumulator never leave the SM (the "tiles
// in SRAM, one fused kernel" design of the tqpw.cn article §4.1-4.2), and K/V
// blocks wholly above the causal diagonal or before the sliding window are
// never loaded (kler.cn page §一.2; window of the zeeklog page).
//
// B200 mapping (one persistent CTA per SM, 512 threads in 4 warpgroups):
//   warps 0-3   softmax warpgroup for Q tile 0 (one thread per query row)
//   warps 4-7   softmax warpgroup for Q tile 1
//   warp  8     TMA producer: Q tiles, then K_j, V_j into a ring of stages
//   warp  9     MMA issuer (one thread) + TMEM owner
//   warps 10-11 idle (they complete the third warpgroup)
//   warps 12-15 epilogue: O = acc / sum to bf16 and the LSE, per unit
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,..).
// P (bf16 or e4m3) is written back over the first columns of its S buffer
// and consumed from TMEM as the A operand of O += P V.
// The two Q tiles of a work unit share every K/V tile: for GQA they are two
// query heads of one K/V group at the same rows; otherwise two consecutive
// 128-row blocks of one head.  While one warpgroup runs the softmax of its
// tile, the tensor core works on the other tile.
//
// Deviations from the pages' sketch: exp2 with scale*log2(e) folded in (same
// value), and the running max is only moved when it grows by more than 8
// (log2 units); with a stale max P stays <= 2^8, and the final O / sum and
// LSE = max + log2(sum) are unchanged mathematically.  This removes most of
// the accumulator rescales.
#include <cfloat>
#include <climits>
#include <cstdio>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace attn {
namespace {

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per K/V block
constexpr int kThreads = 512;  // 4 warpgroups
// Register split (setmaxnreg): the block launches with kLaunchRegs per thread
// (512 threads x 128 fills the register file: 4 warps per SM sub-partition).
// The producer/MMA warpgroup and the epilogue warpgroup give registers back and
// the two softmax warpgroups take them.  Warps go round-robin to the four SM
// sub-partitions, so each holds one warp of every warpgroup, and the shares
// must add up to exactly its launch total or the increase would wait forever:
// 2 * 192 + 88 + 40 = 4 * 128.
// The build checks with ptxas that the kernels launch with kLaunchRegs.
constexpr int kLaunchRegs = 128;
constexpr int kSoftmaxRegs = 192;
constexpr int kIssueRegs = 88;
constexpr int kEpilogueRegs = 40;
static_assert(2 * kSoftmaxRegs + kIssueRegs + kEpilogueRegs == 4 * kLaunchRegs,
              "register split must match the launch total");
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// e4m3 tiles whose rows see few keys ("fine" tiles).  Rounding P to e4m3 (3
// mantissa bits) moves each weight by up to 2^-4 relative; on a row of a
// handful of keys that error does not average out and can reach ~6e-2 in O.
// For a tile whose first row (the row that sees the fewest keys) sees fewer
// than kFineKeys keys, the kernel therefore multiplies V by P in two parts:
// h = e4m3(P) and the rounding residual e4m3(P - h), accumulated into the same
// O, so each weight carries ~7 significant bits.  In those tiles P is scaled
// by 2^kFineShift (the running max is kept exact, so P <= 2^8 <= 448, the
// e4m3 maximum) so that residuals stay above e4m3's subnormal range; the
// scale cancels in O / sum and is taken out of the LSE.  The residual lives in
// TMEM columns [32, 64) of the tile's S buffer (P of 128 keys in e4m3 fills
// columns [0, 32); all 128 columns of S are in registers by then).
constexpr int kFineKeys = 512;
constexpr float kFineShift = 8.0f;
// bf16 tiles take the same two-part product (bf16(P) and bf16(P - bf16(P)),
// the residual in columns [64, 128)) when their first row sees fewer than
// kFineKeysBf16 keys: rounding P to bf16 moves the O of a row of two keys by
// up to ~2^-9 of the spread of its V values, which with the bf16 rounding of O
// can pass 1e-2.  bf16 needs no scaling (its exponent range is fp32's).
constexpr int kFineKeysBf16 = 256;
template <bool FP8>
constexpr uint32_t kFineCol = FP8 ? 32 : 64;
constexpr float kLn2 = 0.6931471805599453f;
// Of every 8 pairs of exponentials, this many are computed by the FMA-pipe
// polynomial instead of the MUFU ex2 unit (balances the two pipes).
#ifndef ATTN_EMU_PAIRS_PER8
#define ATTN_EMU_PAIRS_PER8 0
#endif
// e4m3: 1 of 8.  Without the rounded row sum (plain tiles) its softmax issues
// ~7 instructions per key pair but waits 16 MUFU cycles for the two ex2, so
// one polynomial pair in 8 moves work to idle issue slots (interleaved A/B on
// the e4m3 workload: 1,449 against 1,387 TFLOP/s; 2 and 3 of 8: 1,391, 1,368).
// bf16, MUFU-bound no more than its tensor work, measured best with none.
#ifndef ATTN_EMU_PAIRS_PER8_FP8
#define ATTN_EMU_PAIRS_PER8_FP8 1
#endif
template <bool FP8>
constexpr int kEmuPairsPer8 = FP8 ? ATTN_EMU_PAIRS_PER8_FP8 : ATTN_EMU_PAIRS_PER8;
// P handoff in two parts: after the first ATTN_SPLIT_P x 16 keys of the block
// (0: no split; 2, 4 or 6 of 8) the MMA warp starts O += P V on them while the
// softmax warps compute the rest.
#ifndef ATTN_SPLIT_P
#define ATTN_SPLIT_P 6
#endif
constexpr bool kSplitP = ATTN_SPLIT_P != 0;
constexpr int kSplitKeys = ATTN_SPLIT_P * 16;
static_assert(ATTN_SPLIT_P == 0 || (ATTN_SPLIT_P % 2 == 0 && ATTN_SPLIT_P < 8), "split at 32, 64 or 96 keys");
// Which sum normalises O.  The MMA multiplies V by P rounded to bf16 / e4m3,
// so normalising by the sum of those rounded values makes the weights add to
// exactly one; normalising by the exact fp32 sum (which the LSE needs anyway)
// is off by the mean rounding error of the row's weights: up to 2^-9 / 2^-4
// relative on a row of a few keys -- with the bf16 rounding of O beyond 1e-2
// for bf16 -- but ~2^-9 / sqrt(n) (bf16) or ~2^-4 / sqrt(n) (e4m3) on a row of
// n keys, since round-to-nearest errors are unbiased.  The kernels built for
// tiles whose rows see few keys (FINE) keep the rounded sum (3-4 instructions
// per key pair) and normalise fine tiles by it; other tiles, whose rows see
// >= 256 (bf16) or >= 512 (e4m3) keys, use the exact sum in every kernel: 2e-4
// and 3e-3 of |O| typically.
// ATTN_ROUNDED_SUM=1 keeps the rounded sum everywhere (measurement switch).
#ifndef ATTN_ROUNDED_SUM
#define ATTN_ROUNDED_SUM 0
#endif
static_assert(ATTN_ROUNDED_SUM == 0 || ATTN_ROUNDED_SUM == 1, "row-sum mode 0 or 1");


// E5M2 (with FP8): the 8-bit inputs are e5m2, and P is multiplied in e5m2 too
// (kind::f8f6f4 format code 1; each product keeps one operand type).
template <int D, bool FP8, bool E5M2 = false>
struct Cfg {
  static constexpr int EL = FP8 ? 1 : 2;                 // bytes per element
  static constexpr int ROW_BYTES = D * EL;
  static constexpr int NBOX = ROW_BYTES / 128;           // 128-byte swizzle columns per tile
  static constexpr int BOX_ELEMS = 128 / EL;             // elements per box row
  static constexpr int BOX_BYTES = kBM * 128;            // one box: 128 rows x 128 B
  static constexpr int TILE_BYTES = kBM * ROW_BYTES;
#ifndef ATTN_KV_STAGES_BIG
#define ATTN_KV_STAGES_BIG 4
#define ATTN_KV_STAGES_SMALL 11
#endif
  static constexpr int NS = TILE_BYTES >= 32768 ? ATTN_KV_STAGES_BIG : ATTN_KV_STAGES_SMALL;  // K/V ring stages
  static constexpr int MMA_K = FP8 ? 32 : 16;
  static constexpr int S_KSTEPS = D / MMA_K;
  static constexpr int PV_KSTEPS = kBN / MMA_K;
  static constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O0 = 256, TM_O1 = 256 + D;
  static constexpr uint32_t FMT = FP8 ? (E5M2 ? 1u : 0u) : 1u;  // e4m3 0, e5m2 1; bf16 1
  static constexpr uint32_t IDESC_S = make_idesc(FMT, kBM, kBN, false);
  static constexpr uint32_t IDESC_PV = make_idesc(FMT, kBM, D, true);
  // shared memory: [Q0][Q1][stage 0..NS-1] (1024-aligned) + barriers
  static constexpr int SMEM_TILES = (2 + NS) * TILE_BYTES;
  static constexpr int SMEM_BYTES = SMEM_TILES + 1024 /*align slack*/ + 4096 /*barriers, row statistics*/;
  static_assert(SMEM_BYTES <= 232448, "more than the 227 KB a CTA may use");
  static_assert(NBOX >= 1 && ROW_BYTES % 128 == 0, "rows must be whole 128-byte swizzle rows");
  static_assert(TM_O1 + D <= 512, "TMEM budget");
};

struct Params {
  void* o;
  float* lse;
  int B, Hq, Hkv, Lq, Lk;
  int group;        // Hq / Hkv
  int pair_heads;   // 1: the two tiles are heads 2p, 2p+1 of one group
  int n_pairs;      // units per row group
  int mg_hi;        // this launch covers row groups [mg_hi - n_units / n_pairs, mg_hi)
  int n_units;
  int chunk;        // pairs per chunk of units (whole K/V heads; see get_unit)
  int l2_hints;     // Q loads evict-first, K/V loads evict-last, O stores streaming
  int causal, window;
  float scale_log2;  // logit scale * log2(e) (fp8: times both descales)
  float out_scale;   // 1 (bf16) or v_descale (fp8)

  int* status;
  unsigned long long timeout_ns;
  int stall;  // testing hook: the producer issues no loads, every wait runs out
  // Paged K/V (chunked prefill over a paged cache): sequence b has
  // seq_lens[b] cached tokens (its Lq queries are the last Lq of them),
  // stored in 16-token pages of a pool listed by block_table.
  const int* block_table;
  const int* seq_lens;
  int max_pages, num_pages;
};

constexpr int kPage = 16;  // tokens per page of a paged K/V pool

template <int N>
struct IntC {
  static constexpr int value = N;
};

struct Unit {
  int bh[2];  // b * Hq + head of each tile
  int m0[2];  // first query row of each tile
  int kvbh;   // b * Hkv + kv head
  int kb_lo;  // first K/V block
  int nb;     // number of K/V blocks (0: nothing visible)
  int lk;     // keys of this unit's sequence (Lk, or its cached length when paged)
  // Per-tile fields by a runtime tile index, as selects (an indexed load
  // would put the struct in local memory).
  __device__ __forceinline__ int bh_of(int t) const { return t ? bh[1] : bh[0]; }
  __device__ __forceinline__ int m0_of(int t) const { return t ? m0[1] : m0[0]; }
};

// Visible keys [lo, hi) of query row i (bottom-right causal alignment; window
// of W keys including the query's own position).
__device__ __forceinline__ void key_range(int i, int lk, const Params& p, int& lo, int& hi) {
  if (!p.causal) {
    lo = 0;
    hi = lk;
    return;
  }
  int h = i + (lk - p.Lq) + 1;
  h = h < 0 ? 0 : (h > lk ? lk : h);
  hi = h;
  lo = (p.window > 0 && h - p.window > 0) ? h - p.window : 0;
}

// Units are numbered in chunks of `chunk` pairs (the pairs of whole K/V heads
// whose K and V together fit in a part of L2), and within a chunk so that the
// longest (latest rows under a causal mask) come first.  The CTAs working at
// one time then share the K/V of one chunk, which stays in L2, instead of
// touching every head's.  CTA c takes one unit per round, in snake order (c
// in even rounds, grid - 1 - c in odd rounds), which balances the causal work
// across CTAs without any global queue.
template <bool PAGED>
__device__ __forceinline__ Unit get_unit(int u, const Params& p) {
  Unit w;
  int b_seq;
  const int n_mg = p.n_units / p.n_pairs;  // row groups of this launch
  const int per_chunk = p.chunk * n_mg;
  const int ch = u / per_chunk;
  const int r = u - ch * per_chunk;
  const int cp = min(p.chunk, p.n_pairs - ch * p.chunk);  // pairs in this chunk
  const int mg = p.mg_hi - 1 - r / cp;
  const int pr = ch * p.chunk + r % cp;
  if (p.pair_heads) {
    const int hp_per_b = p.Hq >> 1;
    const int b = pr / hp_per_b, hp = pr % hp_per_b;
    b_seq = b;
    w.bh[0] = b * p.Hq + 2 * hp;
    w.bh[1] = w.bh[0] + 1;
    w.m0[0] = w.m0[1] = mg * kBM;
    w.kvbh = b * p.Hkv + (2 * hp) / p.group;
  } else {
    const int b = pr / p.Hq, h = pr % p.Hq;
    b_seq = b;
    w.bh[0] = w.bh[1] = b * p.Hq + h;
    w.m0[0] = mg * 2 * kBM;
    w.m0[1] = w.m0[0] + kBM;
    w.kvbh = b * p.Hkv + h / p.group;
  }
  w.lk = p.Lk;
  if (PAGED) {
    const int n = p.seq_lens[b_seq], cap = p.max_pages * kPage;
    w.lk = n < 0 ? 0 : (n > cap ? cap : n);
  }
  int lo = INT_MAX, hi = 0;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (w.m0[t] < p.Lq) {
      const int r_last = min(w.m0[t] + kBM - 1, p.Lq - 1);
      int lo0, hi0, lo1, hi1;
      key_range(w.m0[t], w.lk, p, lo0, hi0);
      key_range(r_last, w.lk, p, lo1, hi1);
      if (hi1 > lo0) {  // lo and hi are non-decreasing in the row index
        lo = min(lo, lo0);
        hi = max(hi, hi1);
      }
    }
  }
  if (hi <= lo) {
    w.kb_lo = 0;
    w.nb = 0;
  } else {
    w.kb_lo = lo / kBN;
    w.nb = (hi + kBN - 1) / kBN - w.kb_lo;
  }
  return w;
}

__device__ __forceinline__ int unit_of(int round, int n_units) {
  const int g = (int)gridDim.x, c = (int)blockIdx.x;
#ifdef ATTN_ROUND_ROBIN
  const int u = round * g + c;
#else
  const int u = round * g + ((round & 1) ? g - 1 - c : c);
#endif
  return u < n_units ? u : n_units;  // n_units: no more work
}

struct Smem {
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], p_full[2];
  uint64_t p_half[2];         // first 64 keys of P stored (128 arrivals)
  uint64_t o_full[2], o_empty[2];
  uint64_t drain;
  uint64_t kv_full[12], kv_empty[12];
  uint64_t st_full[2];        // row statistics of a unit written (128 arrivals)
  uint64_t st_empty[2];       // ... and read by the epilogue (128 arrivals)
  uint32_t tmem_base;
  int abort_flag;
  float st_m[2][kBM];         // [tile][row] running max (log2 units) at unit end
  float st_l[2][kBM];         // [tile][row] exact row sum
  float st_r[2][kBM];         // [tile][row] sum of the rounded P
};

static_assert(sizeof(Smem) <= 4096, "barrier/statistics block exceeds its reserve");

// One pair of keys of a softmax row: x = s * scale * log2e - m, P = 2^x (MUFU
// ex2, or for kEmuPairsPer8 of every 8 pairs the FMA-pipe polynomial), packed
// for the MMA, added to the exact row sum and, with RSUM, to the sum of the
// rounded values.  e4m3 pairs go two to a 32-bit word.
// FINE (8-bit P only): also the residual fp8(P - h) into pk_lo, and the sum
// of h + residual, the weight the two products apply together.  E5M2: P and
// its residual in e5m2 (the format of e5m2 inputs), else e4m3.
// EMU: of every 8 pairs, this many take the FMA-pipe polynomial for 2^x.
template <bool FP8, bool RSUM, bool FINE, bool E5M2 = false, int EMU = 0>
__device__ __forceinline__ void p_pair(int q2, const uint32_t (&sr)[kBN], uint64_t sc2, uint64_t nm2,
                                       uint64_t (&rs2)[4], uint64_t (&rr2)[4], uint32_t (&pk)[kBN / 2],
                                       uint32_t (&pk_lo)[kBN / 2]) {
  const uint64_t x2 = fma2(f2(__uint_as_float(sr[2 * q2]), __uint_as_float(sr[2 * q2 + 1])), sc2, nm2);
  float p0, p1;
  if ((q2 & 7) >= 8 - EMU) {
    f2_split(exp2_poly2(x2), p0, p1);
  } else {
    float x0, x1;
    f2_split(x2, x0, x1);
    p0 = ex2_approx(x0);
    p1 = ex2_approx(x1);
  }
  rs2[q2 & 3] = add2(rs2[q2 & 3], f2(p0, p1));
  if (FP8) {
    const uint16_t e = E5M2 ? pack_e5m2x2(p0, p1) : pack_e4m3x2(p0, p1);
    if (q2 & 1) pk[q2 >> 1] |= (uint32_t)e << 16;
    else pk[q2 >> 1] = e;
    float h0, h1;
    unpack_fp8x2<E5M2>(e, h0, h1);
    if (FINE) {
      // P - h is exact in fp32 (h is P rounded to a 3- or 4-bit significand).
      const uint16_t el = E5M2 ? pack_e5m2x2(p0 - h0, p1 - h1) : pack_e4m3x2(p0 - h0, p1 - h1);
      if (q2 & 1) pk_lo[q2 >> 1] |= (uint32_t)el << 16;
      else pk_lo[q2 >> 1] = el;
      float l0, l1;
      unpack_fp8x2<E5M2>(el, l0, l1);
      h0 += l0;
      h1 += l1;
    }
    rr2[q2 & 3] = add2(rr2[q2 & 3], f2(h0, h1));
  } else {
    const uint32_t b = pack_bf16x2(p0, p1);
    pk[q2] = b;
    float h0 = __uint_as_float(b << 16), h1 = __uint_as_float(b & 0xFFFF0000u);
    if (FINE) {
      const uint32_t bl = pack_bf16x2(p0 - h0, p1 - h1);  // P - h is exact in fp32
      pk_lo[q2] = bl;
      h0 += __uint_as_float(bl << 16);
      h1 += __uint_as_float(bl & 0xFFFF0000u);
    }
    if (RSUM) rr2[q2 & 3] = add2(rr2[q2 & 3], f2(h0, h1));
  }
}

template <bool FP8, bool RSUM, bool FINE, int Q_LO, int Q_HI, bool E5M2 = false, int EMU = 0>
__device__ __forceinline__ void p_pairs(const uint32_t (&sr)[kBN], uint64_t sc2, uint64_t nm2, uint64_t (&rs2)[4],
                                        uint64_t (&rr2)[4], uint32_t (&pk)[kBN / 2], uint32_t (&pk_lo)[kBN / 2]) {
#pragma unroll
  for (int q2 = Q_LO; q2 < Q_HI; ++q2) p_pair<FP8, RSUM, FINE, E5M2, EMU>(q2, sr, sc2, nm2, rs2, rr2, pk, pk_lo);
}

// Fine tiles: pairs [Q_LO, Q_HI) in chunks of 8 TMEM columns (e4m3: 16 pairs,
// bf16: 8), each chunk's P and residual stored to TMEM at once (at taddr and taddr + kFineCol; e4m3
// packs two pairs per column, bf16 one), so that the residual adds few live
// registers.
template <bool FP8, bool RSUM, bool E5M2, int Q_LO, int Q_HI>
__device__ __forceinline__ void p_pairs_fine(const uint32_t (&sr)[kBN], uint64_t sc2, uint64_t nm2,
                                             uint64_t (&rs2)[4], uint64_t (&rr2)[4], uint32_t (&pk)[kBN / 2],
                                             uint32_t (&pk_lo)[kBN / 2], uint32_t taddr) {
  if constexpr (Q_LO < Q_HI) {
    constexpr int CH = FP8 ? 16 : 8;  // pairs per chunk: 8 TMEM columns each way
    constexpr int QE = Q_LO + CH < Q_HI ? Q_LO + CH : Q_HI;
    constexpr int C0 = FP8 ? Q_LO / 2 : Q_LO, C1 = FP8 ? QE / 2 : QE;
    p_pairs<FP8, RSUM, true, Q_LO, QE, E5M2>(sr, sc2, nm2, rs2, rr2, pk, pk_lo);
    tmem_st_cols<C0, C1>(taddr, pk);
    tmem_st_cols<C0, C1>(taddr + kFineCol<FP8>, pk_lo);
    p_pairs_fine<FP8, RSUM, E5M2, QE, Q_HI>(sr, sc2, nm2, rs2, rr2, pk, pk_lo, taddr);
  }
}

// Is tile t of unit w a "fine" e4m3 tile (its first row sees < kFineKeys keys)?
// FINE: the kernel is built with the two-part product at all (without it,
// the launch covers no tile that needs it; see run()).
template <bool FP8, bool E5M2, bool FINE>
__device__ __forceinline__ bool tile_fine(const Unit& w, int t, const Params& p) {
  if (!FINE) return false;
  if (FP8 && E5M2) return true;  // 2 mantissa bits: every tile takes the residual product
  const int m0 = w.m0_of(t);
  if (m0 >= p.Lq) return false;
  int lo, hi;
  key_range(m0, w.lk, p, lo, hi);
  return hi - lo < (FP8 ? kFineKeys : kFineKeysBf16);
}

template <int D, bool FP8, bool PAGED, bool E5M2, bool FINE>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg<D, FP8, E5M2>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t tiles_addr = (raw_addr + 1023u) & ~1023u;
  uint8_t* tiles_ptr = smem_raw + (tiles_addr - raw_addr);
  Smem& sm = *reinterpret_cast<Smem*>(tiles_ptr + C::SMEM_TILES);
  auto q_addr = [&](int t) { return tiles_addr + (t ? (uint32_t)C::TILE_BYTES : 0u); };
  const uint32_t kv_addr0 = tiles_addr + 2u * C::TILE_BYTES;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // A launch queued behind this one as a programmatic dependent (the few-key
  // launch) may start on SMs this grid leaves idle; it shares no data with it.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.q_full[t], 1);
      mbar_init(&sm.q_empty[t], 1);
      mbar_init(&sm.s_full[t], 1);
      mbar_init(&sm.p_full[t], 128);
      mbar_init(&sm.p_half[t], 128);
      mbar_init(&sm.o_full[t], 1);
      mbar_init(&sm.o_empty[t], 128);
      mbar_init(&sm.st_full[t], 128);
      mbar_init(&sm.st_empty[t], 128);
    }
    mbar_init(&sm.drain, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitGuard g{&sm.abort_flag, p.status, p.timeout_ns, true};
  const WaitGuard g_drain{&sm.abort_flag, p.status, p.timeout_ns, false};

  // Teardown, run at the end of every role branch (no code is shared between
  // the register regions set by setmaxnreg): all threads meet, then the
  // owner warp releases TMEM.
  auto finish = [&]() {
    tc_fence_before();
    asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
    if (warp == 9) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
    // Launched as a programmatic dependent (the few-key launch after the
    // plain one): complete only after the launch before it, so that stream
    // order holds for both.  Without a prerequisite grid this returns at once.
    asm volatile("griddepcontrol.wait;" ::: "memory");
  };

  // Each role branch sets its own register count first thing, so that no code
  // is reachable under two different counts.
  if (warp == 10 || warp == 11) {
    // spare warps of the third warpgroup
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kIssueRegs));
    finish();
  } else if (warp >= 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kEpilogueRegs));
    // ------------------------------------------------------------ epilogue
    // One thread per query row of each tile: O = acc / sum (bf16) and
    // LSE = (max + log2 sum) ln 2, off the softmax warps' critical path.
    const int r = ((warp & 3) << 5) + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) << 5) << 16;
    uint32_t nunit = 0;
    bool ok = true;
    for (int rnd = 0, u = unit_of(0, p.n_units); u < p.n_units && ok; u = unit_of(++rnd, p.n_units)) {
      const Unit w = get_unit<PAGED>(u, p);
      for (int t = 0; t < 2 && ok; ++t) {
        const int row = w.m0_of(t) + r;
        const bool row_valid = row < p.Lq;
        float m = -INFINITY, l = 0.f, lr = 0.f;
        if (w.nb > 0) {
          ok = mbar_wait(&sm.st_full[t], nunit & 1, g) && mbar_wait(&sm.o_full[t], nunit & 1, g);
          if (!ok) break;
          tc_fence_after();
          m = sm.st_m[t][r];
          l = sm.st_l[t][r];
          lr = sm.st_r[t][r];
          mbar_arrive(&sm.st_empty[t]);  // the softmax may write the next unit's
        }
        const float inv = (lr > 0.f) ? p.out_scale / lr : 0.f;
        __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + ((size_t)w.bh_of(t) * p.Lq + row) * D;
        const uint32_t tO = tmem + (t == 0 ? C::TM_O0 : C::TM_O1) + lane_off;
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          uint32_t raw[16];
          if (w.nb > 0) {
            tmem_ld16(tO + c * 16, raw);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) raw[i] = 0u;
          }
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(raw[2 * i]) * inv, __uint_as_float(raw[2 * i + 1]) * inv);
          if (row_valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 16);
            if (p.l2_hints) {
              __stcs(dst, make_uint4(pk[0], pk[1], pk[2], pk[3]));
              __stcs(dst + 1, make_uint4(pk[4], pk[5], pk[6], pk[7]));
            } else {
              dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
          }
        }
        if (row_valid && p.lse != nullptr)
          p.lse[(size_t)w.bh_of(t) * p.Lq + row] = (l > 0.f) ? (m + log2f(l)) * kLn2 : -INFINITY;
        if (w.nb > 0) {
          tc_fence_before();
          mbar_arrive(&sm.o_empty[t]);
        }
      }
      if (w.nb > 0) ++nunit;
    }
    finish();
  } else if (warp == 8) {
    // ------------------------------------------------------------ producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kIssueRegs));
    if (lane == 0) {
      uint32_t seq = 0, nunit = 0;
      bool ok = !p.stall;
      const uint64_t pol_q = l2_policy_evict_first(), pol_kv = l2_policy_evict_last();
      for (int rnd = 0, u = unit_of(0, p.n_units); u < p.n_units && ok; u = unit_of(++rnd, p.n_units)) {
        const Unit w = get_unit<PAGED>(u, p);
        if (w.nb <= 0) continue;
        for (int t = 0; t < 2 && ok; ++t) {
          if (nunit > 0) ok = mbar_wait(&sm.q_empty[t], (nunit - 1) & 1, g);
          if (!ok) break;
          mbar_arrive_expect_tx(&sm.q_full[t], C::TILE_BYTES);
#pragma unroll
          for (int bx = 0; bx < C::NBOX; ++bx) {
            if (p.l2_hints)
              tma_load_3d_hint(q_addr(t) + bx * C::BOX_BYTES, &tm_q, &sm.q_full[t], bx * C::BOX_ELEMS, w.m0_of(t),
                               w.bh_of(t), pol_q);
            else
              tma_load_3d(q_addr(t) + bx * C::BOX_BYTES, &tm_q, &sm.q_full[t], bx * C::BOX_ELEMS, w.m0_of(t),
                          w.bh_of(t));
          }
        }
        for (int j = 0; j < w.nb && ok; ++j) {
          const int row = (w.kb_lo + j) * kBN;
          for (int kind = 0; kind < 2; ++kind) {
            const uint32_t s = seq % C::NS;
            if (seq >= (uint32_t)C::NS) {
              ok = mbar_wait(&sm.kv_empty[s], ((seq / C::NS) - 1) & 1, g);
              if (!ok) break;
            }
            const uint32_t dst = kv_addr0 + s * C::TILE_BYTES;
            mbar_arrive_expect_tx(&sm.kv_full[s], C::TILE_BYTES);
            const CUtensorMap* m = kind == 0 ? &tm_k : &tm_v;
            if (PAGED) {
              // The block's 128 keys are 8 pages of this K/V head, gathered
              // through the block table into the rows of one tile; pages past
              // the sequence read as zeros (a page id past the pool).
              const int b = w.kvbh / p.Hkv, kvh = w.kvbh % p.Hkv;
              const int npg = (w.lk + kPage - 1) / kPage;
              int ids[kBN / kPage];
#pragma unroll
              for (int i = 0; i < kBN / kPage; ++i) {
                const int pg = row / kPage + i;
                ids[i] = pg < npg ? p.block_table[(size_t)b * p.max_pages + pg] : p.num_pages;
              }
#pragma unroll
              for (int i = 0; i < kBN / kPage; ++i)
#pragma unroll
                for (int bx = 0; bx < C::NBOX; ++bx)
                  tma_load_3d(dst + bx * C::BOX_BYTES + i * (kPage * 128), m, &sm.kv_full[s], bx * C::BOX_ELEMS,
                              kvh, ids[i] * kPage);
            } else {
#pragma unroll
              for (int bx = 0; bx < C::NBOX; ++bx) {
                if (p.l2_hints)
                  tma_load_3d_hint(dst + bx * C::BOX_BYTES, m, &sm.kv_full[s], bx * C::BOX_ELEMS, row, w.kvbh, pol_kv);
                else
                  tma_load_3d(dst + bx * C::BOX_BYTES, m, &sm.kv_full[s], bx * C::BOX_ELEMS, row, w.kvbh);
              }
            }
            ++seq;
          }
        }
        ++nunit;
      }
      // Drain: every load this thread issued has landed before the CTA exits.
      for (uint32_t s = 0; s < (uint32_t)C::NS && s < seq; ++s) {
        const uint32_t last = s + ((seq - 1 - s) / C::NS) * C::NS;
        mbar_wait(&sm.kv_full[s], (last / C::NS) & 1, g_drain);
      }
      if (nunit > 0)
        for (int t = 0; t < 2; ++t) mbar_wait(&sm.q_full[t], (nunit - 1) & 1, g_drain);
    }
    finish();
  } else if (warp == 9) {
    // ----------------------------------------------------------- MMA issue
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kIssueRegs));
    if (lane == 0) {
      // pcnt: K/V blocks whose P of both tiles has been consumed so far
      uint32_t seq = 0, nunit = 0, pcnt = 0;
      bool ok = true;
      auto tS = [&](int t) { return tmem + (t ? C::TM_S1 : C::TM_S0); };
      auto tO = [&](int t) { return tmem + (t ? C::TM_O1 : C::TM_O0); };
      // S_t = Q_t K^T: K-major operands; k-step kk starts kk*MMA_K elements
      // into the 128-byte rows, boxes of 64 (bf16) columns are BOX_BYTES apart.
      // Descriptors are built once per tile and advanced by adding
      // (byte offset >> 4) to their start-address field (no carry: < 256 KB).
      auto issue_s = [&](int t, uint32_t k_stage_addr) {
        const uint64_t a0 = sw128_desc(q_addr(t), 16, 1024);
        const uint64_t b0 = sw128_desc(k_stage_addr, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < C::S_KSTEPS; ++kk) {
          const uint32_t byte_k = kk * C::MMA_K * C::EL;
          const uint32_t off = ((byte_k / 128) * C::BOX_BYTES + (byte_k % 128)) >> 4;
          if (FP8)
            mma_f8_ss(tS(t), a0 + off, b0 + off, C::IDESC_S, kk > 0);
          else
            mma_f16_ss(tS(t), a0 + off, b0 + off, C::IDESC_S, kk > 0);
        }
      };
      // O_t (+)= P_t V: P from TMEM (over S_t), V MN-major, 128-byte column
      // groups BOX_BYTES apart, k-step kk = MMA_K keys of 128-byte rows.
      // k-steps [k_lo, k_hi) of the block's PV_KSTEPS.
      // a_col: TMEM column of P within the S buffer (kFineCol: the residual
      // of a fine e4m3 tile).
      auto issue_pv = [&](int t, uint32_t v_stage_addr, bool acc, int k_lo, int k_hi, uint32_t a_col) {
        const uint64_t b0 = sw128_desc(v_stage_addr, C::BOX_BYTES, 1024);
#pragma unroll
        for (int kk = k_lo; kk < k_hi; ++kk) {
          const uint32_t a = tS(t) + a_col + kk * (C::MMA_K * C::EL / 4);
          const uint32_t off = (kk * C::MMA_K * 128) >> 4;
          if (FP8)
            mma_f8_ts(tO(t), a, b0 + off, C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
          else
            mma_f16_ts(tO(t), a, b0 + off, C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
        }
      };
      for (int rnd = 0, u = unit_of(0, p.n_units); u < p.n_units && ok; u = unit_of(++rnd, p.n_units)) {
        const Unit w = get_unit<PAGED>(u, p);
        if (w.nb <= 0) continue;
        const bool fine0 = tile_fine<FP8, E5M2, FINE>(w, 0, p), fine1 = tile_fine<FP8, E5M2, FINE>(w, 1, p);
        ok = mbar_wait(&sm.q_full[0], nunit & 1, g) && mbar_wait(&sm.q_full[1], nunit & 1, g);
        if (!ok) break;
        // first K block
        uint32_t sk = seq % C::NS;
        ok = mbar_wait(&sm.kv_full[sk], (seq / C::NS) & 1, g);
        if (!ok) break;
        tc_fence_after();
        ++seq;
        // q_empty[t] is committed after the unit's last S of tile t (its last
        // reader of Q_t), so that the next unit's Q and first K/V tiles load
        // while this unit's last softmax and P V run.
        issue_s(0, kv_addr0 + sk * C::TILE_BYTES);
        tc_commit(&sm.s_full[0]);
        if (w.nb == 1) tc_commit(&sm.q_empty[0]);
        issue_s(1, kv_addr0 + sk * C::TILE_BYTES);
        tc_commit(&sm.s_full[1]);
        if (w.nb == 1) tc_commit(&sm.q_empty[1]);
        tc_commit(&sm.kv_empty[sk]);
        for (int j = 0; j < w.nb && ok; ++j) {
          const uint32_t sv = seq % C::NS;
          ok = mbar_wait(&sm.kv_full[sv], (seq / C::NS) & 1, g);
          if (!ok) break;
          ++seq;
          if (PAGED) {
            // Cache slots past the sequence end inside its last page: P is 0
            // there, but the slots may hold anything (0 * NaN = NaN), so their
            // V rows are cleared before P V reads them.
            const int key0 = (w.kb_lo + j) * kBN;
            const int r_lo = w.lk - key0, r_hi = min((w.lk + kPage - 1) / kPage * kPage - key0, kBN);
            if (r_lo > 0 && r_lo < r_hi) {
              for (int rr = r_lo; rr < r_hi; ++rr)
#pragma unroll
                for (int bx = 0; bx < C::NBOX; ++bx)
#pragma unroll
                  for (int ch = 0; ch < 8; ++ch)
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(
                                     kv_addr0 + sv * C::TILE_BYTES + bx * C::BOX_BYTES + rr * 128 + ch * 16),
                                 "r"(0u)
                                 : "memory");
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            }
          }
          const bool has_next = j + 1 < w.nb;
          const uint32_t skn = seq % C::NS;
          for (int t = 0; t < 2 && ok; ++t) {
            ok = mbar_wait(kSplitP ? &sm.p_half[t] : &sm.p_full[t], pcnt & 1, g);
            if (!ok) break;
            if (j == 0 && nunit > 0) {
              ok = mbar_wait(&sm.o_empty[t], (nunit - 1) & 1, g);
              if (!ok) break;
            }
            tc_fence_after();
            // fine tiles: a second product with the residual of P (one loop
            // body for both parts keeps the issuing thread's registers low)
            const int parts = (t ? fine1 : fine0) ? 2 : 1;
            if (kSplitP) {
#pragma unroll 1
              for (int pt = 0; pt < parts; ++pt)
                issue_pv(t, kv_addr0 + sv * C::TILE_BYTES, j > 0 || pt > 0, 0, kSplitKeys / C::MMA_K,
                         pt ? kFineCol<FP8> : 0u);
              ok = mbar_wait(&sm.p_full[t], pcnt & 1, g);
              if (!ok) break;
              tc_fence_after();
#pragma unroll 1
              for (int pt = 0; pt < parts; ++pt)
                issue_pv(t, kv_addr0 + sv * C::TILE_BYTES, true, kSplitKeys / C::MMA_K, C::PV_KSTEPS,
                         pt ? kFineCol<FP8> : 0u);
            } else {
#pragma unroll 1
              for (int pt = 0; pt < parts; ++pt)
                issue_pv(t, kv_addr0 + sv * C::TILE_BYTES, j > 0 || pt > 0, 0, C::PV_KSTEPS, pt ? kFineCol<FP8> : 0u);
            }
            if (!has_next) tc_commit(&sm.o_full[t]);
            if (has_next) {
              if (t == 0) {
                ok = mbar_wait(&sm.kv_full[skn], (seq / C::NS) & 1, g);
                if (!ok) break;
                tc_fence_after();
              }
              issue_s(t, kv_addr0 + skn * C::TILE_BYTES);
              tc_commit(&sm.s_full[t]);
              if (j + 2 == w.nb) tc_commit(&sm.q_empty[t]);
            }
          }
          if (!ok) break;
          ++pcnt;
          tc_commit(&sm.kv_empty[sv]);
          if (has_next) {
            tc_commit(&sm.kv_empty[skn]);
            ++seq;
          }
        }
        if (!ok) break;
        ++nunit;
      }
      // Drain: all issued MMAs complete before TMEM is released.
      tc_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, g_drain);
    }
    __syncwarp();
    finish();
  } else {
    // ------------------------------------------------------------ softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    const int t = warp >> 2;                 // tile of this warpgroup
    const int r = ((warp & 3) << 5) + lane;  // row within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) << 5) << 16;
    const uint32_t tS = tmem + (t == 0 ? C::TM_S0 : C::TM_S1) + lane_off;
    const uint32_t tO = tmem + (t == 0 ? C::TM_O0 : C::TM_O1) + lane_off;
    const float sl2 = p.scale_log2;
    constexpr bool kRsum = FINE || ATTN_ROUNDED_SUM;
    uint32_t scnt = 0, nunit = 0;
    bool ok = true;
    for (int rnd = 0, u = unit_of(0, p.n_units); u < p.n_units && ok; u = unit_of(++rnd, p.n_units)) {
      const Unit w = get_unit<PAGED>(u, p);
      const int row = w.m0_of(t) + r;
      // l_run: exact fp32 row sum (gives the LSE); l_rnd: sum of the rounded P
      // the MMA multiplies (normalises O so its weights sum to one).
      float m_run = -INFINITY, l_run = 0.f, l_rnd = 0.f;
      // fine e4m3 tile: exact running max, P scaled by 2^kFineShift, residual product
      const bool fine = tile_fine<FP8, E5M2, FINE>(w, t, p);
      // (8-bit P only: exact running max and P scaled by 2^kFineShift)
      const float thr = (FP8 && fine) ? 0.f : kRescaleThreshold;
      const float shift = (FP8 && fine) ? kFineShift : 0.f;
      if (w.nb > 0) {
        int lo, hi;
        key_range(row, w.lk, p, lo, hi);
        for (int j = 0; j < w.nb; ++j) {
          ok = mbar_wait(&sm.s_full[t], scnt & 1, g);
          if (!ok) break;
          ++scnt;
          tc_fence_after();
          uint32_t sr[kBN];  // raw fp32 scores of this row
          tmem_ld64x2(tS, sr);
          const int key0 = (w.kb_lo + j) * kBN;
          if (!(lo <= key0 && key0 + kBN <= hi)) {  // diagonal / window-edge / ragged block
#pragma unroll
            for (int c = 0; c < kBN; ++c) {
              const int key = key0 + c;
              if (key < lo || key >= hi) sr[c] = 0xFF800000u;  // -inf
            }
          }
          // row max: 8 independent partial maxima, 3-input max
          float pm[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) pm[i] = fmaxf(__uint_as_float(sr[i]), __uint_as_float(sr[8 + i]));
#pragma unroll
          for (int c = 16; c < kBN; c += 16)
#pragma unroll
            for (int i = 0; i < 8; ++i)
              pm[i] = max3(pm[i], __uint_as_float(sr[c + i]), __uint_as_float(sr[c + 8 + i]));
          const float mx = fmaxf(max3(pm[0], pm[1], pm[2]), max3(max3(pm[3], pm[4], pm[5]), pm[6], pm[7]));
          const float m_blk = mx * sl2;
          float alpha = 1.f;
          if (m_blk > m_run + thr) {
            alpha = ex2_approx(m_run - m_blk);  // m_run = -inf -> 0
            m_run = m_blk;
          }
          l_run *= alpha;
          l_rnd *= alpha;
          const float neg_m = (m_run == -INFINITY) ? 0.f : shift - m_run;
          const uint64_t sc2 = f2(sl2, sl2), nm2 = f2(neg_m, neg_m);
          // P = 2^(s * scale * log2e - m); exact (and rounded) row sums in
          // four independent packed accumulators each.
          uint64_t rs2[4] = {0, 0, 0, 0}, rr2[4] = {0, 0, 0, 0};
          uint32_t pk[kBN / 2];     // P of the block, packed for the MMA
          uint32_t pk_lo[kBN / 2];  // fine tiles: the rounding residual of P
          // Rescale the accumulator when the running max moved.  The previous
          // P.V of this tile has completed: it was issued before this S.
          auto rescale_o = [&]() {
            const bool need = (j > 0) && (alpha != 1.f);
            if (__any_sync(0xffffffffu, need)) {
#pragma unroll
              for (int c = 0; c < D / 32; ++c) {
                uint32_t raw[32];
                tmem_ld32(tO + c * 32, raw);
#pragma unroll
                for (int i = 0; i < 32; ++i) raw[i] = __float_as_uint(__uint_as_float(raw[i]) * alpha);
                tmem_st32(tO + c * 32, raw);
              }
            }
          };
          // P of pairs [Q_LO, Q_HI) into TMEM: bf16 one key pair per column,
          // e4m3 two pairs (and in fine tiles the residual kFineCol columns
          // on; e5m2 tiles are always fine).
          auto p_part = [&](auto q_lo_c, auto q_hi_c) {
            constexpr int Q_LO = decltype(q_lo_c)::value, Q_HI = decltype(q_hi_c)::value;
            constexpr int C0 = FP8 ? Q_LO / 2 : Q_LO, C1 = FP8 ? Q_HI / 2 : Q_HI;
            if (fine) {
              p_pairs_fine<FP8, kRsum, E5M2, Q_LO, Q_HI>(sr, sc2, nm2, rs2, rr2, pk, pk_lo, tS);
            } else {
              // (the exponent polynomial only in the kernels for plain tiles)
              // (plain tiles normalise by the exact sum: no rounded sum here)
              p_pairs<FP8, ATTN_ROUNDED_SUM != 0, false, Q_LO, Q_HI, false, FINE ? 0 : kEmuPairsPer8<FP8>>(
                  sr, sc2, nm2, rs2, rr2, pk, pk_lo);
              tmem_st_cols<C0, C1>(tS, pk);
            }
          };
          if (kSplitP) {
            p_part(IntC<0>{}, IntC<kSplitKeys / 2>{});
            rescale_o();
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&sm.p_half[t]);
            p_part(IntC<kSplitKeys / 2>{}, IntC<kBN / 2>{});
          } else {
            p_part(IntC<0>{}, IntC<kBN / 2>{});
            rescale_o();
          }
          {
            const uint64_t a = add2(add2(rs2[0], rs2[1]), add2(rs2[2], rs2[3]));
            float a0, a1;
            f2_split(a, a0, a1);
            l_run += a0 + a1;
            if (kRsum) {
              const uint64_t b = add2(add2(rr2[0], rr2[1]), add2(rr2[2], rr2[3]));
              float b0, b1;
              f2_split(b, b0, b1);
              l_rnd += b0 + b1;
            }
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&sm.p_full[t]);
        }
        if (!ok) break;
        // Hand the row statistics of this unit to the epilogue warpgroup, once
        // it has taken the previous unit's: a unit of one K/V block can finish
        // while the epilogue is still on the other tile of the unit before.
        if (nunit > 0) {
          ok = mbar_wait(&sm.st_empty[t], (nunit - 1) & 1, g);
          if (!ok) break;
        }
        sm.st_m[t][r] = m_run - shift;  // P carried 2^shift: LSE = m - shift + log2(sum)
        sm.st_l[t][r] = l_run;
        // rounded sum on fine tiles only: the other tiles of a FINE kernel
        // then agree bit for bit with the kernel built without it
        sm.st_r[t][r] = (kRsum && (fine || ATTN_ROUNDED_SUM)) ? l_rnd : l_run;
        mbar_arrive(&sm.st_full[t]);
        ++nunit;
      }
    }
    finish();
  }
}

// --------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
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

// [outer, rows, inner] row-major tensor, box of 128 rows x (128 bytes).
bool encode_3d(CUtensorMap* map, const void* base, bool fp8, uint64_t inner, uint64_t rows, uint64_t outer) {
  auto enc = get_encoder();
  if (!enc) return false;
  const uint64_t el = fp8 ? 1 : 2;
  cuuint64_t dims[3] = {inner, rows, outer};
  cuuint64_t strides[2] = {inner * el, inner * rows * el};
  cuuint32_t box[3] = {(cuuint32_t)(128 / el), (cuuint32_t)kBM, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The K/V page pool [num_pages * 16 tokens, Hkv, D] as a 3-D tensor, box =
// one page of one K/V head, 128 bytes of features (128-byte swizzle).
bool encode_pool(CUtensorMap* map, const void* pool, bool fp8, int D, int num_pages, int Hkv) {
  auto enc = get_encoder();
  if (!enc) return false;
  const uint64_t el = fp8 ? 1 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)num_pages * kPage};
  cuuint64_t strides[2] = {(cuuint64_t)D * el, (cuuint64_t)Hkv * D * el};
  cuuint32_t box[3] = {(cuuint32_t)(128 / el), 1, (cuuint32_t)kPage};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pool),
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// L2 budget of one chunk of units' K and V (the rest of L2 holds the Q and O
// streams and the other CTAs' K/V in flight).
#ifndef ATTN_CHUNK_L2_MB
#define ATTN_CHUNK_L2_MB 32
#endif
constexpr double kChunkL2Bytes = ATTN_CHUNK_L2_MB * 1048576.0;

// Visible-key count of query row i on the host, as key_range().
int host_key_count(int i, int lk, const PrefillArgs& a) {
  if (!a.causal) return lk;
  int h = i + (lk - a.Lq) + 1;
  h = h < 0 ? 0 : (h > lk ? lk : h);
  const int lo = (a.window > 0 && h - a.window > 0) ? h - a.window : 0;
  return h - lo;
}

// dependent: launch as a programmatic dependent of the kernel before it in the
// stream (it reads nothing that kernel writes, and waits for it before exit).
template <int D, bool FP8, bool PAGED, bool E5M2, bool FINE>
int launch_range(const PrefillArgs& a, Params p, int mg_lo, int mg_hi, const CUtensorMap& tq,
                 const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t stream, bool dependent = false) {
  using C = Cfg<D, FP8, E5M2>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail_cuda("cudaGetDevice", err);
  if (dev < 64 && !attr_set[dev]) {
    err = cudaFuncSetAttribute(prefill_kernel<D, FP8, PAGED, E5M2, FINE>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (err != cudaSuccess) return fail_cuda("prefill: cudaFuncSetAttribute", err);
    attr_set[dev] = true;
  }
  p.mg_hi = mg_hi;
  p.n_units = p.n_pairs * (mg_hi - mg_lo);
  // The loads carry L2 policies (Q evict-first, K/V evict-last) and O goes
  // out with streaming stores: K/V stay in L2 for the other units that read
  // them.  On the GQA causal workload that cut the reads from 308 to 245 MB
  // per launch (traffic 1.24x -> 1.01x of the algorithmic bytes) at the same
  // speed (1,041 against 1,035 TFLOP/s, interleaved).
  // With MHA (every query head its own K/V head) the CTAs working at one
  // time, spread over the row groups of all heads, touch more K/V than L2
  // holds (the e4m3 workload read 3x its bytes).  There the units also go in
  // chunks of whole K/V heads whose K and V fit in kChunkL2Bytes: reads fell
  // to the algorithmic bytes and the e4m3 workload gained 2 % (1,482 against
  // 1,455 TFLOP/s, interleaved).  With GQA the K/V of all heads is a quarter
  // the size, and the chunking cost 4-7 % (991 against 1,032 TFLOP/s), so GQA
  // keeps the plain order.
  p.chunk = p.n_pairs;
  p.l2_hints = 1;
  if (p.group == 1) {
    const int lk = PAGED ? a.max_pages * kPage : a.Lk;
    const double kv_bytes = (double)lk * D * (FP8 ? 1 : 2) * 2;
    int heads = kv_bytes > 0 ? (int)(kChunkL2Bytes / kv_bytes) : p.n_pairs;
    heads = heads < 1 ? 1 : heads;
    p.chunk = heads > p.n_pairs ? p.n_pairs : heads;
  }
  const int grid = p.n_units < sm_count() ? p.n_units : sm_count();
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  err = cudaLaunchKernelEx(&cfg, prefill_kernel<D, FP8, PAGED, E5M2, FINE>, tq, tk, tv, p);
  if (err == cudaSuccess) err = cudaGetLastError();
  return err == cudaSuccess ? 0 : fail_cuda("prefill: launch", err);
}

template <int D, bool FP8, bool PAGED, bool E5M2 = false>
int run(const PrefillArgs& a, cudaStream_t stream) {
  Params p{};
  p.o = a.o;
  p.lse = a.lse;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.Lq = a.Lq;
  p.Lk = a.Lk;
  p.group = a.Hq / a.Hkv;
  p.pair_heads = (p.group % 2 == 0) ? 1 : 0;
  int n_mgroups;
  if (p.pair_heads) {
    p.n_pairs = a.B * (a.Hq / 2);
    n_mgroups = (a.Lq + kBM - 1) / kBM;
  } else {
    p.n_pairs = a.B * a.Hq;
    n_mgroups = (a.Lq + 2 * kBM - 1) / (2 * kBM);
  }
  p.causal = a.causal;
  p.window = a.window > 0 ? a.window : 0;
  const float log2e = 1.4426950408889634f;
  p.scale_log2 = a.scale * log2e * (FP8 ? a.q_descale * a.k_descale : 1.f);
  p.out_scale = FP8 ? a.v_descale : 1.f;

  p.status = device_status_word();
  if (!p.status) return fail_cuda("prefill: status word", cudaGetLastError());
  p.timeout_ns = wait_timeout_ns();
  p.stall = (debug_flags() & 2) ? 1 : 0;
  p.block_table = a.block_table;
  p.seq_lens = a.seq_lens;
  p.max_pages = a.max_pages;
  p.num_pages = a.num_pages;

  CUtensorMap tq, tk, tv;
  if constexpr (PAGED) {
    if (!encode_3d(&tq, a.q, FP8, D, a.Lq, (uint64_t)a.B * a.Hq))
      return fail_cuda("prefill: tensor map (q)", cudaErrorInvalidValue);
    if (!encode_pool(&tk, a.k, FP8, D, a.num_pages, a.Hkv) || !encode_pool(&tv, a.v, FP8, D, a.num_pages, a.Hkv))
      return fail_cuda("prefill: tensor map (pool)", cudaErrorInvalidValue);
    // Sequence lengths are device data: one launch that decides per tile.
    return launch_range<D, FP8, PAGED, E5M2, true>(a, p, 0, n_mgroups, tq, tk, tv, stream);
  } else {
    const bool have_k = a.Lk > 0;
    if (!encode_3d(&tq, a.q, FP8, D, a.Lq, (uint64_t)a.B * a.Hq))
      return fail_cuda("prefill: tensor map (q)", cudaErrorInvalidValue);
    // With no keys nothing is loaded from K/V; describe Q instead of an empty tensor.
    const void* kb = have_k ? a.k : a.q;
    const void* vb = have_k ? a.v : a.q;
    const int rows = have_k ? a.Lk : a.Lq;
    const uint64_t outer = have_k ? (uint64_t)a.B * a.Hkv : (uint64_t)a.B * a.Hq;
    if (!encode_3d(&tk, kb, FP8, D, rows, outer)) return fail_cuda("prefill: tensor map (k)", cudaErrorInvalidValue);
    if (!encode_3d(&tv, vb, FP8, D, rows, outer)) return fail_cuda("prefill: tensor map (v)", cudaErrorInvalidValue);
    if constexpr (FP8 && E5M2) {
      return launch_range<D, FP8, PAGED, E5M2, true>(a, p, 0, n_mgroups, tq, tk, tv, stream);
    } else {
      // Tiles that take the two-part product ("fine": the first row sees
      // fewer keys than the threshold) are the leading row groups: a row's key
      // count never decreases along the rows.  They run in a kernel built with
      // that product; the rest in one built without it, whose softmax and MMA
      // issue then carry none of its code (that code alone measured ~6 % on
      // the GQA causal workload).
      const int thr = FP8 ? kFineKeys : kFineKeysBf16;
      int mg_fine = 0;
      while (mg_fine < n_mgroups) {
        bool any = false;
        for (int t = 0; t < 2; ++t) {
          const int m0 = p.pair_heads ? mg_fine * kBM : (2 * mg_fine + t) * kBM;
          if (m0 < a.Lq && host_key_count(m0, a.Lk, a) < thr) any = true;
        }
        if (!any) break;
        ++mg_fine;
      }
      // The plain launch goes first; the few-key launch follows as its
      // programmatic dependent, so that its short units fill the SMs the
      // plain launch's tail leaves idle instead of running on their own.
      int st = 0;
      if (mg_fine < n_mgroups)
        st = launch_range<D, FP8, PAGED, E5M2, false>(a, p, mg_fine, n_mgroups, tq, tk, tv, stream);
      if (st == 0 && mg_fine > 0)
        st = launch_range<D, FP8, PAGED, E5M2, true>(a, p, 0, mg_fine, tq, tk, tv, stream, mg_fine < n_mgroups);
      return st;
    }
  }
}

}  // namespace

int launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
  if (a.paged) {  // bf16 pools only
    if (a.fp8) return -2;
    if (a.D == 128) return run<128, false, true>(a, stream);
    if (a.D == 64) return run<64, false, true>(a, stream);
    return -2;
  }
  if (a.fp8) {
    if (a.D != 128) return -2;
    return a.e5m2 ? run<128, true, false, true>(a, stream) : run<128, true, false>(a, stream);
  }
  if (a.D == 128) return run<128, false, false>(a, stream);
  if (a.D == 64) return run<64, false, false>(a, stream);
  return -2;
}

}  // namespace attn
