// prefill_wide_sm100.cu -- fused attention forward for head dimensions up to
// 256 and for queries/keys of another width than the values (D_qk != D_v),
// the shapes of attention in a latent space: queries and keys projected to a
// latent dimension of 64-256, values to their own dimension (latent
// projection of the page "高效多头潜在注意力解码技术：Flash MLA深度解析"
// (developer.baidu.com), §2.1).  bf16 inputs, for B200 (sm_100a).
//
// Same computation as prefill_sm100.cu (online softmax of the tiled
// FlashAttention loop, page "003-注意力机制详解..." §二; causal / window block
// skipping), with another tiling, because two 128-row accumulators of up to
// 256 columns do not fit the 512 TMEM columns of an SM:
//   * one 128-row Q tile per CTA; K/V blocks of 64 keys (a 64 x 256 bf16 tile
//     is 32 KB, so Q plus two K/V stages fit in shared memory at D = 256);
//   * TMEM: two S buffers of 64 columns and O of D_v columns.  While the
//     softmax warps work on block j in one S buffer, the tensor core computes
//     S of block j + 1 into the other, then O += P_j V_j.
// Roles (320 threads, one persistent CTA per SM):
//   warps 0-3  softmax, one thread per query row (= TMEM lane)
//   warps 4-7  epilogue: O = acc / sum to bf16 and the LSE, per unit
//   warp  8    TMA producer: Q tile, then K_j and V_j into a ring of stages
//   warp  9    MMA issuer (one thread) and TMEM owner
// Units are (batch, head, 128-row block), longest first (later rows of a
// causal mask see more keys), in snake order over the CTAs; the heads of one
// K/V group and row block are neighbours, so their K/V blocks meet in L2.
#include <cfloat>
#include <climits>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace attn {
namespace {

constexpr int kBM = 128;          // query rows per tile
constexpr int kBN = 64;           // keys per K/V block
constexpr int kThreads = 320;
constexpr float kRescaleThreshold = 8.0f;  // log2 units (lazy rescale, as prefill_sm100.cu)
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kTmS0 = 0, kTmS1 = kBN, kTmO = 2 * kBN;
constexpr int kMaxStages = 4;
// Tiles whose first row (the row with the fewest keys) sees fewer than
// kFineKeys keys multiply V by P in two bf16 parts, P rounded and the rounding
// residual (TMEM columns 32-63 of the S buffer; P of 64 keys fills 0-31), so
// the weights of rows of a few keys carry ~16 bits: rounding P to bf16 alone
// moves such a row's O by up to ~2^-9 of the spread of its V values, which
// with the bf16 rounding of O can pass 1e-2.  Rows of many keys average it out.
constexpr int kFineKeys = 256;
constexpr uint32_t kFineCol = 32;

template <int DQK, int DV>
struct WCfg {
  static constexpr int Q_BOX = kBM * 128;                 // one 64-column box of the Q tile: 16 KB
  static constexpr int KV_BOX = kBN * 128;                // one 64-column box of a K or V block: 8 KB
  static constexpr int Q_BYTES = (DQK / 64) * Q_BOX;
  static constexpr int K_BYTES = (DQK / 64) * KV_BOX;
  static constexpr int V_BYTES = (DV / 64) * KV_BOX;
  static constexpr int BAR_BYTES = 4096;
  static constexpr int NS_FIT = (232448 - 1024 - BAR_BYTES - Q_BYTES) / (K_BYTES + V_BYTES);
  static constexpr int NS = NS_FIT < kMaxStages ? NS_FIT : kMaxStages;  // K/V ring stages
  static constexpr int SMEM_TILES = Q_BYTES + NS * (K_BYTES + V_BYTES);
  // Each CTA allocates all 512 TMEM columns, so a second CTA must never fit on
  // an SM (its allocation would wait): at least half the SM's shared memory.
  static constexpr int SMEM_MIN_ONE_CTA = 233472 / 2 - 1024 + 16;
  static constexpr int SMEM_NEED = SMEM_TILES + 1024 + BAR_BYTES;
  static constexpr int SMEM_BYTES = SMEM_NEED > SMEM_MIN_ONE_CTA ? SMEM_NEED : SMEM_MIN_ONE_CTA;
  static constexpr uint32_t IDESC_S = make_idesc(1u, kBM, kBN, false);  // bf16, K-major B
  static constexpr uint32_t IDESC_PV = make_idesc(1u, kBM, DV, true);   // bf16, V MN-major
  static_assert(DQK % 64 == 0 && DV % 64 == 0 && DQK <= 256 && DV <= 256, "64..256 in steps of 64");
  static_assert(NS >= 2, "at least two K/V stages");
  static_assert(SMEM_BYTES <= 232448, "more than the 227 KB a CTA may use");
  static_assert(kTmO + DV <= 512, "TMEM budget");
};

struct WParams {
  void* o;
  float* lse;
  int B, Hq, Hkv, Lq, Lk, group;
  int n_mblocks, n_units;
  int causal, window;
  float scale_log2;
  int* status;
  unsigned long long timeout_ns;
  int stall;
};

struct WUnit {
  int bh, m0, kvbh, kb_lo, nb;
};

__device__ __forceinline__ void wkey_range(int i, const WParams& p, int& lo, int& hi) {
  if (!p.causal) {
    lo = 0;
    hi = p.Lk;
    return;
  }
  int h = i + (p.Lk - p.Lq) + 1;
  h = h < 0 ? 0 : (h > p.Lk ? p.Lk : h);
  hi = h;
  lo = (p.window > 0 && h - p.window > 0) ? h - p.window : 0;
}

// Unit u: row blocks from the last (longest under a causal mask) to the first;
// within a row block, batch-major then head.
__device__ __forceinline__ WUnit wget_unit(int u, const WParams& p) {
  WUnit w;
  const int per_mb = p.B * p.Hq;
  const int mb = p.n_mblocks - 1 - u / per_mb;
  const int r = u % per_mb;
  const int b = r / p.Hq, h = r % p.Hq;
  w.bh = b * p.Hq + h;
  w.kvbh = b * p.Hkv + h / p.group;
  w.m0 = mb * kBM;
  const int r_last = min(w.m0 + kBM - 1, p.Lq - 1);
  int lo0, hi0, lo1, hi1;
  wkey_range(w.m0, p, lo0, hi0);
  wkey_range(r_last, p, lo1, hi1);
  const int lo = lo0, hi = hi1;  // lo and hi are non-decreasing in the row
  if (hi <= lo || hi1 <= lo0) {
    w.kb_lo = 0;
    w.nb = 0;
  } else {
    w.kb_lo = lo / kBN;
    w.nb = (hi + kBN - 1) / kBN - w.kb_lo;
  }
  return w;
}

__device__ __forceinline__ bool wtile_fine(const WUnit& w, const WParams& p) {
  int lo, hi;
  wkey_range(w.m0, p, lo, hi);
  return hi - lo < kFineKeys;
}

__device__ __forceinline__ int wunit_of(int round, int n_units) {
  const int g = (int)gridDim.x, c = (int)blockIdx.x;
  const int u = round * g + ((round & 1) ? g - 1 - c : c);
  return u < n_units ? u : n_units;
}

struct WSmem {
  uint64_t q_full, q_empty;
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done;
  uint64_t o_full, o_empty;
  uint64_t st_full, st_empty;
  uint64_t drain;
  // K and V halves of a stage are released separately: K once its S product
  // completes, V after P V, so the next K loads while P V still runs.
  uint64_t k_full[kMaxStages], v_full[kMaxStages], k_empty[kMaxStages], v_empty[kMaxStages];
  uint32_t tmem_base;
  int abort_flag;
  float st_m[kBM], st_l[kBM], st_r[kBM];
};
static_assert(sizeof(WSmem) <= 4096, "barrier/statistics block exceeds its reserve");

template <int DQK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_wide_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const WParams p) {
  using C = WCfg<DQK, DV>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t tiles_addr = (raw_addr + 1023u) & ~1023u;
  uint8_t* tiles_ptr = smem_raw + (tiles_addr - raw_addr);
  WSmem& sm = *reinterpret_cast<WSmem*>(tiles_ptr + C::SMEM_TILES);
  const uint32_t q_addr = tiles_addr;
  auto k_addr = [&](uint32_t s) { return tiles_addr + C::Q_BYTES + s * (uint32_t)(C::K_BYTES + C::V_BYTES); };
  auto v_addr = [&](uint32_t s) { return k_addr(s) + C::K_BYTES; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.p_full[b], 128);
    }
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.o_empty, 128);
    mbar_init(&sm.st_full, 128);
    mbar_init(&sm.st_empty, 128);
    mbar_init(&sm.drain, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_empty[s], 1);
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

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t seq = 0, nunit = 0;
      bool ok = !p.stall;
      // Q is read once per unit, K/V by every unit of the group and row
      // range: Q evict-first, K/V evict-last in L2 (O goes out streaming).
      // Grouping the units into L2-sized chunks of K/V heads as well cut the
      // 256-wide workload's DRAM reads from 1.62 to 0.41 GB per launch but
      // ran 3-7 % slower; these policies alone cost nothing (1.53-1.60 GB).
      const uint64_t pol_q = l2_policy_evict_first(), pol_kv = l2_policy_evict_last();
      for (int rnd = 0, u = wunit_of(0, p.n_units); u < p.n_units && ok; u = wunit_of(++rnd, p.n_units)) {
        const WUnit w = wget_unit(u, p);
        if (w.nb <= 0) continue;
        if (nunit > 0) ok = mbar_wait(&sm.q_empty, (nunit - 1) & 1, g);
        if (!ok) break;
        mbar_arrive_expect_tx(&sm.q_full, C::Q_BYTES);
#pragma unroll
        for (int bx = 0; bx < DQK / 64; ++bx)
          tma_load_3d_hint(q_addr + bx * C::Q_BOX, &tm_q, &sm.q_full, bx * 64, w.m0, w.bh, pol_q);
        for (int j = 0; j < w.nb && ok; ++j) {
          const int key0 = (w.kb_lo + j) * kBN;
          const uint32_t s = seq % C::NS;
          if (seq >= (uint32_t)C::NS) {
            ok = mbar_wait(&sm.k_empty[s], ((seq / C::NS) - 1) & 1, g);
            if (!ok) break;
          }
          mbar_arrive_expect_tx(&sm.k_full[s], C::K_BYTES);
#pragma unroll
          for (int bx = 0; bx < DQK / 64; ++bx)
            tma_load_3d_hint(k_addr(s) + bx * C::KV_BOX, &tm_k, &sm.k_full[s], bx * 64, key0, w.kvbh, pol_kv);
          if (seq >= (uint32_t)C::NS) {
            ok = mbar_wait(&sm.v_empty[s], ((seq / C::NS) - 1) & 1, g);
            if (!ok) break;
          }
          mbar_arrive_expect_tx(&sm.v_full[s], C::V_BYTES);
#pragma unroll
          for (int bx = 0; bx < DV / 64; ++bx)
            tma_load_3d_hint(v_addr(s) + bx * C::KV_BOX, &tm_v, &sm.v_full[s], bx * 64, key0, w.kvbh, pol_kv);
          ++seq;
        }
        ++nunit;
      }
      // Drain: every load this thread issued has landed before the CTA exits.
      for (uint32_t s = 0; s < (uint32_t)C::NS && s < seq; ++s) {
        const uint32_t last = s + ((seq - 1 - s) / C::NS) * C::NS;
        mbar_wait(&sm.k_full[s], (last / C::NS) & 1, g_drain);
        mbar_wait(&sm.v_full[s], (last / C::NS) & 1, g_drain);
      }
      if (nunit > 0) mbar_wait(&sm.q_full, (nunit - 1) & 1, g_drain);
    }
  } else if (warp == 9) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0) {
      uint32_t seq = 0, nunit = 0, gblk = 0;
      bool ok = true;
      // S = Q K^T into S buffer b: K-major operands, 64-column boxes
      // (Q_BOX / KV_BOX bytes apart), k-step kk = 16 columns = 32 bytes.
      auto issue_s = [&](uint32_t b, uint32_t s) {
        const uint64_t a0 = sw128_desc(q_addr, 16, 1024);
        const uint64_t b0 = sw128_desc(k_addr(s), 16, 1024);
        const uint32_t d = tmem + (b ? kTmS1 : kTmS0);
#pragma unroll
        for (int kk = 0; kk < DQK / 16; ++kk) {
          const uint32_t byte_k = kk * 32;
          const uint32_t offa = ((byte_k / 128) * C::Q_BOX + (byte_k % 128)) >> 4;
          const uint32_t offb = ((byte_k / 128) * C::KV_BOX + (byte_k % 128)) >> 4;
          mma_f16_ss(d, a0 + offa, b0 + offb, C::IDESC_S, kk > 0);
        }
      };
      // O (+)= P V: P (bf16) from TMEM over S buffer b, V MN-major with its
      // 64-feature column groups KV_BOX bytes apart; k-step = 16 keys.
      auto issue_pv = [&](uint32_t b, uint32_t s, bool acc, uint32_t a_col) {
        const uint64_t b0 = sw128_desc(v_addr(s), C::KV_BOX, 1024);
        const uint32_t a_base = tmem + (b ? kTmS1 : kTmS0) + a_col;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_f16_ts(tmem + kTmO, a_base + kk * 8, b0 + ((kk * 16 * 128) >> 4), C::IDESC_PV,
                     (acc || kk > 0) ? 1u : 0u);
      };
      for (int rnd = 0, u = wunit_of(0, p.n_units); u < p.n_units && ok; u = wunit_of(++rnd, p.n_units)) {
        const WUnit w = wget_unit(u, p);
        if (w.nb <= 0) continue;
        const bool fine = wtile_fine(w, p);
        ok = mbar_wait(&sm.q_full, nunit & 1, g);
        if (!ok) break;
        {
          const uint32_t s0 = seq % C::NS;
          ok = mbar_wait(&sm.k_full[s0], (seq / C::NS) & 1, g);
          if (!ok) break;
          tc_fence_after();
          issue_s(gblk & 1, s0);
          tc_commit(&sm.s_full[gblk & 1]);
          tc_commit(&sm.k_empty[s0]);
          if (w.nb == 1) tc_commit(&sm.q_empty);
        }
        for (int j = 0; j < w.nb && ok; ++j) {
          const uint32_t gc = gblk + j;
          const uint32_t s = (seq + j) % C::NS;
          if (j + 1 < w.nb) {
            // S of the next block into the other buffer: its last reader
            // (P V of block j - 1) was issued earlier, and MMAs run in order.
            const uint32_t sn = (seq + j + 1) % C::NS;
            ok = mbar_wait(&sm.k_full[sn], ((seq + j + 1) / C::NS) & 1, g);
            if (!ok) break;
            tc_fence_after();
            issue_s((gc + 1) & 1, sn);
            tc_commit(&sm.s_full[(gc + 1) & 1]);
            tc_commit(&sm.k_empty[sn]);
            if (j + 2 == w.nb) tc_commit(&sm.q_empty);  // last reader of Q issued
          }
          ok = mbar_wait(&sm.p_full[gc & 1], (gc >> 1) & 1, g);
          if (!ok) break;
          if (j == 0 && nunit > 0) {
            ok = mbar_wait(&sm.o_empty, (nunit - 1) & 1, g);
            if (!ok) break;
          }
          ok = mbar_wait(&sm.v_full[s], ((seq + j) / C::NS) & 1, g);
          if (!ok) break;
          tc_fence_after();
          issue_pv(gc & 1, s, j > 0, 0);
          if (fine) issue_pv(gc & 1, s, true, kFineCol);
          tc_commit(&sm.pv_done);
          tc_commit(&sm.v_empty[s]);
        }
        if (!ok) break;
        tc_commit(&sm.o_full);
        seq += w.nb;
        gblk += w.nb;
        ++nunit;
      }
      tc_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, g_drain);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int r = ((warp & 3) << 5) + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) << 5) << 16;
    uint32_t nunit = 0;
    bool ok = true;
    for (int rnd = 0, u = wunit_of(0, p.n_units); u < p.n_units && ok; u = wunit_of(++rnd, p.n_units)) {
      const WUnit w = wget_unit(u, p);
      const int row = w.m0 + r;
      const bool row_valid = row < p.Lq;
      float m = -INFINITY, l = 0.f, lr = 0.f;
      if (w.nb > 0) {
        ok = mbar_wait(&sm.st_full, nunit & 1, g) && mbar_wait(&sm.o_full, nunit & 1, g);
        if (!ok) break;
        tc_fence_after();
        m = sm.st_m[r];
        l = sm.st_l[r];
        lr = sm.st_r[r];
        mbar_arrive(&sm.st_empty);
      }
      const float inv = lr > 0.f ? 1.f / lr : 0.f;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + ((size_t)w.bh * p.Lq + row) * DV;
#pragma unroll 1
      for (int c = 0; c < DV / 16; ++c) {
        uint32_t raw[16];
        if (w.nb > 0) {
          tmem_ld16(tmem + kTmO + lane_off + c * 16, raw);
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
          __stcs(dst, make_uint4(pk[0], pk[1], pk[2], pk[3]));
          __stcs(dst + 1, make_uint4(pk[4], pk[5], pk[6], pk[7]));
        }
      }
      if (row_valid && p.lse != nullptr)
        p.lse[(size_t)w.bh * p.Lq + row] = (l > 0.f) ? (m + log2f(l)) * kLn2 : -INFINITY;
      if (w.nb > 0) {
        tc_fence_before();
        mbar_arrive(&sm.o_empty);
        ++nunit;
      }
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int r = (warp << 5) + lane;  // row within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(warp << 5) << 16;
    const float sl2 = p.scale_log2;
    uint32_t gblk = 0, nunit = 0;
    bool ok = true;
    for (int rnd = 0, u = wunit_of(0, p.n_units); u < p.n_units && ok; u = wunit_of(++rnd, p.n_units)) {
      const WUnit w = wget_unit(u, p);
      if (w.nb <= 0) continue;
      const int row = w.m0 + r;
      int lo, hi;
      wkey_range(row, p, lo, hi);
      const bool fine = wtile_fine(w, p);
      // exact fp32 row sum (LSE) and sum of the bf16-rounded P (normalises O)
      float m_run = -INFINITY, l_run = 0.f, l_rnd = 0.f;
      for (int j = 0; j < w.nb; ++j) {
        const uint32_t gc = gblk + j;
        const uint32_t tS = tmem + ((gc & 1) ? kTmS1 : kTmS0) + lane_off;
        ok = mbar_wait(&sm.s_full[gc & 1], (gc >> 1) & 1, g);
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[kBN];
        tmem_ld64(tS, sr);
        const int key0 = (w.kb_lo + j) * kBN;
        if (!(lo <= key0 && key0 + kBN <= hi)) {
#pragma unroll
          for (int c = 0; c < kBN; ++c) {
            const int key = key0 + c;
            if (key < lo || key >= hi) sr[c] = 0xFF800000u;  // -inf
          }
        }
        float pm[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pm[i] = fmaxf(__uint_as_float(sr[i]), __uint_as_float(sr[8 + i]));
#pragma unroll
        for (int c = 16; c < kBN; c += 16)
#pragma unroll
          for (int i = 0; i < 8; ++i) pm[i] = max3(pm[i], __uint_as_float(sr[c + i]), __uint_as_float(sr[c + 8 + i]));
        const float mx = fmaxf(max3(pm[0], pm[1], pm[2]), max3(max3(pm[3], pm[4], pm[5]), pm[6], pm[7]));
        const float m_blk = mx * sl2;
        float alpha = 1.f;
        if (m_blk > m_run + kRescaleThreshold) {
          alpha = ex2_approx(m_run - m_blk);  // m_run = -inf -> 0
          m_run = m_blk;
        }
        l_run *= alpha;
        l_rnd *= alpha;
        // The accumulator moved with the max: wait for the previous block's
        // P V (the completion of pv_done phase gc - 1), then rescale O.
        const bool need = (j > 0) && (alpha != 1.f);
        if (__any_sync(0xffffffffu, need)) {
          ok = mbar_wait(&sm.pv_done, (gc - 1) & 1, g);
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < DV / 32; ++c) {
            uint32_t raw[32];
            tmem_ld32(tmem + kTmO + lane_off + c * 32, raw);
#pragma unroll
            for (int i = 0; i < 32; ++i) raw[i] = __float_as_uint(__uint_as_float(raw[i]) * alpha);
            tmem_st32(tmem + kTmO + lane_off + c * 32, raw);
          }
        }
        const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
        const uint64_t sc2 = f2(sl2, sl2), nm2 = f2(neg_m, neg_m);
        uint64_t rs2[4] = {0, 0, 0, 0}, rr2[4] = {0, 0, 0, 0};
        uint32_t pk[kBN / 2];
        if (fine) {
#pragma unroll
          for (int q2 = 0; q2 < kBN / 2; ++q2) {
            const uint64_t x2 = fma2(f2(__uint_as_float(sr[2 * q2]), __uint_as_float(sr[2 * q2 + 1])), sc2, nm2);
            float x0, x1;
            f2_split(x2, x0, x1);
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            rs2[q2 & 3] = add2(rs2[q2 & 3], f2(p0, p1));
            const uint32_t bb = pack_bf16x2(p0, p1);
            const float h0 = __uint_as_float(bb << 16), h1 = __uint_as_float(bb & 0xFFFF0000u);
            const uint32_t bl = pack_bf16x2(p0 - h0, p1 - h1);  // P - h is exact in fp32
            pk[q2] = bb;
            sr[q2] = bl;  // the scores of pairs < q2 are spent: reuse their registers
            rr2[q2 & 3] = add2(rr2[q2 & 3], f2(h0 + __uint_as_float(bl << 16),
                                               h1 + __uint_as_float(bl & 0xFFFF0000u)));
          }
          tmem_st32(tS + kFineCol, *reinterpret_cast<const uint32_t(*)[32]>(sr));
        } else {
#pragma unroll
          for (int q2 = 0; q2 < kBN / 2; ++q2) {
            const uint64_t x2 = fma2(f2(__uint_as_float(sr[2 * q2]), __uint_as_float(sr[2 * q2 + 1])), sc2, nm2);
            float x0, x1;
            f2_split(x2, x0, x1);
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            rs2[q2 & 3] = add2(rs2[q2 & 3], f2(p0, p1));
            const uint32_t bb = pack_bf16x2(p0, p1);
            pk[q2] = bb;
            rr2[q2 & 3] = add2(rr2[q2 & 3], f2(__uint_as_float(bb << 16), __uint_as_float(bb & 0xFFFF0000u)));
          }
        }
        tmem_st32(tS, pk);
        {
          float a0, a1, b0, b1;
          f2_split(add2(add2(rs2[0], rs2[1]), add2(rs2[2], rs2[3])), a0, a1);
          f2_split(add2(add2(rr2[0], rr2[1]), add2(rr2[2], rr2[3])), b0, b1);
          l_run += a0 + a1;
          l_rnd += b0 + b1;
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&sm.p_full[gc & 1]);
      }
      if (!ok) break;
      gblk += w.nb;
      if (nunit > 0) {
        ok = mbar_wait(&sm.st_empty, (nunit - 1) & 1, g);
        if (!ok) break;
      }
      sm.st_m[r] = m_run;
      sm.st_l[r] = l_run;
      sm.st_r[r] = l_rnd;
      mbar_arrive(&sm.st_full);
      ++nunit;
    }
  }
  // Teardown: all threads meet, then the owner warp releases TMEM.
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// [outer, rows, inner] row-major bf16 tensor, box of `box_rows` rows x 64
// elements (128 bytes, 128-byte swizzle).
bool encode_wide(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t outer,
                 uint32_t box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if (!enc) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  cuuint64_t dims[3] = {inner, rows, outer};
  cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DQK, int DV>
int run_wide(const WideArgs& a, cudaStream_t stream) {
  using C = WCfg<DQK, DV>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail_cuda("cudaGetDevice", err);
  if (dev < 64 && !attr_set[dev]) {
    err = cudaFuncSetAttribute(prefill_wide_kernel<DQK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM_BYTES);
    if (err != cudaSuccess) return fail_cuda("prefill (wide): cudaFuncSetAttribute", err);
    attr_set[dev] = true;
  }
  WParams p{};
  p.o = a.o;
  p.lse = a.lse;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.Lq = a.Lq;
  p.Lk = a.Lk;
  p.group = a.Hq / a.Hkv;
  p.n_mblocks = (a.Lq + kBM - 1) / kBM;
  p.n_units = a.B * a.Hq * p.n_mblocks;
  p.causal = a.causal;
  p.window = a.window > 0 ? a.window : 0;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.status = device_status_word();
  if (!p.status) return fail_cuda("prefill (wide): status word", cudaGetLastError());
  p.timeout_ns = wait_timeout_ns();
  p.stall = (debug_flags() & 2) ? 1 : 0;
  CUtensorMap tq, tk, tv;
  const bool have_k = a.Lk > 0;
  // With no keys nothing is loaded from K/V; describe Q instead of an empty tensor.
  if (!encode_wide(&tq, a.q, DQK, a.Lq, (uint64_t)a.B * a.Hq, kBM) ||
      !encode_wide(&tk, have_k ? a.k : a.q, DQK, have_k ? a.Lk : a.Lq,
                   have_k ? (uint64_t)a.B * a.Hkv : (uint64_t)a.B * a.Hq, kBN) ||
      !encode_wide(&tv, have_k ? a.v : a.q, have_k ? DV : DQK, have_k ? a.Lk : a.Lq,
                   have_k ? (uint64_t)a.B * a.Hkv : (uint64_t)a.B * a.Hq, kBN))
    return fail_cuda("prefill (wide): tensor map", cudaErrorInvalidValue);
  const int grid = p.n_units < sm_count() ? p.n_units : sm_count();
  prefill_wide_kernel<DQK, DV><<<grid, kThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  err = cudaGetLastError();
  return err == cudaSuccess ? 0 : fail_cuda("prefill (wide): launch", err);
}

template <int DQK>
int run_wide_dv(const WideArgs& a, cudaStream_t stream) {
  switch (a.Dv) {
    case 64: return run_wide<DQK, 64>(a, stream);
    case 128: return run_wide<DQK, 128>(a, stream);
    case 192: return run_wide<DQK, 192>(a, stream);
    case 256: return run_wide<DQK, 256>(a, stream);
    default: return -2;
  }
}

}  // namespace

int launch_prefill_wide(const WideArgs& a, cudaStream_t stream) {
  switch (a.Dqk) {
    case 64: return run_wide_dv<64>(a, stream);
    case 128: return run_wide_dv<128>(a, stream);
    case 192: return run_wide_dv<192>(a, stream);
    case 256: return run_wide_dv<256>(a, stream);
    default: return -2;
  }
}

}  // namespace attn
