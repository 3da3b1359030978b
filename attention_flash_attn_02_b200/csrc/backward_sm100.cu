// backward_sm100.cu -- attention backward (dQ, dK, dV) for B200 (sm_100a).
//
// The backward recomputes the attention weights from the forward's per-row
// LSE instead of storing them (the recomputation of the tqpw.cn article
// §4.1): with P = exp(scale * Q K^T - LSE) (masked entries 0) and
// Dvec = rowsum(dO * O),
//     dV = P^T dO,   dP = dO V^T,   dS = P * (dP - Dvec),
//     dQ = scale * dS K,   dK = scale * dS^T Q.
//
// Three launches:
//   bwd_pre_kernel    one warp per query row: Dvec, the LSE in log2 units
//                     (+inf for rows without keys or past Lq, so their P is
//                     0) and a zeroed fp32 dQ accumulator row.
//   bwd_kernel        one CTA per 128-key K/V tile of one K/V head, looping
//                     over the query heads of its group and the 128-row
//                     query blocks that see the tile.  Per CTA:
//       warp 8       TMA producer and reducer, one thread: K_j and V_j
//                    once; per step the Q_i and dO_i tiles (double
//                    buffered), each loaded into its buffer right after that
//                    buffer's dQ staging from two steps back has been added
//                    to the fp32 dQ accumulator by a bulk tensor reduction
//                    (the loads then do not queue behind other reductions).
//       warp 9       TMEM owner; one thread issues per step
//                      dP^T = V_j dO_i^T                        (TMEM),
//                    then, once P^T and dS^T are written back,
//                      dV += P^T dO_i                           (A from TMEM)
//                      S^T = K_j Q_{i'}^T of the next step (if Q_{i'} is in)
//                      dK += dS^T Q_i                           (A from TMEM)
//                      dQ_i = dS K_j                            (A from smem)
//                    so that the next P^T is formed while dK and dQ_i run.
//       warps 0-7    two warps per TMEM lane quadrant, each over 64 of the
//                    block's 128 queries: P^T of the warp's keys (one thread
//                    per key = TMEM lane) as soon as S^T is there, back to
//                    TMEM as bf16; the previous step's dQ_i, whenever it is
//                    complete, from TMEM (one thread per query row, half of
//                    the features each) into 128-byte-swizzled fp32 staging
//                    boxes in that step's Q buffer (first half of the
//                    features) and dO buffer (second half), which no product
//                    reads once dQ_i is done; then dS^T once dP^T is there,
//                    back to TMEM, and dS (bf16) into a swizzled shared-memory
//                    tile.  At the end each writes its half of dK (times
//                    scale) and dV.
//   bwd_post_kernel   dQ = bf16(scale * accumulator).
// TMEM (512 columns): [0,128) S^T, then P^T packed over columns 0-31 (queries
// 0-63) and 64-95 (queries 64-127); [128,256) dP^T, then dS^T packed the same
// way, then dQ_i; [256,384) dV; [384,512) dK.  So the next step's S^T can be
// computed, and its P^T formed, while dK and dQ_i run and dQ_i is read out;
// only dP^T waits for the read-out.
// Every operand tile is a 128-row, 128-byte-swizzled TMA tile, used K-major
// or MN-major by its descriptor; dS is stored [key][query] so that dQ reads
// it MN-major.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <climits>
#include <cstdint>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace attn {
namespace {

constexpr int kT = 128;          // keys per K/V tile, query rows per Q block
constexpr int kThreads = 384;    // 12 warps
constexpr float kLog2e = 1.4426950408889634f;

// Instruction descriptor (kind::f16, bf16 operands, fp32 accumulator) with
// both major-ness bits: A MN-major (bit 15), B MN-major (bit 16).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

template <int D>
struct BCfg {
  static constexpr int NBOX = D * 2 / 128;               // 64-feature boxes per row
  static constexpr int BOX_BYTES = kT * 128;             // 128 rows x 128 B
  static constexpr int TILE_BYTES = kT * D * 2;          // one 128 x D bf16 tile
  // shared memory: K, V, Q[2], dO[2], dS (each a tile), then small arrays
  static constexpr int OFF_K = 0, OFF_V = TILE_BYTES, OFF_Q = 2 * TILE_BYTES, OFF_DO = 4 * TILE_BYTES;
  static constexpr int OFF_DS = 6 * TILE_BYTES;
  static constexpr int DS_BYTES = kT * kT * 2;           // [128 keys][128 queries] bf16
  static constexpr int SMEM_TILES = OFF_DS + DS_BYTES;
  static constexpr int SMEM_BYTES = 232448;  // all a CTA may use: the tiles, then the small arrays
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 384;
  static constexpr uint32_t ID_S = idesc_bf16(kT, kT, false, false);   // K-major x K-major
  static constexpr uint32_t ID_ACC = idesc_bf16(kT, D, false, true);   // TMEM A, B MN-major
  static constexpr uint32_t ID_DQ = idesc_bf16(kT, D, true, true);     // A and B MN-major
};

struct BParams {
  const float* lse2;   // [B*Hq*Lq] LSE * log2(e), +inf where P must be 0
  const float* dvec;   // [B*Hq*Lq] rowsum(dO * O)
  float* dq_acc;       // [B*Hq*Lq][D] fp32
  __nv_bfloat16* dk;   // [B*Hkv*Lk][D]
  __nv_bfloat16* dv;
  int B, Hq, Hkv, Lq, Lk, group, n_kt;
  int causal, window;
  float scale, scale_log2;
  int* status;
  unsigned long long timeout_ns;
};

struct BSmem {
  uint64_t kv_full, q_full[2], do_full[2];
  uint64_t s_full, dp_full, p_full, dq_full, dq_empty, fin, drain;
  uint64_t stat[2];  // [step & 1]: the step's LSE/Dvec written to shared memory (128 arrivals)
  uint64_t stg_q[2], stg_do[2];  // [step & 1]: a half of the step's dQ staged (128 arrivals each)
  uint32_t tmem_base;
  int abort_flag;
  float lse2[2][kT];  // [buffer][query]
  float dvec[2][kT];
};

// Query rows [r_lo, r_hi) that see some key of tile [k0, k1) (bottom-right
// causal alignment, window of W keys including the query's own position).
__device__ __forceinline__ void query_range(const BParams& p, int k0, int k1, int& r_lo, int& r_hi) {
  if (!p.causal) {
    r_lo = 0;
    r_hi = p.Lq;
    return;
  }
  const int off = p.Lk - p.Lq;  // row r sees keys <= r + off
  r_lo = k0 - off;
  r_hi = p.window > 0 ? (k1 - 1) - off + p.window : p.Lq;  // row r sees keys >= r + off - W + 1
  r_lo = r_lo < 0 ? 0 : r_lo;
  r_hi = r_hi > p.Lq ? p.Lq : r_hi;
}

// The dQ staging (D/32 fp32 boxes of 128 rows x 32 features) fills the step's
// dO and Q buffers exactly.
static_assert(BCfg<128>::TILE_BYTES == 2 * BCfg<128>::BOX_BYTES && BCfg<64>::TILE_BYTES == BCfg<64>::BOX_BYTES,
              "dQ staging fills the step's dO and Q buffers");

template <int D>
constexpr bool bwd_fits() {
  return BCfg<D>::SMEM_TILES + (int)sizeof(BSmem) <= BCfg<D>::SMEM_BYTES;
}
static_assert(bwd_fits<128>() && bwd_fits<64>(), "tiles and barriers exceed the shared memory of a CTA");

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_dq, const BParams p) {
  using C = BCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if ((base & 1023u) != 0) {  // the swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicExch(p.status, kErrBounds);
    return;
  }
  BSmem& sm = *reinterpret_cast<BSmem*>(smem_raw + C::SMEM_TILES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // The tile: key tiles in ascending order across the grid (the first tiles
  // see the most query blocks under a causal mask, so they start first).
  const int j = blockIdx.x / (p.B * p.Hkv);
  const int bkv = blockIdx.x % (p.B * p.Hkv);
  const int b = bkv / p.Hkv, kvh = bkv % p.Hkv;
  const int k0 = j * kT, k1 = min(p.Lk, k0 + kT);
  int r_lo, r_hi;
  query_range(p, k0, k1, r_lo, r_hi);
  const int i_lo = r_lo / kT, i_hi = r_hi > r_lo ? (r_hi + kT - 1) / kT : i_lo;
  const int nib = i_hi - i_lo;                 // query blocks per head
  const int nsteps = nib > 0 ? nib * p.group : 0;

  if (threadIdx.x == 0) {
    mbar_init(&sm.kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.do_full[s], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.dp_full, 1);
    mbar_init(&sm.p_full, 256);
    mbar_init(&sm.dq_full, 1);
    mbar_init(&sm.dq_empty, 256);
    mbar_init(&sm.fin, 1);
    mbar_init(&sm.drain, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.stat[t], 128);
      mbar_init(&sm.stg_q[t], 128);
      mbar_init(&sm.stg_do[t], 128);
    }
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitGuard g{&sm.abort_flag, p.status, p.timeout_ns, true};
  const WaitGuard g_drain{&sm.abort_flag, p.status, p.timeout_ns, false};
  auto finish = [&]() {
    tc_fence_before();
    asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
    if (warp == 9) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  };
  // step s -> (query head, query block)
  auto step_head = [&](int s) { return kvh * p.group + s / nib; };
  auto step_blk = [&](int s) { return i_lo + s % nib; };

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nsteps > 0) {
      bool ok = true;
      mbar_arrive_expect_tx(&sm.kv_full, 2 * C::TILE_BYTES);
      for (int bx = 0; bx < C::NBOX; ++bx) {
        tma_load_3d(base + C::OFF_K + bx * C::BOX_BYTES, &tm_k, &sm.kv_full, bx * 64, k0, bkv);
        tma_load_3d(base + C::OFF_V + bx * C::BOX_BYTES, &tm_v, &sm.kv_full, bx * 64, k0, bkv);
      }
      // Step t's dQ staging, a half at a time, into the fp32 accumulator
      // with bulk tensor reductions (rows past Lq fall outside the tensor map
      // and are not written); each half's buffer is reloaded right after it
      // has been read, so the loads do not queue behind the other half.
      auto reduce_half = [&](int t, int h) {
        const int ts = t & 1;
        if (!mbar_wait(h == 0 ? &sm.stg_q[ts] : &sm.stg_do[ts], (t >> 1) & 1, g)) return false;
        const int bh = b * p.Hq + step_head(t), r0 = step_blk(t) * kT;
        const uint32_t src = base + (h == 0 ? C::OFF_Q : C::OFF_DO) + ts * C::TILE_BYTES;
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx)
          tma_reduce_add_3d(&tm_dq, src + bx * C::BOX_BYTES, h * (D / 2) + bx * 32, r0, bh);
        bulk_commit_group();
        bulk_wait_read<0>();
        return true;
      };
      for (int s = 0; s < nsteps && ok; ++s) {
        const int qs = s & 1;
        const int bh = b * p.Hq + step_head(s), r0 = step_blk(s) * kT;
        if (s >= 2) ok = reduce_half(s - 2, 0);
        if (!ok) break;
        mbar_arrive_expect_tx(&sm.q_full[qs], C::TILE_BYTES);
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_load_3d(base + C::OFF_Q + qs * C::TILE_BYTES + bx * C::BOX_BYTES, &tm_q, &sm.q_full[qs], bx * 64,
                      r0, bh);
        if (s >= 2) ok = reduce_half(s - 2, 1);
        if (!ok) break;
        mbar_arrive_expect_tx(&sm.do_full[qs], C::TILE_BYTES);
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_load_3d(base + C::OFF_DO + qs * C::TILE_BYTES + bx * C::BOX_BYTES, &tm_do, &sm.do_full[qs],
                      bx * 64, r0, bh);
      }
      for (int t = (nsteps > 2 ? nsteps - 2 : 0); t < nsteps && ok; ++t) ok = reduce_half(t, 0) && reduce_half(t, 1);
      bulk_wait_all();  // every reduction has completed
      // Drain: the last loads have landed before the CTA exits.
      mbar_wait(&sm.kv_full, 0, g_drain);
      for (int s = (nsteps > 2 ? nsteps - 2 : 0); s < nsteps; ++s) {
        mbar_wait(&sm.q_full[s & 1], (s >> 1) & 1, g_drain);
        mbar_wait(&sm.do_full[s & 1], (s >> 1) & 1, g_drain);
      }
    }
    finish();
  } else if (warp == 9) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0 && nsteps > 0) {
      bool ok = mbar_wait(&sm.kv_full, 0, g);
      tc_fence_after();
      const uint64_t dk_desc = sw128_desc(base + C::OFF_K, 16, 1024);   // K_j K-major (S^T A)
      const uint64_t dv_desc = sw128_desc(base + C::OFF_V, 16, 1024);   // V_j K-major (dP^T A)
      const uint64_t kmn_desc = sw128_desc(base + C::OFF_K, C::BOX_BYTES, 1024);  // K_j MN-major (dQ B)
      const uint64_t ds_desc = sw128_desc(base + C::OFF_DS, C::BOX_BYTES, 1024);  // dS MN-major (dQ A)
      // packed bf16 P^T / dS^T column of k-step kk (16 queries): queries 0-63
      // at columns 0-31 of their region, queries 64-127 at columns 64-95
      auto a_col = [](int kk) { return (uint32_t)((kk >> 2) * 64 + (kk & 3) * 8); };
      // S^T = K_j Q_i^T of step s into TM_S, k-steps of 16 features
      auto issue_st = [&](int s) {
        const uint64_t q_km = sw128_desc(base + C::OFF_Q + (s & 1) * C::TILE_BYTES, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t bk = kk * 32;
          const uint32_t off = ((bk / 128) * C::BOX_BYTES + (bk % 128)) >> 4;
          mma_f16_ss(tmem + C::TM_S, dk_desc + off, q_km + off, C::ID_S, kk > 0);
        }
        tc_commit(&sm.s_full);
      };
      if (ok) ok = mbar_wait(&sm.q_full[0], 0, g);
      if (ok) {
        tc_fence_after();
        issue_st(0);
      }
      for (int s = 0; s < nsteps && ok; ++s) {
        const int qs = s & 1;
        if (s > 0) {  // dP^T's columns hold the previous dQ until it has been read
          ok = mbar_wait(&sm.dq_empty, (s - 1) & 1, g);
          if (!ok) break;
          tc_fence_after();
        }
        const uint32_t q_tile = base + C::OFF_Q + qs * C::TILE_BYTES;
        const uint32_t do_tile = base + C::OFF_DO + qs * C::TILE_BYTES;
        const uint64_t do_km = sw128_desc(do_tile, 16, 1024);
        ok = mbar_wait(&sm.do_full[qs], (s >> 1) & 1, g);
        if (!ok) break;
        tc_fence_after();
        // dP^T = V_j dO_i^T
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t bk = kk * 32;
          const uint32_t off = ((bk / 128) * C::BOX_BYTES + (bk % 128)) >> 4;
          mma_f16_ss(tmem + C::TM_DP, dv_desc + off, do_km + off, C::ID_S, kk > 0);
        }
        tc_commit(&sm.dp_full);
        ok = mbar_wait(&sm.p_full, s & 1, g);
        if (!ok) break;
        tc_fence_after();
        // dV += P^T dO_i (A from TMEM, 16 queries = 8 columns per k-step; B
        // MN-major, 16 rows = 2 KB per k-step)
        const uint64_t do_mn = sw128_desc(do_tile, C::BOX_BYTES, 1024);
        const uint64_t q_mn = sw128_desc(q_tile, C::BOX_BYTES, 1024);
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk) {
          const uint32_t off = (kk * 16 * 128) >> 4;
          mma_f16_ts(tmem + C::TM_DV, tmem + C::TM_S + a_col(kk), do_mn + off, C::ID_ACC, (s > 0 || kk > 0) ? 1u : 0u);
        }
        // The next step's S^T, before dK and dQ when its Q block is in, so
        // that its P^T is formed while they run (its columns' last reader,
        // dV, was issued above, and MMAs run in issue order); else after them.
        const bool st_next = s + 1 < nsteps;
        const uint32_t q_par = ((s + 1) >> 1) & 1;
        bool st_early = st_next && mbar_test(&sm.q_full[(s + 1) & 1], q_par);
        if (st_early) {
          tc_fence_after();
          issue_st(s + 1);
        }
        // dK += dS^T Q_i (A from TMEM)
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk) {
          const uint32_t off = (kk * 16 * 128) >> 4;
          mma_f16_ts(tmem + C::TM_DK, tmem + C::TM_DP + a_col(kk), q_mn + off, C::ID_ACC, (s > 0 || kk > 0) ? 1u : 0u);
        }
        // dQ_i = dS K_j over the tile's 128 keys (both operands MN-major),
        // into the dP^T columns: issued after dK, their last reader.  Its
        // completion also frees the step's Q and dO buffers (dQ staging).
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk) {
          const uint32_t off = (kk * 16 * 128) >> 4;
          mma_f16_ss(tmem + C::TM_DP, ds_desc + off, kmn_desc + off, C::ID_DQ, kk > 0);
        }
        tc_commit(&sm.dq_full);
        if (st_next && !st_early) {
          ok = mbar_wait(&sm.q_full[(s + 1) & 1], q_par, g);
          if (!ok) break;
          tc_fence_after();
          issue_st(s + 1);
        }
      }
      tc_commit(&sm.fin);  // dK and dV complete
      tc_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, g_drain);
    }
    __syncwarp();
    finish();
  } else if (warp < 8) {
    // -------------------- P^T, dS^T and the dQ_i read-out: two warps per TMEM
    // lane quadrant, each over 64 of the block's 128 queries (or of dQ_i's
    // features)
    const int quad = warp & 3, hf = warp >> 2;
    const int r = quad * 32 + lane;  // TMEM lane: key row (P^T, dS^T), query row (dQ_i)
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const int q0 = hf * 64;  // this warp's queries of the block
    // its S^T and dP^T columns; packed bf16 P^T and dS^T go over the first 32
    const uint32_t c_s = tmem + C::TM_S + hf * 64 + lane_off, c_dp = tmem + C::TM_DP + hf * 64 + lane_off;
    const int key = k0 + r;
    const int off = p.Lk - p.Lq;
    bool ok = true;
    // LSE (log2) and Dvec of query r of step s's block; the threads of the
    // first four warps each load one of the 128 and share it through shared
    // memory.  Step s's values are in place once `stat[s & 1]` completes its
    // phase s / 2 (an mbarrier, so the wait is bounded); step s + 2's go into
    // the same buffer once step s + 1's dP^T is complete, which is after every
    // thread is done with step s (dP^T is issued after all of step s's dS^T).
    auto load_stat = [&](int s, float& l2v, float& dvv) {
      const int q = step_blk(s) * kT + r;
      const size_t row = (size_t)(b * p.Hq + step_head(s)) * p.Lq + q;
      l2v = q < p.Lq ? p.lse2[row] : INFINITY;
      dvv = q < p.Lq ? p.dvec[row] : 0.f;
    };
    auto put_stat = [&](int s, float l2v, float dvv) {
      sm.lse2[s & 1][r] = l2v;
      sm.dvec[s & 1][r] = dvv;
      mbar_arrive(&sm.stat[s & 1]);
    };
    if (nsteps > 0 && hf == 0) {
      float l2v, dvv;
      load_stat(0, l2v, dvv);
      put_stat(0, l2v, dvv);
    }
    // dQ_i of step t: this warp's D/2 features of its query row out of TMEM
    // (the columns then take the next dP^T), then into its half's staging
    // boxes (32 features each) in step t's Q buffer (first half) or dO buffer
    // (second half), which no product reads any more (dQ_i was the step's
    // last): row r's 8 chunks of 16 bytes, XOR-swizzled by the row's low 3
    // bits (the 128-byte swizzle of the reduction's tensor map).
    auto dq_out = [&](int t) {
      tc_fence_after();
      uint32_t v[D / 2];
      if constexpr (D == 128) {
        tmem_ld64(tmem + C::TM_DP + lane_off + hf * 64, v);
      } else {
        tmem_ld32(tmem + C::TM_DP + lane_off + hf * 32, v);
      }
      tc_fence_before();
      mbar_arrive(&sm.dq_empty);
      const uint32_t stage = base + (hf == 0 ? C::OFF_Q : C::OFF_DO) + (t & 1) * C::TILE_BYTES;
#pragma unroll
      for (int bx = 0; bx < D / 64; ++bx)
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t a = stage + bx * C::BOX_BYTES + r * 128 + ((u ^ (r & 7)) << 4);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v[bx * 32 + 4 * u]),
                       "r"(v[bx * 32 + 4 * u + 1]), "r"(v[bx * 32 + 4 * u + 2]), "r"(v[bx * 32 + 4 * u + 3])
                       : "memory");
        }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // staging visible to the TMA unit
      mbar_arrive(hf == 0 ? &sm.stg_q[t & 1] : &sm.stg_do[t & 1]);
    };
    // visible queries of this key: q + off >= key (causal), q + off - W + 1 <= key (window)
    const int q_first = p.causal ? key - off : INT_MIN;
    const int q_last = (p.causal && p.window > 0) ? key - off + p.window - 1 : INT_MAX;
    const bool key_ok = key < p.Lk;
    for (int s = 0; s < nsteps && ok; ++s) {
      const int i = step_blk(s);
      const int buf = s & 1;
      float nl2 = INFINITY, ndv = 0.f;  // the next step's values, loaded early
      if (hf == 0 && s + 1 < nsteps) load_stat(s + 1, nl2, ndv);
      // Wait for S^T, reading the previous step's dQ out meanwhile if it
      // completes first (a bounded wait, like mbar_wait's).
      bool dq_pending = s > 0;
      {
        bool got = false;
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t it = 0; it < (1u << 28); ++it) {
          if (dq_pending && __all_sync(0xffffffffu, mbar_test(&sm.dq_full, (s - 1) & 1))) {
            dq_out(s - 1);
            dq_pending = false;
          }
          got = __all_sync(0xffffffffu, mbar_test(&sm.s_full, s & 1));
          if (got || ((it & 31u) == 31u && __any_sync(0xffffffffu, *g.abort_flag != 0 ||
                                                                        globaltimer_ns() - t0 > g.timeout_ns)))
            break;
        }
        if (!got) {
          if (lane == 0 && !*g.abort_flag) {
            *g.abort_flag = 1;
            atomicExch(p.status, kErrTimeout);
          }
          ok = false;
          break;
        }
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.stat[buf], (s >> 1) & 1, g));
      if (!ok) break;
      tc_fence_after();
      // P^T from S^T (masked entries 0), back to TMEM as bf16.  A key that
      // sees all of the warp's queries needs no per-element test (rows past
      // Lq have LSE +inf, so their P is 0 either way).
      const int qb = i * kT + q0;
      const bool all_vis = __all_sync(0xffffffffu, key_ok && qb >= q_first && qb + 63 <= q_last);
      uint32_t sr[64];  // this warp's 64 S^T columns, loaded together
      tmem_ld32_async(c_s, *reinterpret_cast<uint32_t(*)[32]>(sr));
      tmem_ld32_async(c_s + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
      tmem_ld_wait(sr);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pp[16];
        const float* l2 = &sm.lse2[buf][q0 + c * 32];
        if (all_vis) {
#pragma unroll
          for (int t = 0; t < 32; t += 2) {
            const uint64_t x2 = fma2(f2(__uint_as_float(sr[c * 32 + t]), __uint_as_float(sr[c * 32 + t + 1])),
                                     f2(p.scale_log2, p.scale_log2), f2(-l2[t], -l2[t + 1]));
            float x0, x1;
            f2_split(x2, x0, x1);
            pp[t / 2] = pack_bf16x2(ex2_approx(x0), ex2_approx(x1));
          }
        } else {
#pragma unroll
          for (int t = 0; t < 32; t += 2) {
            float pv[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int q = qb + c * 32 + t + e;
              const bool vis = key_ok && q >= q_first && q <= q_last;
              const float x = fmaf(__uint_as_float(sr[c * 32 + t + e]), p.scale_log2, -l2[t + e]);
              pv[e] = vis ? ex2_approx(x) : 0.f;
            }
            pp[t / 2] = pack_bf16x2(pv[0], pv[1]);
          }
        }
        tmem_st16(c_s + c * 16, pp);
      }
      tmem_st_wait();  // P^T is read back below
      if (dq_pending) {
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.dq_full, (s - 1) & 1, g));
        if (!ok) break;
        dq_out(s - 1);
      }
      // dP^T complete also means the previous dQ product, the dS tile's last
      // reader, is (it was issued before dP^T)
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.dp_full, s & 1, g));
      if (!ok) break;
      tc_fence_after();
      // dS = P (dP - Dvec), with P as rounded for the dV product
      uint32_t dr[64], pw[32];  // dP^T and the packed P^T of this warp's queries, loaded together
      tmem_ld32_async(c_dp, *reinterpret_cast<uint32_t(*)[32]>(dr));
      tmem_ld32_async(c_dp + 32, *reinterpret_cast<uint32_t(*)[32]>(dr + 32));
      tmem_ld32_async(c_s, pw);
      tmem_ld_wait(dr, pw);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t dd[16];
        const float* dv = &sm.dvec[buf][q0 + c * 32];
#pragma unroll
        for (int t = 0; t < 32; t += 2) {
          const uint32_t w = pw[c * 16 + t / 2];
          const float p0 = __uint_as_float(w << 16), p1 = __uint_as_float(w & 0xFFFF0000u);
          dd[t / 2] = pack_bf16x2(p0 * (__uint_as_float(dr[c * 32 + t]) - dv[t]),
                                  p1 * (__uint_as_float(dr[c * 32 + t + 1]) - dv[t + 1]));
        }
        tmem_st16(c_dp + c * 16, dd);
        // dS row (queries q0 + c*32 .. +31 of key r) into the swizzled tile:
        // 64-query boxes, 16-byte chunks XORed with the row's low 3 bits
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t a = base + C::OFF_DS + hf * C::BOX_BYTES + r * 128 + (((c * 4 + u) ^ (r & 7)) << 4);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(dd[4 * u]), "r"(dd[4 * u + 1]),
                       "r"(dd[4 * u + 2]), "r"(dd[4 * u + 3])
                       : "memory");
        }
      }
      tmem_st_wait();
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // dS visible to the tensor core
      tc_fence_before();
      mbar_arrive(&sm.p_full);
      if (hf == 0 && s + 1 < nsteps) put_stat(s + 1, nl2, ndv);
    }
    if (ok && nsteps > 0) {  // the last step's dQ
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.dq_full, (nsteps - 1) & 1, g));
      if (ok) dq_out(nsteps - 1);
    }
    // dK (times scale) and dV of this key row, this warp's D/2 features
    if (ok && nsteps > 0) ok = __all_sync(0xffffffffu, mbar_wait(&sm.fin, 0, g));
    if (ok) {
      tc_fence_after();
      const size_t row = (size_t)bkv * p.Lk + key;
#pragma unroll 1
      for (int c = hf * (D / 64); c < (hf + 1) * (D / 64); ++c) {
        uint32_t kr[32], vr[32];
        if (nsteps > 0) {
          tmem_ld32(tmem + C::TM_DK + lane_off + c * 32, kr);
          tmem_ld32(tmem + C::TM_DV + lane_off + c * 32, vr);
        } else {  // no query sees this tile
#pragma unroll
          for (int t = 0; t < 32; ++t) kr[t] = vr[t] = 0u;
        }
        if (key < p.Lk) {
          uint4* kd = reinterpret_cast<uint4*>(p.dk + row * D + c * 32);
          uint4* vd = reinterpret_cast<uint4*>(p.dv + row * D + c * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t kp[4], vp[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              kp[e] = pack_bf16x2(__uint_as_float(kr[8 * u + 2 * e]) * p.scale,
                                  __uint_as_float(kr[8 * u + 2 * e + 1]) * p.scale);
              vp[e] = pack_bf16x2(__uint_as_float(vr[8 * u + 2 * e]), __uint_as_float(vr[8 * u + 2 * e + 1]));
            }
            kd[u] = make_uint4(kp[0], kp[1], kp[2], kp[3]);
            vd[u] = make_uint4(vp[0], vp[1], vp[2], vp[3]);
          }
        }
      }
    }
    finish();
  } else {
    finish();  // warps 10-11
  }
}

// One warp per query row: Dvec = rowsum(dO * O), LSE in log2 units (+inf
// where the row has no key, so that its P is 0), zeroed dQ accumulator.
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* o, const __nv_bfloat16* dout,
                                                      const float* lse, float* lse2, float* dvec, float* dq_acc,
                                                      long long rows) {
  const long long row = blockIdx.x * 8ll + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float acc = 0.f;
  for (int d = lane * 2; d < D; d += 64) {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(o + row * D + d);
    const __nv_bfloat162 c = *reinterpret_cast<const __nv_bfloat162*>(dout + row * D + d);
    acc += __bfloat162float(a.x) * __bfloat162float(c.x) + __bfloat162float(a.y) * __bfloat162float(c.y);
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  for (int d = lane * 4; d < D; d += 128)
    *reinterpret_cast<float4*>(dq_acc + row * D + d) = make_float4(0.f, 0.f, 0.f, 0.f);
  if (lane == 0) {
    dvec[row] = acc;
    const float l = lse[row];
    lse2[row] = (l == -INFINITY || l != l) ? INFINITY : l * kLog2e;
  }
}

template <int D>
__global__ void __launch_bounds__(256) bwd_post_kernel(const float* dq_acc, __nv_bfloat16* dq, float scale,
                                                       long long n4) {
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n4; i += (long long)gridDim.x * 256) {
    const float4 v = reinterpret_cast<const float4*>(dq_acc)[i];
    uint2 pk;
    pk.x = pack_bf16x2(v.x * scale, v.y * scale);
    pk.y = pack_bf16x2(v.z * scale, v.w * scale);
    reinterpret_cast<uint2*>(dq)[i] = pk;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 bwd_encoder() {
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

// The fp32 dQ accumulator [outer, rows, D] as a 3-D tensor, box 32 features x
// 128 rows (128 bytes a row, 128-byte swizzle), the target of bulk reductions.
bool bwd_encode_acc(CUtensorMap* map, void* base, int D, uint64_t rows, uint64_t outer) {
  auto enc = bwd_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, rows, outer};
  cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)D * 4 * rows};
  cuuint32_t box[3] = {32, (cuuint32_t)kT, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [outer, rows, D] bf16, box 64 features x 128 rows (128-byte swizzle).
bool bwd_encode(CUtensorMap* map, const void* base, int D, uint64_t rows, uint64_t outer) {
  auto enc = bwd_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, rows, outer};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)D * 2 * rows};
  cuuint32_t box[3] = {64, (cuuint32_t)kT, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
int run_bwd(const BackwardArgs& a, cudaStream_t stream) {
  using C = BCfg<D>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail_cuda("cudaGetDevice", err);
  if (dev < 64 && !attr_set[dev]) {
    err = cudaFuncSetAttribute(bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (err != cudaSuccess) return fail_cuda("backward: cudaFuncSetAttribute", err);
    attr_set[dev] = true;
  }
  const long long rows = (long long)a.B * a.Hq * a.Lq;
  float* dq_acc = static_cast<float*>(a.workspace);
  float* lse2 = dq_acc + rows * D;
  float* dvec = lse2 + rows;
  bwd_pre_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dout), a.lse, lse2, dvec,
      dq_acc, rows);
  err = cudaGetLastError();
  if (err != cudaSuccess) return fail_cuda("backward: pre launch", err);
  if (a.Lk > 0) {
    BParams p{};
    p.lse2 = lse2;
    p.dvec = dvec;
    p.dq_acc = dq_acc;
    p.dk = static_cast<__nv_bfloat16*>(a.dk);
    p.dv = static_cast<__nv_bfloat16*>(a.dv);
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.Lq = a.Lq;
    p.Lk = a.Lk;
    p.group = a.Hq / a.Hkv;
    p.n_kt = (a.Lk + kT - 1) / kT;
    p.causal = a.causal;
    p.window = a.window > 0 ? a.window : 0;
    p.scale = a.scale;
    p.scale_log2 = a.scale * kLog2e;
    p.status = device_status_word();
    if (!p.status) return fail_cuda("backward: status word", cudaGetLastError());
    p.timeout_ns = wait_timeout_ns();
    CUtensorMap tq, tk, tv, tdo, tdq;
    if (!bwd_encode(&tq, a.q, D, a.Lq, (uint64_t)a.B * a.Hq) ||
        !bwd_encode(&tdo, a.dout, D, a.Lq, (uint64_t)a.B * a.Hq) ||
        !bwd_encode(&tk, a.k, D, a.Lk, (uint64_t)a.B * a.Hkv) || !bwd_encode(&tv, a.v, D, a.Lk, (uint64_t)a.B * a.Hkv) ||
        !bwd_encode_acc(&tdq, dq_acc, D, a.Lq, (uint64_t)a.B * a.Hq))
      return fail_cuda("backward: tensor map", cudaErrorInvalidValue);
    const long long grid = (long long)p.n_kt * a.B * a.Hkv;
    bwd_kernel<D><<<(unsigned)grid, kThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, tdq, p);
    err = cudaGetLastError();
    if (err != cudaSuccess) return fail_cuda("backward: launch", err);
  }
  const long long n4 = rows * D / 4;
  long long blocks = (n4 + 255) / 256;
  if (blocks > 16ll * sm_count()) blocks = 16ll * sm_count();
  if (blocks < 1) blocks = 1;
  bwd_post_kernel<D><<<(unsigned)blocks, 256, 0, stream>>>(dq_acc, static_cast<__nv_bfloat16*>(a.dq), a.scale, n4);
  err = cudaGetLastError();
  return err == cudaSuccess ? 0 : fail_cuda("backward: post launch", err);
}

}  // namespace

int launch_backward(const BackwardArgs& a, cudaStream_t stream) {
  if (a.D == 128) return run_bwd<128>(a, stream);
  if (a.D == 64) return run_bwd<64>(a, stream);
  return -2;
}

}  // namespace attn
