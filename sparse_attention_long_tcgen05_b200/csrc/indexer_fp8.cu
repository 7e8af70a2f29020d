// indexer_fp8.cu -- lightning-indexer scores on the 5th-generation tensor
// cores (tcgen05, kind::f8f6f4) with the ReLU + weighted head reduction fused
// into the TMEM epilogue.
//
// Definition (DeepSeek-V3.2-Exp report read-through on 53ai.com, section
// "Innovative architecture: core design of DSA"; juhe.plus read-through, step 1
// "Lightning Indexer"): for query token t and every preceding key s <= t,
//     I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]),
// multi-head (j < 64), ReLU-gated, on FP8 inputs. With e4m3 codes and positive
// per-token scales (q = sq[t] * code, k = sk[s] * code) this is
//     I[t,s] = sk[s] * sum_j (w[t,j] * sq[t]) * ReLU(code_q[t,j] . code_k[s]),
// which is what the kernel evaluates: the code dot products on the tensor core
// (exact e4m3 products, f32 accumulation), then the epilogue of
// indexer_epilogue.cuh.
//
// Mapping: one MMA is D[128 keys, G*64] = K_tile[128 x 128 B] * Qgroup[G*64 x 128 B]^T
// with keys on TMEM lanes and (query, head) on TMEM columns, so each epilogue
// thread owns one key and reduces the 64 heads of a query inside its registers.
//
// Roles (352 threads, one CTA per SM, persistent over work units):
//   warp 0    TMA producer: Q group (once per unit), key tiles and their fp32
//             key scales through a 6-stage ring; in paged mode it loads the
//             first 64-key page of each tile and warp 10 the second (a TMA
//             load keeps its issuing warp busy for ~100 cycles, and a paged
//             tile takes four of them)
//   warp 1    TMEM owner and single-thread MMA issuer (2 accumulators in TMEM)
//   warps 2-9 epilogue, two warps per TMEM sub-partition: warps 2-5 reduce
//             queries 0-1 of the group, warps 6-9 queries 2-3;
//             tcgen05.ld -> ReLU * w -> head sum -> * sk -> global.
//             With one query per group (paged decode) each MMA step covers
//             two key tiles, one per 64-column half of a 128-column
//             accumulator, and warps 2-5 reduce the first, warps 6-9 the
//             second, so both halves of the epilogue work.
//   warp 10   second paged producer (idle on contiguous keys)
// A work unit is (group of G query rows, run of 8..64 key tiles of 128, 8..16
// with paged keys); the launcher picks the run length that spreads the units
// most evenly over the CTAs. Launched after another kernel of the same selection, the kernel
// starts at once and only the epilogue, which overwrites the score rows that
// kernel may still read, waits for it (griddepcontrol).
#include "dsa_common.cuh"
#include "dsa_kernels.h"
#include "indexer_epilogue.cuh"

namespace dsa {
namespace {

constexpr int kHeads = 64;
constexpr int kDim = 128;  // e4m3 bytes per head row / per key row
constexpr int kKeyTile = 128;
constexpr int kMaxG = 4;
constexpr int kStages = 6;
constexpr int kTilesPerUnit = 64;        // largest run of key tiles in a work unit
constexpr int kMinTilesPerUnit = 8;      // shortest run the launcher considers
// Paged keys: the producer fetches a unit's page ids one per lane of a warp
// (two 64-token pages per tile), so a paged unit spans at most 16 tiles.
constexpr int kTilesPerUnitPaged = 16;
static_assert(2 * kTilesPerUnitPaged <= 32, "one lane of a warp per page id of a unit");
static_assert(kMinTilesPerUnit <= kTilesPerUnitPaged, "a paged run can be the shortest");
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = 64 + kEpiThreads + 32;   // + warp 10, second paged producer
constexpr int kPageWarp = 2 + kEpiWarps;
constexpr int kQBytes = kHeads * kDim;      // 8 KB per query
constexpr int kKBytes = kKeyTile * kDim;    // 16 KB per key tile
constexpr int kSkBytes = kKeyTile * 4;      // 512 B of key scales per tile
constexpr uint32_t kTmemCols = 512;

struct __align__(1024) Smem {
  uint8_t q[2][kMaxG * kQBytes];     // B operand (query group), double buffered per unit
  uint8_t k[kStages][kKBytes];       // A operand (key tile) ring
  float sk[kStages][kKeyTile];       // key scales of the tile in the same stage
  float wq[kMaxG * kHeads];          // w[t,j] * sq[t] of the current unit
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_drain;                // the MMA issuer's own MMAs have all completed
  uint32_t tmem_base;
};

struct Unit {
  int ng;             // query rows in the group
  int row0;           // first row index
  int qi[kMaxG];      // query indices
  int seq0;           // paged: block-table row (sequence) of the group's query
  int pos[kMaxG];     // their positions (-1: invalid row, fully masked)
  int max_pos;
  int t0, t1;         // key-tile range of the unit
  int t_end;          // tiles [t0, t_end) need an MMA (some query sees them)
};

__device__ __forceinline__ Unit get_unit(const IndexerFp8Args& a, int G, int n_chunks,
                                         int n_tiles, int tpu, int u, bool report_errors) {
  Unit U;
  const int g = u / n_chunks;
  const int c = u - g * n_chunks;
  U.row0 = g * G;
  U.ng = min(G, a.qr.n_rows - U.row0);
  U.max_pos = -1;
  U.seq0 = 0;
#pragma unroll
  for (int i = 0; i < kMaxG; ++i) {
    U.qi[i] = 0;
    U.pos[i] = -1;
    if (i < U.ng) {
      const int r = U.row0 + i;
      int qi = a.qr.rows ? a.qr.rows[r] : a.qr.q_base + r;
      int pos = -1;
      if (qi < 0 || qi >= a.keys.n_q) {
        if (report_errors) report(a.status, DSA_ERR_DEVICE_BOUNDS);
        qi = 0;
      } else if (a.keys.paged) {
        // one query per group in paged mode (G = 1)
        int seq;
        if (!paged_query(a.keys, qi, seq, pos) && report_errors)
          report(a.status, DSA_ERR_DEVICE_BOUNDS);
        U.seq0 = seq;
      } else {
        pos = a.keys.n_keys - a.keys.n_q + qi;
      }
      U.qi[i] = qi;
      U.pos[i] = pos;
      U.max_pos = max(U.max_pos, pos);
    }
  }
  U.t0 = c * tpu;
  U.t1 = min(n_tiles, U.t0 + tpu);
  const int last = U.max_pos >= 0 ? U.max_pos / kKeyTile + 1 : 0;
  U.t_end = max(U.t0, min(U.t1, last));
  return U;
}

// Page id of logical page p of sequence seq, checked; 0 when out of range.
__device__ __forceinline__ int page_of(const IndexerFp8Args& a, int seq, int p,
                                       bool report_errors) {
  int page = a.keys.block_table[static_cast<int64_t>(seq) * a.keys.ld_block_table + p];
  if (page < 0 || page >= a.keys.num_pages) {
    if (report_errors) report(a.status, DSA_ERR_DEVICE_BOUNDS);
    page = 0;
  }
  return page;
}

// kLimitArg: the pipeline waits take their bound from a.wait_ns (a launch after
// the caller changed the bound); otherwise the default bound is a compile-time
// constant and each wait's suspend hint an immediate.
template <bool kLimitArg>
__global__ void __launch_bounds__(kThreads, 1)
indexer_fp8_kernel(const __grid_constant__ IndexerFp8Args a, int G, int n_chunks, int n_tiles,
                   int tpu, int n_units) {
  const uint64_t wait_ns = kLimitArg ? a.wait_ns : kWaitLimitNs;
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~uintptr_t(1023));
  const int warp = warp_id();
  const int lane = threadIdx.x & 31;
  const int N = G * kHeads;
  // Only the epilogue touches memory that a kernel before this one on the
  // stream uses (the score rows a previous top-k may still be reading); it
  // waits for that kernel below. Everything else may start at once.
  griddep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.q_full[i], 1);
      mbar_init(&S.q_empty[i], 1);
      mbar_init(&S.acc_full[i], 1);
      mbar_init(&S.acc_empty[i], kEpiThreads);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&S.k_full[i], 1);
      // released by the MMAs' completion and by every epilogue thread that
      // reads the stage's key scales (half of them with one query per group)
      mbar_init(&S.k_empty[i], 1 + (G == 1 ? kEpiThreads / 2 : kEpiThreads));
    }
    mbar_init(&S.mma_drain, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&a.map_q);
    tma_prefetch_desc(&a.map_k);
    tma_prefetch_desc(&a.map_sk);
  }
  if (warp == 1) tmem_alloc(&S.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;

  if (warp == 0 || (warp == kPageWarp && a.keys.paged)) {
    // ------------------------------------------------------------ producer(s)
    // Lane 0 issues the TMA loads; in paged mode the whole warp first reads the
    // unit's (at most 32) block-table entries in one coalesced load, so no key
    // tile waits on a dependent page lookup. Warp 0 loads the query group,
    // arms the stage's barrier for the whole tile and loads its first page (or
    // the whole contiguous tile); warp 10 loads the second page of a paged tile.
    const bool first = warp == 0;
    int it = 0, ks = 0;
    uint32_t kph = 0;
    bool ok = true;
    // loads issued per buffer / stage, so the drain below knows which phases
    // to wait for
    uint32_t q_fills[2] = {0u, 0u};
    uint32_t k_fills[kStages];
#pragma unroll
    for (int i = 0; i < kStages; ++i) k_fills[i] = 0u;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++it) {
      const Unit U = get_unit(a, G, n_chunks, n_tiles, tpu, u, first && lane == 0);
      const int qb = it & 1;
      const uint32_t qph = (it >> 1) & 1;
      if (first) {
        if (!mbar_wait_warp(&S.q_empty[qb], qph ^ 1, a.status, wait_ns)) { ok = false; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(&S.q_full[qb], U.ng * kQBytes);
#pragma unroll
          for (int i = 0; i < kMaxG; ++i)   // constant indices keep U in registers
            if (i < U.ng)
              tma_load_3d(S.q[qb] + i * kQBytes, &a.map_q, 0, 0, U.qi[i], &S.q_full[qb]);
        }
        ++q_fills[qb];
      }
      int pg = -1;     // page of logical page 2 t0 + lane, if it holds a key <= max_pos
      if (a.keys.paged) {
        const int p = 2 * U.t0 + lane;
        if (lane < 2 * (U.t_end - U.t0) && p * 64 <= U.max_pos)
          pg = page_of(a, U.seq0, p, first);
      }
      for (int t = U.t0; t < U.t_end; ++t) {
        if (!mbar_wait_warp(&S.k_empty[ks], kph ^ 1, a.status, wait_ns)) { ok = false; break; }
        const int i0 = 2 * (t - U.t0);
        const int pg0 = __shfl_sync(0xffffffffu, pg, i0 & 31);
        const int pg1 = __shfl_sync(0xffffffffu, pg, (i0 + 1) & 31);
        if (lane == 0) {
          if (first) mbar_arrive_expect_tx(&S.k_full[ks], kKBytes + kSkBytes);
          if (!a.keys.paged) {
            tma_load_2d(S.k[ks], &a.map_k, 0, t * kKeyTile, &S.k_full[ks]);
            tma_load_1d(S.sk[ks], &a.map_sk, t * kKeyTile, &S.k_full[ks]);
          } else if (first) {
            tma_load_2d(S.k[ks], &a.map_k, 0, pg0 * 64, &S.k_full[ks]);
            tma_load_1d(S.sk[ks], &a.map_sk, pg0 * 64, &S.k_full[ks]);
          } else {
            const int pg1u = pg1 >= 0 ? pg1 : pg0;   // second page past max_pos: reuse the first
            tma_load_2d(S.k[ks] + kKBytes / 2, &a.map_k, 0, pg1u * 64, &S.k_full[ks]);
            tma_load_1d(S.sk[ks] + 64, &a.map_sk, pg1u * 64, &S.k_full[ks]);
          }
        }
#pragma unroll
        for (int i = 0; i < kStages; ++i) k_fills[i] += i == ks ? 1u : 0u;
        if (++ks == kStages) { ks = 0; kph ^= 1; }
      }
    }
    // Drain: after a give-up the consumers may never have waited for the last
    // loads; wait (with the default bound) until every load this warp issued
    // has landed, so no copy is still writing shared memory when the CTA
    // exits. On the normal path each of these phases completed long ago.
    if (lane == 0) {
      if (first)
        for (int b = 0; b < 2; ++b)
          if (q_fills[b]) mbar_wait(&S.q_full[b], (q_fills[b] - 1u) & 1u, a.status);
#pragma unroll
      for (int i = 0; i < kStages; ++i)
        if (k_fills[i]) mbar_wait(&S.k_full[i], (k_fills[i] - 1u) & 1u, a.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = make_idesc(static_cast<uint32_t>(N), 0, 0, 0, 0);
      int it = 0, ks = 0, ab = 0;
      uint32_t kph = 0, aph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++it) {
        const Unit U = get_unit(a, G, n_chunks, n_tiles, tpu, u, false);
        const int qb = it & 1;
        const uint32_t qph = (it >> 1) & 1;
        if (!mbar_wait(&S.q_full[qb], qph, a.status, wait_ns)) break;
        tc_fence_after();
        const uint64_t bdesc = sw128_desc(smem_u32(S.q[qb]), 16, 1024);
        if (G == 1) {
          // two key tiles per step, into the two 64-column halves of a
          // 128-column accumulator
          for (int t = U.t0; t < U.t_end && ok; t += 2) {
            const int nt = min(2, U.t_end - t);
            if (!mbar_wait(&S.acc_empty[ab], aph ^ 1, a.status, wait_ns)) { ok = false; break; }
            for (int h = 0; h < nt && ok; ++h) {
              const int kss = ks + h < kStages ? ks + h : ks + h - kStages;
              const uint32_t kp = ks + h < kStages ? kph : kph ^ 1u;
              if (!mbar_wait(&S.k_full[kss], kp, a.status, wait_ns)) ok = false;
            }
            if (!ok) break;
            tc_fence_after();
            for (int h = 0; h < nt; ++h) {
              const int kss = ks + h < kStages ? ks + h : ks + h - kStages;
              const uint64_t adesc = sw128_desc(smem_u32(S.k[kss]), 16, 1024);
              const uint32_t d = tmem_base + static_cast<uint32_t>(ab * 2 * N + h * N);
#pragma unroll
              for (int kk = 0; kk < kDim / 32; ++kk)
                mma_f8(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, kk > 0 ? 1u : 0u);
              mma_commit(&S.k_empty[kss]);
            }
            mma_commit(&S.acc_full[ab]);
            for (int h = 0; h < nt; ++h)
              if (++ks == kStages) { ks = 0; kph ^= 1; }
            if (++ab == 2) { ab = 0; aph ^= 1; }
          }
          mma_commit(&S.q_empty[qb]);
          continue;
        }
        for (int t = U.t0; t < U.t_end; ++t) {
          if (!mbar_wait(&S.k_full[ks], kph, a.status) ||
              !mbar_wait(&S.acc_empty[ab], aph ^ 1, a.status, wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = sw128_desc(smem_u32(S.k[ks]), 16, 1024);
          const uint32_t d = tmem_base + static_cast<uint32_t>(ab * N);
#pragma unroll
          for (int kk = 0; kk < kDim / 32; ++kk)
            mma_f8(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, kk > 0 ? 1u : 0u);
          mma_commit(&S.k_empty[ks]);
          mma_commit(&S.acc_full[ab]);
          if (++ks == kStages) { ks = 0; kph ^= 1; }
          if (++ab == 2) { ab = 0; aph ^= 1; }
        }
        mma_commit(&S.q_empty[qb]);
      }
      // Drain: the MMAs issued so far (possibly none) complete before TMEM is
      // freed and before the operands' shared memory goes away.
      mma_commit(&S.mma_drain);
      mbar_wait(&S.mma_drain, 0, a.status);
    }
    __syncwarp();
  } else if (warp >= 2 && warp < kPageWarp) {
    // ------------------------------------------------------------ epilogue
    const int sub = warp & 3;              // TMEM sub-partition of this warp
    const int half = (warp - 2) >> 2;      // 0: queries 0-1, 1: queries 2-3
    const int et = threadIdx.x - 64;       // 0..255
    int ab = 0, ks = 0;
    uint32_t aph = 0, kph = 0;
    // After a timed-out wait the warp stops waiting and computing but keeps
    // walking the same units, so every epilogue warp meets every named barrier.
    bool ok = true;
    griddep_wait();
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
      const Unit U = get_unit(a, G, n_chunks, n_tiles, tpu, u, false);
      named_bar_sync(1, kEpiThreads);
      for (int i = et; i < U.ng * kHeads; i += kEpiThreads) {
        const int g = i / kHeads;
        const int qi = g == 0 ? U.qi[0] : g == 1 ? U.qi[1] : g == 2 ? U.qi[2] : U.qi[3];
        // odd heads staged at half weight: their ReLU is taken as d + |d| (chain_step)
        S.wq[i] = a.w[static_cast<int64_t>(qi) * a.ld_w + (i % kHeads)] * a.q_scale[qi] *
                  ((i & 1) ? 0.5f : 1.f);
      }
      named_bar_sync(1, kEpiThreads);
      if (G == 1) {
        // one query; half h reduces the second key tile of each step if h = 1
        float* const srow = a.scores + static_cast<int64_t>(U.row0) * a.ld_scores;
        const int my_pos = U.pos[0];
        if (a.write_masked)
          for (int t = max(U.t0, U.t_end) + half; t < U.t1; t += 2) {
            const int s = t * kKeyTile + sub * 32 + lane;
            if (s < a.n_cols) srow[s] = -INFINITY;
          }
        for (int t = U.t0; t < U.t_end && ok; t += 2) {
          const int nt = min(2, U.t_end - t);
          const bool mine = half < nt;
          const int s = (t + half) * kKeyTile + sub * 32 + lane;
          float sk = 0.f;
          if (mine) {
            const int kss = ks + half < kStages ? ks + half : ks + half - kStages;
            const uint32_t kp = ks + half < kStages ? kph : kph ^ 1u;
            if (!mbar_wait_warp(&S.k_full[kss], kp, a.status, wait_ns)) { ok = false; break; }
            sk = S.sk[kss][sub * 32 + lane];
            mbar_arrive(&S.k_empty[kss]);
          }
          if (!mbar_wait_warp(&S.acc_full[ab], aph, a.status, wait_ns)) { ok = false; break; }
          tc_fence_after();
          if (mine) {
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) +
                                   static_cast<uint32_t>(ab * 2 * N + half * N);
            uint32_t r0[32], r1[32];
            tmem_ld32(tbase, r0);
            tmem_ld32(tbase + 32, r1);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&S.acc_empty[ab]);
            const float s0 = indexer_score_from_dots(r0, r1, &S.wq[0], sk);
            if (s < a.n_cols) srow[s] = s <= my_pos ? s0 : -INFINITY;
          } else {
            tc_fence_before();
            mbar_arrive(&S.acc_empty[ab]);
          }
          for (int h = 0; h < nt; ++h)
            if (++ks == kStages) { ks = 0; kph ^= 1; }
          if (++ab == 2) { ab = 0; aph ^= 1; }
        }
        continue;
      }
      const int g0 = 2 * half;                          // first query of this warp
      const int nq = max(0, min(2, U.ng - g0));         // queries this warp reduces
      // this warp's two rows, selected with constant indices so U stays in registers
      const int pos0 = half ? U.pos[2] : U.pos[0];
      const int pos1 = half ? U.pos[3] : U.pos[1];
      float* const srow0 = a.scores + static_cast<int64_t>(U.row0 + g0) * a.ld_scores;
      float* const srow1 = srow0 + a.ld_scores;
      for (int t = U.t0; t < U.t1 && ok; ++t) {
        const int s = t * kKeyTile + sub * 32 + lane;
        if (t >= U.t_end) {
          if (a.write_masked && s < a.n_cols) {
            if (nq > 0) srow0[s] = -INFINITY;
            if (nq > 1) srow1[s] = -INFINITY;
          }
          continue;
        }
        // this tile's key scale (the stage also holds the key codes)
        if (!mbar_wait_warp(&S.k_full[ks], kph, a.status, wait_ns)) { ok = false; break; }
        const float sk = S.sk[ks][sub * 32 + lane];
        mbar_arrive(&S.k_empty[ks]);
        if (++ks == kStages) { ks = 0; kph ^= 1; }
        if (!mbar_wait_warp(&S.acc_full[ab], aph, a.status, wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tbase = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) +
                               static_cast<uint32_t>(ab * N + g0 * kHeads);
        if (nq == 2) {
          uint32_t r0[32], r1[32], r2[32], r3[32];
          tmem_ld32(tbase, r0);
          tmem_ld32(tbase + 32, r1);
          tmem_ld32(tbase + 64, r2);
          tmem_ld32(tbase + 96, r3);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(&S.acc_empty[ab]);
          const float s0 = indexer_score_from_dots(r0, r1, &S.wq[g0 * kHeads], sk);
          const float s1 = indexer_score_from_dots(r2, r3, &S.wq[(g0 + 1) * kHeads], sk);
          if (s < a.n_cols) {
            srow0[s] = s <= pos0 ? s0 : -INFINITY;
            srow1[s] = s <= pos1 ? s1 : -INFINITY;
          }
        } else if (nq == 1) {
          uint32_t r0[32], r1[32];
          tmem_ld32(tbase, r0);
          tmem_ld32(tbase + 32, r1);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(&S.acc_empty[ab]);
          const float s0 = indexer_score_from_dots(r0, r1, &S.wq[g0 * kHeads], sk);
          if (s < a.n_cols) srow0[s] = s <= pos0 ? s0 : -INFINITY;
        } else {
          tc_fence_before();
          mbar_arrive(&S.acc_empty[ab]);
        }
        if (++ab == 2) { ab = 0; aph ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

// Tiles per work unit: the run length (kMinTilesPerUnit..max_tpu) whose units
// spread most evenly over the persistent CTAs, counting a unit's set-up (the
// query group's load and the weights' staging, during which the tensor pipe
// waits) as one tile. Long runs pay the set-up less often: at 128K, runs of up
// to 32 tiles instead of 16 took the indexer from 117.0 to 112.5 ms, up to 64
// to 111.0 (up to 128 was slower again). Short runs keep every SM busy when a block of rows has few key
// tiles (148 rows near the start of a sequence form 37 groups: runs of 32
// tiles there would leave three quarters of the SMs idle).
int balanced_tiles_per_unit(int n_groups, int n_tiles, int num_sms, int max_tpu) {
  int best = max_tpu;
  long long best_cost = -1;
  for (int tpu = max_tpu; tpu >= kMinTilesPerUnit; --tpu) {
    const long long units = static_cast<long long>(n_groups) * ((n_tiles + tpu - 1) / tpu);
    const long long grid = units < num_sms ? units : num_sms;
    const long long per_cta = (units + grid - 1) / grid;
    const long long cost = per_cta * ((tpu < n_tiles ? tpu : n_tiles) + 1);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = tpu;
    }
  }
  return best;
}

cudaError_t launch_indexer_fp8(const IndexerFp8Args& a, int num_sms, bool pdl,
                               cudaStream_t stream) {
  const int G = a.keys.paged ? 1 : kMaxG;
  const int n_groups = (a.qr.n_rows + G - 1) / G;
  const int n_tiles = (a.n_cols + kKeyTile - 1) / kKeyTile;
  if (n_groups <= 0 || n_tiles <= 0) return cudaSuccess;
  const int tpu = balanced_tiles_per_unit(n_groups, n_tiles, num_sms,
                                          a.keys.paged ? kTilesPerUnitPaged : kTilesPerUnit);
  const int n_chunks = (n_tiles + tpu - 1) / tpu;
  const long long n_units_ll = static_cast<long long>(n_groups) * n_chunks;
  if (n_units_ll > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int n_units = static_cast<int>(n_units_ll);
  const size_t smem = sizeof(Smem) + 1024;
  const bool limit_arg = a.wait_ns != kWaitLimitNs;
  auto kernel = limit_arg ? indexer_fp8_kernel<true> : indexer_fp8_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_units < num_sms ? n_units : num_sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, a, G, n_chunks, n_tiles, tpu, n_units);
}

}  // namespace dsa
