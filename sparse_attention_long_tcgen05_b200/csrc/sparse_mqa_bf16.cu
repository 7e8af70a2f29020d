// sparse_mqa_bf16.cu -- MQA-mode sparse attention over the selected latent KV
// rows on the 5th-generation tensor cores (tcgen05, kind::f16, bf16 -> f32).
//
// What it computes (DeepSeek-V3.2-Exp report read-through on 53ai.com, section
// "Innovative architecture: core design of DSA" and Figure 1; paperbridge.wiki
// summary, section "DeepSeek Sparse Attention"): for query token t with its
// selected key positions idx_t (k = 2048 in DeepSeek-V3.2), all 128 query
// heads attend to the same selected latent rows (MQA mode of MLA):
//     O[t,h] = sum_i softmax_i(scale * q[t,h] . kv[i]) * kv[i, 0:512],  i in idx_t
// with a 576-wide key (512 latent + 64 rope) and the 512-wide latent as value.
//
// B200 design. The fp32 output of 128 heads x 512 values would fill all 512
// TMEM columns of one SM, so one query runs on a CLUSTER OF TWO CTAs that split
// the 576 key dimensions: CTA0 owns dims [0,256), CTA1 [256,512), and the 64 rope
// dims are split by key (see below). Each CTA
//   - keeps its slice of Q in TMEM (the MMA's A operand read from tensor
//     memory) and gathers only its column range of the selected rows with
//     per-thread 16-byte cp.async copies written straight into the
//     128-byte-swizzled tiles the MMAs read, so the pair reads each selected
//     row once (TMA tile::gather4 requests, one per four 128-byte row pieces,
//     were slower: their issue rate, ~35 cycles per request, set the pace);
//   - computes a partial S_r = Q[:, dims_r] K[:, dims_r]^T for all 128 heads
//     (M=128, N=64 keys) into TMEM;
//   - owns the softmax of 64 of the heads. TMEM lane 32s+i (i < 16) of SM
//     sub-partition s holds one of its own heads, lane 32s+16+i one of the
//     peer's; Q rows are staged in that order, so S, P and O rows follow it.
//     The CTA sends the peer the 8 KB partial S of the peer's heads (fp16: the
//     partials of a 288-dim dot product of bf16 rows stay far inside fp16's
//     range, and its 11-bit rounding lies well below the bf16 rounding P gets
//     right after; halving these bytes cut the 128K attention from 146 to
//     138 ms on B200), adds
//     the peer's partial for its own heads, runs the online softmax and
//     writes the bf16 P rows of its heads into its own P tile, from where
//     they are copied into the peer's (8 KB), together with the per-head
//     rescale factors. Every transfer is a bulk copy out of this CTA's shared
//     memory into the peer's, counted on the peer's transaction barrier: a
//     few asynchronous operations per block, which leaves the SM's
//     asynchronous copy path to the gather;
//   - accumulates its half of the value columns, O[:, 256r : 256r+256] += P V_r
//     for all 128 heads, where V_r lies inside its own gathered columns.
// Measured on B200, cluster shared-memory traffic runs at ~20 B/cycle per SM
// and direction, so the exchange is kept to the 16 KB per 64-key block that
// the split requires, and QK^T of block j+1 is issued as soon as S_j has been
// read, so that the partial S of block j+1 travels while block j's softmax runs.
// The softmax keeps a stale running max and rescales O in TMEM only when the
// block max exceeds it by more than 2^8 (exact: the final normalisation uses
// the same max); the owner of a head sends its factor to the peer, whose O
// rows for that head are rescaled there.
//
// Roles per CTA (1024 threads, 8 warps per SM sub-partition):
//   warps 0-15   plan (each scans two 64-entry blocks of the query's index row:
//                physical rows, valid masks);
//   warps 0-15, 17-18  copy the selected rows (all lanes, cp.async; three
//                groups of six warps, each taking every third block);
//   warp 16      owns TMEM and issues the MMAs;
//   warps 20-23  softmax of the CTA's own heads (TMEM lanes 32s .. 32s+15);
//   warps 24-27  send the peer's partial S (lanes 32s+16 .. 32s+31), as fp16;
//   warps 28-31  take in the peer's P rows and rescale factors, rescale the
//                peer's O rows here, and write those rows at the end.
// The 64 rope dims are needed only by QK^T. Each CTA gathers them for its own
// 32 keys of a block (CTA r: keys 32r .. 32r+31) into a ring of their own,
// released as soon as QK^T has read it, and adds their term to those 32
// columns of its partial S; with 64 value-row pieces of 512 bytes plus 8
// instructions of four 128-byte rope pieces, each CTA issues 72 warp-wide copy
// instructions per block.
#include <cuda_fp16.h>

#include "dsa_common.cuh"
#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int kH = 128;              // query heads = MMA M
constexpr int kBK = 64;              // keys per block = QK^T MMA N
constexpr int kStages = 4;           // ring of the four 64-dim value chunks of a key block
constexpr int kRopeStages = 4;       // ring of the rope chunk of this CTA's 32 keys
constexpr int kChunkKV = kBK * 128;  // one 64-dim chunk of a key block: 64 rows x 128 B
constexpr int kMaxK = 2048;
constexpr int kMaxBlocks = kMaxK / kBK;
static_assert(kMaxBlocks <= 32, "one lane of a warp per key block in the plan's compaction");
// Warp roles. Three groups of six warps copy the selected rows (a block's 72
// row-piece instructions round-robin over the warps of its group).
constexpr int kPlanWarps = 16;       // warps 0-15 scan the index row (two blocks each)
constexpr int kMmaWarp = 16;
constexpr int kGatherIssuers = 19;   // warps 0-15 and 17-19 (all meet on named barrier 2)
constexpr int kGroups = 3;           // issuer groups, block j to group j % kGroups
constexpr int kGroupWarps = 6;       // warps per group (issuer 18, warp 19, takes no block)
// A group's leader starts block j once block j - kStages has left its ring
// stage, waiting on the stage's barrier by phase parity. Its previous wait,
// for block j - kGroups, ended after block j - kGroups - kStages had left, and
// blocks leave in order, so block j - 2 kStages has left too when
// kGroups <= kStages: the phase waited for is then the newest one with that
// parity. With more groups than stages a wait could find an older completed
// phase of the same parity and return before the stage is free.
static_assert(kGroups <= kStages && kGroups <= kRopeStages,
              "a copy group must not run two uses ahead on a ring stage");
constexpr int kSoftmaxWarp0 = 20;    // 20..23
constexpr int kSendWarp0 = 24;       // 24..27
constexpr int kRecvWarp0 = 28;       // 28..31
constexpr int kThreads = 32 * 32;
// setmaxnreg: the block is launched with 64 registers per thread (65,536);
// warps 0-19 drop to 48, the softmax warps rise to 128 and the exchange warps
// to 72: 20 x 48 + 4 x 128 + 8 x 72 = 2048 per 32 threads, all 65,536, and
// per SM sub-partition 5 x 48 + 128 + 2 x 72 = 512 x 32 = 16,384.
constexpr uint32_t kRegsSmall = 48;
constexpr uint32_t kRegsSoftmax = 128;
constexpr uint32_t kRegsExchange = 72;
constexpr uint32_t kTmemCols = 512;  // O: [0,256), S: [256,320), Q: [320,480)
constexpr uint32_t kColO = 0;
constexpr uint32_t kColS = 256;
constexpr uint32_t kColQ = 320;
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kRxSBytes = 64 * kBK * 2;        // the peer's partial S of our 64 heads (fp16)
constexpr uint32_t kRxPBytes = 64 * 128 + 64 * 4;   // the peer's 64 P rows + rescale factors

struct __align__(1024) Smem {
  uint8_t kv[kStages][4][kChunkKV];           // 128 KB value-chunk ring
  uint8_t rope[kRopeStages][kChunkKV / 2];    // 16 KB: rope dims of this CTA's 32 keys
  uint8_t p[2][kH * 128];                     // 2 x 16 KB: P [128 rows x 64 keys] bf16
  uint32_t rx_s[64 * kBK / 2];                // 8 KB: the peer's partial S of our heads (fp16 pairs)
  uint32_t tx_s[64 * kBK / 2];                // 8 KB: our partial S of the peer's heads (fp16 pairs)
  int32_t rows[kMaxK];                        // KV row of every index entry (0 if invalid)
  uint32_t bmask[kMaxBlocks][2];              // valid entries of block b
  uint32_t mask[kMaxBlocks][2];               // valid entries of the j-th non-empty block
  int32_t blk[kMaxBlocks];                    // block number of the j-th non-empty block
  __align__(16) float rx_alpha[2][64];        // the peer's rescale factors of its heads
  __align__(16) float tx_alpha[2][64];        // our rescale factors, copied to the peer
  float rx_done[4][32];                       // softmax warps' last use of rx_s (see below)
  float rx_l[64];                             // the peer's final row sums of its heads
  int32_t n_blocks;
  int32_t gather_n;                           // blocks the gather walks (issuer 0's view)
  int32_t gather_go[kGroups][2];              // group leader: stage ready (1) or give up (0)
  uint64_t plan_full, q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t rope_full[kRopeStages], rope_empty[kRopeStages];
  uint64_t s_full, s_empty;
  uint64_t p_full[2], p_empty[2];
  uint64_t o_full;
  uint64_t rxs_full;   // the peer's partial S of this block has landed in rx_s
  uint64_t rxs_free;   // the peer has read its rx_s (we may send the next block)
  uint64_t rxp_full[2];   // the peer's P rows and factors of a block have landed
  uint64_t l_full;     // the peer's row sums have landed
  uint32_t tmem_base;
};

// 2^x with the ex2.approx instruction (flush-to-zero; 2^-inf = 0). P is
// rounded to bf16 right after, far coarser than the instruction's error.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Maximum of 32 values as a balanced tree (5 dependent steps instead of 32).
__device__ __forceinline__ float max_tree32(const float (&x)[32]) {
  float m[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) m[i] = fmaxf(x[2 * i], x[2 * i + 1]);
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
  return m[0];
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Writes this CTA's 256 O columns of one head per thread pair, scaled by inv,
// from TMEM lanes (t_lane lane) + (t & 15); thread t covers columns
// 64c + 32 (t >> 4) .. +31 for c = 0..3. zero: write zeros.
__device__ __forceinline__ void write_o_rows(uint32_t t_lane, __nv_bfloat16* orow, int hh,
                                             float inv, bool zero) {
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint32_t o[32];
    tmem_ld16x2_32(t_lane + kColO + 64 * c, o);
    tmem_wait_ld();
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      pk[i] = pack_bf16x2(zero ? 0.f : __uint_as_float(o[2 * i]) * inv,
                          zero ? 0.f : __uint_as_float(o[2 * i + 1]) * inv);
    uint4* dst = reinterpret_cast<uint4*>(orow + 64 * c + 32 * hh);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
  }
}

// Multiplies the 256 O columns of TMEM lanes (t_lane lane) + (t & 15) by alpha.
__device__ __forceinline__ void rescale_o_rows(uint32_t t_lane, float alpha) {
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint32_t o[32];
    tmem_ld16x2_32(t_lane + kColO + 64 * c, o);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
    tmem_st16x2_32(t_lane + kColO + 64 * c, o);
  }
  tmem_wait_st();
}

// Stages 64-dim Q chunks cs[] of this thread's Q row into TMEM columns 32 c of
// taddr_q: chunk c < 4 is dims col0 + 64c .., chunk 4 the rope dims 512 ..;
// all loads are issued before the first store.
template <int N>
__device__ __forceinline__ void stage_q_chunks(uint32_t taddr_q, const uint4* qrow, int col0,
                                               const int (&cs)[N]) {
  uint4 qv[8 * N];
#pragma unroll
  for (int k = 0; k < N; ++k) {
    const uint4* src = qrow + (cs[k] < 4 ? col0 + 64 * cs[k] : 512) / 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) qv[8 * k + i] = __ldg(src + i);
  }
#pragma unroll
  for (int k = 0; k < N; ++k) {
    {
      uint32_t w[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        w[4 * i + 0] = qv[8 * k + i].x;
        w[4 * i + 1] = qv[8 * k + i].y;
        w[4 * i + 2] = qv[8 * k + i].z;
        w[4 * i + 3] = qv[8 * k + i].w;
      }
      tmem_st32(taddr_q + 32 * cs[k], w);
    }
  }
  tmem_wait_st();
}

// kDense: dense causal attention (the baseline DSA replaces) -- query t attends
// to every key 0..t, walked as consecutive 64-key blocks (rows computed, or one
// 64-token page per block), masked past t in the last block; no index rows.
template <bool kDense>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
sparse_mqa_bf16_kernel(const __grid_constant__ AttnBf16Args a) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~uintptr_t(1023));
  const int warp = warp_id();
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();     // 0 or 1
  const uint32_t peer = rank ^ 1u;
  const int col0 = 256 * static_cast<int>(rank);
  // dense: the longest queries (the latest positions) are launched first
  const int qi = kDense ? a.keys.n_q - 1 - static_cast<int>(blockIdx.x >> 1)
                        : static_cast<int>(blockIdx.x >> 1);

  int pos, seq = 0;
  bool q_ok = true;
  if (a.keys.paged) {
    q_ok = paged_query(a.keys, qi, seq, pos);
  } else {
    pos = a.keys.n_keys - a.keys.n_q + qi;
  }
  const int nb = (a.k + kBK - 1) / kBK;

  // The planning warps issue their index-row loads first, so the loads
  // overlap the barrier set-up and the cluster sync below.
  int e_in[4] = {-1, -1, -1, -1};
  if (!kDense && warp < kPlanWarps) {
    const int32_t* irow = a.idx + static_cast<int64_t>(qi) * a.ld_idx;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int b = 2 * warp + (i >> 1);
      const int jj = b * kBK + (i & 1) * 32 + lane;
      if (b < nb && jj < a.k) e_in[i] = __ldg(irow + jj);
    }
  }

  if (threadIdx.x == 0) {
    mbar_init(&S.plan_full, 1);
    mbar_init(&S.q_full, 12);          // softmax, send and receive warps (one arrival each)
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&S.kv_full[i], kGroupWarps);   // one arrival per warp of the block's group
      mbar_init(&S.kv_empty[i], 1);
    }
    for (int i = 0; i < kRopeStages; ++i) {
      mbar_init(&S.rope_full[i], kGroupWarps);
      mbar_init(&S.rope_empty[i], 1);
    }
    mbar_init(&S.s_full, 1);
    mbar_init(&S.s_empty, 8);         // softmax and send warps (one arrival each)
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.p_full[b], 8);          // softmax and receive warps (one arrival each)
      mbar_init(&S.p_empty[b], 2);         // this CTA's PV and the peer's PV are done
      mbar_init(&S.rxp_full[b], 1);
    }
    mbar_init(&S.o_full, 1);
    mbar_init(&S.rxs_full, 1);        // one expect-tx arrival; the peer's st.async bytes
    mbar_init(&S.rxs_free, 4);        // one arrival per peer softmax warp
    mbar_init(&S.l_full, 1);
    fence_barrier_init();
    if (!q_ok) report(a.status, DSA_ERR_DEVICE_BOUNDS);
  }
  if (warp == kMmaWarp) tmem_alloc(&S.tmem_base, kTmemCols);
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;

  if (warp < kSoftmaxWarp0) {
    regs_dec<kRegsSmall>();
    if (kDense && warp < kPlanWarps) {
      // ---------------------------------------------------------- dense plan
      // blocks 0 .. pos / 64; with paged keys every block's page id is checked
      // first, and a query with a page id out of range is reported and left
      // empty (zero output), since its keys cannot be read
      int nblk = pos >= 0 ? (pos >> 6) + 1 : 0;
      bool bad = false;
      if (a.keys.paged) {
        const int32_t* bt = a.keys.block_table + static_cast<int64_t>(seq) * a.keys.ld_block_table;
        for (int b = warp * 32 + lane; b < nblk; b += kPlanWarps * 32) {
          const int pg = __ldg(bt + b);
          bad |= pg < 0 || pg >= a.keys.num_pages;
        }
      }
      const bool wbad = __any_sync(0xffffffffu, bad);
      if (lane == 0) S.bmask[warp][0] = wbad ? 1u : 0u;   // per-warp vote (unused when dense)
      named_bar_sync(1, kPlanWarps * 32);
      if (warp == 0) {
        const bool any_bad =
            __any_sync(0xffffffffu, lane < kPlanWarps && S.bmask[lane][0] != 0u);
        if (lane == 0) {
          if (any_bad && rank == 0) report(a.status, DSA_ERR_DEVICE_BOUNDS);
          S.n_blocks = any_bad ? 0 : nblk;
          mbar_arrive(&S.plan_full);
        }
      }
    }
    if (!kDense && warp < kPlanWarps) {
      // ---------------------------------------------------------- plan (warps 0-15)
      // warp w scans blocks 2w and 2w+1; e[2i + half] holds entry
      // (2w + i) * 64 + 32 half + lane
      int e[4];
      bool bad = false;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        e[i] = e_in[i];
        bad |= e[i] > pos;
        e[i] = (e[i] >= 0 && e[i] <= pos) ? e[i] : -1;
      }
      int pg[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        pg[i] = (a.keys.paged && e[i] >= 0)
                    ? __ldg(a.keys.block_table +
                            static_cast<int64_t>(seq) * a.keys.ld_block_table + (e[i] >> 6))
                    : 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        int r = 0;
        if (e[i] >= 0) {
          if (!a.keys.paged) {
            r = e[i];
          } else if (pg[i] < 0 || pg[i] >= a.keys.num_pages) {
            bad = true;
            e[i] = -1;      // an unusable page: skip the entry
          } else {
            r = pg[i] * 64 + (e[i] & 63);
          }
        }
        S.rows[(2 * warp + (i >> 1)) * kBK + (i & 1) * 32 + lane] = r;
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t m0 = __ballot_sync(0xffffffffu, e[2 * i] >= 0);
        const uint32_t m1 = __ballot_sync(0xffffffffu, e[2 * i + 1] >= 0);
        if (lane == 0) {
          S.bmask[2 * warp + i][0] = m0;
          S.bmask[2 * warp + i][1] = m1;
        }
      }
      if (rank == 0 && __any_sync(0xffffffffu, bad) && lane == 0)
        report(a.status, DSA_ERR_DEVICE_BOUNDS);
      named_bar_sync(1, kPlanWarps * 32);
      if (warp == 0) {
        // compaction of the non-empty blocks: lane b looks at block b
        const uint32_t m0 = lane < nb ? S.bmask[lane][0] : 0u;
        const uint32_t m1 = lane < nb ? S.bmask[lane][1] : 0u;
        const bool live = (m0 | m1) != 0u;
        const uint32_t bal = __ballot_sync(0xffffffffu, live);
        if (live) {
          const int slot = __popc(bal & ((1u << lane) - 1u));
          S.mask[slot][0] = m0;
          S.mask[slot][1] = m1;
          S.blk[slot] = lane;
        }
        if (lane == 0) S.n_blocks = __popc(bal);
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.plan_full);
      }
    }
    if (warp != kMmaWarp) {
      // ---------------------------------------------------------- gather (3 groups of 6 warps)
      // Block j's selected rows are copied with 16-byte cp.async straight into
      // the 128-byte-swizzled K-major tiles the MMAs read: the CTA's 256 value
      // columns of each of the 64 rows (one 512-byte row per warp instruction,
      // lane l copying 16 bytes of 64-dim chunk l / 8) and the 64 rope columns
      // of this CTA's 32 keys (four rows per instruction). The block's 72
      // instructions go round-robin to the six warps of the block's group: 18
      // of the 19 issuing warps form three groups, group g taking blocks
      // j = g mod 3. A warp releases its block to the MMA as soon as its own
      // copies of it have landed, after a proxy fence that makes them visible
      // to the tensor core, so three blocks are in flight and no block waits
      // for the next one to be issued (one group of 19 warps releasing block
      // j-1 after issuing j: 134.8 ms at 128K; two groups 127.8; three 125.2).
      // Only a group's first warp waits on the ring's barriers; the others
      // sleep on the group's hardware named barrier (taking no issue slots from
      // the softmax warps) and learn from a shared flag whether to go on, so
      // all of a group's warps take the same number of barrier steps.
      const int issuer = warp < kMmaWarp ? warp : warp - 1;
      if (issuer == 0) {
        const bool ok = mbar_wait_warp(&S.plan_full, 0, a.status);
        if (lane == 0) S.gather_n = ok ? S.n_blocks : 0;
      }
      named_bar_sync(2, kGatherIssuers * 32);
      const int n = S.gather_n;
      const int c_l = lane >> 3;            // 64-dim chunk (value) / row of four (rope)
      const int i_l = lane & 7;             // 16-byte unit within the 128-byte row piece
      const char* const kv_b = reinterpret_cast<const char*>(a.kv);
      const int64_t ld_b = a.ld_kv * 2;
      const int64_t val_off = static_cast<int64_t>(col0 + 64 * c_l + 8 * i_l) * 2;
      const int64_t rope_off = static_cast<int64_t>(512 + 8 * i_l) * 2;
      constexpr int n_items = kBK + kBK / 8;   // 64 value rows + 8 rope instructions
      // copies of block jj have landed in this warp: release them to the MMA
      auto release = [&](int jj) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&S.kv_full[jj % kStages]);
          mbar_arrive(&S.rope_full[jj % kRopeStages]);
        }
      };
      // Groups of issuing warps take every kGroups-th block; a group releases
      // its block as soon as its own copies have landed, so no block waits for
      // the issue of the next one.
      const int grp = issuer / kGroupWarps;
      const int li = issuer - grp * kGroupWarps;
      for (int j = grp; j < n && grp < kGroups; j += kGroups) {
        const int st = j % kStages;
        const int rs = j % kRopeStages;
        const int use = (j / kGroups) & 1;
        if (li == 0) {
          bool ok = mbar_wait_warp(&S.kv_empty[st], static_cast<uint32_t>((j / kStages) & 1) ^ 1u,
                                   a.status);
          if (ok)
            ok = mbar_wait_warp(&S.rope_empty[rs],
                                static_cast<uint32_t>((j / kRopeStages) & 1) ^ 1u, a.status);
          if (lane == 0) S.gather_go[grp][use] = ok ? 1 : 0;
        }
        named_bar_sync(3 + grp, kGroupWarps * 32);
        if (S.gather_go[grp][use] == 0) break;
        const int* rb = kDense ? nullptr : S.rows + S.blk[j] * kBK;
        int64_t dense_base = 0;
        if (kDense)
          dense_base = a.keys.paged
                           ? static_cast<int64_t>(__ldg(a.keys.block_table +
                                                        static_cast<int64_t>(seq) *
                                                            a.keys.ld_block_table + j)) * kBK
                           : static_cast<int64_t>(j) * kBK;
        auto kv_row = [&](int r) -> int64_t {
          if (!kDense) return rb[r];
          if (a.keys.paged) return dense_base + r;
          return min(dense_base + r, static_cast<int64_t>(pos));
        };
        const uint32_t kv_st = smem_u32(S.kv[st][c_l]);
        const uint32_t rope_st = smem_u32(S.rope[rs]);
        for (int p = li; p < n_items; p += kGroupWarps) {
          if (p < kBK) {
            const int r = p;
            const char* src = kv_b + kv_row(r) * ld_b + val_off;
            cp_async16(kv_st + r * 128 + ((i_l ^ (r & 7)) << 4), src);
          } else {
            const int rr = 4 * (p - kBK) + c_l;
            const char* src = kv_b + kv_row(32 * rank + rr) * ld_b + rope_off;
            cp_async16(rope_st + rr * 128 + ((i_l ^ (rr & 7)) << 4), src);
          }
        }
        cp_async_commit();
        cp_async_wait_group<0>();
        release(j);
      }
      cp_async_wait_group<0>();
    } else {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t idesc_qk = make_idesc(kBK, 1, 1, 0, 0);   // bf16, A (TMEM) and B K-major
      const uint32_t idesc_rope = make_idesc(kBK / 2, 1, 1, 0, 0);   // this CTA's 32 keys
      const uint32_t idesc_pv = make_idesc(256, 1, 1, 0, 1);   // bf16, K-major P, MN-major V
      bool ok = mbar_wait_warp(&S.plan_full, 0, a.status);
      const int n = ok ? S.n_blocks : 0;
      ok = ok && mbar_wait_warp(&S.q_full, 0, a.status);
      tc_fence_after();
      // QK^T of block jj into S once the softmax and send warps have read S_{jj-1}
      auto issue_qk = [&](int jj) -> bool {
        const int st = jj % kStages;
        const int rs = jj % kRopeStages;
        if (!mbar_wait_warp(&S.kv_full[st], static_cast<uint32_t>(jj / kStages) & 1u,
                            a.status))
          return false;
        if (!mbar_wait_warp(&S.rope_full[rs], static_cast<uint32_t>(jj / kRopeStages) & 1u,
                            a.status))
          return false;
        if (!mbar_wait_warp(&S.s_empty, static_cast<uint32_t>((jj & 1) ^ 1), a.status))
          return false;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t d = tmem_base + kColS;
          for (int c = 0; c < 4; ++c) {
            const uint64_t kd = sw128_desc(smem_u32(S.kv[st][c]), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ts(d, tmem_base + kColQ + c * 32 + kk * 8, kd + 2 * kk, idesc_qk,
                          (c | kk) != 0 ? 1u : 0u);
          }
          // rope term of this CTA's 32 keys, into their S columns
          const uint64_t rd = sw128_desc(smem_u32(S.rope[rs]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(d + 32u * rank, tmem_base + kColQ + 4 * 32 + kk * 8, rd + 2 * kk,
                        idesc_rope, 1u);
          mma_commit(&S.s_full);
          mma_commit(&S.rope_empty[rs]);
        }
        __syncwarp();
        return true;
      };
      // O += P V of block jj once every P row of it is in place
      auto issue_pv = [&](int jj) -> bool {
        const int b = jj & 1;
        if (!mbar_wait_warp(&S.p_full[b], static_cast<uint32_t>(jj >> 1) & 1u, a.status))
          return false;
        tc_fence_after();
        if (lane == 0) {
          const int st = jj % kStages;
          const uint64_t pdesc = sw128_desc(smem_u32(S.p[b]), 16, 1024);
          const uint64_t vdesc = sw128_desc(smem_u32(S.kv[st][0]), kChunkKV, 1024);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_bf16(tmem_base + kColO, pdesc + 2 * kk, vdesc + 128 * kk, idesc_pv,
                     (jj > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&S.kv_empty[st]);
          mma_commit(&S.p_empty[b]);
          // the peer may overwrite its rows of this P tile
          mma_commit_cluster(mapa_shared(smem_u32(&S.p_empty[b]), peer));
        }
        __syncwarp();
        return true;
      };
      ok = ok && (n == 0 || issue_qk(0));
      for (int j = 0; j < n && ok; ++j) {
        if (j + 1 < n && !issue_qk(j + 1)) ok = false;
        if (ok && !issue_pv(j)) ok = false;
      }
      if (lane == 0) mma_commit(&S.o_full);
    }
  } else if (warp < kSendWarp0) {
    regs_inc<kRegsSoftmax>();
    const int s = warp & 3;                     // TMEM sub-partition
    const int i16 = lane & 15;
    const int hh = lane >> 4;                   // key half (S) / column half (O)
    const int o = 16 * s + i16;                 // index among the owner's 64 heads
    const uint32_t sw = static_cast<uint32_t>(i16 & 7);
    const uint32_t lane_q = static_cast<uint32_t>(32 * s) << 16;
    // Q -> TMEM (32x32b: thread = lane 32s + lane). Row order: lane 32s+i is
    // own head 64 rank + 16s + i, lane 32s+16+i the peer's head.
    const uint4* qrow = reinterpret_cast<const uint4*>(
        a.q + static_cast<int64_t>(qi) * a.ld_q +
        static_cast<int64_t>(64 * static_cast<int>(rank ^ static_cast<uint32_t>(lane >> 4)) +
                             16 * s + (lane & 15)) * 576);
    {
      const int cs[3] = {0, 3, 4};   // the send and receive warps stage 1 and 2
      stage_q_chunks(tmem_base + lane_q + kColQ, qrow, col0, cs);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.q_full);
    }
    bool ok = mbar_wait_warp(&S.plan_full, 0, a.status);
    const int n = ok ? S.n_blocks : 0;
    {
      // ---------------------------------------------------------- softmax of own heads
      // thread t: head 64 rank + o in TMEM lane 32s + (t & 15), keys 32 hh .. +31
      const int head = 64 * static_cast<int>(rank) + o;
      const uint32_t t_lane = tmem_base + lane_q;
      const uint32_t m_own = static_cast<uint32_t>(32 * s + i16);   // our P row of the head
      const uint32_t prow_off = (m_own >> 3) * 1024 + (m_own & 7) * 128;
      // this warp's 16 P rows 32s .. 32s+15 are bytes [4096 s, +2048) of a P
      // tile; in the peer they are rows 32s+16 .. 32s+31, bytes [4096 s + 2048, +2048)
      const uint32_t p_peer0 = mapa_shared(smem_u32(S.p[0]), peer) + 4096u * s + 2048u;
      const uint32_t rxp_full_peer0 = mapa_shared(smem_u32(&S.rxp_full[0]), peer);
      const uint32_t alpha_peer0 = mapa_shared(smem_u32(&S.rx_alpha[0][16 * s]), peer);
      const uint32_t rxs_free_peer = mapa_shared(smem_u32(&S.rxs_free), peer);
      const float sl2 = a.scale_log2;
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < n && ok; ++j) {
        const int b = j & 1;                       // P tile of this block
        uint32_t mk;                               // valid keys among this thread's 32
        if (kDense) {
          const int nv = pos - (j * kBK + 32 * hh) + 1;
          mk = nv >= 32 ? 0xffffffffu : (nv <= 0 ? 0u : (1u << nv) - 1u);
        } else {
          mk = S.mask[j][hh];
        }
        // own partial S of the block
        if (!mbar_wait_warp(&S.s_full, static_cast<uint32_t>(j & 1), a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[32];
        tmem_ld16x2_32(t_lane + kColS, v);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.s_empty);
        // the peer's partial for our heads
        if (warp == kSoftmaxWarp0 && lane == 0) mbar_arrive_expect_tx(&S.rxs_full, kRxSBytes);
        if (!mbar_wait_cluster_warp(&S.rxs_full, static_cast<uint32_t>(j & 1), a.status)) {
          ok = false;
          break;
        }
        float x[32];
        const uint4* rp = reinterpret_cast<const uint4*>(S.rx_s + o * (kBK / 2));
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 pv = rp[(4 * hh + c) ^ static_cast<int>(sw)];
          const uint32_t w4[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w4[i]));
            x[8 * c + 2 * i] = __uint_as_float(v[8 * c + 2 * i]) + f.x;
            x[8 * c + 2 * i + 1] = __uint_as_float(v[8 * c + 2 * i + 1]) + f.y;
          }
        }
        // block row max over both key halves (threads t and t ^ 16 share a head)
        if (mk != 0xffffffffu) {
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = ((mk >> i) & 1u) ? x[i] : -INFINITY;
        }
        float bm = max_tree32(x);
        // Tell the peer that rx_s may be refilled. The store of bm needs every
        // value this thread loaded from rx_s, so it cannot issue before all of
        // those loads have returned; after __syncwarp that holds for all lanes,
        // and the arrive (issued in order after it) can be relaxed -- a
        // cluster-scope release here costs ~1.3K cycles on B200.
        *reinterpret_cast<volatile float*>(&S.rx_done[warp - kSoftmaxWarp0][lane]) = bm;
        __syncwarp();
        if (lane == 31) mbar_arrive_cluster_relaxed(rxs_free_peer);
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16)) * sl2;   // scale > 0
        const float m_new = fmaxf(m_used, bm);
        const bool rescale = m_new > m_used + kRescaleLog2;
        const float m_next = rescale ? m_new : m_used;
        const float alpha = rescale ? fast_exp2(m_used - m_next) : 1.f;
        // PV of block j-2 done in both CTAs: P tile b free here and in the peer
        if (!mbar_wait_cluster_warp(&S.p_empty[b], static_cast<uint32_t>((j >> 1) & 1) ^ 1u,
                                    a.status)) {
          ok = false;
          break;
        }
        if (j > 0 && __any_sync(0xffffffffu, rescale)) {
          // O stable: PV of block j-1 done
          if (!mbar_wait_cluster_warp(&S.p_empty[b ^ 1],
                                      static_cast<uint32_t>((j - 1) >> 1) & 1u, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          rescale_o_rows(t_lane, alpha);
        }
        if (hh == 0) S.tx_alpha[b][o] = alpha;
        uint8_t* prow = S.p[b] + prow_off;
        l *= alpha;
        m_used = m_next;
        const float neg_m = -m_used;
        float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t w4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float p0 = fast_exp2(fmaf(x[8 * c + 2 * i], sl2, neg_m));
            const float p1 = fast_exp2(fmaf(x[8 * c + 2 * i + 1], sl2, neg_m));
            ps[i] += p0 + p1;
            w4[i] = pack_bf16x2(p0, p1);
          }
          const uint32_t cc = (static_cast<uint32_t>(4 * hh + c) ^ sw) << 4;
          *reinterpret_cast<uint4*>(prow + cc) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
        // P rows and factors visible to the async proxy (our MMA, the copy to
        // the peer); any O rescale of this thread ordered before the release
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          const uint32_t bb = static_cast<uint32_t>(b);
          const uint32_t rxp_full_peer = rxp_full_peer0 + 8u * bb;
          bulk_copy_to_cluster(p_peer0 + bb * (kH * 128), smem_u32(S.p[b]) + 4096u * s, 2048,
                               rxp_full_peer);
          bulk_copy_to_cluster(alpha_peer0 + 256u * bb, smem_u32(&S.tx_alpha[b][16 * s]), 64,
                               rxp_full_peer);
          mbar_arrive(&S.p_full[b]);
        }
      }
      // epilogue: O / l -> bf16 for own heads, lse; the peer gets l for its rows
      const float lt = l + __shfl_xor_sync(0xffffffffu, l, 16);
      if (hh == 0)
        st_async_b32(mapa_shared(smem_u32(&S.rx_l[o]), peer), __float_as_uint(lt),
                     mapa_shared(smem_u32(&S.l_full), peer));
      if (mbar_wait_warp(&S.o_full, 0, a.status)) {
        tc_fence_after();
        const bool zero = !ok || n == 0 || !(lt > 0.f);
        write_o_rows(t_lane, a.out + (static_cast<int64_t>(qi) * kH + head) * 512 + col0, hh,
                     zero ? 0.f : 1.f / lt, zero);
        if (hh == 0 && a.lse != nullptr)
          a.lse[static_cast<int64_t>(qi) * kH + head] =
              zero ? -INFINITY : (m_used + log2f(lt)) * 0.69314718055994531f;
      }
    }
  } else {
    regs_inc<kRegsExchange>();
    const int s = warp & 3;                     // TMEM sub-partition
    const int i16 = lane & 15;
    const int hh = lane >> 4;                   // key half (S) / column half (O)
    const int o = 16 * s + i16;                 // index among the owner's 64 heads
    const uint32_t sw = static_cast<uint32_t>(i16 & 7);
    const uint32_t lane_q = static_cast<uint32_t>(32 * s) << 16;
    // Q -> TMEM (32x32b: thread = lane 32s + lane). Row order: lane 32s+i is
    // own head 64 rank + 16s + i, lane 32s+16+i the peer's head.
    const uint4* qrow = reinterpret_cast<const uint4*>(
        a.q + static_cast<int64_t>(qi) * a.ld_q +
        static_cast<int64_t>(64 * static_cast<int>(rank ^ static_cast<uint32_t>(lane >> 4)) +
                             16 * s + (lane & 15)) * 576);
    {
      const int cs[1] = {warp < kRecvWarp0 ? 1 : 2};
      stage_q_chunks(tmem_base + lane_q + kColQ, qrow, col0, cs);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.q_full);
    }
    bool ok = mbar_wait_warp(&S.plan_full, 0, a.status);
    const int n = ok ? S.n_blocks : 0;
    if (warp < kRecvWarp0) {
      // ---------------------------------------------------------- send the peer's partial S
      // thread t: the peer's head o in TMEM lane 32s + 16 + (t & 15), keys 32 hh .. +31
      const uint32_t t_lane = tmem_base + lane_q + (16u << 16);
      uint8_t* tx_row = reinterpret_cast<uint8_t*>(S.tx_s + o * (kBK / 2));
      // this warp's rows 16s .. 16s+15 of tx_s go to the same rows of the peer's rx_s
      const uint32_t tx_warp = smem_u32(S.tx_s + 16 * s * (kBK / 2));
      const uint32_t rxs_peer_warp = mapa_shared(smem_u32(S.rx_s + 16 * s * (kBK / 2)), peer);
      const uint32_t rxs_full_peer = mapa_shared(smem_u32(&S.rxs_full), peer);
      for (int j = 0; j < n && ok; ++j) {
        if (!mbar_wait_warp(&S.s_full, static_cast<uint32_t>(j & 1), a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[32];
        tmem_ld16x2_32(t_lane + kColS, v);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.s_empty);
        // the peer has read block j-1 out of its rx_s (so our copy out of tx_s is done)
        if (!mbar_wait_cluster_warp(&S.rxs_free, static_cast<uint32_t>((j & 1) ^ 1),
                                    a.status)) {
          ok = false;
          break;
        }
        uint32_t hv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const __half2 h = __floats2half2_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          hv[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t cc = (static_cast<uint32_t>(4 * hh + c) ^ sw) << 4;
          *reinterpret_cast<uint4*>(tx_row + cc) = make_uint4(hv[4 * c], hv[4 * c + 1],
                                                              hv[4 * c + 2], hv[4 * c + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) bulk_copy_to_cluster(rxs_peer_warp, tx_warp, 16 * kBK * 2, rxs_full_peer);
      }
    } else {
      // ---------------------------------------------------------- the peer's P rows
      // thread t: the peer's head in TMEM lane 32s + 16 + (t & 15)
      const int head = 64 * static_cast<int>(peer) + o;
      const uint32_t t_lane = tmem_base + lane_q + (16u << 16);
      for (int j = 0; j < n && ok; ++j) {
        const int b = j & 1;
        if (warp == kRecvWarp0 && lane == 0) mbar_arrive_expect_tx(&S.rxp_full[b], kRxPBytes);
        if (!mbar_wait_cluster_warp(&S.rxp_full[b], static_cast<uint32_t>(j >> 1) & 1u,
                                    a.status)) {
          ok = false;
          break;
        }
        const float alpha = S.rx_alpha[b][o];
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          // O stable: PV of block j-1 done
          if (!mbar_wait_cluster_warp(&S.p_empty[b ^ 1],
                                      static_cast<uint32_t>((j - 1) >> 1) & 1u, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          rescale_o_rows(t_lane, alpha);
        }
        fence_proxy_async_smem();   // the peer's rows, seen here, before the MMA reads them
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.p_full[b]);
      }
      if (warp == kRecvWarp0 && lane == 0) mbar_arrive_expect_tx(&S.l_full, 64 * 4);
      const bool l_ok = mbar_wait_cluster_warp(&S.l_full, 0, a.status);
      const float lt = l_ok ? S.rx_l[o] : 0.f;
      if (mbar_wait_warp(&S.o_full, 0, a.status)) {
        tc_fence_after();
        const bool zero = !ok || !l_ok || n == 0 || !(lt > 0.f);
        write_o_rows(t_lane, a.out + (static_cast<int64_t>(qi) * kH + head) * 512 + col0, hh,
                     zero ? 0.f : 1.f / lt, zero);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still touch its shared memory
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_attn_bf16(const AttnBf16Args& a, cudaStream_t stream) {
  if (a.keys.n_q <= 0) return cudaSuccess;
  if (a.k > kMaxK) return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem) + 1024;
  if (a.idx == nullptr) {   // dense causal attention
    cudaError_t e = cudaFuncSetAttribute(sparse_mqa_bf16_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    sparse_mqa_bf16_kernel<true><<<2 * a.keys.n_q, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
  }
  cudaError_t e = cudaFuncSetAttribute(sparse_mqa_bf16_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  sparse_mqa_bf16_kernel<false><<<2 * a.keys.n_q, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
