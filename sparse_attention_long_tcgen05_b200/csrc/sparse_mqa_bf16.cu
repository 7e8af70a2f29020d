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
// the 576 key dimensions: CTA0 owns dims [0,256), CTA1 owns [256,576). Each CTA
//   - keeps its slice of Q in TMEM (the MMA's A operand read from tensor
//     memory), which leaves shared memory to a 4-deep ring of key blocks;
//   - gathers only its column range of the selected rows with TMA tile::gather4
//     (four 128-byte row pieces per request, 128B-swizzled on arrival, no
//     multicast), so the pair reads each selected row exactly once. A request
//     keeps its issuing warp busy ~90 cycles and the measured gather rate grows
//     with the number of issuing warps, so 19 warps share the requests;
//   - computes a partial S_r = Q[:, dims_r] K[:, dims_r]^T (M=128 heads,
//     N=64 keys) into TMEM;
//   - sends S_r to the peer (st.async into the peer's shared memory, counted on
//     the peer's transaction barrier) and adds the peer's partial:
//     S = S_0 + S_1 is bit-identical in both CTAs (fp32 addition commutes), so
//     both run the same online softmax;
//   - accumulates its half of the value columns, O[:, 256r : 256r+256] += P V_r,
//     where V_r lies inside its own gathered columns (dims [256r, 256r+256)).
// The softmax keeps a stale running max and rescales O in TMEM only when the
// block max exceeds it by more than 2^8 (exact: the final normalisation uses
// the same max).
//
// Roles per CTA (896 threads, 7 warps per SM sub-partition):
//   warps 0-15   plan (each scans two 64-entry blocks of the query's index row:
//                physical rows, valid masks);
//   warps 0-15, 17-19  issue the gather requests (lane 0 of each);
//   warp 16      owns TMEM and issues the MMAs;
//   warps 20-27  softmax, two warps per TMEM sub-partition: warps 20+s and 24+s
//                share the 32 heads (TMEM lanes) of sub-partition s and split
//                the 64 key columns of a block and the 256 output columns in
//                halves; they stage Q into TMEM, exchange with the peer CTA,
//                write P and, at the end, O.
// setmaxnreg gives the softmax warpgroups 152 registers and the others 40.
#include "dsa_common.cuh"
#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int kH = 128;              // query heads = MMA M
constexpr int kBK = 64;              // keys per block = QK^T MMA N
constexpr int kStages = 4;
constexpr int kMaxCh = 5;            // 64-dim chunks per CTA (CTA1: 5, CTA0: 4)
constexpr int kChunkKV = kBK * 128;  // one 64-dim chunk of a key block: 64 rows x 128 B
constexpr int kMaxK = 2048;
constexpr int kMaxBlocks = kMaxK / kBK;
// Warp roles (28 warps, 7 per SM sub-partition). One TMA tile::gather4 request
// moves four 128-byte row pieces and keeps its issuing warp busy ~90 cycles;
// measured on B200, the gather rate grows with the number of issuing warps
// (not lanes), so 19 warps issue them. Registers are moved to the softmax
// warps with setmaxnreg: 20 warps x 40 + 8 warps x 152 = 896 threads x 72.
constexpr int kPlanWarps = 16;       // warps 0-15 scan the index row (two blocks each)
constexpr int kMmaWarp = 16;
constexpr int kGatherIssuers = 19;   // warps 0-15 and 17-19 issue gather4 requests
constexpr int kSoftmaxWarp0 = 20;    // warps 20..27
constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = (kSoftmaxWarp0 + 8) * 32;
constexpr uint32_t kRegsSmall = 40;
constexpr uint32_t kRegsSoftmax = 152;
constexpr uint32_t kTmemCols = 512;  // O: [0,256), S: [256,320), Q: [320,480)
constexpr uint32_t kColO = 0;
constexpr uint32_t kColS = 256;
constexpr uint32_t kColQ = 320;
constexpr float kRescaleLog2 = 8.0f;

struct __align__(1024) Smem {
  uint8_t kv[kStages][kMaxCh][kChunkKV];      // 160 KB key-block ring
  uint8_t p[kH * 128];                        // 16 KB: P [128 heads x 64 keys] bf16
  float recv[kH * kBK];                       // 32 KB: peer's partial S
  int32_t rows[kMaxK];                        // KV row of every index entry (0 if invalid)
  uint32_t bmask[kMaxBlocks][2];              // valid entries of block b
  uint32_t mask[kMaxBlocks][2];               // valid entries of the j-th non-empty block
  int32_t blk[kMaxBlocks];                    // block number of the j-th non-empty block
  float red[2][kH][2];                        // per-half row maxima (double buffered by block)
  float lsum[kH][2];                          // per-half row sums (end of query)
  int32_t n_blocks;
  uint64_t plan_full, q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full, s_empty;
  uint64_t p_full, p_empty;
  uint64_t o_full;
  uint64_t rx_full;   // the peer has written its partial into recv
  uint64_t rx_free;   // the peer has read its own recv (we may write into it)
  uint64_t pair[4];   // the two softmax warps of sub-partition s have posted red/lsum
  uint32_t tmem_base;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// 16 TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
sparse_mqa_bf16_kernel(const __grid_constant__ AttnBf16Args a) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~uintptr_t(1023));
  const int warp = warp_id();
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();     // 0 or 1
  const uint32_t peer = rank ^ 1u;
  const int nch = 4 + static_cast<int>(rank);  // 64-dim chunks owned by this CTA
  const int col0 = 256 * static_cast<int>(rank);
  const int qi = blockIdx.x >> 1;

  int pos;
  bool q_ok = true;
  if (a.keys.paged) {
    const int ctx = a.keys.ctx_lens[qi];
    q_ok = ctx >= 1 && ctx <= a.keys.max_pages * 64;
    pos = q_ok ? ctx - 1 : -1;
  } else {
    pos = a.keys.n_keys - a.keys.n_q + qi;
  }
  const int nb = (a.k + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    mbar_init(&S.plan_full, 1);
    mbar_init(&S.q_full, kSoftmaxThreads);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&S.kv_full[i], 1);   // the expect-tx arrival; gather4 bytes complete it
      mbar_init(&S.kv_empty[i], 1);
    }
    mbar_init(&S.s_full, 1);
    mbar_init(&S.s_empty, kSoftmaxThreads);
    mbar_init(&S.p_full, kSoftmaxThreads);
    mbar_init(&S.p_empty, 1);
    mbar_init(&S.o_full, 1);
    mbar_init(&S.rx_full, 1);    // one expect-tx arrival; the peer's st.async bytes complete it
    mbar_init(&S.rx_free, 8);    // one arrival per peer softmax warp
    for (int i = 0; i < 4; ++i) mbar_init(&S.pair[i], 64);
    fence_barrier_init();
    if (!q_ok) report(a.status, DSA_ERR_DEVICE_BOUNDS);
  }
  if (threadIdx.x == 32) tma_prefetch_desc(&a.map_kv);
  if (warp == kMmaWarp) tmem_alloc(&S.tmem_base, kTmemCols);
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;

  if (warp < kSoftmaxWarp0) {
  regs_dec<kRegsSmall>();
  if (warp < kPlanWarps) {
    // ------------------------------------------------------------ plan (warps 0-15)
    const int32_t* irow = a.idx + static_cast<int64_t>(qi) * a.ld_idx;
    // warp w scans blocks 2w and 2w+1; e[2i + half] holds entry
    // (2w + i) * 64 + 32 half + lane
    int e[4];
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int b = 2 * warp + (i >> 1);
      const int jj = b * kBK + (i & 1) * 32 + lane;
      e[i] = (b < nb && jj < a.k) ? __ldg(irow + jj) : -1;
      bad |= e[i] > pos;
      e[i] = (e[i] >= 0 && e[i] <= pos) ? e[i] : -1;
    }
    int pg[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      pg[i] = (a.keys.paged && e[i] >= 0)
                  ? __ldg(a.keys.block_table + static_cast<int64_t>(qi) * a.keys.ld_block_table +
                          (e[i] >> 6))
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
    if (threadIdx.x == 0) {
      int nvb = 0;
      for (int b = 0; b < nb; ++b) {
        const uint32_t m0 = S.bmask[b][0], m1 = S.bmask[b][1];
        if ((m0 | m1) != 0u) {
          S.mask[nvb][0] = m0;
          S.mask[nvb][1] = m1;
          S.blk[nvb] = b;
          ++nvb;
        }
      }
      S.n_blocks = nvb;
      mbar_arrive(&S.plan_full);
    }
  }
  if (warp != kMmaWarp) {
    // ------------------------------------------------------------ gather (19 issuing warps)
    // Block j's 16 groups of 4 rows x nch 64-dim chunks are split over the
    // issuers: issuer i requests pieces p = i, i + 19, ... (group p / nch,
    // chunk p % nch), each landing as 4 swizzled 128-byte rows of the stage.
    const int issuer = warp < kMmaWarp ? warp : warp - 1;
    if (lane == 0) {
      bool ok = mbar_wait(&S.plan_full, 0, a.status);
      const int n = ok ? S.n_blocks : 0;
      const int n_req = (kBK / 4) * nch;
      for (int j = 0; j < n; ++j) {
        const int st = j % kStages;
        const uint32_t ph = static_cast<uint32_t>(j / kStages) & 1u;
        if (!mbar_wait(&S.kv_empty[st], ph ^ 1u, a.status)) break;
        if (issuer == 0) mbar_arrive_expect_tx(&S.kv_full[st], nch * kChunkKV);
        const int* rb = S.rows + S.blk[j] * kBK;
        for (int p = issuer; p < n_req; p += kGatherIssuers) {
          const int g = p / nch, c = p - g * nch;
          const int4 r4 = *reinterpret_cast<const int4*>(rb + 4 * g);
          tma_gather4(S.kv[st][c] + g * 512, &a.map_kv, col0 + 64 * c, r4.x, r4.y, r4.z, r4.w,
                      &S.kv_full[st]);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc_qk = make_idesc(kBK, 1, 1, 0, 0);   // bf16, A (TMEM) and B K-major
    const uint32_t idesc_pv = make_idesc(256, 1, 1, 0, 1);   // bf16, K-major P, MN-major V
    const uint64_t pdesc = sw128_desc(smem_u32(S.p), 16, 1024);
    bool ok = mbar_wait_warp(&S.plan_full, 0, a.status);
    const int n = ok ? S.n_blocks : 0;
    ok = ok && mbar_wait_warp(&S.q_full, 0, a.status);
    tc_fence_after();
    auto issue_pv = [&](int pst, int jj) -> bool {
      if (!mbar_wait_warp(&S.p_full, static_cast<uint32_t>(jj & 1), a.status)) return false;
      tc_fence_after();
      if (lane == 0) {
        const uint64_t vdesc = sw128_desc(smem_u32(S.kv[pst][0]), kChunkKV, 1024);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          mma_bf16(tmem_base + kColO, pdesc + 2 * kk, vdesc + 128 * kk, idesc_pv,
                   (jj > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&S.kv_empty[pst]);
        mma_commit(&S.p_empty);
      }
      __syncwarp();
      return true;
    };
    int j = 0, prev_st = 0;
    for (; j < n && ok; ++j) {
      const int st = j % kStages;
      const uint32_t ph = static_cast<uint32_t>(j / kStages) & 1u;
      if (!mbar_wait_warp(&S.kv_full[st], ph, a.status) ||
          !mbar_wait_warp(&S.s_empty, static_cast<uint32_t>((j & 1) ^ 1), a.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t d = tmem_base + kColS;
        for (int c = 0; c < nch; ++c) {
          const uint64_t kd = sw128_desc(smem_u32(S.kv[st][c]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(d, tmem_base + kColQ + c * 32 + kk * 8, kd + 2 * kk, idesc_qk,
                        (c | kk) != 0 ? 1u : 0u);
        }
        mma_commit(&S.s_full);
      }
      __syncwarp();
      if (j > 0 && !issue_pv(prev_st, j - 1)) {
        ok = false;
        break;
      }
      prev_st = st;
    }
    if (ok && n > 0) issue_pv(prev_st, n - 1);
    if (lane == 0) mma_commit(&S.o_full);
  }
  } else {
    regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax (warps 20-27)
    const int sub = warp & 3;                              // TMEM sub-partition
    const int hf = (warp - kSoftmaxWarp0) >> 2;            // column half of this warp
    const int h = sub * 32 + lane;                         // head = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    uint64_t* pair_bar = &S.pair[sub];   // both warps of the sub-partition, 64 arrivals per use
    {
      // Q -> TMEM: this CTA's slice of q[t, h, :] as raw bf16 pairs; the two
      // warps of a sub-partition stage alternate 64-dim chunks
      const uint4* src = reinterpret_cast<const uint4*>(
          a.q + static_cast<int64_t>(qi) * a.ld_q + static_cast<int64_t>(h) * 576 + col0);
      uint4 qv[24];
#pragma unroll
      for (int i = 0; i < 24; ++i) {
        const int c = hf + 2 * (i >> 3);        // chunks hf, hf+2, hf+4
        qv[i] = c < nch ? __ldg(src + c * 8 + (i & 7)) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int cc = 0; cc < 3; ++cc) {
        const int c = hf + 2 * cc;
        if (c < nch) {
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            w[4 * i + 0] = qv[cc * 8 + i].x;
            w[4 * i + 1] = qv[cc * 8 + i].y;
            w[4 * i + 2] = qv[cc * 8 + i].z;
            w[4 * i + 3] = qv[cc * 8 + i].w;
          }
          tmem_st32(tmem_base + lane_off + kColQ + 32 * c, w);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&S.q_full);
    }
    // this warp's 16-byte chunks of row h of the exchange buffer: 8*hf .. 8*hf+7
    const uint32_t sw = static_cast<uint32_t>(h & 7);
    const uint32_t recv_row = smem_u32(S.recv) + static_cast<uint32_t>(h) * 256u;
    const uint32_t recv_peer = mapa_shared(recv_row, peer);
    const uint32_t rx_full_peer = mapa_shared(smem_u32(&S.rx_full), peer);
    const uint32_t rx_free_peer = mapa_shared(smem_u32(&S.rx_free), peer);
    uint8_t* prow = S.p + (h >> 3) * 1024 + (h & 7) * 128;
    const float sl2 = a.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = mbar_wait_warp(&S.plan_full, 0, a.status);
    const int n = ok ? S.n_blocks : 0;
    int j = 0;
    for (; j < n && ok; ++j) {
      const uint32_t mk = S.mask[j][hf];          // valid keys among this warp's 32 columns
      // own partial S for this warp's columns
      if (!mbar_wait_warp(&S.s_full, static_cast<uint32_t>(j & 1), a.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[32];
      {
        uint32_t (&v0)[16] = *reinterpret_cast<uint32_t(*)[16]>(&v[0]);
        uint32_t (&v1)[16] = *reinterpret_cast<uint32_t(*)[16]>(&v[16]);
        tmem_ld16(tmem_base + lane_off + kColS + 32 * hf, v0);
        tmem_ld16(tmem_base + lane_off + kColS + 32 * hf + 16, v1);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(&S.s_empty);
      // this block's expected bytes from the peer (all 32 KB of it)
      if (h == 0 && hf == 0) mbar_arrive_expect_tx(&S.rx_full, kH * kBK * 4);
      // send ours once the peer has consumed the previous block
      if (!mbar_wait_cluster_warp(&S.rx_free, static_cast<uint32_t>((j & 1) ^ 1), a.status)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t cc = (static_cast<uint32_t>(8 * hf + c) ^ sw) << 4;
        st_async_v4(recv_peer + cc, v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3],
                    rx_full_peer);
      }
      // receive the peer's partial and add (fp32 addition is commutative:
      // both CTAs get identical S)
      if (!mbar_wait_cluster_warp(&S.rx_full, static_cast<uint32_t>(j & 1), a.status)) {
        ok = false;
        break;
      }
      float x[32];
      const float4* rp = reinterpret_cast<const float4*>(S.recv + h * kBK);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 pv = rp[(8 * hf + c) ^ static_cast<int>(sw)];
        x[4 * c + 0] = __uint_as_float(v[4 * c + 0]) + pv.x;
        x[4 * c + 1] = __uint_as_float(v[4 * c + 1]) + pv.y;
        x[4 * c + 2] = __uint_as_float(v[4 * c + 2]) + pv.z;
        x[4 * c + 3] = __uint_as_float(v[4 * c + 3]) + pv.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(rx_free_peer);   // values already consumed
      // row max of this half (masked), combined with the other half
      float bm = -INFINITY;
      if (mk == 0xffffffffu) {
#pragma unroll
        for (int i = 0; i < 32; ++i) bm = fmaxf(bm, x[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          x[i] = ((mk >> i) & 1u) ? x[i] : -INFINITY;
          bm = fmaxf(bm, x[i]);
        }
      }
      S.red[j & 1][h][hf] = bm;
      mbar_arrive(pair_bar);
      if (!mbar_wait_warp(pair_bar, static_cast<uint32_t>(j & 1), a.status)) {
        ok = false;
        break;
      }
      bm = fmaxf(bm, S.red[j & 1][h][hf ^ 1]) * sl2;   // scale > 0: max commutes with it
      const float m_new = fmaxf(m_used, bm);
      const bool rescale = m_new > m_used + kRescaleLog2;
      const float m_next = rescale ? m_new : m_used;
      const float alpha = rescale ? exp2f(m_used - m_next) : 1.f;
      // previous PV done: P buffer free, O stable
      if (!mbar_wait_warp(&S.p_empty, static_cast<uint32_t>((j & 1) ^ 1), a.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
        // this warp's 128 of the 256 output columns
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          const uint32_t col = kColO + 128 * hf + 32 * c;
          tmem_ld32(tmem_base + lane_off + col, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem_base + lane_off + col, o);
        }
        tmem_wait_st();
      }
      l *= alpha;
      m_used = m_next;
      const float neg_m = -m_used;
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t w4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float p0 = exp2f(fmaf(x[8 * c + 2 * i], sl2, neg_m));
          const float p1 = exp2f(fmaf(x[8 * c + 2 * i + 1], sl2, neg_m));
          psum += p0 + p1;
          w4[i] = pack_bf16x2(p0, p1);
        }
        *reinterpret_cast<uint4*>(prow + ((static_cast<uint32_t>(4 * hf + c) ^ sw) << 4)) =
            make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      l += psum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&S.p_full);
    }
    // epilogue: O / l -> bf16, lse (l summed over both halves)
    S.lsum[h][hf] = l;
    mbar_arrive(pair_bar);
    const bool pair_ok = mbar_wait_warp(pair_bar, static_cast<uint32_t>(j & 1), a.status);
    ok = ok && pair_ok;
    const float lt = S.lsum[h][0] + S.lsum[h][1];
    if (mbar_wait_warp(&S.o_full, 0, a.status)) {
      tc_fence_after();
      const float inv = (ok && lt > 0.f) ? 1.f / lt : 0.f;
      __nv_bfloat16* orow = a.out + (static_cast<int64_t>(qi) * kH + h) * 512 +
                            static_cast<int64_t>(col0 + 128 * hf);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem_base + lane_off + kColO + 128 * hf + 32 * c, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(j > 0 ? __uint_as_float(o[2 * i]) * inv : 0.f,
                              j > 0 ? __uint_as_float(o[2 * i + 1]) * inv : 0.f);
        uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
      if (rank == 0 && hf == 0 && a.lse != nullptr)
        a.lse[static_cast<int64_t>(qi) * kH + h] =
            (ok && lt > 0.f) ? (m_used + log2f(lt)) * 0.69314718055994531f : -INFINITY;
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
  cudaError_t e = cudaFuncSetAttribute(sparse_mqa_bf16_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  sparse_mqa_bf16_kernel<<<2 * a.keys.n_q, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
