// sparse_mqa_bwd.cu -- gradient of the MQA-mode sparse attention with respect to
// the queries and the latent KV rows, on the 5th-generation tensor cores
// (tcgen05, kind::f16, bf16 -> f32).
//
// What it computes (wiki-for-amaranth engineering report, section "DeepSeek
// Sparse Attention (DSA)", stage B: in sparse training the main model learns
// through the attention over the selected keys only, the indexer's input being
// detached, so no gradient reaches the selection). For query t with selected
// rows i in idx_t (K_i = kv[i, 0:576], V_i = kv[i, 0:512]), the forward's
// log-sum-exp lse[h] and the upstream gradient dO = d loss / d O:
//     P[h,i]  = exp(scale q[h].K_i - lse[h])
//     dP[h,i] = dO[h].V_i                 D[h] = dO[h].O[h]
//     dZ[h,i] = scale P[h,i] (dP[h,i] - D[h])
//     dq[h]   = sum_i dZ[h,i] K_i
//     dkv[i] += sum_h dZ[h,i] q[h]  (+ sum_h P[h,i] dO[h] in columns 0..511)
// dq is written (bf16); dkv is accumulated (fp32 reductions: a latent row is
// selected by many queries). D is computed first by a small row-dot kernel, as
// its two halves over value dims [0,256) and [256,512).
//
// B200 design. As in the forward, one query runs on a cluster of two CTAs that
// split the 512 latent dims (CTA r owns [256r, 256r+256)); the rope dims of the
// keys are split by key (CTA r gathers them for keys 32r .. 32r+31), and both
// CTAs hold all 64 rope dims of q. For the whole query each CTA keeps in shared
// memory its q slice (128 heads x 320 dims) and its dO slice (128 x 256), both
// 128-byte-swizzled, and per 64-key block it gathers its 256 value dims of the
// 64 rows plus the rope dims of its 32 keys with 16-byte cp.async. Per block:
//   1. partial S_r = q_r K_r^T and dP_r = dO_r V_r^T over the CTA's dims
//      (M=128 heads, N=64 keys) into TMEM;
//   2. each CTA sends its partial S and dP - D rows (fp16, 32 KB; D split into
//      the halves over each CTA's value dims, so the rounding is relative to
//      dP - D, which cancels where one key dominates) straight into the peer's
//      P and dZ tiles with st.async, adds the peer's partials to its own and
//      computes P and scale*dZ for all 128 heads (bf16) in place, each thread
//      overwriting the bytes it has just read: one exchange per block;
//   3. dq_r += dZ K_r (N=256 value dims; the rope dims, over the CTA's 32 keys,
//      into a partial that the pair sums at the end); the K tile is then free
//      for the next block's gather;
//   4. dkv^T tiles, 128 dims at a time: dkv^T[d,i] = sum_h q[h,d] dZ[h,i] +
//      dO[h,d] P[h,i] (M=128 dims, N=64 keys, K=128 heads, both operands
//      MN-major straight from the tiles above), and the 64 rope dims (M padded
//      to 128; the extra rows are never read), into the TMEM columns of S and dP
//      (free by then) and 64 spare ones;
//   5. eight of the gather warps, idle from the moment the next block's rows
//      have landed, read those tiles (TMEM lane = dim, column = key), release
//      the S and dP columns to the next block's MMAs as soon as each is read,
//      and add them into dkv with fp32 reductions, 32 consecutive dims of one
//      row per warp instruction; a CTA adds the rope dims of its own 32 keys
//      only. The reductions (576 fp32 adds per selected pair) thus stay off the
//      chain MMA -> exchange -> P / dZ -> MMA that sets the pace.
// TMEM (512 columns): dq [0,256), rope dq partial [256,320), S [320,384),
// dP [384,448), rope dkv tile [448,512).
//
// Roles (20 warps):
//   warps 0-7    plan (four 64-entry blocks of the index row each), then with
//                warps 9-11 the cp.async gather; after gathering block j they
//                drain block j-1's dkv tiles (warps w and w+4: TMEM
//                sub-partition w, key columns 0-31 and 32-63);
//   warp 8       owns TMEM and issues the MMAs;
//   warps 12-19  exchange and P / dZ (thread = head = TMEM lane; warps 12-15
//                keys 0-31 of each block, 16-19 keys 32-63); warps 16-19 then
//                write dq.
#include <cuda_fp16.h>

#include "dsa_common.cuh"
#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int kH = 128;               // query heads
constexpr int kBK = 64;               // keys per block
constexpr int kMaxK = 2048;
constexpr int kMaxBlocks = kMaxK / kBK;
static_assert(kMaxBlocks <= 32, "one lane of a warp per key block in the plan's compaction");
constexpr int kTile = kH * 128;       // 64 dims of 128 head rows: 16 KB
constexpr int kChunkKV = kBK * 128;   // 64 dims of a block's 64 rows: 8 KB
constexpr int kPlanWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kGatherWarps = 11;      // warps 0-7 and 9-11
constexpr int kSoftWarp0 = 12;        // 12..19: exchange, P and dZ
constexpr int kThreads = 20 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDQ = 0;
constexpr uint32_t kColDQR = 256;
constexpr uint32_t kColS = 320;
constexpr uint32_t kColDP = 384;
constexpr uint32_t kColX = 448;
constexpr uint32_t kRxBytes = 2 * kTile;      // the peer's partial S and dP rows (fp16)
constexpr uint32_t kRqBytes = 64 * 64 * 4;    // the peer's rope dq partial of our 64 heads
constexpr int kQItems = 9 * kH * 8;           // 16-byte pieces of the q and dO slices
constexpr int kKvItems = kBK * 32 + 32 * 8;   // 16-byte pieces of a block's K tile

struct __align__(1024) Smem {
  uint8_t q[5][kTile];        // q slice: chunks 0-3 value dims col0 + 64c .., 4 the rope dims
  uint8_t dout[4][kTile];     // dO slice; follows q, so the padded rope MMA reads stay inside
  uint8_t kv[4][kChunkKV];    // value dims col0 .. col0+255 of the block's 64 rows
  uint8_t rope[kChunkKV / 2]; // rope dims of this CTA's 32 keys of the block
  uint8_t p[kTile];           // P (bf16); first the peer's partial S rows (fp16)
  uint8_t dz[kTile];          // scale * dZ (bf16); first the peer's partial dP rows (fp16)
  int32_t rows[kMaxK];        // KV row of every index entry (0 if invalid)
  uint32_t bmask[kMaxBlocks][2];
  uint32_t mask[kMaxBlocks][2];   // valid entries of the j-th non-empty block
  int32_t blk[kMaxBlocks];        // block number of the j-th non-empty block
  int32_t n_blocks;
  uint64_t plan_full, q_full, kv_full, kv_empty, s_full, sdp_full, rx_full, pdz_full;
  uint64_t peer_free;   // the peer's MMAs of a block are done: its P / dZ tiles may be written
  uint64_t dkv_full, s_free, dp_free, x_free, dq_full, rq_full;
  uint32_t tmem_base;
};
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory of one CTA on sm_100");

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_half2(uint32_t lo, uint32_t hi) {
  const __half2 h = __floats2half2_rn(__uint_as_float(lo), __uint_as_float(hi));
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Offset of 16-byte unit u of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw_off(int r, int u) {
  return static_cast<uint32_t>(r * 128 + ((u ^ (r & 7)) << 4));
}

// One of the eight workers draining block j's dkv^T tiles: TMEM sub-partition
// s (lanes = dims 32s ..), key columns 32 half .. 32 half + 31. Both value
// tiles are read before anything else, so that the next block's S and dP MMAs
// can take their columns at once; the fp32 reductions follow (the key's KV row
// broadcast from the lane that read it); then the rope tile (lanes 0-63; this
// CTA's 32 keys, 16 per worker), whose columns are needed only by the next
// block's dkv MMAs.
__device__ __forceinline__ bool drain_block(Smem& S, const AttnBwdArgs& a, uint32_t tmem_base,
                                            int s, int half, int lane, int j, uint32_t rank,
                                            int col0) {
  if (!mbar_wait_warp(&S.dkv_full, static_cast<uint32_t>(j) & 1u, a.status)) return false;
  tc_fence_after();
  const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(32 * s) << 16);
  const int* rb = S.rows + S.blk[j] * kBK;
  const int64_t ld = a.ld_dkv;
  const int dl = 32 * s + lane;
  {
    uint32_t v0[32], v1[32];
    tmem_ld32(t_lane + kColS + 32 * half, v0);
    tmem_ld32(t_lane + kColDP + 32 * half, v1);
    tmem_wait_ld();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&S.s_free);
      mbar_arrive(&S.dp_free);
    }
    const int my_row = rb[32 * half + lane];
    const uint32_t mk = S.mask[j][half];
    float* const d0 = a.d_kv + col0 + dl;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int64_t row = __shfl_sync(0xffffffffu, my_row, i);
      if ((mk >> i) & 1u) {
        float* const p = d0 + row * ld;
        atomicAdd(p, __uint_as_float(v0[i]));
        atomicAdd(p + 128, __uint_as_float(v1[i]));
      }
    }
  }
  uint32_t x[16];
  if (s < 2) {
    tmem_ld16(t_lane + kColX + 32u * rank + 16 * half, x);
    tmem_wait_ld();
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(&S.x_free);
  if (s < 2) {
    const int r_row = rb[32 * static_cast<int>(rank) + 16 * half + (lane & 15)];
    const uint32_t mr = (S.mask[j][rank] >> (16 * half)) & 0xffffu;
    float* const dr = a.d_kv + 512 + dl;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int64_t row = __shfl_sync(0xffffffffu, r_row, i);
      if ((mr >> i) & 1u) atomicAdd(dr + row * ld, __uint_as_float(x[i]));
    }
  }
  return true;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
sparse_mqa_bwd_kernel(const __grid_constant__ AttnBwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~uintptr_t(1023));
  const int warp = warp_id();
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int col0 = 256 * static_cast<int>(rank);
  const int qi = static_cast<int>(blockIdx.x >> 1);
  const int pos = a.n_keys - a.n_q + qi;
  const int nb = (a.k + kBK - 1) / kBK;

  int e_in[8];
  if (warp < kPlanWarps) {
    const int32_t* irow = a.idx + static_cast<int64_t>(qi) * a.ld_idx;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int b = 4 * warp + (i >> 1);
      const int jj = b * kBK + (i & 1) * 32 + lane;
      e_in[i] = (b < nb && jj < a.k) ? __ldg(irow + jj) : -1;
    }
  }

  if (threadIdx.x == 0) {
    mbar_init(&S.plan_full, 1);
    mbar_init(&S.q_full, kGatherWarps);
    mbar_init(&S.kv_full, kGatherWarps);
    mbar_init(&S.kv_empty, 1);
    mbar_init(&S.s_full, 1);
    mbar_init(&S.sdp_full, 1);
    mbar_init(&S.rx_full, 1);       // one expect-tx arrival; the peer's st.async bytes
    mbar_init(&S.pdz_full, 8);
    mbar_init(&S.peer_free, 1);     // the peer's MMA commit
    mbar_init(&S.dkv_full, 1);
    mbar_init(&S.s_free, 8);
    mbar_init(&S.dp_free, 8);
    mbar_init(&S.x_free, 8);
    mbar_init(&S.dq_full, 1);
    mbar_init(&S.rq_full, 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) tmem_alloc(&S.tmem_base, kTmemCols);
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;

  if (warp < kSoftWarp0 && warp != kMmaWarp) {
    if (warp < kPlanWarps) {
      // ---------------------------------------------------------- plan (warps 0-7)
      // warp w scans blocks 4w .. 4w+3; e_in[2i + half] is entry
      // (4w + i) * 64 + 32 half + lane
      bool bad = false;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = e_in[i];
        bad |= e > pos;
        const bool valid = e >= 0 && e <= pos;
        const int b = 4 * warp + (i >> 1);
        S.rows[b * kBK + (i & 1) * 32 + lane] = valid ? e : 0;
        const uint32_t m = __ballot_sync(0xffffffffu, valid);
        if (lane == 0) S.bmask[b][i & 1] = m;
      }
      if (rank == 0 && __any_sync(0xffffffffu, bad) && lane == 0)
        report(a.status, DSA_ERR_DEVICE_BOUNDS);
      named_bar_sync(1, kPlanWarps * 32);
      if (warp == 0) {
        // compaction of the non-empty blocks: lane b looks at block b
        const uint32_t m0 = S.bmask[lane][0];
        const uint32_t m1 = S.bmask[lane][1];
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
    // ------------------------------------------------------------ gather (11 warps)
    // The q and dO slices once, then per block the K tile, all with 16-byte
    // cp.async written straight into the swizzled tiles the MMAs read; a warp
    // releases its copies after they have landed and a proxy fence.
    const int g = warp < kMmaWarp ? warp : warp - 1;
    {
      const char* qb = reinterpret_cast<const char*>(a.q + static_cast<int64_t>(qi) * a.ld_q);
      const char* ob = reinterpret_cast<const char*>(a.d_out + static_cast<int64_t>(qi) * kH * 512);
      for (int p = g * 32 + lane; p < kQItems; p += kGatherWarps * 32) {
        const int c = p >> 10;            // chunk: 0-4 q, 5-8 dO
        const int r = (p >> 3) & (kH - 1);
        const int u = p & 7;
        if (c < 5) {
          const int d = (c < 4 ? col0 + 64 * c : 512) + 8 * u;
          cp_async16(smem_u32(S.q[c]) + sw_off(r, u), qb + (static_cast<int64_t>(r) * 576 + d) * 2);
        } else {
          const int d = col0 + 64 * (c - 5) + 8 * u;
          cp_async16(smem_u32(S.dout[c - 5]) + sw_off(r, u),
                     ob + (static_cast<int64_t>(r) * 512 + d) * 2);
        }
      }
      cp_async_commit();
      cp_async_wait_group<0>();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.q_full);
    }
    const bool ok0 = mbar_wait_warp(&S.plan_full, 0, a.status);
    const int n = ok0 ? S.n_blocks : 0;
    const char* kvb = reinterpret_cast<const char*>(a.kv);
    const int64_t ldb = a.ld_kv * 2;
    // warps 0-7 also drain: block j-1's dkv tiles land about when the copies
    // of block j have been issued and have landed
    const bool drains = warp < kPlanWarps;
    bool dok = true;
    int gathered = 0;
    for (int j = 0; j < n; ++j) {
      if (j > 0 && !mbar_wait_warp(&S.kv_empty, static_cast<uint32_t>(j - 1) & 1u, a.status))
        break;
      const int* rb = S.rows + S.blk[j] * kBK;
      for (int p = g * 32 + lane; p < kKvItems; p += kGatherWarps * 32) {
        if (p < kBK * 32) {
          const int r = p >> 5;
          const int c = (p >> 3) & 3;
          const int u = p & 7;
          cp_async16(smem_u32(S.kv[c]) + sw_off(r, u),
                     kvb + rb[r] * ldb + static_cast<int64_t>(col0 + 64 * c + 8 * u) * 2);
        } else {
          const int rr = (p - kBK * 32) >> 3;
          const int u = p & 7;
          cp_async16(smem_u32(S.rope) + sw_off(rr, u),
                     kvb + rb[32 * static_cast<int>(rank) + rr] * ldb +
                         static_cast<int64_t>(512 + 8 * u) * 2);
        }
      }
      cp_async_commit();
      cp_async_wait_group<0>();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.kv_full);
      gathered = j + 1;
      if (drains && j > 0 && dok) dok = drain_block(S, a, tmem_base, warp & 3, warp >> 2, lane, j - 1, rank, col0);
    }
    cp_async_wait_group<0>();
    if (drains && dok && n > 0 && gathered == n)
      drain_block(S, a, tmem_base, warp & 3, warp >> 2, lane, n - 1, rank, col0);
  } else if (warp == kMmaWarp) {
    // -------------------------------------------------------------- MMA issuer
    const uint32_t id_s = make_idesc(kBK, 1, 1, 0, 0);        // K-major A and B
    const uint32_t id_sr = make_idesc(kBK / 2, 1, 1, 0, 0);   // this CTA's 32 keys
    const uint32_t id_dq = make_idesc(256, 1, 1, 0, 1);       // K-major dZ, MN-major K tile
    const uint32_t id_dqr = make_idesc(64, 1, 1, 0, 1);
    const uint32_t id_kv = make_idesc(kBK, 1, 1, 1, 1);       // MN-major q / dO and dZ / P
    bool ok = mbar_wait_warp(&S.plan_full, 0, a.status);
    const int n = ok ? S.n_blocks : 0;
    ok = ok && mbar_wait_warp(&S.q_full, 0, a.status);
    const uint32_t tS = tmem_base + kColS;
    const uint32_t tDP = tmem_base + kColDP;
    const uint32_t tX = tmem_base + kColX;
    const uint32_t peer_free_remote = mapa_shared(smem_u32(&S.peer_free), peer);
    for (int j = 0; j < n && ok; ++j) {
      const uint32_t ph = static_cast<uint32_t>(j) & 1u;
      const uint32_t pp = ph ^ 1u;
      ok = mbar_wait_warp(&S.kv_full, ph, a.status);
      // the drain has read block j-1's first dkv tile out of the S columns
      if (ok && j > 0) ok = mbar_wait_warp(&S.s_free, pp, a.status);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        const uint64_t rd = sw128_desc(smem_u32(S.rope), 16, 1024);
        const uint64_t qr = sw128_desc(smem_u32(S.q[4]), 16, 1024);
        for (int c = 0; c < 4; ++c) {
          const uint64_t qd = sw128_desc(smem_u32(S.q[c]), 16, 1024);
          const uint64_t kd = sw128_desc(smem_u32(S.kv[c]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tS, qd + 2 * kk, kd + 2 * kk, id_s, (c | kk) != 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tS + 32u * rank, qr + 2 * kk, rd + 2 * kk, id_sr, 1u);
        mma_commit(&S.s_full);   // the partial S travels while dP is computed
      }
      __syncwarp();
      // ... and the second out of the dP columns
      if (j > 0 && !mbar_wait_warp(&S.dp_free, pp, a.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        for (int c = 0; c < 4; ++c) {
          const uint64_t od = sw128_desc(smem_u32(S.dout[c]), 16, 1024);
          const uint64_t kd = sw128_desc(smem_u32(S.kv[c]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tDP, od + 2 * kk, kd + 2 * kk, id_s, (c | kk) != 0 ? 1u : 0u);
        }
        mma_commit(&S.sdp_full);
      }
      __syncwarp();
      ok = mbar_wait_warp(&S.pdz_full, ph, a.status);
      if (ok && j > 0) ok = mbar_wait_warp(&S.x_free, pp, a.status);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        // dq += dZ K (value dims), rope partial over this CTA's 32 keys
        const uint64_t za = sw128_desc(smem_u32(S.dz), 16, 1024);
        const uint64_t vb = sw128_desc(smem_u32(S.kv[0]), kChunkKV, 1024);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          mma_bf16(tmem_base + kColDQ, za + 2 * kk, vb + 128 * kk, id_dq,
                   (j > 0 || kk > 0) ? 1u : 0u);
        const uint64_t rb = sw128_desc(smem_u32(S.rope), kChunkKV, 1024);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_bf16(tmem_base + kColDQR, za + 4 * rank + 2 * kk, rb + 128 * kk, id_dqr,
                   (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&S.kv_empty);
        // dkv^T tiles: lanes = dims, columns = keys
        const uint64_t zb = sw128_desc(smem_u32(S.dz), kTile, 1024);
        const uint64_t pb = sw128_desc(smem_u32(S.p), kTile, 1024);
        for (int t = 0; t < 2; ++t) {
          const uint32_t d = t ? tDP : tS;
          const uint64_t qa = sw128_desc(smem_u32(S.q[2 * t]), kTile, 1024);
          const uint64_t oa = sw128_desc(smem_u32(S.dout[2 * t]), kTile, 1024);
#pragma unroll
          for (int kk = 0; kk < kH / 16; ++kk)
            mma_bf16(d, qa + 128 * kk, zb + 128 * kk, id_kv, kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kH / 16; ++kk) mma_bf16(d, oa + 128 * kk, pb + 128 * kk, id_kv, 1u);
        }
        const uint64_t qa4 = sw128_desc(smem_u32(S.q[4]), kTile, 1024);
#pragma unroll
        for (int kk = 0; kk < kH / 16; ++kk)
          mma_bf16(tX, qa4 + 128 * kk, zb + 128 * kk, id_kv, kk > 0 ? 1u : 0u);
        mma_commit(&S.dkv_full);
        mma_commit_cluster(peer_free_remote);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(&S.dq_full);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ exchange, P and dZ
    // warps 12-15 take keys 0-31 of every block, warps 16-19 keys 32-63
    const int s = warp & 3;                   // TMEM sub-partition
    const int kh = (warp - kSoftWarp0) >> 2;  // key half
    const int m = 32 * s + lane;              // head = TMEM lane = tile row
    const int dl = m;
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(32 * s) << 16);
    const int sw = m & 7;
    const uint32_t row_off = static_cast<uint32_t>((m >> 3) * 1024 + (m & 7) * 128);
    uint8_t* const prow = S.p + row_off;
    uint8_t* const zrow = S.dz + row_off;
    const uint32_t p_peer = mapa_shared(smem_u32(S.p) + row_off, peer);
    const uint32_t z_peer = mapa_shared(smem_u32(S.dz) + row_off, peer);
    const uint32_t rx_full_peer = mapa_shared(smem_u32(&S.rx_full), peer);
    const float sl2 = a.scale_log2;
    const float sc = a.scale;
    const float lse2 = a.lse[static_cast<int64_t>(qi) * kH + m] * 1.4426950408889634f;
    // this CTA's half of D (over its value dims): the pair exchanges its
    // partial of dP - D, so the fp16 rounding is relative to dP - D itself,
    // which vanishes where one key takes all the probability
    const float dlt = a.delta[(static_cast<int64_t>(qi) * kH + m) * 2 + rank];
    bool ok = mbar_wait_warp(&S.plan_full, 0, a.status);
    const int n = ok ? S.n_blocks : 0;
    for (int j = 0; j < n && ok; ++j) {
      const uint32_t ph = static_cast<uint32_t>(j) & 1u;
      if (warp == kSoftWarp0 && lane == 0) mbar_arrive_expect_tx(&S.rx_full, kRxBytes);
      if (!mbar_wait_warp(&S.s_full, ph, a.status)) {
        ok = false;
        break;
      }
      // the peer's MMAs of block j-1 are done: its P and dZ tiles take our partials
      if (j > 0 && !mbar_wait_cluster_warp(&S.peer_free, ph ^ 1u, a.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {   // partial S, 16 keys at a time
        const int hf = 2 * kh + hh;
        uint32_t v[16];
        tmem_ld16(t_lane + kColS + 16 * hf, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint32_t off = static_cast<uint32_t>(((2 * hf + c) ^ sw) << 4);
          st_async_v4(p_peer + off,
                      make_uint4(pack_half2(v[8 * c], v[8 * c + 1]), pack_half2(v[8 * c + 2], v[8 * c + 3]),
                                 pack_half2(v[8 * c + 4], v[8 * c + 5]),
                                 pack_half2(v[8 * c + 6], v[8 * c + 7])),
                      rx_full_peer);
        }
      }
      if (!mbar_wait_warp(&S.sdp_full, ph, a.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {   // partial dP - D
        const int hf = 2 * kh + hh;
        uint32_t u[16];
        tmem_ld16(t_lane + kColDP + 16 * hf, u);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint32_t off = static_cast<uint32_t>(((2 * hf + c) ^ sw) << 4);
          uint32_t du[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) du[e] = __float_as_uint(__uint_as_float(u[8 * c + e]) - dlt);
          st_async_v4(z_peer + off,
                      make_uint4(pack_half2(du[0], du[1]), pack_half2(du[2], du[3]),
                                 pack_half2(du[4], du[5]), pack_half2(du[6], du[7])),
                      rx_full_peer);
        }
      }
      if (!mbar_wait_cluster_warp(&S.rx_full, ph, a.status)) {
        ok = false;
        break;
      }
      const uint32_t mkh = S.mask[j][kh];
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        const int hf = 2 * kh + hh;
        uint32_t v[16], u[16];
        tmem_ld16(t_lane + kColS + 16 * hf, v);
        tmem_ld16(t_lane + kColDP + 16 * hf, u);
        tmem_wait_ld();
        const uint32_t mk = (mkh >> (16 * hh)) & 0xffffu;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint32_t off = static_cast<uint32_t>(((2 * hf + c) ^ sw) << 4);
          const uint4 rs = *reinterpret_cast<const uint4*>(prow + off);
          const uint4 rp = *reinterpret_cast<const uint4*>(zrow + off);
          const uint32_t ws[4] = {rs.x, rs.y, rs.z, rs.w};
          const uint32_t wp[4] = {rp.x, rp.y, rp.z, rp.w};
          uint32_t pw[4], zw[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int kk = 8 * c + 2 * i;
            const float2 fs = __half22float2(*reinterpret_cast<const __half2*>(&ws[i]));
            const float2 fp = __half22float2(*reinterpret_cast<const __half2*>(&wp[i]));
            const float x0 = __uint_as_float(v[kk]) + fs.x;
            const float x1 = __uint_as_float(v[kk + 1]) + fs.y;
            const float y0 = (__uint_as_float(u[kk]) - dlt) + fp.x;   // dP - D
            const float y1 = (__uint_as_float(u[kk + 1]) - dlt) + fp.y;
            const float p0 = ((mk >> kk) & 1u) ? fast_exp2(fmaf(x0, sl2, -lse2)) : 0.f;
            const float p1 = ((mk >> (kk + 1)) & 1u) ? fast_exp2(fmaf(x1, sl2, -lse2)) : 0.f;
            pw[i] = pack_bf16x2(p0, p1);
            zw[i] = pack_bf16x2(p0 * y0 * sc, p1 * y1 * sc);
          }
          *reinterpret_cast<uint4*>(prow + off) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
          *reinterpret_cast<uint4*>(zrow + off) = make_uint4(zw[0], zw[1], zw[2], zw[3]);
        }
      }
      // P and dZ rows visible to the tensor core; our TMEM reads ordered first
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.pdz_full);
    }
    if (kh == 1) {
      // dq of head dl: value dims col0 .. col0+255 here; the rope dims of the
      // CTA's own 64 heads (64 rank ..) with the peer's partial added
      const bool got = mbar_wait_warp(&S.dq_full, 0, a.status);
      const bool live = ok && got && n > 0;
      if (got) tc_fence_after();
      __nv_bfloat16* const dqrow = a.d_q + (static_cast<int64_t>(qi) * kH + dl) * 576;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t v[32];
        if (live) {
          tmem_ld32(t_lane + kColDQ + 32 * c, v);
          tmem_wait_ld();
        }
        uint4* dst = reinterpret_cast<uint4*>(dqrow + col0 + 32 * c);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = live ? make_uint4(pack_bf16x2(__uint_as_float(v[8 * i]), __uint_as_float(v[8 * i + 1])),
                                     pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3])),
                                     pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5])),
                                     pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7])))
                        : make_uint4(0u, 0u, 0u, 0u);
      }
      const bool own = (s >> 1) == static_cast<int>(rank);   // heads 64 rank .. 64 rank + 63
      // slot of head dl in its owner's exchange area (the owner's P tile)
      const uint32_t slot_off = static_cast<uint32_t>((dl & 63) * 256);
      if (!own) {
        // the peer's last MMAs are done: its P tile takes our partials
        if (live && mbar_wait_cluster_warp(&S.peer_free, static_cast<uint32_t>(n - 1) & 1u, a.status)) {
          const uint32_t dst = mapa_shared(smem_u32(S.p) + slot_off, peer);
          const uint32_t bar = mapa_shared(smem_u32(&S.rq_full), peer);
#pragma unroll 1
          for (int h = 0; h < 2; ++h) {
            uint32_t r[32];
            tmem_ld32(t_lane + kColDQR + 32 * h, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 8; ++i)
              st_async_v4(dst + 128 * h + 16 * i,
                          make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]), bar);
          }
        }
      } else {
        if (live && s == 2 * static_cast<int>(rank) && lane == 0)
          mbar_arrive_expect_tx(&S.rq_full, kRqBytes);
        const bool x_ok = live && mbar_wait_cluster_warp(&S.rq_full, 0, a.status);
        const float* px = reinterpret_cast<const float*>(S.p + slot_off);
        uint4* dst = reinterpret_cast<uint4*>(dqrow + 512);
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          uint32_t r[32];
          if (x_ok) {
            tmem_ld32(t_lane + kColDQR + 32 * h, r);
            tmem_wait_ld();
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              f[e] = x_ok ? __uint_as_float(r[8 * i + e]) + px[32 * h + 8 * i + e] : 0.f;
            dst[4 * h + i] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                        pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
          }
        }
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

// D[row] = dO[row] . O[row], as its two halves over value dims [0,256) and
// [256,512) (one per CTA of the pair): delta[2 row + r]. One warp per row.
__global__ void __launch_bounds__(256) mqa_bwd_delta_kernel(const __nv_bfloat16* __restrict__ out,
                                                            const __nv_bfloat16* __restrict__ d_out,
                                                            float* __restrict__ delta,
                                                            int64_t rows) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int lane = threadIdx.x & 31;
  const uint4* o = reinterpret_cast<const uint4*>(out + r * 512);
  const uint4* g = reinterpret_cast<const uint4*>(d_out + r * 512);
  float acc[2] = {0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 2; ++i) {   // half i: dims 256 i + 8 lane ..
    const uint4 ov = __ldg(o + lane + 32 * i);
    const uint4 gv = __ldg(g + lane + 32 * i);
    const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 a2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ow[e]));
      const float2 b2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[e]));
      acc[i] = fmaf(a2.x, b2.x, acc[i]);
      acc[i] = fmaf(a2.y, b2.y, acc[i]);
    }
  }
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], w);
    acc[1] += __shfl_xor_sync(0xffffffffu, acc[1], w);
  }
  if (lane == 0) {
    delta[2 * r] = acc[0];
    delta[2 * r + 1] = acc[1];
  }
}

}  // namespace

cudaError_t launch_attn_bwd(const AttnBwdArgs& a, cudaStream_t stream) {
  if (a.n_q <= 0) return cudaSuccess;
  if (a.k > kMaxK) return cudaErrorInvalidValue;
  const int64_t rows = static_cast<int64_t>(a.n_q) * kH;   // delta holds 2 rows floats
  mqa_bwd_delta_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
      a.out, a.d_out, a.delta, rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(Smem) + 1024;
  e = cudaFuncSetAttribute(sparse_mqa_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  sparse_mqa_bwd_kernel<<<2 * a.n_q, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
