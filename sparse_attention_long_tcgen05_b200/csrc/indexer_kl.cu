// indexer_kl.cu -- the lightning indexer's KL training signal over each
// query's selected keys, on the 5th-generation tensor cores (tcgen05,
// kind::f16, bf16 -> f32).
//
// The indexer learns to match the main attention's distribution through a
// KL-divergence loss, over every preceding key in the dense warm-up and with
// only the top-k keys selected in sparse training (wiki-for-amaranth report,
// section "DeepSeek Sparse Attention (DSA)"; juhe.plus read-through, stages
// "Dense Warm-up" and "Sparse Training"; 53ai.com read-through, continued
// pre-training). For query t with selected keys i (the rows of idx_t):
//     p_i = (1/H) sum_h exp(scale * q[t,h] . kv[i] - lse[t,h])   (main attention, heads averaged)
//     r_i = softmax_i(I[t, i])                                   (the indexer, same keys)
//     loss_t = sum_i p_i (log p_i - log r_i),   grad_i = r_i - p_i  (d loss / d I[t, i])
// lse is the forward's log-sum-exp of the same selection, so p sums to 1 over
// it; with a selection of every key 0..t this is the dense warm-up signal.
//
// One CTA per query, 512 threads. All 576 key dims fit one SM here (no output
// accumulator is needed, so Q's 288 TMEM columns and two 64-column S buffers
// share the 512 columns):
//   warps 0-7    plan (index row -> physical rows, valid masks, non-empty
//                blocks), then copy each block's 64 selected rows (1152 B each)
//                with 16-byte cp.async into nine 128-byte-swizzled 64-dim
//                tiles, three stages (216 KB: the copies are latency-bound,
//                and with two stages the copy of block j could start only
//                once S of block j-2 was done -- 95.7 -> 72.6 ms at 128K);
//   warp 8       owns TMEM and issues S = Q K^T (M = 128 heads, N = 64 keys,
//                K = 576 in 36 steps of 16) into the S buffer of the block;
//   warps 12-15  stage Q in TMEM (thread = head), then per block read S, form
//                exp(scale s - lse) for their 32 heads and sum them over the
//                heads (a shuffle transpose-reduce within the warp, then the
//                four warps' partial sums in shared memory) into p, which
//                waits in the gradient row (L2-resident global memory, leaving
//                the shared memory to the copies); at the end the indexer's
//                softmax, the loss and the gradient, written over p.
#include "dsa_common.cuh"
#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int kH = 128;
constexpr int kBK = 64;
constexpr int kMaxK = 2048;
constexpr int kMaxBlocks = kMaxK / kBK;
constexpr int kChunks = 9;                      // 64-dim chunks of a 576-wide row
constexpr int kChunkBytes = kBK * 128;          // one chunk of a block: 64 rows x 128 B
constexpr int kStages = 3;
constexpr int kGatherWarps = 8;                 // warps 0-7
constexpr int kMmaWarp = 8;
constexpr int kEpiWarp0 = 12;                   // warps 12-15 = TMEM sub-partitions 0-3
constexpr int kThreads = 16 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0;                   // Q: 288 columns (bf16 pairs)
constexpr uint32_t kColS = 288;                 // S buffers: [288, 352), [352, 416)

struct __align__(1024) Smem {
  uint8_t kv[kStages][kChunks][kChunkBytes];    // 216 KB
  int32_t rows[kMaxK];                          // KV row of every index entry (0 if invalid)
  float part[4][kBK];                           // per-warp head sums of one block
  uint32_t bmask[kMaxBlocks][2];                // valid entries of block b
  uint32_t mask[kMaxBlocks][2];                 // valid entries of the j-th non-empty block
  int32_t blk[kMaxBlocks];                      // block number of the j-th non-empty block
  float red[4][2];                              // cross-warp reductions of the final pass
  int32_t n_blocks;
  int32_t n_epi;                                // the epilogue warps' common block count
  uint64_t plan_full, q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t mma_drain;
  uint32_t tmem_base;
};
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory of one CTA on sm_100");

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Sum over the 32 lanes of a warp of 64 values per lane (lane l's v[i] is the
// value of key i for the lane's head): five butterfly rounds that each halve
// the keys a lane keeps; afterwards lane l holds the sums of keys 2l, 2l+1 in
// v[0], v[1].
__device__ __forceinline__ void transpose_reduce64(float (&v)[64], int lane) {
#pragma unroll
  for (int r = 0; r < 5; ++r) {
    const int o = 16 >> r;              // lane offset of this round
    const int half = 32 >> r;           // keys kept after this round
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) indexer_kl_kernel(const KlArgs a) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~uintptr_t(1023));
  const int warp = warp_id();
  const int lane = threadIdx.x & 31;
  const int qi = blockIdx.x;

  int pos, seq = 0;
  bool q_ok = true;
  if (a.keys.paged) {
    q_ok = paged_query(a.keys, qi, seq, pos);
  } else {
    pos = a.keys.n_keys - a.keys.n_q + qi;
  }
  const int nb = (a.k + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    mbar_init(&S.plan_full, 1);
    mbar_init(&S.q_full, 4 * 32);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&S.kv_full[i], kGatherWarps);
      mbar_init(&S.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_empty[i], 4 * 32);
    }
    mbar_init(&S.mma_drain, 1);
    fence_barrier_init();
    if (!q_ok) report(a.status, DSA_ERR_DEVICE_BOUNDS);
  }
  if (warp == kMmaWarp) tmem_alloc(&S.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;

  if (warp < kGatherWarps) {
    // ------------------------------------------------------------ plan
    // warp w scans blocks 4w .. 4w+3 (two 32-entry halves each)
    bool bad = false;
    const int32_t* irow = a.idx + static_cast<int64_t>(qi) * a.ld_idx;
    for (int b = 4 * warp; b < 4 * warp + 4; ++b) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int jj = b * kBK + 32 * h + lane;
        int e = (b < nb && jj < a.k) ? __ldg(irow + jj) : -1;
        bad |= e > pos;
        e = (e >= 0 && e <= pos) ? e : -1;
        int r = 0;
        if (e >= 0) {
          if (!a.keys.paged) {
            r = e;
          } else {
            const int pg = __ldg(a.keys.block_table +
                                 static_cast<int64_t>(seq) * a.keys.ld_block_table + (e >> 6));
            if (pg < 0 || pg >= a.keys.num_pages) {
              bad = true;
              e = -1;
            } else {
              r = pg * 64 + (e & 63);
            }
          }
        }
        if (b < kMaxBlocks) S.rows[b * kBK + 32 * h + lane] = r;
        const uint32_t m = __ballot_sync(0xffffffffu, e >= 0);
        if (lane == 0 && b < kMaxBlocks) S.bmask[b][h] = m;
      }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) report(a.status, DSA_ERR_DEVICE_BOUNDS);
    named_bar_sync(1, kGatherWarps * 32);
    if (warp == 0) {
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
    named_bar_sync(1, kGatherWarps * 32);
    // ------------------------------------------------------------ gather
    // Block j: 64 rows x (two 512-byte value halves + one 128-byte rope
    // piece): 128 + 16 warp instructions, round-robin over the 8 warps; lane l
    // copies 16 bytes (64-dim chunk l / 8 of the half, 16-byte unit l % 8).
    const int n = S.n_blocks;
    const int c_l = lane >> 3, i_l = lane & 7;
    const char* const kv_b = reinterpret_cast<const char*>(a.kv);
    const int64_t ld_b = a.ld_kv * 2;
    constexpr int n_items = 2 * kBK + kBK / 4;
    auto release = [&](int jj) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.kv_full[jj % kStages]);
    };
    int issued = 0;
    for (int j = 0; j < n; ++j) {
      const int st = j % kStages;
      if (!mbar_wait_warp(&S.kv_empty[st], static_cast<uint32_t>((j / kStages) & 1) ^ 1u,
                          a.status))
        break;
      const int* rb = S.rows + S.blk[j] * kBK;
      for (int p = warp; p < n_items; p += kGatherWarps) {
        if (p < 2 * kBK) {
          const int r = p >> 1, c = 4 * (p & 1) + c_l;     // row, 64-dim chunk 0..7
          const char* src = kv_b + static_cast<int64_t>(rb[r]) * ld_b + (64 * c + 8 * i_l) * 2;
          cp_async16(smem_u32(S.kv[st][c]) + r * 128 + ((i_l ^ (r & 7)) << 4), src);
        } else {
          const int r = 4 * (p - 2 * kBK) + c_l;           // rope dims 512..575 of row r
          const char* src = kv_b + static_cast<int64_t>(rb[r]) * ld_b + (512 + 8 * i_l) * 2;
          cp_async16(smem_u32(S.kv[st][8]) + r * 128 + ((i_l ^ (r & 7)) << 4), src);
        }
      }
      cp_async_commit();
      ++issued;
      if (j > 0) {
        cp_async_wait_group<1>();
        release(j - 1);
      }
    }
    // the last block, and a drain after a give-up: every copy lands first
    cp_async_wait_group<0>();
    if (issued > 0) release(issued - 1);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = mbar_wait_warp(&S.plan_full, 0, a.status);
    const int n = ok ? S.n_blocks : 0;
    ok = ok && mbar_wait_warp(&S.q_full, 0, a.status);
    tc_fence_after();
    const uint32_t idesc = make_idesc(kBK, 1, 1, 0, 0);   // bf16, A (TMEM) and B K-major
    for (int j = 0; j < n && ok; ++j) {
      const int st = j % kStages;
      const int b = j & 1;
      if (!mbar_wait_warp(&S.kv_full[st], static_cast<uint32_t>(j / kStages) & 1u, a.status) ||
          !mbar_wait_warp(&S.s_empty[b], static_cast<uint32_t>((j >> 1) & 1) ^ 1u, a.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t d = tmem_base + kColS + 64u * static_cast<uint32_t>(b);
        for (int c = 0; c < kChunks; ++c) {
          const uint64_t kd = sw128_desc(smem_u32(S.kv[st][c]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(d, tmem_base + kColQ + c * 32 + kk * 8, kd + 2 * kk, idesc,
                        (c | kk) != 0 ? 1u : 0u);
        }
        mma_commit(&S.s_full[b]);
        mma_commit(&S.kv_empty[st]);
      }
      __syncwarp();
    }
    // Drain: the MMAs issued so far complete before TMEM is freed and before
    // their operands' shared memory goes away.
    if (lane == 0) {
      mma_commit(&S.mma_drain);
      mbar_wait(&S.mma_drain, 0, a.status);
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    const int sub = warp & 3;                       // heads 32 sub .. 32 sub + 31
    const int head = 32 * sub + lane;
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(32 * sub) << 16);
    const int et = threadIdx.x - kEpiWarp0 * 32;    // 0..127
    {
      // Q row of this head -> TMEM columns 32c .. 32c+31 for 64-dim chunk c
      const uint4* qrow = reinterpret_cast<const uint4*>(
          a.q + static_cast<int64_t>(qi) * a.ld_q + static_cast<int64_t>(head) * 576);
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = __ldg(qrow + 8 * c + i);
          w[4 * i] = v.x;
          w[4 * i + 1] = v.y;
          w[4 * i + 2] = v.z;
          w[4 * i + 3] = v.w;
        }
        tmem_st32(t_lane + kColQ + 32 * c, w);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&S.q_full);
    }
    const float sl2 = a.scale_log2;
    const float l2 = a.lse[static_cast<int64_t>(qi) * kH + head] * 1.4426950408889634f;
    float* const grow = a.grad + static_cast<int64_t>(qi) * a.ld_grad;
    bool ok = mbar_wait_warp(&S.plan_full, 0, a.status);
    // one block count for all four warps (read once, after the plan), so they
    // take the same named-barrier steps whatever their own waits did
    if (et == 0) S.n_epi = ok ? S.n_blocks : 0;
    named_bar_sync(2, 4 * 32);
    const int n = S.n_epi;
    ok = ok && n == S.n_blocks;
    // After a timed-out wait the warp stops waiting and computing but keeps
    // walking the blocks, so all four warps meet every named barrier.
    for (int j = 0; j < n; ++j) {
      const int b = j & 1;
      if (ok && !mbar_wait_warp(&S.s_full[b], static_cast<uint32_t>(j >> 1) & 1u, a.status))
        ok = false;
      float v[64];
      if (ok) {
        tc_fence_after();
        const uint32_t sb = t_lane + kColS + 64u * static_cast<uint32_t>(b);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t r[32];
          tmem_ld32(sb + 32u * static_cast<uint32_t>(h), r);
          tmem_wait_ld();
          const uint32_t mk = S.mask[j][h];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            v[32 * h + i] =
                ((mk >> i) & 1u) ? fast_exp2(fmaf(__uint_as_float(r[i]), sl2, -l2)) : 0.f;
        }
        tc_fence_before();
        mbar_arrive(&S.s_empty[b]);
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) v[i] = 0.f;
      }
      transpose_reduce64(v, lane);                   // lane l: keys 2l, 2l+1 of these 32 heads
      S.part[sub][2 * lane] = v[0];
      S.part[sub][2 * lane + 1] = v[1];
      named_bar_sync(2, 4 * 32);
      // the target of the block's entries waits in the gradient row (global
      // memory, L2-resident) until the final pass overwrites it with r - p
      // (entries past k exist only in the last block's padding: nothing of
      // them is stored, so a gradient row exactly k wide stays in bounds)
      if (et < kBK && S.blk[j] * kBK + et < a.k)
        grow[S.blk[j] * kBK + et] =
            (S.part[0][et] + S.part[1][et] + S.part[2][et] + S.part[3][et]) * (1.f / kH);
      named_bar_sync(2, 4 * 32);
    }
    // ---------------------------------------------------------- loss and gradient
    // r = softmax of the selected entries' indexer scores (entries the plan
    // found valid); loss = sum p (log p - log r); grad = r - p.
    const float* srow = a.sel + static_cast<int64_t>(qi) * a.ld_sel;
    const int32_t* irow = a.idx + static_cast<int64_t>(qi) * a.ld_idx;
    auto valid = [&](int i) {
      const int e = __ldg(irow + i);
      return e >= 0 && e <= pos && q_ok;
    };
    const int ew = et >> 5;                         // 0..3
    float m = -INFINITY;
    for (int i = et; i < a.k; i += 128)
      if (valid(i)) m = fmaxf(m, srow[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) S.red[ew][0] = m;
    named_bar_sync(2, 4 * 32);
    m = fmaxf(fmaxf(S.red[0][0], S.red[1][0]), fmaxf(S.red[2][0], S.red[3][0]));
    float z = 0.f;
    for (int i = et; i < a.k; i += 128)
      if (valid(i)) z += expf(srow[i] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane == 0) S.red[ew][1] = z;
    named_bar_sync(2, 4 * 32);
    z = (S.red[0][1] + S.red[1][1]) + (S.red[2][1] + S.red[3][1]);
    const float log_z = logf(z);
    float kl = 0.f;
    __threadfence_block();   // every thread's targets in grow seen by the others
    named_bar_sync(2, 4 * 32);
    for (int i = et; i < a.k; i += 128) {
      float g = 0.f;
      if (valid(i) && ok) {
        const float lr = (srow[i] - m) - log_z;     // log r_i
        const float p = grow[i];
        g = expf(lr) - p;
        if (p > 0.f) kl += p * (logf(p) - lr);
      }
      grow[i] = g;
    }
    named_bar_sync(2, 4 * 32);                      // S.red reused below
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kl += __shfl_xor_sync(0xffffffffu, kl, o);
    if (lane == 0) S.red[ew][0] = kl;
    named_bar_sync(2, 4 * 32);
    if (et == 0) a.loss[qi] = ok ? (S.red[0][0] + S.red[1][0]) + (S.red[2][0] + S.red[3][0])
                                 : NAN;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_indexer_kl(const KlArgs& a, cudaStream_t stream) {
  if (a.keys.n_q <= 0) return cudaSuccess;
  if (a.k > kMaxK) return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(indexer_kl_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  indexer_kl_kernel<<<a.keys.n_q, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
