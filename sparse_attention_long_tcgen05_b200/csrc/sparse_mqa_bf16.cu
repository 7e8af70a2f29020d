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
// B200 design. The fp32 output of 128 heads x 512 values fills all 512 TMEM
// columns of one SM, so one query runs on a CLUSTER OF TWO CTAs that split the
// 576 key dimensions: CTA0 owns dims [0,256), CTA1 owns [256,576). Each CTA
//   - gathers only its column range of the selected rows (TMA tile::gather4,
//     no multicast), so the pair reads each selected row exactly once;
//   - computes a partial S_r = Q[:, dims_r] K[:, dims_r]^T (M=128 heads,
//     N=64 keys) into TMEM;
//   - sends S_r to the peer through distributed shared memory and adds the
//     peer's partial: S = S_0 + S_1 is bit-identical in both CTAs (fp32
//     addition commutes), so both run the same online softmax;
//   - accumulates its half of the value columns, O[:, 256r : 256r+256] += P V_r,
//     where V_r lies inside its own gathered columns (dims [256r, 256r+256)).
// The softmax keeps a stale running max and rescales O in TMEM only when the
// block max exceeds it by more than 2^8 (exact: the final normalisation uses
// the same max).
//
// Roles per CTA (192 threads): warp 0 gathers (TMA), warp 1 owns TMEM and
// issues MMAs, warps 2-5 (one thread per head = TMEM lane) run the softmax,
// the DSMEM exchange and the epilogue.
#include "dsa_common.cuh"
#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int kH = 128;              // query heads = MMA M
constexpr int kBK = 64;              // keys per block = QK^T MMA N
constexpr int kStages = 2;
constexpr int kMaxCh = 5;            // 64-dim chunks per CTA (CTA1: 5, CTA0: 4)
constexpr int kChunkQ = kH * 128;    // one 64-dim chunk of Q: 128 rows x 128 B
constexpr int kChunkKV = kBK * 128;  // one 64-dim chunk of a key block: 64 rows x 128 B
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;  // O: [0,256), S: [256,384)
constexpr uint32_t kColO = 0;
constexpr uint32_t kColS = 256;
constexpr float kRescaleLog2 = 8.0f;

struct __align__(1024) Smem {
  uint8_t q[kMaxCh][kChunkQ];                 // 80 KB
  uint8_t kv[kStages][kMaxCh][kChunkKV];      // 80 KB
  uint8_t p[kH * 128];                        // 16 KB: P [128 heads x 64 keys] bf16
  float recv[kH * kBK];                       // 32 KB: peer's partial S
  uint64_t q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full, p_empty;
  uint64_t o_full;
  uint64_t rx_full;   // the peer has written its partial into recv
  uint64_t rx_free;   // the peer has read its own recv (we may write into it)
  uint32_t tmem_base;
};

// The 64 index entries of block b: lane holds entries b*64+lane and
// b*64+32+lane; masks of the entries that name a key the query may see.
struct BlockEntries {
  int e0, e1;
  uint32_t m0, m1;
};

__device__ __forceinline__ BlockEntries block_entries(const AttnBf16Args& a, int qi, int pos,
                                                      int b, int lane) {
  BlockEntries E;
  const int32_t* row = a.idx + static_cast<int64_t>(qi) * a.ld_idx;
  const int j0 = b * kBK + lane, j1 = j0 + 32;
  E.e0 = j0 < a.k ? row[j0] : -1;
  E.e1 = j1 < a.k ? row[j1] : -1;
  E.m0 = __ballot_sync(0xffffffffu, E.e0 >= 0 && E.e0 <= pos);
  E.m1 = __ballot_sync(0xffffffffu, E.e1 >= 0 && E.e1 <= pos);
  return E;
}

// Row of the KV tensor map holding logical key e of query qi (0 if invalid).
__device__ __forceinline__ int kv_row(const AttnBf16Args& a, int qi, int e, bool valid) {
  if (!valid) return 0;
  if (!a.keys.paged) return e;
  int page = a.keys.block_table[static_cast<int64_t>(qi) * a.keys.ld_block_table + (e >> 6)];
  if (page < 0 || page >= a.keys.num_pages) {
    report(a.status, DSA_ERR_DEVICE_BOUNDS);
    page = 0;
  }
  return page * 64 + (e & 63);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
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
    mbar_init(&S.q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&S.kv_full[i], 1);
      mbar_init(&S.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_empty[i], 128);
    }
    mbar_init(&S.p_full, 128);
    mbar_init(&S.p_empty, 1);
    mbar_init(&S.o_full, 1);
    mbar_init(&S.rx_full, 128);
    mbar_init(&S.rx_free, 128);
    fence_barrier_init();
    if (!q_ok) report(a.status, DSA_ERR_DEVICE_BOUNDS);
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&a.map_q);
    tma_prefetch_desc(&a.map_kv);
  }
  if (warp == 1) tmem_alloc(&S.tmem_base, kTmemCols);
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ gather (TMA)
    if (lane == 0) {
      mbar_arrive_expect_tx(&S.q_full, nch * kChunkQ);
      for (int c = 0; c < nch; ++c)
        tma_load_3d(S.q[c], &a.map_q, col0 + 64 * c, 0, qi, &S.q_full);
    }
    int st = 0;
    uint32_t ph = 0;
    for (int b = 0; b < nb; ++b) {
      const BlockEntries E = block_entries(a, qi, pos, b, lane);
      if ((E.m0 | E.m1) == 0u) continue;
      if (rank == 0 && ((E.e0 > pos) || (E.e1 > pos))) report(a.status, DSA_ERR_DEVICE_BOUNDS);
      const int r0 = kv_row(a, qi, E.e0, (E.m0 >> lane) & 1u);
      const int r1 = kv_row(a, qi, E.e1, (E.m1 >> lane) & 1u);
      if (!mbar_wait_warp(&S.kv_empty[st], ph ^ 1, a.status)) break;
      if (lane == 0) mbar_arrive_expect_tx(&S.kv_full[st], nch * kChunkKV);
#pragma unroll 1
      for (int g = 0; g < kBK / 4; ++g) {
        const int src = (4 * g) & 31;
        const int v = (4 * g) < 32 ? r0 : r1;
        const int y0 = __shfl_sync(0xffffffffu, v, src + 0);
        const int y1 = __shfl_sync(0xffffffffu, v, src + 1);
        const int y2 = __shfl_sync(0xffffffffu, v, src + 2);
        const int y3 = __shfl_sync(0xffffffffu, v, src + 3);
        if (lane == 0)
          for (int c = 0; c < nch; ++c)
            tma_gather4(S.kv[st][c] + g * 512, &a.map_kv, col0 + 64 * c, y0, y1, y2, y3,
                        &S.kv_full[st]);
      }
      if (++st == kStages) { st = 0; ph ^= 1; }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc_qk = make_idesc(kBK, 1, 1, 0, 0);   // bf16, K-major A and B
    const uint32_t idesc_pv = make_idesc(256, 1, 1, 0, 1);   // bf16, K-major P, MN-major V
    const uint64_t pdesc = sw128_desc(smem_u32(S.p), 16, 1024);
    bool ok = mbar_wait_warp(&S.q_full, 0, a.status);
    tc_fence_after();
    int st = 0, sb = 0, j = 0, prev_st = 0;
    uint32_t ph = 0, sph = 0;
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
    for (int b = 0; b < nb && ok; ++b) {
      const BlockEntries E = block_entries(a, qi, pos, b, lane);
      if ((E.m0 | E.m1) == 0u) continue;
      if (!mbar_wait_warp(&S.kv_full[st], ph, a.status) ||
          !mbar_wait_warp(&S.s_empty[sb], sph ^ 1, a.status)) { ok = false; break; }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t d = tmem_base + kColS + static_cast<uint32_t>(sb * kBK);
        for (int c = 0; c < nch; ++c) {
          const uint64_t qd = sw128_desc(smem_u32(S.q[c]), 16, 1024);
          const uint64_t kd = sw128_desc(smem_u32(S.kv[st][c]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(d, qd + 2 * kk, kd + 2 * kk, idesc_qk, (c | kk) != 0 ? 1u : 0u);
        }
        mma_commit(&S.s_full[sb]);
      }
      __syncwarp();
      if (j > 0 && !issue_pv(prev_st, j - 1)) { ok = false; break; }
      prev_st = st;
      if (++st == kStages) { st = 0; ph ^= 1; }
      if (++sb == 2) { sb = 0; sph ^= 1; }
      ++j;
    }
    if (ok && j > 0) issue_pv(prev_st, j - 1);
    if (lane == 0) mma_commit(&S.o_full);
  } else {
    // ------------------------------------------------------------ softmax / exchange / epilogue
    const int sub = warp & 3;
    const int h = sub * 32 + lane;                         // head = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    const uint32_t recv_local = smem_u32(S.recv) + static_cast<uint32_t>(h) * 256u;
    const uint32_t recv_peer = mapa_shared(recv_local, peer);
    const uint32_t rx_full_peer = mapa_shared(smem_u32(&S.rx_full), peer);
    const uint32_t rx_free_peer = mapa_shared(smem_u32(&S.rx_free), peer);
    const uint32_t sw = static_cast<uint32_t>(h & 7);
    uint8_t* prow = S.p + (h >> 3) * 1024 + (h & 7) * 128;
    float m_used = -INFINITY, l = 0.f;
    int sb = 0, j = 0;
    uint32_t sph = 0;
    bool ok = true;
    for (int b = 0; b < nb && ok; ++b) {
      const BlockEntries E = block_entries(a, qi, pos, b, lane);
      if ((E.m0 | E.m1) == 0u) continue;
      // own partial S for this block
      if (!mbar_wait_warp(&S.s_full[sb], sph, a.status)) { ok = false; break; }
      tc_fence_after();
      uint32_t v[64];
      {
        uint32_t (&v0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[0]);
        uint32_t (&v1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[32]);
        tmem_ld32(tmem_base + lane_off + kColS + sb * kBK, v0);
        tmem_ld32(tmem_base + lane_off + kColS + sb * kBK + 32, v1);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(&S.s_empty[sb]);
      // send it to the peer once the peer has consumed the previous block
      if (!mbar_wait_cluster_warp(&S.rx_free, static_cast<uint32_t>((j & 1) ^ 1), a.status)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int c = 0; c < 16; ++c)
        st_cluster_v4(recv_peer + ((static_cast<uint32_t>(c) ^ sw) << 4), v[4 * c], v[4 * c + 1],
                      v[4 * c + 2], v[4 * c + 3]);
      mbar_arrive_cluster(rx_full_peer);
      // receive the peer's partial and add (same order of operands is not
      // needed: fp32 addition is commutative, both CTAs get identical S)
      if (!mbar_wait_cluster_warp(&S.rx_full, static_cast<uint32_t>(j & 1), a.status)) {
        ok = false;
        break;
      }
      float x[64];
      const float4* rp = reinterpret_cast<const float4*>(S.recv + h * kBK);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 pv = rp[c ^ static_cast<int>(sw)];
        x[4 * c + 0] = __uint_as_float(v[4 * c + 0]) + pv.x;
        x[4 * c + 1] = __uint_as_float(v[4 * c + 1]) + pv.y;
        x[4 * c + 2] = __uint_as_float(v[4 * c + 2]) + pv.z;
        x[4 * c + 3] = __uint_as_float(v[4 * c + 3]) + pv.w;
      }
      mbar_arrive_cluster(rx_free_peer);
      // scaled logits (log2 domain), masked
      float bm = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const uint32_t valid = i < 32 ? (E.m0 >> i) & 1u : (E.m1 >> (i - 32)) & 1u;
        x[i] = valid ? x[i] * a.scale_log2 : -INFINITY;
        bm = fmaxf(bm, x[i]);
      }
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
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem_base + lane_off + kColO + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem_base + lane_off + kColO + 32 * c, o);
        }
        tmem_wait_st();
      }
      l *= alpha;
      m_used = m_next;
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t w4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float p0 = exp2f(x[8 * c + 2 * i] - m_used);
          const float p1 = exp2f(x[8 * c + 2 * i + 1] - m_used);
          psum += p0 + p1;
          w4[i] = pack_bf16x2(p0, p1);
        }
        *reinterpret_cast<uint4*>(prow + ((static_cast<uint32_t>(c) ^ sw) << 4)) =
            make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      l += psum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&S.p_full);
      if (++sb == 2) { sb = 0; sph ^= 1; }
      ++j;
    }
    // epilogue: O / l -> bf16, lse
    if (mbar_wait_warp(&S.o_full, 0, a.status)) {
      tc_fence_after();
      const float inv = (ok && l > 0.f) ? 1.f / l : 0.f;
      __nv_bfloat16* orow =
          a.out + (static_cast<int64_t>(qi) * kH + h) * 512 + static_cast<int64_t>(col0);
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem_base + lane_off + kColO + 32 * c, o);
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
      if (rank == 0 && a.lse != nullptr)
        a.lse[static_cast<int64_t>(qi) * kH + h] =
            (ok && l > 0.f) ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still touch its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_attn_bf16(const AttnBf16Args& a, cudaStream_t stream) {
  if (a.keys.n_q <= 0) return cudaSuccess;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(sparse_mqa_bf16_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  sparse_mqa_bf16_kernel<<<2 * a.keys.n_q, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
