// topk.cu -- exact per-row top-k selection over float32 score rows.
//
// Fine-grained token selection (juhe.plus read-through, step 2 "Fine-grained
// Token Selection"; DeepSeek-V3.2-Exp report read-through on 53ai.com, section
// "Innovative architecture: core design of DSA"): query t keeps the k keys
// s <= t with the highest indexer score. Ties go to the lower s, -0.0 equals
// +0.0, NaN ranks below every number; the kept s are written in ascending
// order, padded with -1 when t+1 < k.
//
// One CTA (1024 threads) per row, scores compared as order-preserving uint32
// keys, rows read as float4 where their alignment allows. Two passes over the
// row:
//   1. a histogram of the top 12 key bits finds the bin b1 holding the k-th
//      largest key;
//   2. an ordered collection (warp ballots, one block scan per 8192 scores)
//      copies every key in a bin >= b1 -- the sure winners and the contenders
//      of bin b1 -- with its index into shared memory, in index order.
// The rest runs in shared memory: two 10-bit digits of the contenders give the
// exact k-th key T and how many keys equal to T are kept; a stable compaction
// of the collected list emits key > T plus the lowest-index keys == T.
// If the collection would not fit (heavy ties), the row falls back to a
// three-digit select with a compaction over the row in global memory.
#include "dsa_common.cuh"
#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kPer = 8;                     // scores per lane per chunk
constexpr int kChunk = kThreads * kPer;     // scores per block-scan
constexpr int kCap = 14336;                 // collected (index, key) pairs

struct TopkSmem {
  uint32_t hist[4096];
  uint32_t warp_sums[kWarps + 1];
  uint32_t found[2];
  uint32_t m_pub;                           // pair mode: this CTA's collected count
  int32_t lidx[kCap];
  uint32_t lkey[kCap];
};

// Monotone map float -> uint32: a < b  <=>  key(a) < key(b); -0.0 -> key(+0.0);
// NaN -> 0 (below -inf, whose key is 0x007fffff).
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix sum of one value per thread; also the total.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_sums,
                                                    uint32_t& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[w] = x;
  __syncthreads();
  if (w == 0) {
    const uint32_t s = warp_sums[lane];
    uint32_t t = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_sums[lane] = t - s;         // exclusive prefix of warp totals
    if (lane == 31) warp_sums[32] = t;
  }
  __syncthreads();
  const uint32_t r = warp_sums[w] + x - v;
  total = warp_sums[32];
  __syncthreads();
  return r;
}

// Exclusive prefix over the 32 warps of one value per warp (lane 0's `v`);
// returns it to every lane of the warp, and the block total.
__device__ __forceinline__ uint32_t warp_excl_scan(uint32_t v, uint32_t* warp_sums,
                                                   uint32_t& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (lane == 0) warp_sums[w] = v;
  __syncthreads();
  if (w == 0) {
    const uint32_t s = warp_sums[lane];
    uint32_t t = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_sums[lane] = t - s;
    if (lane == 31) warp_sums[32] = t;
  }
  __syncthreads();
  const uint32_t r = warp_sums[w];
  total = warp_sums[32];
  __syncthreads();
  return r;
}

// Given a histogram over `nb` bins and the rank `k_rem` (1-based, from the
// top) being looked for, find the bin holding it: out[0] = bin, out[1] = rank
// inside that bin.
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nb, uint32_t k_rem,
                                         uint32_t* warp_sums, uint32_t* out) {
  const int per = nb / kThreads;  // 1, 2 or 4
  const int hi = nb - 1 - threadIdx.x * per;
  uint32_t local = 0;
  for (int i = 0; i < per; ++i) local += hist[hi - i];
  uint32_t total;
  uint32_t cum = block_excl_scan(local, warp_sums, total);
  for (int i = 0; i < per; ++i) {
    const uint32_t c = hist[hi - i];
    if (cum < k_rem && cum + c >= k_rem) {
      out[0] = static_cast<uint32_t>(hi - i);
      out[1] = k_rem - cum;
    }
    cum += c;
  }
  __syncthreads();
}

__device__ __forceinline__ void clear_hist(uint32_t* hist, int nb) {
  for (int i = threadIdx.x; i < nb; i += kThreads) hist[i] = 0;
  __syncthreads();
}

// Ordered selection over `m` (index, key) pairs produced by `get(e)`, given the
// threshold key T and the number of keys == T to keep: writes the kept indices
// in the pairs' order to out[0..]. Pairs are taken kPer per lane, lane-major
// inside a warp's 256-pair segment, so one block scan covers kChunk pairs.
template <class Get>
__device__ __forceinline__ void ordered_emit(int m, uint32_t T, uint32_t take_eq, int k,
                                             int32_t* out, float* sel, const float* row,
                                             uint32_t* warp_sums, Get get) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t run_gt = 0, run_eq = 0;
  for (int c0 = 0; c0 < m; c0 += kChunk) {
    uint32_t bgt[kPer], beq[kPer];
    int id[kPer];
    uint32_t cgt = 0, ceq = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int e = c0 + w * (32 * kPer) + j * 32 + lane;
      uint32_t key = 0;
      id[j] = -1;
      if (e < m) get(e, id[j], key);
      const bool in = e < m;
      bgt[j] = __ballot_sync(0xffffffffu, in && key > T);
      beq[j] = __ballot_sync(0xffffffffu, in && key == T);
      cgt += __popc(bgt[j]);
      ceq += __popc(beq[j]);
    }
    uint32_t total;
    const uint32_t ex = warp_excl_scan(cgt | (ceq << 16), warp_sums, total);
    uint32_t gt_b = run_gt + (ex & 0xffffu);
    uint32_t eq_b = run_eq + (ex >> 16);
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const uint32_t g_me = gt_b + __popc(bgt[j] & lt);
      const uint32_t e_me = eq_b + __popc(beq[j] & lt);
      const bool gt = (bgt[j] >> lane) & 1u;
      const bool eq = (beq[j] >> lane) & 1u;
      if (gt || (eq && e_me < take_eq)) {
        const uint32_t o = g_me + min(e_me, take_eq);
        out[o] = id[j];
        if (sel != nullptr) sel[o] = row[id[j]];   // the kept key's score, as ranked
      }
      gt_b += __popc(bgt[j]);
      eq_b += __popc(beq[j]);
    }
    run_gt += total & 0xffffu;
    run_eq += total >> 16;
    if (run_gt + min(run_eq, take_eq) >= static_cast<uint32_t>(k)) break;
  }
}

// Exact select without the shared-memory collection (rows with heavy ties):
// digits 11/11/10 over the row in global memory, then an ordered compaction of
// the row.
__device__ void select_in_global(const float* row, int n, int k, int32_t* out, float* sel,
                                 TopkSmem& S) {
  clear_hist(S.hist, 2048);
  for (int i = threadIdx.x; i < n; i += kThreads) atomicAdd(&S.hist[order_key(row[i]) >> 21], 1u);
  __syncthreads();
  find_bin(S.hist, 2048, static_cast<uint32_t>(k), S.warp_sums, S.found);
  uint32_t prefix = S.found[0];
  uint32_t k_rem = S.found[1];
  clear_hist(S.hist, 2048);
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const uint32_t key = order_key(row[i]);
    if ((key >> 21) == prefix) atomicAdd(&S.hist[(key >> 10) & 2047u], 1u);
  }
  __syncthreads();
  find_bin(S.hist, 2048, k_rem, S.warp_sums, S.found);
  prefix = (prefix << 11) | S.found[0];
  k_rem = S.found[1];
  clear_hist(S.hist, 1024);
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const uint32_t key = order_key(row[i]);
    if ((key >> 10) == prefix) atomicAdd(&S.hist[key & 1023u], 1u);
  }
  __syncthreads();
  find_bin(S.hist, 1024, k_rem, S.warp_sums, S.found);
  const uint32_t T = (prefix << 10) | S.found[0];
  const uint32_t take_eq = S.found[1];
  ordered_emit(n, T, take_eq, k, out, sel, row, S.warp_sums, [&](int e, int& id, uint32_t& key) {
    id = e;
    key = order_key(row[e]);
  });
}

// kPair: each row runs on a cluster of two CTAs (used when the rows are at
// most half the SMs, e.g. a decode batch): each CTA histograms and collects
// one half of the row, the histograms are added through distributed shared
// memory, the second CTA appends its contenders after the first's in the
// first CTA's shared memory, and the first CTA finishes as in the one-CTA
// form. Halves split at a multiple of 4, so both read the row as float4 where
// it allows; the contenders stay in index order, so the result is the same.
template <bool kPair>
__global__ void __launch_bounds__(kThreads, 1) topk_kernel(const TopkArgs a) {
  extern __shared__ uint8_t smem_raw[];
  TopkSmem& S = *reinterpret_cast<TopkSmem*>(smem_raw);
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const int r = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int tid = threadIdx.x;
  const int lane = tid & 31, w = tid >> 5;
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld_scores;
  int32_t* out = a.idx + static_cast<int64_t>(r) * a.ld_idx;
  float* sel = a.sel ? a.sel + static_cast<int64_t>(r) * a.ld_sel : nullptr;
  griddep_launch_dependents();
  griddep_wait();   // the score rows come from the kernel before this one
  int pos;
  if (a.row_pos) {
    pos = a.row_pos[r];
  } else if (a.keys.paged) {
    int seq;
    paged_query(a.keys, a.pos_base + r, seq, pos);   // -1 when out of range
  } else {
    pos = a.pos_base + r;
  }
  if (pos < 0 || pos >= a.ld_scores) {
    if (rank != 0) return;                         // (both CTAs take this branch)
    if (tid == 0) report(a.status, DSA_ERR_DEVICE_BOUNDS);
    for (int j = tid; j < a.k; j += kThreads) {
      out[j] = -1;
      if (sel != nullptr) sel[j] = -INFINITY;
    }
    return;
  }
  const int n = pos + 1;
  const int k = a.k;
  if (n <= k) {
    if (rank != 0) return;
    for (int j = tid; j < k; j += kThreads) {
      out[j] = j < n ? j : -1;
      if (sel != nullptr) sel[j] = j < n ? row[j] : -INFINITY;
    }
    return;
  }

  // Rows that start on a 16-byte boundary with a row pitch of whole float4s
  // are read as float4: the float4 holding the last score stays inside the
  // row, and a lane keeps four loads in flight where it had one.
  const bool vec = (reinterpret_cast<uintptr_t>(row) & 15u) == 0 && (a.ld_scores & 3) == 0;
  const float4* row4 = reinterpret_cast<const float4*>(row);
  // this CTA's part of the row: [lo, hi)
  int lo = 0, hi = n;
  if (kPair) {
    const int h0 = min(n, (((n + 1) >> 1) + 3) & ~3);
    lo = rank == 0 ? 0 : h0;
    hi = rank == 0 ? h0 : n;
  }

  // ---- pass 1: histogram of the top 12 key bits
  clear_hist(S.hist, 4096);
  if (vec) {
    const int hi4 = (hi + 3) >> 2;
    for (int c = (lo >> 2) + tid; c < hi4; c += 4 * kThreads) {
      float4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int q = c + j * kThreads;
        v[j] = q < hi4 ? row4[q] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = 4 * (c + j * kThreads);
        if (i < hi) atomicAdd(&S.hist[order_key(v[j].x) >> 20], 1u);
        if (i + 1 < hi) atomicAdd(&S.hist[order_key(v[j].y) >> 20], 1u);
        if (i + 2 < hi) atomicAdd(&S.hist[order_key(v[j].z) >> 20], 1u);
        if (i + 3 < hi) atomicAdd(&S.hist[order_key(v[j].w) >> 20], 1u);
      }
    }
  } else {
    for (int i = lo + tid; i < hi; i += kThreads) atomicAdd(&S.hist[order_key(row[i]) >> 20], 1u);
  }
  __syncthreads();
  if (kPair) {
    // add the peer's histogram: read it, let both CTAs finish reading, add
    const uint32_t peer_hist = mapa_shared(smem_u32(S.hist), rank ^ 1u);
    uint32_t ph[4096 / kThreads];
    cluster_sync();                                // both histograms complete
#pragma unroll
    for (int i = 0; i < 4096 / kThreads; ++i)
      ph[i] = ld_shared_cluster_u32(peer_hist + 4u * static_cast<uint32_t>(tid + i * kThreads));
    cluster_sync();                                // both CTAs have read the peer's
#pragma unroll
    for (int i = 0; i < 4096 / kThreads; ++i) S.hist[tid + i * kThreads] += ph[i];
    __syncthreads();
  }
  find_bin(S.hist, 4096, static_cast<uint32_t>(k), S.warp_sums, S.found);
  const uint32_t b1 = S.found[0];
  const uint32_t k_rem = S.found[1];
  const uint32_t collect = static_cast<uint32_t>(k) - k_rem + S.hist[b1];
  if (collect > static_cast<uint32_t>(kCap)) {   // uniform: every thread read the same values
    if (rank == 0) select_in_global(row, n, k, out, sel, S);
    return;
  }

  // ---- pass 2: collect keys in bins >= b1 with their indices, in index order.
  // Warp w takes scores [c0 + 256 w, c0 + 256 w + 256) of a chunk: two slices
  // of 128, lane l holding scores 4l..4l+3 of a slice (float4 rows) or, for
  // other rows, scores j*32 + l.
  // float4 rows load the next chunk before the block scan of this one.
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t base = 0;
  float4 nxt[kPer / 4];
  if (vec) {
#pragma unroll
    for (int h = 0; h < kPer / 4; ++h) {
      const int i0 = lo + w * (32 * kPer) + h * 128 + 4 * lane;
      nxt[h] = i0 < hi ? row4[i0 >> 2] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  for (int c0 = lo; c0 < hi; c0 += kChunk) {
    uint32_t bal[kPer], key[kPer];
    uint32_t cnt = 0;
    const int wbase = c0 + w * (32 * kPer);
    if (vec) {
      float4 cur[kPer / 4];
#pragma unroll
      for (int h = 0; h < kPer / 4; ++h) {
        cur[h] = nxt[h];
        const int i1 = wbase + kChunk + h * 128 + 4 * lane;
        nxt[h] = i1 < hi ? row4[i1 >> 2] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int h = 0; h < kPer / 4; ++h) {
        const int i0 = wbase + h * 128 + 4 * lane;
        const float4 v = cur[h];
        key[4 * h + 0] = i0 < hi ? order_key(v.x) : 0u;
        key[4 * h + 1] = i0 + 1 < hi ? order_key(v.y) : 0u;
        key[4 * h + 2] = i0 + 2 < hi ? order_key(v.z) : 0u;
        key[4 * h + 3] = i0 + 3 < hi ? order_key(v.w) : 0u;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          bal[4 * h + e] = __ballot_sync(0xffffffffu, i0 + e < hi && (key[4 * h + e] >> 20) >= b1);
      }
    } else {
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = wbase + j * 32 + lane;
        key[j] = i < hi ? order_key(row[i]) : 0u;
        bal[j] = __ballot_sync(0xffffffffu, i < hi && (key[j] >> 20) >= b1);
      }
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) cnt += __popc(bal[j]);
    uint32_t total;
    uint32_t off = base + warp_excl_scan(cnt, S.warp_sums, total);
    if (vec) {
#pragma unroll
      for (int h = 0; h < kPer / 4; ++h) {
        uint32_t p = off;
#pragma unroll
        for (int e = 0; e < 4; ++e) p += __popc(bal[4 * h + e] & lt);
        const int i0 = wbase + h * 128 + 4 * lane;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if ((bal[4 * h + e] >> lane) & 1u) {
            S.lidx[p] = i0 + e;
            S.lkey[p] = key[4 * h + e];
            ++p;
          }
          off += __popc(bal[4 * h + e]);
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        if ((bal[j] >> lane) & 1u) {
          const uint32_t p = off + __popc(bal[j] & lt);
          S.lidx[p] = wbase + j * 32 + lane;
          S.lkey[p] = key[j];
        }
        off += __popc(bal[j]);
      }
    }
    base += total;
  }
  __syncthreads();
  int m = static_cast<int>(base);
  if (kPair) {
    // the second CTA appends its contenders after the first CTA's, in the
    // first CTA's shared memory (the two counts add up to `collect`, which
    // fits the buffer); then the first CTA goes on alone
    if (tid == 0) S.m_pub = base;
    cluster_sync();
    if (rank == 1) {
      const uint32_t m0 = ld_shared_cluster_u32(mapa_shared(smem_u32(&S.m_pub), 0u));
      const uint32_t pidx = mapa_shared(smem_u32(S.lidx), 0u);
      const uint32_t pkey = mapa_shared(smem_u32(S.lkey), 0u);
      for (int e = tid; e < m; e += kThreads) {
        st_shared_cluster_u32(pidx + 4u * (m0 + static_cast<uint32_t>(e)),
                              static_cast<uint32_t>(S.lidx[e]));
        st_shared_cluster_u32(pkey + 4u * (m0 + static_cast<uint32_t>(e)), S.lkey[e]);
      }
    } else {
      m += static_cast<int>(ld_shared_cluster_u32(mapa_shared(smem_u32(&S.m_pub), 1u)));
    }
    cluster_sync();                                // the appended list is in place
    if (rank == 1) return;
  }

  // ---- exact threshold among the contenders of bin b1 (shared memory only)
  clear_hist(S.hist, 1024);
  for (int e = tid; e < m; e += kThreads) {
    const uint32_t kk = S.lkey[e];
    if ((kk >> 20) == b1) atomicAdd(&S.hist[(kk >> 10) & 1023u], 1u);
  }
  __syncthreads();
  find_bin(S.hist, 1024, k_rem, S.warp_sums, S.found);
  const uint32_t p2 = (b1 << 10) | S.found[0];
  const uint32_t k_rem2 = S.found[1];
  clear_hist(S.hist, 1024);
  for (int e = tid; e < m; e += kThreads) {
    const uint32_t kk = S.lkey[e];
    if ((kk >> 10) == p2) atomicAdd(&S.hist[kk & 1023u], 1u);
  }
  __syncthreads();
  find_bin(S.hist, 1024, k_rem2, S.warp_sums, S.found);
  const uint32_t T = (p2 << 10) | S.found[0];
  const uint32_t take_eq = S.found[1];

  // ---- ordered emit from the collected list
  ordered_emit(m, T, take_eq, k, out, sel, row, S.warp_sums, [&](int e, int& id, uint32_t& kk) {
    id = S.lidx[e];
    kk = S.lkey[e];
  });
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, bool pdl, bool pair, cudaStream_t stream) {
  if (a.n_rows <= 0) return cudaSuccess;
  const size_t smem = sizeof(TopkSmem);
  auto kernel = pair ? topk_kernel<true> : topk_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pair ? 2 * a.n_rows : a.n_rows);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (pair) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 2;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

}  // namespace dsa
