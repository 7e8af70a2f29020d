// topk.cu -- exact per-row top-k selection over float32 score rows.
//
// Fine-grained token selection (juhe.plus read-through, step 2 "Fine-grained
// Token Selection"; DeepSeek-V3.2-Exp report read-through on 53ai.com, section
// "Innovative architecture: core design of DSA"): query t keeps the k keys
// s <= t with the highest indexer score. Ties go to the lower s, -0.0 equals
// +0.0, NaN ranks below every number; the kept s are written in ascending
// order, padded with -1 when t+1 < k.
//
// One CTA (1024 threads) per row: a three-digit MSB radix select (11/11/10
// bits) over order-preserving uint32 keys finds the k-th largest key T and how
// many keys equal to T are kept; a final stable compaction in index order
// emits key > T, plus the first (lowest-index) keys == T.
#include "dsa_common.cuh"
#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

// Monotone map float -> uint32: a < b  <=>  key(a) < key(b); -0.0 -> key(+0.0);
// NaN -> 0 (below -inf, whose key is 0x007fffff).
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix sum; also returns the block total.
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
    uint32_t s = warp_sums[lane];
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

// Given a histogram over `nb` bins of the candidates still in play and the
// rank `k_rem` (1-based, from the top) being looked for, find the bin holding
// it. Writes the bin and the rank inside that bin to out[0], out[1].
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nb, uint32_t k_rem,
                                         uint32_t* warp_sums, uint32_t* out) {
  const int per = nb / kThreads;  // 1 or 2
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

__global__ void __launch_bounds__(kThreads, 1) topk_kernel(const TopkArgs a) {
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t warp_sums[kWarps + 1];
  __shared__ uint32_t found[2];

  const int r = blockIdx.x;
  const int tid = threadIdx.x;
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld_scores;
  int32_t* out = a.idx + static_cast<int64_t>(r) * a.ld_idx;
  const int pos = a.row_pos ? a.row_pos[r] - a.pos_minus : a.pos_base + r;
  if (pos < 0) {
    if (tid == 0) report(a.status, DSA_ERR_DEVICE_BOUNDS);
    for (int j = tid; j < a.k; j += kThreads) out[j] = -1;
    return;
  }
  const int n = pos + 1;
  const int k = a.k;
  if (n <= k) {
    for (int j = tid; j < k; j += kThreads) out[j] = j < n ? j : -1;
    return;
  }

  // ---- digit 1: bits 31..21
  for (int i = tid; i < 2048; i += kThreads) hist[i] = 0;
  __syncthreads();
  for (int i = tid; i < n; i += kThreads) atomicAdd(&hist[order_key(row[i]) >> 21], 1u);
  __syncthreads();
  find_bin(hist, 2048, static_cast<uint32_t>(k), warp_sums, found);
  uint32_t prefix = found[0];
  uint32_t k_rem = found[1];

  // ---- digit 2: bits 20..10
  for (int i = tid; i < 2048; i += kThreads) hist[i] = 0;
  __syncthreads();
  for (int i = tid; i < n; i += kThreads) {
    const uint32_t key = order_key(row[i]);
    if ((key >> 21) == prefix) atomicAdd(&hist[(key >> 10) & 2047u], 1u);
  }
  __syncthreads();
  find_bin(hist, 2048, k_rem, warp_sums, found);
  prefix = (prefix << 11) | found[0];
  k_rem = found[1];

  // ---- digit 3: bits 9..0
  for (int i = tid; i < 1024; i += kThreads) hist[i] = 0;
  __syncthreads();
  for (int i = tid; i < n; i += kThreads) {
    const uint32_t key = order_key(row[i]);
    if ((key >> 10) == prefix) atomicAdd(&hist[key & 1023u], 1u);
  }
  __syncthreads();
  find_bin(hist, 1024, k_rem, warp_sums, found);
  const uint32_t T = (prefix << 10) | found[0];
  const uint32_t take_eq = found[1];   // keys == T kept, lowest indices first

  // ---- stable compaction in index order
  uint32_t run_gt = 0, run_eq = 0;
  for (int base = 0; base < n; base += kThreads) {
    const int i = base + tid;
    uint32_t gt = 0, eq = 0;
    if (i < n) {
      const uint32_t key = order_key(row[i]);
      gt = key > T;
      eq = key == T;
    }
    uint32_t total;
    const uint32_t ex = block_excl_scan(gt | (eq << 16), warp_sums, total);
    const uint32_t gt_before = run_gt + (ex & 0xffffu);
    const uint32_t eq_before = run_eq + (ex >> 16);
    if (gt || (eq && eq_before < take_eq))
      out[gt_before + min(eq_before, take_eq)] = i;
    run_gt += total & 0xffffu;
    run_eq += total >> 16;
    if (run_gt + min(run_eq, take_eq) >= static_cast<uint32_t>(k)) break;
  }
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t stream) {
  if (a.n_rows <= 0) return cudaSuccess;
  topk_kernel<<<a.n_rows, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
