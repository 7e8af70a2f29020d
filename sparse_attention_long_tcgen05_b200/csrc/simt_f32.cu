// simt_f32.cu -- float32 CUDA-core kernels for small problems (the tiny
// correctness workload: H_I=4, d_I=32, 8 heads, d=64, separate V). Same
// definitions as the tensor-core path, no FP8 and no scales:
//   indexer  I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]),  s <= t
//            (53ai.com read-through, section "Innovative architecture: core
//            design of DSA");
//   attention O[t,h] = softmax_i(scale * q[t,h] . K[idx_i]) V[idx_i] over the
//            selected rows, shared by every head (MQA mode, same section).
#include "dsa_common.cuh"
#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int kIdxThreads = 128;
constexpr int kAttnThreads = 128;

__global__ void __launch_bounds__(kIdxThreads) indexer_f32_kernel(const IndexerF32Args a) {
  extern __shared__ float sm[];
  float* qs = sm;                       // [heads * dim]
  float* ws = sm + a.heads * a.dim;     // [heads]
  const int r = blockIdx.x;
  int qi = a.qr.rows ? a.qr.rows[r] : a.qr.q_base + r;
  int pos = -1;
  if (qi < 0 || qi >= a.keys.n_q) {
    if (threadIdx.x == 0) report(a.status, DSA_ERR_DEVICE_BOUNDS);
    qi = 0;
  } else {
    pos = a.keys.n_keys - a.keys.n_q + qi;
  }
  const float* q = a.q + static_cast<int64_t>(qi) * a.ld_q;
  for (int i = threadIdx.x; i < a.heads * a.dim; i += blockDim.x) qs[i] = q[i];
  for (int i = threadIdx.x; i < a.heads; i += blockDim.x)
    ws[i] = a.w[static_cast<int64_t>(qi) * a.ld_w + i];
  __syncthreads();
  const int s = blockIdx.y * blockDim.x + threadIdx.x;
  if (s >= a.n_cols) return;
  float out = -INFINITY;
  if (s <= pos) {
    const float4* kr = reinterpret_cast<const float4*>(a.k + static_cast<int64_t>(s) * a.ld_k);
    float acc = 0.f;
    for (int j = 0; j < a.heads; ++j) {
      const float* qj = qs + j * a.dim;
      float dot = 0.f;
      for (int d4 = 0; d4 < a.dim / 4; ++d4) {
        const float4 kv = kr[d4];
        dot = fmaf(qj[4 * d4 + 0], kv.x, dot);
        dot = fmaf(qj[4 * d4 + 1], kv.y, dot);
        dot = fmaf(qj[4 * d4 + 2], kv.z, dot);
        dot = fmaf(qj[4 * d4 + 3], kv.w, dot);
      }
      acc = fmaf(ws[j], fmaxf(dot, 0.f), acc);
    }
    out = acc;
  }
  a.scores[static_cast<int64_t>(r) * a.ld_scores + s] = out;
}

__device__ __forceinline__ float block_reduce(float v, float* red, bool is_max) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float y = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, y) : v + y;
  }
  if (lane == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kAttnThreads / 32; ++i) r = is_max ? fmaxf(r, red[i]) : r + red[i];
  __syncthreads();
  return r;
}

// One CTA per (query, head). Sparse: the query's k selected entries; dense
// (idx null): entry j is key j for j <= pos, and k covers every key.
__global__ void __launch_bounds__(kAttnThreads) attn_f32_kernel(const AttnF32Args a) {
  extern __shared__ float sm[];
  float* qs = sm;                        // [d_qk]
  float* p = sm + a.d_qk;                // [k]
  int* rows = reinterpret_cast<int*>(p + a.k);  // [k]
  __shared__ float red[kAttnThreads / 32];
  const int qi = blockIdx.x;
  const int h = blockIdx.y;
  const int pos = a.keys.n_keys - a.keys.n_q + qi;
  const float* q = a.q + static_cast<int64_t>(qi) * a.ld_q + static_cast<int64_t>(h) * a.d_qk;
  for (int i = threadIdx.x; i < a.d_qk; i += blockDim.x) qs[i] = q[i];
  __syncthreads();
  const int32_t* idx = a.idx ? a.idx + static_cast<int64_t>(qi) * a.ld_idx : nullptr;
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < a.k; j += blockDim.x) {
    const int e = idx ? idx[j] : (j <= pos ? j : -1);
    float z = -INFINITY;
    int row = -1;
    if (e > pos) {
      report(a.status, DSA_ERR_DEVICE_BOUNDS);
    } else if (e >= 0) {
      row = e;
      const float* kr = a.kv + static_cast<int64_t>(e) * a.ld_kv;
      float dot = 0.f;
      for (int d = 0; d < a.d_qk; ++d) dot = fmaf(qs[d], kr[d], dot);
      z = a.scale * dot;
    }
    p[j] = z;
    rows[j] = row;
    mx = fmaxf(mx, z);
  }
  mx = block_reduce(mx, red, true);
  float sum = 0.f;
  for (int j = threadIdx.x; j < a.k; j += blockDim.x) {
    const float e = rows[j] >= 0 ? expf(p[j] - mx) : 0.f;
    p[j] = e;
    sum += e;
  }
  sum = block_reduce(sum, red, false);   // also orders the p[] writes
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  float* o = a.out + (static_cast<int64_t>(qi) * a.heads + h) * a.d_v;
  for (int d = threadIdx.x; d < a.d_v; d += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < a.k; ++j) {
      const int row = rows[j];
      if (row < 0) continue;
      const float v = a.v ? a.v[static_cast<int64_t>(row) * a.ld_v + d]
                          : a.kv[static_cast<int64_t>(row) * a.ld_kv + d];
      acc = fmaf(p[j], v, acc);
    }
    o[d] = acc * inv;
  }
  if (threadIdx.x == 0 && a.lse)
    a.lse[static_cast<int64_t>(qi) * a.heads + h] = sum > 0.f ? mx + logf(sum) : -INFINITY;
}

}  // namespace

cudaError_t launch_indexer_f32(const IndexerF32Args& a, cudaStream_t stream) {
  if (a.qr.n_rows <= 0 || a.n_cols <= 0) return cudaSuccess;
  dim3 grid(a.qr.n_rows, (a.n_cols + kIdxThreads - 1) / kIdxThreads);
  const size_t smem = static_cast<size_t>(a.heads * a.dim + a.heads) * sizeof(float);
  indexer_f32_kernel<<<grid, kIdxThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_attn_f32(const AttnF32Args& a, cudaStream_t stream) {
  if (a.keys.n_q <= 0) return cudaSuccess;
  dim3 grid(a.keys.n_q, a.heads);
  const size_t smem = static_cast<size_t>(a.d_qk + 2 * a.k) * sizeof(float);
  attn_f32_kernel<<<grid, kAttnThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
