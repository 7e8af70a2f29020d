// dsa_kernels.h -- internal launch interface between the C ABI (dsa_api.cu)
// and the kernels. Not installed; not part of the ABI.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace dsa {

// Query rows handled by one indexer launch: row r is query
// rows ? rows[r] : q_base + r.
struct QueryRows {
  const int32_t* rows;
  int32_t q_base;
  int32_t n_rows;
};

// Position of query i and the key-side mapping.
struct KeySide {
  int32_t paged;               // 0 contiguous, 1 paged (64-token pages)
  int32_t n_q;                 // queries in the problem
  int32_t n_keys;              // contiguous: key rows
  const int32_t* block_table;  // paged
  int64_t ld_block_table;
  int32_t max_pages;
  int32_t num_pages;
  const int32_t* ctx_lens;     // paged
};

// ---------------------------------------------------------------- indexer

struct IndexerFp8Args {
  CUtensorMap map_q;   // 3-D {d=128, heads=64, n_q} e4m3, box {128,64,1}, 128B swizzle
  CUtensorMap map_k;   // 2-D {128, key rows}, box {128, 128} (contiguous) or {128, 64} (paged)
  CUtensorMap map_sk;  // 1-D {key rows} f32 key scales, box {128} (contiguous) or {64} (paged)
  const float* q_scale;
  const float* w;
  int64_t ld_w;
  const float* k_scale;
  KeySide keys;
  QueryRows qr;
  float* scores;
  int64_t ld_scores;
  int32_t n_cols;
  int32_t write_masked;  // also write -inf for tiles wholly past every query
  int* status;
};

// pdl: launch with programmatic stream serialization, so the kernel's set-up
// overlaps the end of the kernel before it on the stream. Only for a launch
// that follows another kernel of this library issued by the same call.
cudaError_t launch_indexer_fp8(const IndexerFp8Args& a, int num_sms, bool pdl,
                               cudaStream_t stream);

struct IndexerF32Args {
  const float* q;
  int64_t ld_q;
  const float* k;
  int64_t ld_k;
  const float* w;
  int64_t ld_w;
  int32_t heads, dim;
  KeySide keys;
  QueryRows qr;
  float* scores;
  int64_t ld_scores;
  int32_t n_cols;
  int* status;
};

cudaError_t launch_indexer_f32(const IndexerF32Args& a, cudaStream_t stream);

// ---------------------------------------------------------------- top-k

struct TopkArgs {
  const float* scores;
  int64_t ld_scores;
  const int32_t* row_pos;  // pos = row_pos[r] - pos_minus, or pos_base + r when null
  int32_t pos_minus;
  int32_t pos_base;
  int32_t n_rows;
  int32_t k;
  int32_t* idx;
  int64_t ld_idx;
  int* status;
};

// pdl: as for launch_indexer_fp8.
cudaError_t launch_topk(const TopkArgs& a, bool pdl, cudaStream_t stream);

// ---------------------------------------------------------------- attention

struct AttnBf16Args {
  CUtensorMap map_kv;      // 2-D {576, kv rows} bf16, box {64, 1}, 128B swizzle (gather4)
  const __nv_bfloat16* q;  // [n_q, 128, 576], 16-byte aligned rows
  int64_t ld_q;            // elements between query tokens
  const int32_t* idx;
  int64_t ld_idx;
  int32_t k;
  KeySide keys;
  float scale_log2;     // softmax scale * log2(e)
  __nv_bfloat16* out;   // [n_q, 128, 512]
  float* lse;           // [n_q, 128] or null
  int* status;
};

cudaError_t launch_attn_bf16(const AttnBf16Args& a, cudaStream_t stream);

struct AttnF32Args {
  const float* q;
  int64_t ld_q;
  const float* kv;
  int64_t ld_kv;
  const float* v;   // nullable
  int64_t ld_v;
  int32_t heads, d_qk, d_v;
  float scale;
  const int32_t* idx;
  int64_t ld_idx;
  int32_t k;
  KeySide keys;
  float* out;
  float* lse;
  int* status;
};

cudaError_t launch_attn_f32(const AttnF32Args& a, cudaStream_t stream);

// Position of query i (shared host/device definition of the ABI rule).
__host__ __device__ __forceinline__ int32_t query_pos(const KeySide& ks, int32_t qi) {
  return ks.paged ? ks.ctx_lens[qi] - 1 : ks.n_keys - ks.n_q + qi;
}

}  // namespace dsa
