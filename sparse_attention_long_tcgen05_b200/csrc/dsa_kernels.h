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
  const int32_t* block_table;  // paged: [n_seq, ld_block_table]
  int64_t ld_block_table;
  int32_t max_pages;
  int32_t num_pages;
  const int32_t* ctx_lens;     // paged: [n_seq]
  const int32_t* q_seq;        // paged, nullable: sequence of each query (else query i -> i)
  const int32_t* q_pos;        // paged, nullable: position of each query (else ctx - 1)
  int32_t n_seq;               // paged: sequences
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
  uint64_t wait_ns;      // bound of each pipeline wait (mbarrier) before giving up
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
  // position of row r: row_pos[r] when row_pos is set; else, for paged keys,
  // that of query pos_base + r (paged_query); else pos_base + r
  const int32_t* row_pos;
  int32_t pos_base;
  KeySide keys;
  int32_t n_rows;
  int32_t k;
  int32_t* idx;
  int64_t ld_idx;
  float* sel;              // nullable: the kept keys' scores, laid out like idx (-inf padding)
  int64_t ld_sel;
  int* status;
};

// pdl: as for launch_indexer_fp8. pair: each row on a cluster of two CTAs
// (for calls with at most half as many rows as SMs); same results.
cudaError_t launch_topk(const TopkArgs& a, bool pdl, bool pair, cudaStream_t stream);

// ---------------------------------------------------------------- attention

struct AttnBf16Args {
  const __nv_bfloat16* kv; // latent KV rows [rows, 576] (contiguous, or pages of 64 rows)
  int64_t ld_kv;           // elements between KV rows (a multiple of 8: 16-byte rows)
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

// Gradient of the sparse MQA attention (contiguous keys; query i at position
// n_keys - n_q + i): D = rowsum(dO * O), then dq (written) and dkv (accumulated).
struct AttnBwdArgs {
  const __nv_bfloat16* q;      // [n_q, 128, 576], query tokens ld_q apart
  int64_t ld_q;
  const __nv_bfloat16* kv;     // latent KV rows [n_keys, 576], ld_kv apart
  int64_t ld_kv;
  const int32_t* idx;          // [n_q, ld_idx] selected key positions (-1 skipped)
  int64_t ld_idx;
  int32_t k;
  int32_t n_q, n_keys;
  float scale;                 // softmax scale
  float scale_log2;            // scale * log2(e)
  const float* lse;            // [n_q, 128] the forward's natural-log LSE
  const __nv_bfloat16* out;    // [n_q, 128, 512] the forward's output
  const __nv_bfloat16* d_out;  // [n_q, 128, 512] upstream gradient
  float* delta;                // [n_q, 128, 2] written: rowsum(dO * O) over dims [0,256), [256,512)
  __nv_bfloat16* d_q;          // [n_q, 128, 576] written
  float* d_kv;                 // [n_keys, ld_dkv] accumulated (columns 0..575)
  int64_t ld_dkv;
  int* status;
};

cudaError_t launch_attn_bwd(const AttnBwdArgs& a, cudaStream_t stream);

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

// ---------------------------------------------------------------- indexer KL signal

struct KlArgs {
  const __nv_bfloat16* q;   // [n_q, 128, 576]
  int64_t ld_q;
  const __nv_bfloat16* kv;  // latent KV rows [rows, 576] (contiguous, or pages of 64 rows)
  int64_t ld_kv;
  const int32_t* idx;       // [n_q, ld_idx] selected key positions (-1 skipped)
  int64_t ld_idx;
  int32_t k;
  KeySide keys;
  float scale_log2;         // softmax scale * log2(e)
  const float* lse;         // [n_q, 128] the forward's natural-log LSE over the selection
  const float* sel;         // [n_q, ld_sel] indexer scores of the selected entries
  int64_t ld_sel;
  float* loss;              // [n_q]
  float* grad;              // [n_q, ld_grad]
  int64_t ld_grad;
  int* status;
};

cudaError_t launch_indexer_kl(const KlArgs& a, cudaStream_t stream);

// Sequence and position of paged query qi (the rule of the ABI's PAGED
// layout): the sequence is q_seq[qi] (qi when q_seq is null), whose ctx_lens
// cached tokens include the query's own; the position is q_pos[qi] (ctx - 1
// when q_pos is null). Returns false -- with seq 0 and pos -1 -- when the
// sequence, its length or the position is out of range.
__device__ __forceinline__ bool paged_query(const KeySide& ks, int32_t qi, int32_t& seq,
                                            int32_t& pos) {
  seq = ks.q_seq ? ks.q_seq[qi] : qi;
  pos = -1;
  if (seq < 0 || seq >= ks.n_seq) {
    seq = 0;
    return false;
  }
  const int32_t ctx = ks.ctx_lens[seq];
  if (ctx < 1 || ctx > ks.max_pages * 64) return false;
  const int32_t p = ks.q_pos ? ks.q_pos[qi] : ctx - 1;
  if (p < 0 || p >= ctx) return false;
  pos = p;
  return true;
}

}  // namespace dsa
