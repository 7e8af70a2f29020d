// dsa_api.cu -- the C ABI declared in include/dsa.h: host-side validation,
// TMA tensor-map encoding, workspace carving and stream-ordered launches of the
// DSA kernels. Nothing here computes a step of the method; every step runs in
// the kernels. No device memory is allocated on these paths.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "dsa.h"
#include "dsa_kernels.h"

// Per-device status word written by the kernels' checks (first error wins).
__device__ int g_dsa_status;

namespace {

thread_local int32_t t_last_cuda_error = 0;
std::atomic<int64_t> g_launches{0};

// Bound of each pipeline wait of the indexer kernel (dsa_set_wait_limit_ns).
constexpr int64_t kDefaultWaitNs = 1000LL * 1000LL * 1000LL;
std::atomic<int64_t> g_wait_ns{kDefaultWaitNs};

constexpr int kMaxDevices = 64;
constexpr int kKMax = 2048;
constexpr int kPage = 64;
constexpr int kDenseF32MaxKeys = 4096;

struct DeviceInfo {
  bool init = false;
  int* status = nullptr;
  int num_sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

dsa_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int32_t>(e);
  return DSA_ERR_CUDA;
}

#define DSA_TRY_CUDA(expr)                          \
  do {                                              \
    cudaError_t e_ = (expr);                        \
    if (e_ != cudaSuccess) return cuda_fail(e_);    \
  } while (0)

// A kernel launch through one of the dsa::launch_* helpers, counted.
#define DSA_LAUNCH(expr)                            \
  do {                                              \
    cudaError_t e_ = (expr);                        \
    if (e_ != cudaSuccess) return cuda_fail(e_);    \
    g_launches.fetch_add(1, std::memory_order_relaxed); \
  } while (0)

#define DSA_TRY(expr)                               \
  do {                                              \
    dsa_status s_ = (expr);                         \
    if (s_ != DSA_OK) return s_;                    \
  } while (0)

// NVTX ranges around each call and each score block, for a timeline profiler;
// on only when the environment variable DSA_NVTX is set to a non-zero value
// (read once). Off, a range costs one branch.
bool nvtx_on() {
  static const bool on = [] {
    const char* v = std::getenv("DSA_NVTX");
    return v != nullptr && v[0] != '\0' && v[0] != '0';
  }();
  return on;
}

struct NvtxRange {
  bool pushed;
  explicit NvtxRange(const char* name) : pushed(nvtx_on()) {
    if (pushed) nvtxRangePushA(name);
  }
  ~NvtxRange() {
    if (pushed) nvtxRangePop();
  }
};

// Device status word address and SM count of the current device (set up once
// per device, with that device current).
dsa_status device_info(DeviceInfo** out) {
  int dev = 0;
  DSA_TRY_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return DSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    void* p = nullptr;
    DSA_TRY_CUDA(cudaGetSymbolAddress(&p, g_dsa_status));
    DSA_TRY_CUDA(cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev));
    int major = 0, minor = 0;
    DSA_TRY_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    DSA_TRY_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    if (major != 10 || minor != 0) return DSA_ERR_UNSUPPORTED;   // sm_100a only
    d.status = static_cast<int*>(p);
    d.init = true;
  }
  *out = &d;
  return DSA_OK;
}

// ---------------------------------------------------------------- tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// rank-D tiled map; dims/box innermost first; strides (bytes) of dims 1..D-1.
dsa_status make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
                    const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
                    CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cuda_fail(cudaErrorNotSupported);
  cuuint64_t d[5], s[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) s[i] = strides[i];
  CUresult r = fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, s, b, e,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- validation

dsa_status check_layout(const dsa_kv_layout& kv, int32_t n_q, int32_t n_keys) {
  if (kv.kind == DSA_KV_CONTIGUOUS) {
    if (n_q < 1 || n_keys < n_q) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
  }
  if (kv.kind != DSA_KV_PAGED) return DSA_ERR_INVALID_ARG;
  if (kv.page_size != kPage) return DSA_ERR_UNSUPPORTED;
  if (n_q < 1 || kv.block_table == nullptr || kv.ctx_lens == nullptr || kv.max_pages < 1 ||
      kv.num_pages < 1 || kv.ld_block_table < kv.max_pages || kv.n_seq < 0)
    return DSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(kv.max_pages) * kPage > 0x7fffffffLL) return DSA_ERR_INVALID_ARG;
  // without q_seq, query b is sequence b: there must be a sequence per query
  if (kv.q_seq == nullptr && kv.n_seq != 0 && kv.n_seq < n_q) return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

dsa::KeySide key_side(const dsa_kv_layout& kv, int32_t n_q, int32_t n_keys) {
  dsa::KeySide k{};
  k.paged = kv.kind == DSA_KV_PAGED;
  k.n_q = n_q;
  k.n_keys = n_keys;
  k.block_table = kv.block_table;
  k.ld_block_table = kv.ld_block_table;
  k.max_pages = kv.max_pages;
  k.num_pages = kv.num_pages;
  k.ctx_lens = kv.ctx_lens;
  k.q_seq = kv.q_seq;
  k.q_pos = kv.q_pos;
  k.n_seq = kv.n_seq > 0 ? kv.n_seq : n_q;
  return k;
}

bool is_fp8_indexer(const dsa_indexer_in& in) {
  return in.dtype == DSA_E4M3 && in.heads == 64 && in.dim == 128;
}

dsa_status check_indexer(const dsa_indexer_in* in) {
  if (in == nullptr) return DSA_ERR_INVALID_ARG;
  DSA_TRY(check_layout(in->kv, in->n_q, in->n_keys));
  if (in->q == nullptr || in->k == nullptr || in->w == nullptr) return DSA_ERR_INVALID_ARG;
  if (in->heads < 1 || in->dim < 1) return DSA_ERR_INVALID_ARG;
  if (in->ld_q < static_cast<int64_t>(in->heads) * in->dim || in->ld_k < in->dim ||
      in->ld_w < in->heads)
    return DSA_ERR_INVALID_ARG;
  if (in->dtype == DSA_E4M3) {
    if (!is_fp8_indexer(*in)) return DSA_ERR_UNSUPPORTED;
    if (in->q_scale == nullptr || in->k_scale == nullptr) return DSA_ERR_INVALID_ARG;
    if (!aligned16(in->q) || !aligned16(in->k) || !aligned16(in->k_scale) || in->ld_q % 16 ||
        in->ld_k % 16)
      return DSA_ERR_INVALID_ARG;
    return DSA_OK;
  }
  if (in->dtype == DSA_F32) {
    if (in->kv.kind != DSA_KV_CONTIGUOUS) return DSA_ERR_UNSUPPORTED;
    if (in->heads > 64 || in->dim > 128 || in->dim % 4) return DSA_ERR_UNSUPPORTED;
    if (in->q_scale != nullptr || in->k_scale != nullptr) return DSA_ERR_INVALID_ARG;
    if (!aligned16(in->k) || in->ld_k % 4) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
  }
  return DSA_ERR_UNSUPPORTED;
}

bool is_bf16_attn(const dsa_attn_in& in) {
  return in.dtype == DSA_BF16 && in.heads == 128 && in.d_qk == 576 && in.d_v == 512;
}

dsa_status check_attn(const dsa_attn_in* in) {
  if (in == nullptr) return DSA_ERR_INVALID_ARG;
  DSA_TRY(check_layout(in->kv_layout, in->n_q, in->n_keys));
  if (in->q == nullptr || in->kv == nullptr) return DSA_ERR_INVALID_ARG;
  if (in->heads < 1 || in->d_qk < 1 || in->d_v < 1) return DSA_ERR_INVALID_ARG;
  if (!(in->scale > 0.f) || !std::isfinite(in->scale)) return DSA_ERR_INVALID_ARG;
  if (in->ld_q < static_cast<int64_t>(in->heads) * in->d_qk || in->ld_kv < in->d_qk)
    return DSA_ERR_INVALID_ARG;
  if (in->dtype == DSA_BF16) {
    if (!is_bf16_attn(*in) || in->v != nullptr) return DSA_ERR_UNSUPPORTED;
    if (!aligned16(in->q) || !aligned16(in->kv) || (in->ld_q * 2) % 16 || (in->ld_kv * 2) % 16)
      return DSA_ERR_INVALID_ARG;
    return DSA_OK;
  }
  if (in->dtype == DSA_F32) {
    if (in->kv_layout.kind != DSA_KV_CONTIGUOUS) return DSA_ERR_UNSUPPORTED;
    if (in->heads > 128 || in->d_qk > 256 || in->d_v > 256) return DSA_ERR_UNSUPPORTED;
    if (in->v == nullptr && in->d_v > in->d_qk) return DSA_ERR_INVALID_ARG;
    if (in->v != nullptr && in->ld_v < in->d_v) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
  }
  return DSA_ERR_UNSUPPORTED;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// Query rows per indexer launch inside the fused prefill. The score block of
// one launch (rows x keys floats) stays resident in the 126 MB L2 between the
// indexer that writes it and the top-k that reads it: at most 80 MiB. Its rows
// are a multiple of 148 where that fits, so the top-k launch (one CTA per row)
// fills the 148 SMs of a B200 in whole waves.
constexpr int64_t kBlockFloatsMax = int64_t(20) << 20;  // 80 MiB of scores
constexpr int64_t kRowGrain = 148;

int32_t forward_chunk_rows(int32_t n_q, int32_t n_cols) {
  const int64_t cols = n_cols > 0 ? n_cols : 1;
  if (int64_t(n_q) * cols <= kBlockFloatsMax) return n_q;
  int64_t c = kBlockFloatsMax / cols;
  c = c >= kRowGrain ? (c / kRowGrain) * kRowGrain : (c < 128 ? 128 : (c / 4) * 4);
  return c > n_q ? n_q : static_cast<int32_t>(c);
}

struct ForwardPlan {
  int32_t n_cols;      // columns of a score row
  int32_t chunk;       // query rows per indexer launch
  size_t scores_bytes;
  size_t idx_bytes;
};

ForwardPlan forward_plan(const dsa_indexer_in& ind, int32_t k) {
  ForwardPlan p{};
  p.n_cols = ind.kv.kind == DSA_KV_PAGED ? ind.kv.max_pages * kPage : ind.n_keys;
  p.chunk = forward_chunk_rows(ind.n_q, p.n_cols);
  p.scores_bytes = round256(static_cast<size_t>(p.chunk) * p.n_cols * sizeof(float));
  p.idx_bytes = round256(static_cast<size_t>(ind.n_q) * k * sizeof(int32_t));
  return p;
}

// ---------------------------------------------------------------- launchers

dsa_status run_indexer(const dsa_indexer_in& in, const int32_t* rows, int32_t q_base,
                       int32_t n_rows, float* scores, int64_t ld_scores, int32_t n_cols,
                       int write_masked, bool pdl, DeviceInfo* dev, cudaStream_t stream) {
  const dsa::KeySide ks = key_side(in.kv, in.n_q, in.n_keys);
  if (in.dtype == DSA_E4M3) {
    dsa::IndexerFp8Args a{};
    {
      const uint64_t dims[3] = {128, 64, static_cast<uint64_t>(in.n_q)};
      const uint64_t strides[2] = {128, static_cast<uint64_t>(in.ld_q)};
      const uint32_t box[3] = {128, 64, 1};
      DSA_TRY(make_map(&a.map_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, in.q, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B));
    }
    {
      const uint64_t rows_k = ks.paged ? static_cast<uint64_t>(in.kv.num_pages) * kPage
                                       : static_cast<uint64_t>(in.n_keys);
      const uint64_t dims[2] = {128, rows_k};
      const uint64_t strides[1] = {static_cast<uint64_t>(in.ld_k)};
      const uint32_t box[2] = {128, ks.paged ? 64u : 128u};
      DSA_TRY(make_map(&a.map_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, in.k, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B));
      const uint64_t sdims[1] = {rows_k};
      const uint32_t sbox[1] = {ks.paged ? 64u : 128u};
      DSA_TRY(make_map(&a.map_sk, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, in.k_scale, sdims, nullptr,
                       sbox, CU_TENSOR_MAP_SWIZZLE_NONE));
    }
    a.q_scale = in.q_scale;
    a.w = in.w;
    a.ld_w = in.ld_w;
    a.k_scale = in.k_scale;
    a.keys = ks;
    a.qr = {rows, q_base, n_rows};
    a.scores = scores;
    a.ld_scores = ld_scores;
    a.n_cols = n_cols;
    a.write_masked = write_masked;
    a.wait_ns = static_cast<uint64_t>(g_wait_ns.load(std::memory_order_relaxed));
    a.status = dev->status;
    DSA_LAUNCH(dsa::launch_indexer_fp8(a, dev->num_sms, pdl, stream));
    return DSA_OK;
  }
  dsa::IndexerF32Args a{};
  a.q = static_cast<const float*>(in.q);
  a.ld_q = in.ld_q;
  a.k = static_cast<const float*>(in.k);
  a.ld_k = in.ld_k;
  a.w = in.w;
  a.ld_w = in.ld_w;
  a.heads = in.heads;
  a.dim = in.dim;
  a.keys = ks;
  a.qr = {rows, q_base, n_rows};
  a.scores = scores;
  a.ld_scores = ld_scores;
  a.n_cols = n_cols;
  a.status = dev->status;
  DSA_LAUNCH(dsa::launch_indexer_f32(a, stream));
  return DSA_OK;
}

// Top-k over n_rows score rows. Row r's position: row_pos[r] when row_pos is
// set; else, with paged keys (keys != nullptr), that of query pos_base + r;
// else pos_base + r.
dsa_status run_topk(const float* scores, int64_t ld_scores, const int32_t* row_pos,
                    int32_t pos_base, const dsa::KeySide* keys, int32_t n_rows, int32_t k,
                    int32_t* idx, int64_t ld_idx, float* sel, int64_t ld_sel, bool pdl,
                    DeviceInfo* dev, cudaStream_t stream) {
  dsa::TopkArgs a{};
  a.scores = scores;
  a.ld_scores = ld_scores;
  a.row_pos = row_pos;
  a.pos_base = pos_base;
  if (keys != nullptr) a.keys = *keys;
  a.n_rows = n_rows;
  a.k = k;
  a.idx = idx;
  a.ld_idx = ld_idx;
  a.sel = sel;
  a.ld_sel = ld_sel;
  a.status = dev->status;
  // few rows (a decode batch): two CTAs per row so the row's two passes use
  // twice the SMs
  const bool pair = 2 * static_cast<int64_t>(n_rows) <= dev->num_sms;
  DSA_LAUNCH(dsa::launch_topk(a, pdl, pair, stream));
  return DSA_OK;
}

dsa_status run_attn(const dsa_attn_in& in, const int32_t* idx, int64_t ld_idx, int32_t k,
                    void* out, float* lse, DeviceInfo* dev, cudaStream_t stream) {
  const dsa::KeySide ks = key_side(in.kv_layout, in.n_q, in.n_keys);
  if (in.dtype == DSA_BF16) {
    dsa::AttnBf16Args a{};
    a.q = static_cast<const __nv_bfloat16*>(in.q);
    a.ld_q = in.ld_q;
    a.kv = static_cast<const __nv_bfloat16*>(in.kv);
    a.ld_kv = in.ld_kv;
    a.idx = idx;
    a.ld_idx = ld_idx;
    a.k = k;
    a.keys = ks;
    a.scale_log2 = in.scale * 1.4426950408889634f;
    a.out = static_cast<__nv_bfloat16*>(out);
    a.lse = lse;
    a.status = dev->status;
    DSA_LAUNCH(dsa::launch_attn_bf16(a, stream));
    return DSA_OK;
  }
  dsa::AttnF32Args a{};
  a.q = static_cast<const float*>(in.q);
  a.ld_q = in.ld_q;
  a.kv = static_cast<const float*>(in.kv);
  a.ld_kv = in.ld_kv;
  a.v = static_cast<const float*>(in.v);
  a.ld_v = in.ld_v;
  a.heads = in.heads;
  a.d_qk = in.d_qk;
  a.d_v = in.d_v;
  a.scale = in.scale;
  a.idx = idx;
  a.ld_idx = ld_idx;
  a.k = k;
  a.keys = ks;
  a.out = static_cast<float*>(out);
  a.lse = lse;
  a.status = dev->status;
  DSA_LAUNCH(dsa::launch_attn_f32(a, stream));
  return DSA_OK;
}

// Indexer -> top-k over bounded blocks of `chunk` query rows, the scores of
// one block living only in `scores` (chunk x n_cols floats). Prefill block
// rows see keys 0..off+q0+rows-1; paged rows see their sequence's pages.
// sel (nullable) receives the kept keys' scores, laid out like idx.
dsa_status run_select(const dsa_indexer_in& ind, int32_t k, int32_t* idx, int64_t ld_idx,
                      float* scores, int32_t n_cols, int32_t chunk, DeviceInfo* dev,
                      cudaStream_t stream, float* sel = nullptr, int64_t ld_sel = 0) {
  const int32_t n_q = ind.n_q;
  const bool paged = ind.kv.kind == DSA_KV_PAGED;
  const int32_t off = paged ? 0 : ind.n_keys - n_q;  // position of query 0 (contiguous)
  for (int32_t q0 = 0; q0 < n_q; q0 += chunk) {
    NvtxRange range("dsa score block (indexer + top-k)");
    const int32_t rows = n_q - q0 < chunk ? n_q - q0 : chunk;
    int32_t* out = idx + static_cast<int64_t>(q0) * ld_idx;
    float* sel_out = sel ? sel + static_cast<int64_t>(q0) * ld_sel : nullptr;
    const int32_t cols = paged ? n_cols : off + q0 + rows;  // keys any row of the block sees
    DSA_TRY(run_indexer(ind, nullptr, q0, rows, scores, cols, cols, 0, q0 > 0, dev, stream));
    if (paged) {  // row r is query q0 + r at its own position in its sequence
      const dsa::KeySide ks = key_side(ind.kv, n_q, ind.n_keys);
      DSA_TRY(run_topk(scores, cols, nullptr, q0, &ks, rows, k, out, ld_idx, sel_out, ld_sel, true,
                       dev, stream));
    } else {
      DSA_TRY(run_topk(scores, cols, nullptr, off + q0, nullptr, rows, k, out, ld_idx, sel_out,
                       ld_sel, true, dev, stream));
    }
  }
  return DSA_OK;
}

}  // namespace

extern "C" {

DSA_API dsa_status dsa_indexer_scores(const dsa_indexer_in* in, const int32_t* rows,
                                      int32_t n_rows, float* scores, int64_t ld_scores,
                                      int32_t n_cols, void* ws, size_t ws_bytes,
                                      dsa_stream_t stream) {
  NvtxRange range("dsa_indexer_scores");
  (void)ws;
  (void)ws_bytes;
  DSA_TRY(check_indexer(in));
  if (scores == nullptr || n_rows < 1 || n_cols < 1 || ld_scores < n_cols)
    return DSA_ERR_INVALID_ARG;
  if (rows == nullptr && n_rows > in->n_q) return DSA_ERR_INVALID_ARG;
  if (in->kv.kind == DSA_KV_PAGED && static_cast<int64_t>(n_cols) > int64_t(in->kv.max_pages) * kPage)
    return DSA_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  DSA_TRY(device_info(&dev));
  return run_indexer(*in, rows, 0, n_rows, scores, ld_scores, n_cols, 1, false, dev,
                     reinterpret_cast<cudaStream_t>(stream));
}

DSA_API dsa_status dsa_topk(const float* scores, int64_t ld_scores, const int32_t* row_pos,
                            int32_t n_rows, int32_t k, int32_t* idx, int64_t ld_idx,
                            dsa_stream_t stream) {
  NvtxRange range("dsa_topk");
  if (scores == nullptr || row_pos == nullptr || idx == nullptr || n_rows < 1 || ld_scores < 1)
    return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kKMax || ld_idx < k) return DSA_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  DSA_TRY(device_info(&dev));
  return run_topk(scores, ld_scores, row_pos, 0, nullptr, n_rows, k, idx, ld_idx, nullptr, 0,
                  false, dev, reinterpret_cast<cudaStream_t>(stream));
}

DSA_API dsa_status dsa_sparse_mqa_fwd(const dsa_attn_in* in, const int32_t* idx, int64_t ld_idx,
                                      int32_t k, void* out, float* lse, void* ws,
                                      size_t ws_bytes, dsa_stream_t stream) {
  NvtxRange range("dsa_sparse_mqa_fwd");
  (void)ws;
  (void)ws_bytes;
  DSA_TRY(check_attn(in));
  if (idx == nullptr || out == nullptr || k < 1 || k > kKMax || ld_idx < k)
    return DSA_ERR_INVALID_ARG;
  if (in->dtype == DSA_BF16 && !aligned16(out)) return DSA_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  DSA_TRY(device_info(&dev));
  return run_attn(*in, idx, ld_idx, k, out, lse, dev, reinterpret_cast<cudaStream_t>(stream));
}

DSA_API dsa_status dsa_dense_mqa_fwd(const dsa_attn_in* in, void* out, float* lse,
                                     dsa_stream_t stream) {
  NvtxRange range("dsa_dense_mqa_fwd");
  DSA_TRY(check_attn(in));
  if (out == nullptr) return DSA_ERR_INVALID_ARG;
  if (in->dtype == DSA_BF16 && !aligned16(out)) return DSA_ERR_INVALID_ARG;
  // the fp32 kernel keeps one probability per key in shared memory
  if (in->dtype == DSA_F32 && in->n_keys > kDenseF32MaxKeys) return DSA_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  DSA_TRY(device_info(&dev));
  return run_attn(*in, nullptr, 0, in->dtype == DSA_F32 ? in->n_keys : 0, out, lse, dev,
                  reinterpret_cast<cudaStream_t>(stream));
}

DSA_API dsa_status dsa_indexer_kl(const dsa_attn_in* attn, const int32_t* idx, int64_t ld_idx,
                                  int32_t k, const float* lse, const float* sel_scores,
                                  int64_t ld_sel, float* loss, float* grad, int64_t ld_grad,
                                  dsa_stream_t stream) {
  NvtxRange range("dsa_indexer_kl");
  DSA_TRY(check_attn(attn));
  if (attn->dtype != DSA_BF16) return DSA_ERR_UNSUPPORTED;
  if (idx == nullptr || lse == nullptr || sel_scores == nullptr || loss == nullptr ||
      grad == nullptr || k < 1 || k > kKMax || ld_idx < k || ld_sel < k || ld_grad < k)
    return DSA_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  DSA_TRY(device_info(&dev));
  dsa::KlArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(attn->q);
  a.ld_q = attn->ld_q;
  a.kv = static_cast<const __nv_bfloat16*>(attn->kv);
  a.ld_kv = attn->ld_kv;
  a.idx = idx;
  a.ld_idx = ld_idx;
  a.k = k;
  a.keys = key_side(attn->kv_layout, attn->n_q, attn->n_keys);
  a.scale_log2 = attn->scale * 1.4426950408889634f;
  a.lse = lse;
  a.sel = sel_scores;
  a.ld_sel = ld_sel;
  a.loss = loss;
  a.grad = grad;
  a.ld_grad = ld_grad;
  a.status = dev->status;
  DSA_LAUNCH(dsa::launch_indexer_kl(a, reinterpret_cast<cudaStream_t>(stream)));
  return DSA_OK;
}

DSA_API dsa_status dsa_sparse_mqa_bwd(const dsa_attn_in* in, const int32_t* idx, int64_t ld_idx,
                                      int32_t k, const void* out, const float* lse,
                                      const void* d_out, void* d_q, float* d_kv, int64_t ld_dkv,
                                      float* delta, dsa_stream_t stream) {
  NvtxRange range("dsa_sparse_mqa_bwd");
  DSA_TRY(check_attn(in));
  if (in->dtype != DSA_BF16 || in->kv_layout.kind != DSA_KV_CONTIGUOUS) return DSA_ERR_UNSUPPORTED;
  if (idx == nullptr || out == nullptr || lse == nullptr || d_out == nullptr || d_q == nullptr ||
      d_kv == nullptr || delta == nullptr || k < 1 || k > kKMax || ld_idx < k || ld_dkv < 576)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(d_out) || !aligned16(d_q)) return DSA_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  DSA_TRY(device_info(&dev));
  dsa::AttnBwdArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(in->q);
  a.ld_q = in->ld_q;
  a.kv = static_cast<const __nv_bfloat16*>(in->kv);
  a.ld_kv = in->ld_kv;
  a.idx = idx;
  a.ld_idx = ld_idx;
  a.k = k;
  a.n_q = in->n_q;
  a.n_keys = in->n_keys;
  a.scale = in->scale;
  a.scale_log2 = in->scale * 1.4426950408889634f;
  a.lse = lse;
  a.out = static_cast<const __nv_bfloat16*>(out);
  a.d_out = static_cast<const __nv_bfloat16*>(d_out);
  a.delta = delta;
  a.d_q = static_cast<__nv_bfloat16*>(d_q);
  a.d_kv = d_kv;
  a.ld_dkv = ld_dkv;
  a.status = dev->status;
  DSA_LAUNCH(dsa::launch_attn_bwd(a, reinterpret_cast<cudaStream_t>(stream)));
  return DSA_OK;
}

DSA_API dsa_status dsa_workspace_size(int32_t op, const dsa_indexer_in* indexer,
                                      const dsa_attn_in* attn, int32_t n_rows, int32_t n_cols,
                                      int32_t k, size_t* bytes) {
  (void)attn;
  (void)n_rows;
  (void)n_cols;
  if (bytes == nullptr) return DSA_ERR_INVALID_ARG;
  *bytes = 0;
  switch (op) {
    case DSA_OP_INDEXER_SCORES:
    case DSA_OP_TOPK:
    case DSA_OP_SPARSE_MQA:
      return DSA_OK;
    case DSA_OP_FORWARD:
    case DSA_OP_SELECT: {
      DSA_TRY(check_indexer(indexer));
      if (k < 1 || k > kKMax) return DSA_ERR_INVALID_ARG;
      const ForwardPlan p = forward_plan(*indexer, k);
      *bytes = p.scores_bytes + (op == DSA_OP_FORWARD ? p.idx_bytes : 0);
      return DSA_OK;
    }
    default:
      return DSA_ERR_INVALID_ARG;
  }
}

DSA_API dsa_status dsa_forward(const dsa_indexer_in* indexer, const dsa_attn_in* attn,
                               int32_t k, int32_t* idx_out, void* out, float* lse, void* ws,
                               size_t ws_bytes, dsa_stream_t stream_) {
  NvtxRange range("dsa_forward");
  DSA_TRY(check_indexer(indexer));
  DSA_TRY(check_attn(attn));
  if (out == nullptr || k < 1 || k > kKMax) return DSA_ERR_INVALID_ARG;
  if (indexer->n_q != attn->n_q || indexer->kv.kind != attn->kv_layout.kind)
    return DSA_ERR_INVALID_ARG;
  const bool paged = indexer->kv.kind == DSA_KV_PAGED;
  if (!paged && indexer->n_keys != attn->n_keys) return DSA_ERR_INVALID_ARG;
  if (paged && (indexer->kv.block_table != attn->kv_layout.block_table ||
                indexer->kv.ld_block_table != attn->kv_layout.ld_block_table ||
                indexer->kv.max_pages != attn->kv_layout.max_pages ||
                indexer->kv.ctx_lens != attn->kv_layout.ctx_lens ||
                indexer->kv.q_seq != attn->kv_layout.q_seq ||
                indexer->kv.q_pos != attn->kv_layout.q_pos ||
                indexer->kv.n_seq != attn->kv_layout.n_seq))
    return DSA_ERR_INVALID_ARG;
  const bool fp8 = indexer->dtype == DSA_E4M3 && attn->dtype == DSA_BF16;
  const bool f32 = indexer->dtype == DSA_F32 && attn->dtype == DSA_F32;
  if (!fp8 && !f32) return DSA_ERR_UNSUPPORTED;
  if (attn->dtype == DSA_BF16 && !aligned16(out)) return DSA_ERR_INVALID_ARG;
  const ForwardPlan p = forward_plan(*indexer, k);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) ||
      ws_bytes < p.scores_bytes + p.idx_bytes)
    return DSA_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo* dev = nullptr;
  DSA_TRY(device_info(&dev));
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int32_t* idx = idx_out ? idx_out
                         : reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + p.scores_bytes);
  DSA_TRY(run_select(*indexer, k, idx, k, static_cast<float*>(ws), p.n_cols, p.chunk, dev,
                     stream));
  return run_attn(*attn, idx, k, k, out, lse, dev, stream);
}

DSA_API dsa_status dsa_select(const dsa_indexer_in* indexer, int32_t k, int32_t* idx,
                              int64_t ld_idx, void* ws, size_t ws_bytes, dsa_stream_t stream) {
  NvtxRange range("dsa_select");
  DSA_TRY(check_indexer(indexer));
  if (idx == nullptr || k < 1 || k > kKMax || ld_idx < k) return DSA_ERR_INVALID_ARG;
  const ForwardPlan p = forward_plan(*indexer, k);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < p.scores_bytes)
    return DSA_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo* dev = nullptr;
  DSA_TRY(device_info(&dev));
  return run_select(*indexer, k, idx, ld_idx, static_cast<float*>(ws), p.n_cols, p.chunk, dev,
                    reinterpret_cast<cudaStream_t>(stream));
}

DSA_API dsa_status dsa_select_scored(const dsa_indexer_in* indexer, int32_t k, int32_t* idx,
                                     int64_t ld_idx, float* sel_scores, int64_t ld_sel,
                                     void* ws, size_t ws_bytes, dsa_stream_t stream) {
  NvtxRange range("dsa_select_scored");
  DSA_TRY(check_indexer(indexer));
  if (idx == nullptr || sel_scores == nullptr || k < 1 || k > kKMax || ld_idx < k || ld_sel < k)
    return DSA_ERR_INVALID_ARG;
  const ForwardPlan p = forward_plan(*indexer, k);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < p.scores_bytes)
    return DSA_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo* dev = nullptr;
  DSA_TRY(device_info(&dev));
  return run_select(*indexer, k, idx, ld_idx, static_cast<float*>(ws), p.n_cols, p.chunk, dev,
                    reinterpret_cast<cudaStream_t>(stream), sel_scores, ld_sel);
}

DSA_API int64_t dsa_launch_counter(void) { return g_launches.load(); }

DSA_API dsa_status dsa_set_wait_limit_ns(int64_t ns) {
  g_wait_ns.store(ns > 0 ? ns : kDefaultWaitNs, std::memory_order_relaxed);
  return DSA_OK;
}

DSA_API dsa_status dsa_check_status(dsa_stream_t stream) {
  DeviceInfo* dev = nullptr;
  DSA_TRY(device_info(&dev));
  DSA_TRY_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  int v = 0;
  DSA_TRY_CUDA(cudaMemcpyFromSymbol(&v, g_dsa_status, sizeof(int)));
  if (v != 0) {
    const int zero = 0;
    DSA_TRY_CUDA(cudaMemcpyToSymbol(g_dsa_status, &zero, sizeof(int)));
  }
  return static_cast<dsa_status>(v);
}

DSA_API const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported dtype/dims/layout combination";
    case DSA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small or misaligned";
    case DSA_ERR_CUDA: return "CUDA runtime error";
    case DSA_ERR_DEVICE_BOUNDS: return "device saw an index or page id out of range";
    case DSA_ERR_TIMEOUT: return "a bounded device wait ran out";
  }
  return "unknown status";
}

DSA_API int32_t dsa_last_cuda_error(void) { return t_last_cuda_error; }

DSA_API int32_t dsa_version(void) { return 201; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free selection (dsa_select_noalloc). For callers that cannot hand
// the library a workspace -- a plugin whose host owns all device memory through
// its own pool, or a loop that must not call cudaMalloc because it can
// synchronise the device -- the score rows of one block of queries live in this
// fixed file-scope array instead. It is 16 MiB on every GPU that loads the
// library, kept until the process exits. Host code must not pass its name to a
// kernel (on the host it names a stand-in, not device memory): the device
// address is looked up once per device below and passed explicitly.

namespace {

static __device__ __align__(256) float
    g_noalloc_scratch[DSA_NOALLOC_SCRATCH_BYTES / sizeof(float)];

struct NoallocScratch {
  bool init = false;
  float* ptr = nullptr;
};
NoallocScratch g_noalloc[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device; the first call on
// a device looks it up (with that device current) and caches it.
dsa_status noalloc_scratch(float** out) {
  int dev = 0;
  DSA_TRY_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return DSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocScratch& s = g_noalloc[dev];
  if (!s.init) {
    void* p = nullptr;
    DSA_TRY_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    s.ptr = static_cast<float*>(p);
    s.init = true;
  }
  *out = s.ptr;
  return DSA_OK;
}

}  // namespace

extern "C" DSA_API dsa_status dsa_select_noalloc(const dsa_indexer_in* indexer, int32_t k,
                                                 int32_t* idx, int64_t ld_idx,
                                                 dsa_stream_t stream_) {
  DSA_TRY(check_indexer(indexer));
  if (idx == nullptr || k < 1 || k > kKMax || ld_idx < k) return DSA_ERR_INVALID_ARG;
  const bool paged = indexer->kv.kind == DSA_KV_PAGED;
  const int64_t n_cols = paged ? static_cast<int64_t>(indexer->kv.max_pages) * kPage
                               : static_cast<int64_t>(indexer->n_keys);
  const int64_t cap = DSA_NOALLOC_SCRATCH_BYTES / sizeof(float);
  if (n_cols > cap) return DSA_ERR_WORKSPACE_TOO_SMALL;  // one score row must fit
  DeviceInfo* dev = nullptr;
  DSA_TRY(device_info(&dev));
  float* scratch = nullptr;
  DSA_TRY(noalloc_scratch(&scratch));
  int64_t block = cap / n_cols;            // query rows whose scores fit at once
  if (block >= 4) block -= block % 4;
  if (block > indexer->n_q) block = indexer->n_q;
  // Every score the top-k reads (columns 0..pos of each row of a block) is
  // written by the indexer launch just before it, so nothing needs clearing.
  return run_select(*indexer, k, idx, ld_idx, scratch, static_cast<int32_t>(n_cols),
                    static_cast<int32_t>(block), dev, reinterpret_cast<cudaStream_t>(stream_));
}
