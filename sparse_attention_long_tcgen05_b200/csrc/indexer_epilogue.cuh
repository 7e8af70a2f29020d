// indexer_epilogue.cuh -- the one definition of how a lightning-indexer score
// is formed from the 64 per-head code dot products of one (query, key) pair.
// Every kernel that produces or ranks indexer scores calls this function, so
// scores written by the standalone indexer and scores ranked inside the fused
// forward are bit-identical.
//
//   score = sk * sum_{j=0..63} wq[j] * max(dot_j, 0)       (j ascending, fmaf)
//
// with wq[j] = w[t,j] * sq[t] (the query's head weight times its FP8 scale) and
// sk the key's FP8 scale. Multi-head ReLU gating as described in the
// DeepSeek-V3.2-Exp report read-through (53ai.com), section "Innovative
// architecture: core design of DSA".
#pragma once

#include <cstdint>

namespace dsa {

__device__ __forceinline__ float indexer_score_from_dots(const uint32_t (&lo)[32],
                                                         const uint32_t (&hi)[32],
                                                         const float* __restrict__ wq,
                                                         float sk) {
  float acc = 0.f;
#pragma unroll
  for (int j = 0; j < 32; ++j) acc = fmaf(wq[j], fmaxf(__uint_as_float(lo[j]), 0.f), acc);
#pragma unroll
  for (int j = 0; j < 32; ++j) acc = fmaf(wq[32 + j], fmaxf(__uint_as_float(hi[j]), 0.f), acc);
  return acc * sk;
}

}  // namespace dsa
