// indexer_epilogue.cuh -- the one definition of how a lightning-indexer score
// is formed from the 64 per-head code dot products of one (query, key) pair.
// Every kernel that produces or ranks indexer scores calls this function, so
// scores written by the standalone indexer and scores ranked inside the fused
// forward are bit-identical.
//
//   score = sk * (((A.x + A.y) + (B.x + B.y)) + ((C.x + C.y) + (D.x + D.y))),
//   A, B, C, D = sums over heads [0,16), [16,32), [32,48), [48,64), each kept
//   as an (even head, odd head) pair of running fp32 sums updated in ascending
//   j with a packed fused multiply-add:  (x, y) <- (wq[j] * max(d_j, 0) + x,
//                                                  wq[j+1] * max(d_j+1, 0) + y)
//
// with wq[j] = w[t,j] * sq[t] (the query's head weight times its FP8 scale;
// staged halved for odd j, see chain_step) and
// sk the key's FP8 scale. Multi-head ReLU gating as described in the
// DeepSeek-V3.2-Exp report read-through (53ai.com), section "Innovative
// architecture: core design of DSA". Two independent chains per half of the
// heads keep the multiply-add latency off the critical path; the packed form
// halves the multiply-add issue slots. Each chain's operations and their order
// are fixed by this definition, whether its inputs come from one TMEM load of
// all 64 heads or two loads of 32.
#pragma once

#include <cstdint>

namespace dsa {

__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void unpack_f32x2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// acc <- w * x + acc on two fp32 lanes at once
__device__ __forceinline__ uint64_t ffma2(uint64_t w, uint64_t x, uint64_t acc) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(w), "l"(x), "l"(acc));
  return r;
}

// One step of a chain pair: (x, y) <- (w[0] * max(d0, 0) + x, w[1] * max(d1, 0) + y).
// The odd head's ReLU is evaluated as d + |d| = 2 max(d, 0) with its weight
// staged at half (wq[j] = w[t,j] sq[t] / 2 for odd j): both factors are exact
// (scaling by a power of two), so the product and the fused multiply-add round
// exactly as w * max(d, 0) would, while the add runs on the FMA pipe and the
// max of the even head on the ALU pipe, which takes a max at half rate.
__device__ __forceinline__ uint64_t chain_step(float w0, float w1, uint32_t d0, uint32_t d1,
                                               uint64_t acc) {
  const float x0 = __uint_as_float(d0), x1 = __uint_as_float(d1);
  return ffma2(pack_f32x2(w0, w1), pack_f32x2(fmaxf(x0, 0.f), x1 + fabsf(x1)), acc);
}

// Chains over 32 consecutive heads: x from dots[0..15] (weights wq[0..15]),
// y from dots[16..31] (weights wq[16..31]), each in ascending head order.
// Called with the dot products of heads 0..31 for chains A, B and of heads
// 32..63 for chains C, D (raw TMEM words; wq 16-byte aligned shared memory).
__device__ __forceinline__ void indexer_chains32(const uint32_t (&dots)[32],
                                                 const float* __restrict__ wq, uint64_t& x,
                                                 uint64_t& y) {
  const float4* w4 = reinterpret_cast<const float4*>(wq);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 wa = w4[q];
    const float4 wb = w4[4 + q];
    x = chain_step(wa.x, wa.y, dots[4 * q + 0], dots[4 * q + 1], x);
    y = chain_step(wb.x, wb.y, dots[16 + 4 * q + 0], dots[16 + 4 * q + 1], y);
    x = chain_step(wa.z, wa.w, dots[4 * q + 2], dots[4 * q + 3], x);
    y = chain_step(wb.z, wb.w, dots[16 + 4 * q + 2], dots[16 + 4 * q + 3], y);
  }
}

// The score from the four finished chains and the key's scale.
__device__ __forceinline__ float indexer_finish(uint64_t a, uint64_t b, uint64_t c, uint64_t d,
                                                float sk) {
  float ax, ay, bx, by, cx, cy, dx, dy;
  unpack_f32x2(a, ax, ay);
  unpack_f32x2(b, bx, by);
  unpack_f32x2(c, cx, cy);
  unpack_f32x2(d, dx, dy);
  return (((ax + ay) + (bx + by)) + ((cx + cy) + (dx + dy))) * sk;
}

// lo: dot products of heads 0..31, hi: heads 32..63 (raw TMEM words);
// wq: 64 head weights (16-byte aligned, shared memory).
__device__ __forceinline__ float indexer_score_from_dots(const uint32_t (&lo)[32],
                                                         const uint32_t (&hi)[32],
                                                         const float* __restrict__ wq,
                                                         float sk) {
  uint64_t a = 0, b = 0, c = 0, d = 0;  // (+0.0f, +0.0f) pairs
  indexer_chains32(lo, wq, a, b);
  indexer_chains32(hi, wq + 32, c, d);
  return indexer_finish(a, b, c, d, sk);
}

}  // namespace dsa
