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
// with wq[j] = w[t,j] * sq[t] (the query's head weight times its FP8 scale) and
// sk the key's FP8 scale. Multi-head ReLU gating as described in the
// DeepSeek-V3.2-Exp report read-through (53ai.com), section "Innovative
// architecture: core design of DSA". The four independent chains of eight
// multiply-adds each hide the FMA latency with two epilogue warps per
// scheduler; the packed form halves the multiply-add issue slots.
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

// lo: dot products of heads 0..31, hi: heads 32..63 (raw TMEM words);
// wq: 64 head weights (16-byte aligned, shared memory).
__device__ __forceinline__ float indexer_score_from_dots(const uint32_t (&lo)[32],
                                                         const uint32_t (&hi)[32],
                                                         const float* __restrict__ wq,
                                                         float sk) {
  uint64_t a = 0, b = 0, c = 0, d = 0;  // (+0.0f, +0.0f) pairs
  const float4* w4 = reinterpret_cast<const float4*>(wq);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 wa = w4[q];
    const float4 wb = w4[4 + q];
    const float4 wc = w4[8 + q];
    const float4 wd = w4[12 + q];
    a = ffma2(pack_f32x2(wa.x, wa.y),
              pack_f32x2(fmaxf(__uint_as_float(lo[4 * q + 0]), 0.f),
                         fmaxf(__uint_as_float(lo[4 * q + 1]), 0.f)),
              a);
    b = ffma2(pack_f32x2(wb.x, wb.y),
              pack_f32x2(fmaxf(__uint_as_float(lo[16 + 4 * q + 0]), 0.f),
                         fmaxf(__uint_as_float(lo[16 + 4 * q + 1]), 0.f)),
              b);
    c = ffma2(pack_f32x2(wc.x, wc.y),
              pack_f32x2(fmaxf(__uint_as_float(hi[4 * q + 0]), 0.f),
                         fmaxf(__uint_as_float(hi[4 * q + 1]), 0.f)),
              c);
    d = ffma2(pack_f32x2(wd.x, wd.y),
              pack_f32x2(fmaxf(__uint_as_float(hi[16 + 4 * q + 0]), 0.f),
                         fmaxf(__uint_as_float(hi[16 + 4 * q + 1]), 0.f)),
              d);
    a = ffma2(pack_f32x2(wa.z, wa.w),
              pack_f32x2(fmaxf(__uint_as_float(lo[4 * q + 2]), 0.f),
                         fmaxf(__uint_as_float(lo[4 * q + 3]), 0.f)),
              a);
    b = ffma2(pack_f32x2(wb.z, wb.w),
              pack_f32x2(fmaxf(__uint_as_float(lo[16 + 4 * q + 2]), 0.f),
                         fmaxf(__uint_as_float(lo[16 + 4 * q + 3]), 0.f)),
              b);
    c = ffma2(pack_f32x2(wc.z, wc.w),
              pack_f32x2(fmaxf(__uint_as_float(hi[4 * q + 2]), 0.f),
                         fmaxf(__uint_as_float(hi[4 * q + 3]), 0.f)),
              c);
    d = ffma2(pack_f32x2(wd.z, wd.w),
              pack_f32x2(fmaxf(__uint_as_float(hi[16 + 4 * q + 2]), 0.f),
                         fmaxf(__uint_as_float(hi[16 + 4 * q + 3]), 0.f)),
              d);
  }
  float ax, ay, bx, by, cx, cy, dx, dy;
  unpack_f32x2(a, ax, ay);
  unpack_f32x2(b, bx, by);
  unpack_f32x2(c, cx, cy);
  unpack_f32x2(d, dx, dy);
  return (((ax + ay) + (bx + by)) + ((cx + cy) + (dx + dy))) * sk;
}

}  // namespace dsa
