// rdft4.cuh — the p4 group-axis butterflies on packed fp16 pairs.
//
// Flash EQ-Linear, technical summary "Specializzazione per il Gruppo di
// Rotazione p4": the 4-point DFT has entries 0 and +-1 only, so the
// non-redundant bins of a real fibre (v0, v1, v2, v3) are sums and
// differences:
//   V0 = (v0+v2) + (v1+v3),  V2 = (v0+v2) - (v1+v3),
//   Re V1 = v0 - v2,         Im V1 = v3 - v1.
// The kernels store -Im V1 = v1 - v3 (one subtraction fewer per pair); every
// consumer of that plane carries the sign instead (weight tiles, MMA negate
// bits).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace feql {

__device__ __forceinline__ __half2 as_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }
__device__ __forceinline__ uint32_t as_u32(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }

// One 16-byte chunk = two channels x four group elements (fp16), i.e. words
// (c0: v0 v1), (c0: v2 v3), (c1: v0 v1), (c1: v2 v3).  Returns the four bins of
// both channels scaled by 1/4, as packed pairs (channel c0 in the low half):
//   b0 = V0/4, b2 = V2/4, b1r = Re V1/4, b1n = -Im V1/4.
// A power-of-two scale is exact, and with it every bin of a finite fp16 fibre
// is finite (|V_k| <= 4 max|v_s|), so the operand planes hold the transform of
// any fp16 input.  The first stage forms (v0 +- v2)/4 with one rounding each:
// c = v2/4 is exact (v2 in the normal range), then fma(v0, 1/4, +-c); the
// second stage adds and subtracts those quarter sums.  Consumers undo the
// scale exactly in fp32.
__device__ __forceinline__ void rdft4_pair_q(const uint4 &v, uint32_t &b0, uint32_t &b2,
                                             uint32_t &b1r, uint32_t &b1n) {
  const __half2 k = __float2half2_rn(0.25f);
  const __half2 a0 = as_h2(v.x), c0 = as_h2(v.y), a1 = as_h2(v.z), c1 = as_h2(v.w);
  const __half2 e0 = __hmul2(c0, k), e1 = __hmul2(c1, k);
  const __half2 s0 = __hfma2(a0, k, e0), d0 = __hfma2(a0, k, __hneg2(e0));
  const __half2 s1 = __hfma2(a1, k, e1), d1 = __hfma2(a1, k, __hneg2(e1));
  const __half2 p = __lows2half2(s0, s1), q = __highs2half2(s0, s1);
  b0 = as_u32(__hadd2(p, q));
  b2 = as_u32(__hsub2(p, q));
  b1r = as_u32(__lows2half2(d0, d1));
  b1n = as_u32(__highs2half2(d0, d1));
}

}  // namespace feql
