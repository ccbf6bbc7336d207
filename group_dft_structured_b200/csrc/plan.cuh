// plan.cuh — tiling plans and the private layout of the Fourier-weight buffer.
//
// The forward pass and the dX pass are the same computation on different
// weights (dX is the forward of W'[c,d,u] = W[d,c,(-u) mod 4], whose Fourier
// bins are conj(What_k)^T), so one "direction plan" describes either:
// Ci = contraction channels, Do = output channels.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace feql {

constexpr int kT = 4;            // group order (p4)
constexpr int kBM = 128;         // tokens per tile = tcgen05 M
constexpr int kCK = 16;          // channels per K-chunk (one K=16 fp16 MMA step)
constexpr int kCK32 = 8;         // channels per K-chunk in split-TF32 mode (one K=8 tf32 step)
constexpr int kMaxBD = 128;      // largest output-channel tile (complex bin N = 2*BD <= 256)

__host__ __device__ inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ inline int64_t align_up(int64_t a, int64_t b) { return cdiv(a, b) * b; }

// Tensor-core direction plan (fp16 data).
struct TcPlan {
  int Ci, Do;        // contraction / output channels
  int BD;            // output channels per tile (multiple of 16, <= 128)
  int nD;            // output-channel tiles
  int nK;            // K-chunks of kCK channels
  int chunk_bytes;   // bytes of the weight tiles for one (tile, chunk): 5*BD rows x 32 B
  int64_t bytes;     // nD * nK * chunk_bytes
};

// Output-channel tile: short contractions (<= 4 chunks) are epilogue-bound, so
// they take BD <= 64 and the four accumulators (4*BD <= 256 columns) can be
// double-buffered in TMEM; long contractions take BD up to 128 so that fewer
// tiles re-read and re-transform the input.
__host__ __device__ inline TcPlan make_tc_plan(int Ci, int Do) {
  TcPlan p;
  p.Ci = Ci;
  p.Do = Do;
  p.nK = static_cast<int>(cdiv(Ci, kCK));
  p.nD = static_cast<int>(cdiv(Do, p.nK <= 4 ? kMaxBD / 2 : kMaxBD));
  p.BD = static_cast<int>(align_up(cdiv(Do, p.nD), 16));
  p.chunk_bytes = 5 * p.BD * kCK * 2;
  p.bytes = static_cast<int64_t>(p.nD) * p.nK * p.chunk_bytes;
  return p;
}

// Split-TF32 direction plan (fp32 data, FEQL_FP32_3XTF32): chunks of 8
// channels (a K-major row of 8 tf32 values is 32 bytes, the fp16 row's size),
// the same output tiles, and per (tile, chunk) two 5-plane weight tiles: the
// tf32-rounded bins (hi) and the tf32-rounded remainders (lo).
__host__ __device__ inline TcPlan make_tc_plan_tf32(int Ci, int Do) {
  TcPlan p;
  p.Ci = Ci;
  p.Do = Do;
  p.nK = static_cast<int>(cdiv(Ci, kCK32));
  p.nD = static_cast<int>(cdiv(Do, Ci <= 4 * kCK ? kMaxBD / 2 : kMaxBD));
  p.BD = static_cast<int>(align_up(cdiv(Do, p.nD), 16));
  p.chunk_bytes = 2 * 5 * p.BD * 32;
  p.bytes = static_cast<int64_t>(p.nD) * p.nK * p.chunk_bytes;
  return p;
}

// Byte offset of element (row, k) inside one weight chunk: K-major rows of
// 16 fp16 (32 B) with the 32-byte swizzle (16-byte half-row index XOR bit 2
// of the row), i.e. exactly the shared-memory image the MMA reads.
__host__ __device__ inline int sw32_offset(int row, int k) {
  return row * 32 + ((((k >> 3) ^ (row >> 2)) & 1) << 4) + (k & 7) * 2;
}

// The same for 32-bit elements (8 per row): tf32 tiles.
__host__ __device__ inline int sw32_offset4(int row, int k) {
  return row * 32 + ((((k >> 2) ^ (row >> 2)) & 1) << 4) + (k & 3) * 4;
}

// Layout of the opaque What buffer.
//   fp16 tensor-core modes: [fwd chunks][dx chunks], each direction laid out
//       [tile j][chunk kc][rows 0..5BD) with rows (every bin divided by 4)
//       [0,BD) What0 | [BD,2BD) What2 | [2BD,3BD) Re1 | [3BD,4BD) Im1 | [4BD,5BD) -Re1
//   so that rows [2BD,4BD) = (Re1 ; Im1) multiply Re X1 and the overlapping
//   window [3BD,5BD) = (Im1 ; -Re1) multiplies the stored -Im X1 plane.
//   SIMT modes: fp32 planes [dir][bin p][Do][Ci], p = (0, 2, Re 1, Im 1).
//   Split-TF32 mode: [fwd chunks][dx chunks] of make_tc_plan_tf32 tiles, each
//       chunk the hi tile (rows as above, tf32 in 32-bit words, 32-byte
//       swizzle) followed by the lo tile; bins not scaled.
enum WhatKind { kWhatSimt = 0, kWhatF16 = 1, kWhatTF32 = 2 };

struct WhatLayout {
  bool tc;
  TcPlan fwd, dx;
  int64_t off_fwd, off_dx, bytes;
};

__host__ __device__ inline WhatLayout make_what_layout(int C, int D, int kind) {
  WhatLayout L;
  const bool tc = kind != kWhatSimt;
  L.tc = tc;
  L.fwd = kind == kWhatTF32 ? make_tc_plan_tf32(C, D) : make_tc_plan(C, D);
  L.dx = kind == kWhatTF32 ? make_tc_plan_tf32(D, C) : make_tc_plan(D, C);
  if (tc) {
    L.off_fwd = 0;
    L.off_dx = align_up(L.fwd.bytes, 1024);
    L.bytes = L.off_dx + align_up(L.dx.bytes, 1024);
  } else {
    L.off_fwd = 0;
    L.off_dx = static_cast<int64_t>(4) * C * D * 4;
    L.bytes = 2 * L.off_dx;
  }
  return L;
}

}  // namespace feql
