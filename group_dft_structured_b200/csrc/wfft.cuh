// wfft.cuh — weight transform: non-redundant bins of the 4-point real DFT of
// W along the group axis, written in the layout each pass consumes.
//
// Flash EQ-Linear, technical summary "Approccio Algoritmico" and
// "Specializzazione per il Gruppo di Rotazione p4": for real W the bins are
//   What0 = w0+w1+w2+w3, What2 = w0-w1+w2-w3, What1 = (w0-w2) + i (w3-w1),
// and What3 = conj(What1) is never stored.  The dX pass uses conj(What)^T.
#pragma once

#include <cuda_fp16.h>

#include "plan.cuh"
#include "sm100.cuh"

namespace feql {

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }

// Bins of W[o_orig... ] for output channel o and contraction channel i of a
// direction: dir 0 (forward) reads W[o][i][:], dir 1 (dX) reads W[i][o][:]
// and conjugates (Im1 -> -Im1).
template <typename T>
__device__ __forceinline__ void weight_bins(const T *__restrict__ W, int C, int dir, int o, int i,
                                            float &b0, float &b2, float &b1r, float &b1i) {
  const int d = dir == 0 ? o : i;
  const int c = dir == 0 ? i : o;
  const T *w = W + (static_cast<int64_t>(d) * C + c) * kT;
  const float w0 = to_f32(w[0]), w1 = to_f32(w[1]), w2 = to_f32(w[2]), w3 = to_f32(w[3]);
  b0 = (w0 + w2) + (w1 + w3);
  b2 = (w0 + w2) - (w1 + w3);
  b1r = w0 - w2;
  b1i = dir == 0 ? (w3 - w1) : (w1 - w3);
}

// Tensor-core layout (fp16): one thread per element of the tiled buffer.
// The bins are stored divided by 4 (exact), so that every bin of a finite fp16
// weight is finite; the passes' epilogues undo the scale in fp32.
__global__ void wfft_tc_kernel(const __half *__restrict__ W, uint8_t *__restrict__ What,
                               WhatLayout L, int C) {
  const int64_t n_fwd = L.fwd.bytes / 2, n_dx = L.dx.bytes / 2;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n_fwd + n_dx;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int dir = e < n_fwd ? 0 : 1;
    const TcPlan &P = dir == 0 ? L.fwd : L.dx;
    const int64_t le = dir == 0 ? e : e - n_fwd;
    const int rows = 5 * P.BD;
    const int64_t chunk = le / (rows * kCK);
    const int rem = static_cast<int>(le % (rows * kCK));
    const int row = rem / kCK, k = rem % kCK;
    const int j = static_cast<int>(chunk / P.nK), kc = static_cast<int>(chunk % P.nK);
    // which plane (What0, What2, Re1, Im1, -Re1), which output channel
    const int sub = row / P.BD;
    const int o = j * P.BD + row % P.BD;
    const int i = kc * kCK + k;
    float v = 0.f;
    if (o < P.Do && i < P.Ci) {
      float b0, b2, b1r, b1i;
      weight_bins(W, C, dir, o, i, b0, b2, b1r, b1i);
      if (sub == 0) v = b0;
      else if (sub == 1) v = b2;
      else if (sub == 2) v = b1r;
      else if (sub == 3) v = b1i;
      else v = -b1r;
    }
    const int64_t base = (dir == 0 ? L.off_fwd : L.off_dx) + chunk * P.chunk_bytes;
    *reinterpret_cast<__half *>(What + base + sw32_offset(row, k)) = __float2half_rn(0.25f * v);
  }
}

// Split-TF32 layout: per (tile, chunk of 8 input channels) the hi tile (the
// bins rounded to tf32) then the lo tile (the remainders rounded to tf32),
// each 5*BD rows of 8 words with the 32-byte swizzle.  One thread per word.
__global__ void wfft_tf32_kernel(const float *__restrict__ W, uint8_t *__restrict__ What,
                                 WhatLayout L, int C) {
  const int64_t n_fwd = L.fwd.bytes / 4, n_dx = L.dx.bytes / 4;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n_fwd + n_dx;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int dir = e < n_fwd ? 0 : 1;
    const TcPlan &P = dir == 0 ? L.fwd : L.dx;
    const int64_t le = dir == 0 ? e : e - n_fwd;
    const int rows = 5 * P.BD;
    const int64_t chunk = le / (2 * rows * kCK32);
    const int rem = static_cast<int>(le % (2 * rows * kCK32));
    const int half = rem / (rows * kCK32);  // 0: hi tile, 1: lo tile
    const int row = (rem % (rows * kCK32)) / kCK32, k = rem % kCK32;
    const int j = static_cast<int>(chunk / P.nK), kc = static_cast<int>(chunk % P.nK);
    const int sub = row / P.BD;
    const int o = j * P.BD + row % P.BD;
    const int i = kc * kCK32 + k;
    float v = 0.f;
    if (o < P.Do && i < P.Ci) {
      float b0, b2, b1r, b1i;
      weight_bins(W, C, dir, o, i, b0, b2, b1r, b1i);
      if (sub == 0) v = b0;
      else if (sub == 1) v = b2;
      else if (sub == 2) v = b1r;
      else if (sub == 3) v = b1i;
      else v = -b1r;
    }
    const uint32_t hi = tf32_rna(v);
    const uint32_t word = half == 0 ? hi : tf32_rna(v - __uint_as_float(hi));
    const int64_t base = (dir == 0 ? L.off_fwd : L.off_dx) + chunk * P.chunk_bytes +
                         half * (rows * 32);
    *reinterpret_cast<uint32_t *>(What + base + sw32_offset4(row, k)) = word;
  }
}

// SIMT layout: fp32 planes [dir][p][o][i].
template <typename T>
__global__ void wfft_simt_kernel(const T *__restrict__ W, float *__restrict__ What, int C, int D) {
  const int64_t per_dir = static_cast<int64_t>(C) * D;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < 2 * per_dir;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int dir = e < per_dir ? 0 : 1;
    const int64_t le = dir == 0 ? e : e - per_dir;
    const int Ci = dir == 0 ? C : D;
    const int o = static_cast<int>(le / Ci), i = static_cast<int>(le % Ci);
    float b0, b2, b1r, b1i;
    weight_bins(W, C, dir, o, i, b0, b2, b1r, b1i);
    float *P = What + dir * 4 * per_dir;
    P[0 * per_dir + le] = b0;
    P[1 * per_dir + le] = b2;
    P[2 * per_dir + le] = b1r;
    P[3 * per_dir + le] = b1i;
  }
}

}  // namespace feql
