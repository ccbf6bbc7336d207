// simt.cuh — CUDA-core (fp32 FMA) kernels of the three passes.
//
// Same algorithm as the tensor-core path (Flash EQ-Linear, technical summary
// "Approccio Algoritmico"): 4-point rDFT of the activations in the load
// phase, the per-bin products in registers, inverse rDFT (+ bias) before the
// store.  Used for the fp32 SIMT mode and as an fp16 cross-check.
#pragma once

#include <cuda_fp16.h>

#include "plan.cuh"
#include "wfft.cuh"

namespace feql {

constexpr int kSimtTile = 64;   // tokens x outputs per block
constexpr int kSimtK = 16;      // channels (or tokens, for dW) per smem chunk
constexpr int kSimtThreads = 256;

template <typename T>
struct Vec4;
template <>
struct Vec4<float> {
  __device__ static void load(const float *p, float (&v)[4]) {
    const float4 q = *reinterpret_cast<const float4 *>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
  }
  __device__ static void store(float *p, const float (&v)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};
template <>
struct Vec4<__half> {
  __device__ static void load(const __half *p, float (&v)[4]) {
    const uint2 q = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&q.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&q.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  }
  __device__ static void store(__half *p, const float (&v)[4]) {
    __half2 a = __floats2half2_rn(v[0], v[1]);
    __half2 b = __floats2half2_rn(v[2], v[3]);
    uint2 q;
    q.x = *reinterpret_cast<uint32_t *>(&a);
    q.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = q;
  }
};

// 4-point rDFT of one group fibre: (V0, V2, Re V1, Im V1).
__device__ __forceinline__ void rdft4(const float (&v)[4], float (&o)[4]) {
  const float a = v[0] + v[2], b = v[1] + v[3];
  o[0] = a + b;
  o[1] = a - b;
  o[2] = v[0] - v[2];
  o[3] = v[3] - v[1];
}

// Inverse: y_t = (Y0 + (-1)^t Y2)/4 + Re(Y1 i^t)/2.
__device__ __forceinline__ void irdft4(float Y0, float Y2, float Y1r, float Y1i, float (&y)[4]) {
  const float e = 0.25f * (Y0 + Y2), o = 0.25f * (Y0 - Y2);
  const float hr = 0.5f * Y1r, hi = 0.5f * Y1i;
  y[0] = e + hr;
  y[1] = o - hi;
  y[2] = e - hr;
  y[3] = o + hi;
}

// Forward / dX: out[n][o][:] = irdft( sum_i What_k[o][i] * rdft(in[n][i][:]) ) (+ bias[o]).
template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
simt_fwd_kernel(const T *__restrict__ in, const float *__restrict__ Wp, const T *__restrict__ bias,
                T *__restrict__ out, int64_t N, int Ci, int Do) {
  __shared__ float Xs[4][kSimtK][kSimtTile + 1];
  __shared__ float Ws[4][kSimtK][kSimtTile + 1];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kSimtTile;
  const int o0 = blockIdx.y * kSimtTile;
  const int64_t plane = static_cast<int64_t>(Do) * Ci;

  float acc[4][4][4];  // [bin][i][j]
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[p][i][j] = 0.f;

  for (int c0 = 0; c0 < Ci; c0 += kSimtK) {
#pragma unroll
    for (int q = 0; q < (kSimtTile * kSimtK) / kSimtThreads; ++q) {
      const int e = tid + q * kSimtThreads;
      const int nn = e / kSimtK, kk = e % kSimtK;
      float v[4] = {0.f, 0.f, 0.f, 0.f}, f[4];
      if (n0 + nn < N && c0 + kk < Ci) Vec4<T>::load(in + ((n0 + nn) * Ci + c0 + kk) * kT, v);
      rdft4(v, f);
#pragma unroll
      for (int p = 0; p < 4; ++p) Xs[p][kk][nn] = f[p];
    }
#pragma unroll
    for (int q = 0; q < (4 * kSimtTile * kSimtK) / kSimtThreads; ++q) {
      const int e = tid + q * kSimtThreads;
      const int p = e / (kSimtTile * kSimtK);
      const int oo = (e / kSimtK) % kSimtTile, kk = e % kSimtK;
      float w = 0.f;
      if (o0 + oo < Do && c0 + kk < Ci) w = Wp[p * plane + static_cast<int64_t>(o0 + oo) * Ci + c0 + kk];
      Ws[p][kk][oo] = w;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kSimtK; ++kk) {
      float xv[4][4], wv[4][4];
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          xv[p][i] = Xs[p][kk][ty + 16 * i];
          wv[p][i] = Ws[p][kk][tx + 16 * i];
        }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[0][i][j] = fmaf(xv[0][i], wv[0][j], acc[0][i][j]);
          acc[1][i][j] = fmaf(xv[1][i], wv[1][j], acc[1][i][j]);
          acc[2][i][j] = fmaf(xv[2][i], wv[2][j], acc[2][i][j]);
          acc[2][i][j] = fmaf(-xv[3][i], wv[3][j], acc[2][i][j]);
          acc[3][i][j] = fmaf(xv[2][i], wv[3][j], acc[3][i][j]);
          acc[3][i][j] = fmaf(xv[3][i], wv[2][j], acc[3][i][j]);
        }
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t n = n0 + ty + 16 * i;
    if (n >= N) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int o = o0 + tx + 16 * j;
      if (o >= Do) continue;
      float y[4];
      irdft4(acc[0][i][j], acc[1][i][j], acc[2][i][j], acc[3][i][j], y);
      if (bias != nullptr) {
        const float bv = to_f32(bias[o]);
        y[0] += bv; y[1] += bv; y[2] += bv; y[3] += bv;
      }
      Vec4<T>::store(out + (n * Do + o) * kT, y);
    }
  }
}

// dW partial sums over one token split:
//   G0 = sum dY0 X0, G2 = sum dY2 X2, G1 = sum dY1 conj(X1)
//   (G1r = dY1r X1r + dY1i X1i, G1i = dY1i X1r - dY1r X1i),
// written as fp32 ws[split][bin][D][C]; db partials ws_db[split][D].
template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
simt_dw_partial_kernel(const T *__restrict__ x, const T *__restrict__ dy, float *__restrict__ ws,
                       float *__restrict__ ws_db, int64_t N, int C, int D, int64_t split_len) {
  __shared__ float Ys[4][kSimtK][kSimtTile + 1];
  __shared__ float Xs[4][kSimtK][kSimtTile + 1];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int d0 = blockIdx.x * kSimtTile, c0 = blockIdx.y * kSimtTile;
  const int split = blockIdx.z;
  const int64_t t_begin = split * split_len;
  const int64_t t_end = t_begin + split_len < N ? t_begin + split_len : N;
  const bool do_db = blockIdx.y == 0;

  float acc[4][4][4];
  float dbacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[p][i][j] = 0.f;

  for (int64_t t0 = t_begin; t0 < t_end; t0 += kSimtK) {
#pragma unroll
    for (int q = 0; q < (kSimtTile * kSimtK) / kSimtThreads; ++q) {
      const int e = tid + q * kSimtThreads;
      const int nn = e / kSimtTile, cc = e % kSimtTile;
      float v[4] = {0.f, 0.f, 0.f, 0.f}, f[4];
      if (t0 + nn < t_end && d0 + cc < D) Vec4<T>::load(dy + ((t0 + nn) * D + d0 + cc) * kT, v);
      rdft4(v, f);
#pragma unroll
      for (int p = 0; p < 4; ++p) Ys[p][nn][cc] = f[p];
      float u[4] = {0.f, 0.f, 0.f, 0.f}, g[4];
      if (t0 + nn < t_end && c0 + cc < C) Vec4<T>::load(x + ((t0 + nn) * C + c0 + cc) * kT, u);
      rdft4(u, g);
#pragma unroll
      for (int p = 0; p < 4; ++p) Xs[p][nn][cc] = g[p];
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kSimtK; ++kk) {
      float yv[4][4], xv[4][4];
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          yv[p][i] = Ys[p][kk][ty + 16 * i];
          xv[p][i] = Xs[p][kk][tx + 16 * i];
        }
      if (do_db && tx == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) dbacc[i] += yv[0][i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[0][i][j] = fmaf(yv[0][i], xv[0][j], acc[0][i][j]);
          acc[1][i][j] = fmaf(yv[1][i], xv[1][j], acc[1][i][j]);
          acc[2][i][j] = fmaf(yv[2][i], xv[2][j], acc[2][i][j]);
          acc[2][i][j] = fmaf(yv[3][i], xv[3][j], acc[2][i][j]);
          acc[3][i][j] = fmaf(yv[3][i], xv[2][j], acc[3][i][j]);
          acc[3][i][j] = fmaf(-yv[2][i], xv[3][j], acc[3][i][j]);
        }
    }
    __syncthreads();
  }

  const int64_t plane = static_cast<int64_t>(D) * C;
  float *wsp = ws + static_cast<int64_t>(split) * 4 * plane;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int d = d0 + ty + 16 * i;
    if (d >= D) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + tx + 16 * j;
      if (c >= C) continue;
#pragma unroll
      for (int p = 0; p < 4; ++p) wsp[p * plane + static_cast<int64_t>(d) * C + c] = acc[p][i][j];
    }
    if (do_db && tx == 0) ws_db[static_cast<int64_t>(split) * D + d] = dbacc[i];
  }
}

// Deterministic reduction over splits (fixed order), inverse rDFT, cast:
//   dW[d][c][u] = (G0 + (-1)^u G2)/4 + Re(G1 i^u)/2,  db[d] = sum of partials.
template <typename T>
__global__ void dw_reduce_kernel(const float *__restrict__ ws, const float *__restrict__ ws_db,
                                 T *__restrict__ dW, T *__restrict__ db, int splits, int C, int D) {
  const int64_t plane = static_cast<int64_t>(D) * C;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < plane + D;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (e < plane) {
      float g[4] = {0.f, 0.f, 0.f, 0.f};
      for (int s = 0; s < splits; ++s) {
        const float *p = ws + static_cast<int64_t>(s) * 4 * plane + e;
#pragma unroll
        for (int k = 0; k < 4; ++k) g[k] += p[k * plane];
      }
      float w[4];
      irdft4(g[0], g[1], g[2], g[3], w);
      Vec4<T>::store(dW + e * kT, w);
    } else if (db != nullptr) {
      const int d = static_cast<int>(e - plane);
      float s = 0.f;
      for (int k = 0; k < splits; ++k) s += ws_db[static_cast<int64_t>(k) * D + d];
      db[d] = static_cast<T>(s);
    }
  }
}

}  // namespace feql
