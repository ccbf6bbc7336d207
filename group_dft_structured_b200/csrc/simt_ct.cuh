// simt_ct.cuh — the EQ-Linear layer of a cyclic group C_T of any order
// 2 <= T <= 16 on the CUDA cores (fp32 arithmetic; fp32 or fp16 data).
//
// Flash EQ-Linear (arXiv abstract) states the method for a cyclic group of
// order T: along the group axis a real DFT keeps bins k = 0 .. floor(T/2) (the
// others are their conjugates), bin 0 and, for even T, bin T/2 are real, the
// rest complex, so a layer is 2T-2 (even T) or 2T-1 (odd T) real channel
// products instead of the T^2 of the unrolled circulant.  The twiddles
// e^{-2 pi i k t / T} are not dyadic for most T (T = 3, 5, 6, 12 ...), so the
// kernels take them from a per-block table (sincospi).  The tensor-core
// kernels cover T = 4 (p4) and T = 8 in fp16; these kernels cover every other
// order and the fp32 modes.
//
// Planes of a fibre (kPlanes = T real numbers): bin 0, then bin T/2 for even
// T, then (Re, Im) of each complex bin k = 1 .. ceil(T/2) - 1.
//   forward   Y_k[n,d] = sum_c W^_k[d,c] X^_k[n,c]            (complex product)
//   dX        the same with conj(W^_k)^T (contraction over d)
//   dW        G_k[d,c] = sum_n dY^_k[n,d] conj(X^_k[n,c]),  dW = irDFT(G),  db = sum dY^_0
//   inverse   y_t = (Y_0 + [T even] (-1)^t Y_{T/2} + 2 sum_k Re(Y_k e^{2 pi i k t / T})) / T
#pragma once

#include <cuda_fp16.h>

#include "plan.cuh"

namespace feql {

constexpr int kCtMaxT = 16;
constexpr int kCtTile = 32;     // tokens x outputs (or d x c for dW) per block
constexpr int kCtK = 8;         // channels (or tokens, for dW) per shared-memory chunk
constexpr int kCtThreads = 256; // 16 x 16 threads, 2 x 2 outputs each

template <int T>
struct CtBins {
  static constexpr int kBins = T / 2 + 1;                 // kept bins 0 .. T/2
  static constexpr bool kNyquist = (T % 2) == 0;          // bin T/2 is real
  static constexpr int kComplex = kBins - 1 - (kNyquist ? 1 : 0);
  static constexpr int kFirstComplexPlane = kNyquist ? 2 : 1;
  static constexpr int kPlanes = T;
};

template <typename Ty>
__device__ __forceinline__ float ct_load(const Ty *p);
template <>
__device__ __forceinline__ float ct_load<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ct_load<__half>(const __half *p) { return __half2float(*p); }

template <typename Ty>
__device__ __forceinline__ Ty ct_cast(float v);
template <>
__device__ __forceinline__ float ct_cast<float>(float v) { return v; }
template <>
__device__ __forceinline__ __half ct_cast<__half>(float v) { return __float2half_rn(v); }

// cs[k][t] = cos(2 pi k t / T), sn[k][t] = sin(2 pi k t / T) for k <= T/2.
template <int T>
__device__ __forceinline__ void ct_twiddles(float (*cs)[T], float (*sn)[T]) {
  for (int e = threadIdx.x; e < CtBins<T>::kBins * T; e += blockDim.x) {
    const int k = e / T, t = e % T;
    float s, c;
    sincospif(2.0f * static_cast<float>((k * t) % T) / static_cast<float>(T), &s, &c);
    cs[k][t] = c;
    sn[k][t] = s;
  }
}

// The planes of one real fibre v[0..T-1].
template <int T>
__device__ __forceinline__ void ct_planes(const float (&v)[T], const float (*cs)[T],
                                          const float (*sn)[T], float (&o)[T]) {
  using B = CtBins<T>;
  float s0 = 0.f;
#pragma unroll
  for (int t = 0; t < T; ++t) s0 += v[t];
  o[0] = s0;
  if (B::kNyquist) {
    float sh = 0.f;
#pragma unroll
    for (int t = 0; t < T; ++t) sh += (t & 1) ? -v[t] : v[t];
    o[1] = sh;
  }
#pragma unroll
  for (int j = 0; j < B::kComplex; ++j) {
    const int k = j + 1;
    float re = 0.f, im = 0.f;
#pragma unroll
    for (int t = 0; t < T; ++t) {
      re = fmaf(v[t], cs[k][t], re);
      im = fmaf(-v[t], sn[k][t], im);
    }
    o[B::kFirstComplexPlane + 2 * j] = re;
    o[B::kFirstComplexPlane + 2 * j + 1] = im;
  }
}

// Group values from the planes of a product (no 1/T yet applied).
template <int T>
__device__ __forceinline__ void ct_inverse(const float (&F)[T], const float (*cs)[T],
                                           const float (*sn)[T], float (&y)[T]) {
  using B = CtBins<T>;
#pragma unroll
  for (int t = 0; t < T; ++t) {
    float acc = F[0];
    if (B::kNyquist) acc += (t & 1) ? -F[1] : F[1];
#pragma unroll
    for (int j = 0; j < B::kComplex; ++j) {
      const int k = j + 1;
      const float re = F[B::kFirstComplexPlane + 2 * j], im = F[B::kFirstComplexPlane + 2 * j + 1];
      acc += 2.f * (re * cs[k][t] - im * sn[k][t]);
    }
    y[t] = acc * (1.f / static_cast<float>(T));
  }
}

// Weight planes of both directions, fp32 [dir][plane][Do][Ci]: dir 0 W^_k[d][c]
// (Ci = C), dir 1 conj(W^_k)[c][d] (Ci = D).
template <int T, typename Ty>
__global__ void ct_simt_wfft_kernel(const Ty *__restrict__ W, float *__restrict__ What, int C,
                                    int D) {
  __shared__ float cs[CtBins<T>::kBins][T], sn[CtBins<T>::kBins][T];
  ct_twiddles<T>(cs, sn);
  __syncthreads();
  const int64_t per = static_cast<int64_t>(C) * D;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < per;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int d = static_cast<int>(e / C), c = static_cast<int>(e % C);
    float v[T], pl[T];
#pragma unroll
    for (int t = 0; t < T; ++t) v[t] = ct_load<Ty>(W + e * T + t);
    ct_planes<T>(v, cs, sn, pl);
#pragma unroll
    for (int p = 0; p < T; ++p) {
      const bool im = p >= CtBins<T>::kFirstComplexPlane && ((p - CtBins<T>::kFirstComplexPlane) & 1);
      What[p * per + static_cast<int64_t>(d) * C + c] = pl[p];                           // forward
      What[(T + p) * per + static_cast<int64_t>(c) * D + d] = im ? -pl[p] : pl[p];       // dX
    }
  }
}

// Forward / dX: out[n][o][:] = irDFT( per bin sum_i Wp_k[o][i] * rDFT(in[n][i][:]) ) (+ bias).
template <int T, typename Ty>
__global__ void __launch_bounds__(kCtThreads)
ct_simt_fwd_kernel(const Ty *__restrict__ in, const float *__restrict__ Wp,
                   const Ty *__restrict__ bias, Ty *__restrict__ out, int64_t N, int Ci, int Do) {
  using B = CtBins<T>;
  __shared__ float cs[B::kBins][T], sn[B::kBins][T];
  __shared__ float Xs[T][kCtK][kCtTile + 1];
  __shared__ float Ws[T][kCtK][kCtTile + 1];
  ct_twiddles<T>(cs, sn);
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kCtTile;
  const int o0 = blockIdx.y * kCtTile;
  const int64_t plane = static_cast<int64_t>(Do) * Ci;
  float acc[T][2][2];
#pragma unroll
  for (int p = 0; p < T; ++p)
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j) acc[p][i][j] = 0.f;
  __syncthreads();

  for (int c0 = 0; c0 < Ci; c0 += kCtK) {
    {  // one fibre per thread: token nn, channel kk
      const int nn = tid / kCtK, kk = tid % kCtK;
      float v[T], f[T];
#pragma unroll
      for (int t = 0; t < T; ++t) v[t] = 0.f;
      if (n0 + nn < N && c0 + kk < Ci) {
        const Ty *src = in + ((n0 + nn) * Ci + c0 + kk) * T;
#pragma unroll
        for (int t = 0; t < T; ++t) v[t] = ct_load<Ty>(src + t);
      }
      ct_planes<T>(v, cs, sn, f);
#pragma unroll
      for (int p = 0; p < T; ++p) Xs[p][kk][nn] = f[p];
    }
    for (int e = tid; e < T * kCtTile * kCtK; e += kCtThreads) {
      const int p = e / (kCtTile * kCtK);
      const int oo = (e / kCtK) % kCtTile, kk = e % kCtK;
      float w = 0.f;
      if (o0 + oo < Do && c0 + kk < Ci) w = Wp[p * plane + static_cast<int64_t>(o0 + oo) * Ci + c0 + kk];
      Ws[p][kk][oo] = w;
    }
    __syncthreads();
#pragma unroll 2
    for (int kk = 0; kk < kCtK; ++kk) {
      float xv[T][2], wv[T][2];
#pragma unroll
      for (int p = 0; p < T; ++p)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          xv[p][i] = Xs[p][kk][ty + 16 * i];
          wv[p][i] = Ws[p][kk][tx + 16 * i];
        }
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          acc[0][i][j] = fmaf(xv[0][i], wv[0][j], acc[0][i][j]);
          if (B::kNyquist) acc[1][i][j] = fmaf(xv[1][i], wv[1][j], acc[1][i][j]);
#pragma unroll
          for (int q = 0; q < B::kComplex; ++q) {
            const int r = B::kFirstComplexPlane + 2 * q;
            const float xr = xv[r][i], xi = xv[r + 1][i], wr = wv[r][j], wi = wv[r + 1][j];
            acc[r][i][j] = fmaf(xr, wr, fmaf(-xi, wi, acc[r][i][j]));
            acc[r + 1][i][j] = fmaf(xr, wi, fmaf(xi, wr, acc[r + 1][i][j]));
          }
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int64_t n = n0 + ty + 16 * i;
      const int o = o0 + tx + 16 * j;
      if (n >= N || o >= Do) continue;
      float F[T], y[T];
#pragma unroll
      for (int p = 0; p < T; ++p) F[p] = acc[p][i][j];
      ct_inverse<T>(F, cs, sn, y);
      const float bv = bias != nullptr ? ct_load<Ty>(bias + o) : 0.f;
      Ty *dst = out + (n * Do + o) * T;
#pragma unroll
      for (int t = 0; t < T; ++t) dst[t] = ct_cast<Ty>(y[t] + bv);
    }
}

// dW partial sums: block (d tile, c tile, token split); per chunk of kCtK
// tokens the planes of dy (d fibres) and x (c fibres) go to shared memory;
// each thread accumulates G_k for 2 d x 2 c.  ws: [split][plane][D][C] fp32,
// ws_db: [split][D] (written by the blocks of c tile 0).
template <int T, typename Ty>
__global__ void __launch_bounds__(kCtThreads)
ct_simt_dw_kernel(const Ty *__restrict__ x, const Ty *__restrict__ dy, float *__restrict__ ws,
                  float *__restrict__ ws_db, int64_t N, int C, int D, int64_t split_len,
                  int tiles_d, int tiles_c) {
  using B = CtBins<T>;
  __shared__ float cs[B::kBins][T], sn[B::kBins][T];
  __shared__ float Ds[T][kCtK][kCtTile + 1];
  __shared__ float Xs[T][kCtK][kCtTile + 1];
  ct_twiddles<T>(cs, sn);
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int tile = blockIdx.x % (tiles_d * tiles_c), split = blockIdx.x / (tiles_d * tiles_c);
  const int d0 = (tile / tiles_c) * kCtTile, c0 = (tile % tiles_c) * kCtTile;
  const int64_t t_begin = static_cast<int64_t>(split) * split_len;
  const int64_t t_end = t_begin + split_len < N ? t_begin + split_len : N;
  float acc[T][2][2];
#pragma unroll
  for (int p = 0; p < T; ++p)
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j) acc[p][i][j] = 0.f;
  float dbs = 0.f;  // thread (token row, d) partial of db, for c tile 0
  __syncthreads();

  for (int64_t n0 = t_begin; n0 < t_end; n0 += kCtK) {
    {  // one dy fibre and one x fibre per thread: token kk, channel mm
      const int kk = tid / kCtTile, mm = tid % kCtTile;
      const int64_t n = n0 + kk;
      float v[T], f[T];
#pragma unroll
      for (int t = 0; t < T; ++t) v[t] = 0.f;
      if (n < t_end && d0 + mm < D) {
        const Ty *src = dy + (n * D + d0 + mm) * T;
#pragma unroll
        for (int t = 0; t < T; ++t) v[t] = ct_load<Ty>(src + t);
      }
      ct_planes<T>(v, cs, sn, f);
      dbs += f[0];
#pragma unroll
      for (int p = 0; p < T; ++p) Ds[p][kk][mm] = f[p];
#pragma unroll
      for (int t = 0; t < T; ++t) v[t] = 0.f;
      if (n < t_end && c0 + mm < C) {
        const Ty *src = x + (n * C + c0 + mm) * T;
#pragma unroll
        for (int t = 0; t < T; ++t) v[t] = ct_load<Ty>(src + t);
      }
      ct_planes<T>(v, cs, sn, f);
#pragma unroll
      for (int p = 0; p < T; ++p) Xs[p][kk][mm] = f[p];
    }
    __syncthreads();
#pragma unroll 2
    for (int kk = 0; kk < kCtK; ++kk) {
      float dv[T][2], xv[T][2];
#pragma unroll
      for (int p = 0; p < T; ++p)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          dv[p][i] = Ds[p][kk][ty + 16 * i];
          xv[p][i] = Xs[p][kk][tx + 16 * i];
        }
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          acc[0][i][j] = fmaf(dv[0][i], xv[0][j], acc[0][i][j]);
          if (B::kNyquist) acc[1][i][j] = fmaf(dv[1][i], xv[1][j], acc[1][i][j]);
#pragma unroll
          for (int q = 0; q < B::kComplex; ++q) {
            const int r = B::kFirstComplexPlane + 2 * q;
            const float yr = dv[r][i], yi = dv[r + 1][i], xr = xv[r][j], xi = xv[r + 1][j];
            acc[r][i][j] = fmaf(yr, xr, fmaf(yi, xi, acc[r][i][j]));          // Re dY conj(X)
            acc[r + 1][i][j] = fmaf(yi, xr, fmaf(-yr, xi, acc[r + 1][i][j]));  // Im
          }
        }
    }
    __syncthreads();
  }
  const int64_t plane = static_cast<int64_t>(D) * C;
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int d = d0 + ty + 16 * i, c = c0 + tx + 16 * j;
      if (d >= D || c >= C) continue;
#pragma unroll
      for (int p = 0; p < T; ++p)
        ws[(static_cast<int64_t>(split) * T + p) * plane + static_cast<int64_t>(d) * C + c] =
            acc[p][i][j];
    }
  if (tile % tiles_c == 0) {  // db: the kCtK token rows of each d column, in a fixed order
    __shared__ float sdb[kCtK][kCtTile];
    sdb[tid / kCtTile][tid % kCtTile] = dbs;
    __syncthreads();
    if (tid < kCtTile && d0 + tid < D) {
      float s = 0.f;
      for (int r = 0; r < kCtK; ++r) s += sdb[r][tid];
      ws_db[static_cast<int64_t>(split) * D + d0 + tid] = s;
    }
  }
}

// Fixed-order sum of the split partials, then dW[d][c][:] = irDFT(G[d][c]) and db.
template <int T, typename Ty>
__global__ void ct_simt_dw_reduce_kernel(const float *__restrict__ ws, const float *__restrict__ ws_db,
                                         Ty *__restrict__ dW, Ty *__restrict__ db, int splits,
                                         int C, int D) {
  __shared__ float cs[CtBins<T>::kBins][T], sn[CtBins<T>::kBins][T];
  ct_twiddles<T>(cs, sn);
  __syncthreads();
  const int64_t plane = static_cast<int64_t>(D) * C;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < plane + D;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (e < plane) {
      float G[T], y[T];
#pragma unroll
      for (int p = 0; p < T; ++p) G[p] = 0.f;
      for (int s = 0; s < splits; ++s)
#pragma unroll
        for (int p = 0; p < T; ++p) G[p] += ws[(static_cast<int64_t>(s) * T + p) * plane + e];
      ct_inverse<T>(G, cs, sn, y);
#pragma unroll
      for (int t = 0; t < T; ++t) dW[e * T + t] = ct_cast<Ty>(y[t]);
    } else if (db != nullptr) {
      const int64_t d = e - plane;
      float s = 0.f;
      for (int sp = 0; sp < splits; ++sp) s += ws_db[static_cast<int64_t>(sp) * D + d];
      db[d] = ct_cast<Ty>(s);
    }
  }
}

}  // namespace feql
