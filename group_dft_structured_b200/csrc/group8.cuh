// group8.cuh — the EQ-Linear layer of a group of order T = 8 or 6 on the
// sm_100a tensor cores, fp16 data with fp32 accumulation: the cyclic group C_8
// (Cyclic8), the point group D4 of p4m (Dihedral4) and the cyclic group C_6
// (Cyclic6).
//
// Flash EQ-Linear states the method for a cyclic group of any order T (arXiv
// abstract: cost 2(T-1)/T^2 of the dense layer), builds kernels for p4 and
// names reflection groups as future work (technical summary, "Limitazioni e
// Lavoro Futuro").  A channel fibre is T fp16 values and its Fourier transform
// has T real components (planes); per 16 channels the layer is one tensor-core
// MMA per real bin and two per complex bin (8 for the order-8 groups, 6 for
// C_6) into T BD accumulator columns.  The kernels are templates over a group
// policy that supplies the order, the transform, its inverse, the weight
// planes and the MMA tables, and over the fibre geometry of its order
// (G8Geo: 16-byte fibres in swizzled 128-byte rows, or 12-byte fibres in
// plain 96-byte rows).
//
// C_8: the real 8-point DFT keeps bins 0..4: bins 0 and 4 are real, 1, 2, 3
// complex: 2 + 3*4 = 14 real N x C x D products instead of 64.
//   a_s = v_s + v_{s+4},  b_s = v_s - v_{s+4}                   (s = 0..3)
//   V0 = a0+a1+a2+a3,  V4 = a0-a1+a2-a3,  V2 = (a0-a2) + i(a3-a1)
//   h = c(b1-b3),  g = c(b1+b3),  c = sqrt(2)/2
//   V1 = (b0+h) - i(b2+g),  V3 = (b0-h) + i(b2-g)
// planes V0, V4 and, per complex bin, Re V_k and -Im V_k; inverse
//   y_t = (Y0 + (-1)^t Y4)/8 + (1/4) sum_{k=1..3} (Re Y_k cos(pi k t/4) - Im Y_k sin(pi k t/4)).
//
// D4 (elements (r, m): rotation r * 90 degrees after reflection m, stored at
// 4 m + r): four irreps of dimension one (A1 = 1, A2 = (-1)^m, B1 = (-1)^r,
// B2 = (-1)^(r+m)) and E(r, m) = R(r * 90 deg) diag(1, -1)^m of dimension two.
// x^(rho) = sum_g x(g) rho(g); the layer is y^(rho) = x^(rho) W^(rho), a 2 x 2
// block product for E: 4 + 8 = 12 real products instead of 64.  With
// P = a0+a2, Q = a1+a3, C = a0-a2, S = a1-a3 of the rotations a_r = x(r, 0)
// and the same of the reflected half b_r = x(r, 1):
//   A1 = (Pa+Qa) + (Pb+Qb)   A2 = (Pa+Qa) - (Pb+Qb)
//   B1 = (Pa-Qa) + (Pb-Qb)   B2 = (Pa-Qa) - (Pb-Qb)
//   E = [[Ca+Cb, Sb-Sa], [Sa+Sb, Ca-Cb]]
// planes A1, A2, B1, B2, E00, E01, E10, E11; inverse
//   x(g) = 1/8 (sum over the 1-dim irreps chi(g) x^) + 1/4 tr(E(g)^T x^(E)).
#pragma once

#include <cuda_fp16.h>

#include "plan.cuh"
#include "sm100.cuh"

namespace feql {

constexpr float kC8 = 0.70710678118654752f;  // sqrt(2)/2

// Fibre geometry.  A TMA box row holds 8 channels x T group elements of one
// token (16 T bytes).  T = 8: 128-byte rows under the 128-byte swizzle, one
// 16-byte chunk per channel fibre; T = 6: 96-byte rows without swizzle,
// 12-byte fibres (a channel pair is 24 bytes, 8-byte aligned).
template <int T>
struct G8Geo;

template <>
struct G8Geo<8> {
  static constexpr int kRow = 128;
  // Channel pair p of the row as packed pairs: v[t] = (channel 2p, channel
  // 2p+1) at group element t.  Chunk c of the row (channel c) sits at chunk
  // c ^ (r & 7) (128-byte swizzle); each pair is two 16-byte loads of its own.
  __device__ static void pair(const uint8_t *row, int p, int r, __half2 (&v)[8]) {
    const uint4 w0 = *reinterpret_cast<const uint4 *>(row + (((2 * p) ^ (r & 7)) << 4));
    const uint4 w1 = *reinterpret_cast<const uint4 *>(row + (((2 * p + 1) ^ (r & 7)) << 4));
    const uint32_t a[4] = {w0.x, w0.y, w0.z, w0.w}, b[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t lo = __byte_perm(a[e], b[e], 0x5410), hi = __byte_perm(a[e], b[e], 0x7632);
      v[2 * e] = *reinterpret_cast<const __half2 *>(&lo);
      v[2 * e + 1] = *reinterpret_cast<const __half2 *>(&hi);
    }
  }
  // Fibres of channels 4h..4h+3 (packed fp16 pairs) into box row r.
  __device__ static void put4(uint8_t *row, int h, int r, const uint32_t (&f)[4][4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint4 *>(row + (((4 * h + i) ^ (r & 7)) << 4)) =
          make_uint4(f[i][0], f[i][1], f[i][2], f[i][3]);
  }
  // One fibre to global memory (16-byte aligned).
  __device__ static void store(__half *dst, const uint32_t (&h)[4]) {
    *reinterpret_cast<uint4 *>(dst) = make_uint4(h[0], h[1], h[2], h[3]);
  }
};

// 96-byte rows: the row is read as six 16-byte chunks (24 words, channel c in
// words 3c..3c+2) and the fibres extracted with static indices; 16-byte
// accesses of neighbouring rows (a 24-word pitch) conflict at most two ways.
template <>
struct G8Geo<6> {
  static constexpr int kRow = 96;
  __device__ static void pairs(const uint8_t *row, int, __half2 (&v)[4][6]) {
    uint32_t w[24];
#pragma unroll
    for (int k = 0; k < 6; ++k) {
      const uint4 c = *reinterpret_cast<const uint4 *>(row + 16 * k);
      w[4 * k] = c.x;
      w[4 * k + 1] = c.y;
      w[4 * k + 2] = c.z;
      w[4 * k + 3] = c.w;
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
#pragma unroll
      for (int e = 0; e < 3; ++e) {
        const uint32_t a = w[6 * p + e], b = w[6 * p + 3 + e];  // channels 2p, 2p + 1
        const uint32_t lo = __byte_perm(a, b, 0x5410), hi = __byte_perm(a, b, 0x7632);
        v[p][2 * e] = *reinterpret_cast<const __half2 *>(&lo);
        v[p][2 * e + 1] = *reinterpret_cast<const __half2 *>(&hi);
      }
    }
  }
  // Channels 4h..4h+3 are words 12h..12h+11 of the row: three 16-byte chunks.
  __device__ static void put4(uint8_t *row, int h, int, const uint32_t (&f)[4][3]) {
    uint4 *dst = reinterpret_cast<uint4 *>(row + 48 * h);
    dst[0] = make_uint4(f[0][0], f[0][1], f[0][2], f[1][0]);
    dst[1] = make_uint4(f[1][1], f[1][2], f[2][0], f[2][1]);
    dst[2] = make_uint4(f[2][2], f[3][0], f[3][1], f[3][2]);
  }
  // (4-byte aligned: fibres start at multiples of 12 bytes)
  __device__ static void store(__half *dst, const uint32_t (&h)[3]) {
    uint32_t *w = reinterpret_cast<uint32_t *>(dst);
    w[0] = h[0];
    w[1] = h[1];
    w[2] = h[2];
  }
};

// One tensor-core MMA of a table: accumulator column block, A operand plane,
// B operand start (weight row block or x plane), N = 2 blocks (wide) or 1, and
// whether it accumulates onto an MMA of the same K-step (chained).
struct G8Mma {
  int acc, a, b, wide, chained;
};

// ---------------------------------------------------------------------------
// Cyclic group C_8
// ---------------------------------------------------------------------------
struct Cyclic8 {
  static constexpr int kT = 8;        // group order: fibre length, planes, accumulator blocks
  static constexpr int kFwdMmas = 8;  // entries of the fwd() and dw() tables
  static constexpr int kDwMmas = 8;
  // Weight rows per output channel of a chunk: What0, What4 and for each complex
  // bin k = 1, 2, 3 at row block r_k = 2 + 3(k-1): Re_k, Im_k, -Re_k, so that
  // the window (Re_k ; Im_k) multiplies Re X_k and (Im_k ; -Re_k) the stored
  // -Im X_k plane.
  static constexpr int kWRows = 11;
  // forward / dX: Y0, Y4 (N = BD), then per complex bin [Re Y_k | Im Y_k] (N = 2 BD)
  __host__ __device__ static constexpr G8Mma fwd(int e) {
    switch (e) {
      case 0: return G8Mma{0, 0, 0, 0, 0};
      case 1: return G8Mma{1, 1, 1, 0, 0};
      case 2: return G8Mma{2, 2, 2, 1, 0};
      case 3: return G8Mma{2, 3, 3, 1, 1};
      case 4: return G8Mma{4, 4, 5, 1, 0};
      case 5: return G8Mma{4, 5, 6, 1, 1};
      case 6: return G8Mma{6, 6, 8, 1, 0};
      default: return G8Mma{6, 7, 9, 1, 1};
    }
  }
  // dW (columns in CT units): G0, G4, then per complex bin a = Re dY_k [Re X_k | -Im X_k]
  // and b = -Im dY_k [Re X_k | -Im X_k]: Re G_k = a[c] + b[CT + c], Im G_k = a[CT + c] - b[c]
  static constexpr int kDwBlocks = 14;
  __host__ __device__ static constexpr G8Mma dw(int e) {
    switch (e) {
      case 0: return G8Mma{0, 0, 0, 0, 0};
      case 1: return G8Mma{1, 1, 1, 0, 0};
      case 2: return G8Mma{2, 2, 2, 1, 0};
      case 3: return G8Mma{4, 3, 2, 1, 0};
      case 4: return G8Mma{6, 4, 4, 1, 0};
      case 5: return G8Mma{8, 5, 4, 1, 0};
      case 6: return G8Mma{10, 6, 6, 1, 0};
      default: return G8Mma{12, 7, 6, 1, 0};
    }
  }

  // Plane values of one real fibre v[0..7] (fp32): V0, V4, Re V1, -Im V1, ..., -Im V3.
  __device__ static void planes(const float (&v)[8], float (&o)[8]) {
    const float a0 = v[0] + v[4], a1 = v[1] + v[5], a2 = v[2] + v[6], a3 = v[3] + v[7];
    const float b0 = v[0] - v[4], b1 = v[1] - v[5], b2 = v[2] - v[6], b3 = v[3] - v[7];
    const float h = kC8 * (b1 - b3), g = kC8 * (b1 + b3);
    o[0] = (a0 + a2) + (a1 + a3);
    o[1] = (a0 + a2) - (a1 + a3);
    o[2] = b0 + h;
    o[3] = b2 + g;
    o[4] = a0 - a2;
    o[5] = a1 - a3;
    o[6] = b0 - h;
    o[7] = g - b2;
  }

  // The same for two channels at once on packed fp16 pairs, every plane divided
  // by 8: v[t] = (channel q, channel q+1) at group element t; o[p] packs plane
  // p / 8 (three to four roundings per output).  Bin 0 sums eight values, so
  // the unscaled planes of inputs above 65504 / 8 would overflow fp16; the
  // first butterfly stage takes the 1/8 (exact outside the subnormals).
  __device__ static void planes_h2(const __half2 (&v)[8], __half2 (&o)[8]) {
    const __half2 c = __float2half2_rn(kC8), q = __float2half2_rn(0.125f);
    __half2 a[4], b[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const __half2 u = __hmul2(v[t + 4], q);
      a[t] = __hfma2(v[t], q, u);
      b[t] = __hfma2(v[t], q, __hneg2(u));
    }
    const __half2 a0 = a[0], a1 = a[1], a2 = a[2], a3 = a[3];
    const __half2 b0 = b[0], b1 = b[1], b2 = b[2], b3 = b[3];
    const __half2 e02 = __hadd2(a0, a2), e13 = __hadd2(a1, a3);
    const __half2 h = __hmul2(c, __hsub2(b1, b3)), g = __hmul2(c, __hadd2(b1, b3));
    o[0] = __hadd2(e02, e13);
    o[1] = __hsub2(e02, e13);
    o[2] = __hadd2(b0, h);
    o[3] = __hadd2(b2, g);
    o[4] = __hsub2(a0, a2);
    o[5] = __hsub2(a1, a3);
    o[6] = __hsub2(b0, h);
    o[7] = __hsub2(g, b2);
  }

  // Group values, times s, from the accumulator blocks Y0, Y4, Re Y1, Im Y1,
  // ..., Im Y3 (s undoes the scale of the fp16 planes and weights).
  __device__ static void inverse(const float (&F)[8], float (&y)[8], float s) {
    const float r1 = F[2], i1 = F[3], r2 = F[4], i2 = F[5], r3 = F[6], i3 = F[7];
    const float e = 0.125f * s, h = 0.25f * s;
    const float P = e * (F[0] + F[1]), Q = e * (F[0] - F[1]);
    const float u = kC8 * (r1 - r3), w = kC8 * (i1 + i3);  // the +-c terms of bins 1 and 3
    y[0] = P + h * (r1 + r2 + r3);
    y[1] = Q + h * (u - w - i2);
    y[2] = P + h * (i3 - i1 - r2);
    y[3] = Q + h * (i2 - u - w);
    y[4] = P + h * (r2 - r1 - r3);
    y[5] = Q + h * (w - u - i2);
    y[6] = P + h * (i1 - r2 - i3);
    y[7] = Q + h * (u + w + i2);
  }

  // Weight rows of one fibre W[d][c][0..7] for pass direction dir (0: forward,
  // What_k[d][c]; 1: dX, conj(What_k)[c][d], i.e. Im negated).
  __device__ static void weight_rows(const float (&w)[8], int dir, float (&rows)[kWRows]) {
    float pl[8];
    planes(w, pl);  // planes hold -Im; weights want Im (conjugated for dX)
    const float s = dir == 0 ? -1.f : 1.f;
    rows[0] = pl[0];
    rows[1] = pl[1];
#pragma unroll
    for (int bk = 0; bk < 3; ++bk) {
      rows[2 + 3 * bk] = pl[2 + 2 * bk];
      rows[3 + 3 * bk] = s * pl[3 + 2 * bk];
      rows[4 + 3 * bk] = -pl[2 + 2 * bk];
    }
  }

  // dW planes G0, G4, Re G1, Im G1, ..., Im G3 from the accumulator blocks of one column.
  __device__ static void dw_planes(const float (&a)[kDwBlocks], float (&G)[8]) {
    G[0] = a[0];
    G[1] = a[1];
#pragma unroll
    for (int bk = 0; bk < 3; ++bk) {
      G[2 + 2 * bk] = a[2 + 4 * bk] + a[5 + 4 * bk];
      G[3 + 2 * bk] = a[3 + 4 * bk] - a[4 + 4 * bk];
    }
  }
};

// ---------------------------------------------------------------------------
// Point group D4 of p4m
// ---------------------------------------------------------------------------
struct Dihedral4 {
  static constexpr int kT = 8;
  static constexpr int kFwdMmas = 8;
  static constexpr int kDwMmas = 8;
  // Weight rows per output channel of a chunk: A1, A2, B1, B2, then the 2 x 2
  // block of E with W^(E)[k][j] at row block 4 + 2k + j, so that the window
  // (W^[k][0] ; W^[k][1]) multiplies the plane x^(E)[i][k] into [Y^[i][0] | Y^[i][1]].
  static constexpr int kWRows = 8;
  // forward / dX: the four 1-dim irreps (N = BD), then Y^(E)[i][.] += x^(E)[i][k] W^(E)[k][.]
  __host__ __device__ static constexpr G8Mma fwd(int e) {
    switch (e) {
      case 0: return G8Mma{0, 0, 0, 0, 0};
      case 1: return G8Mma{1, 1, 1, 0, 0};
      case 2: return G8Mma{2, 2, 2, 0, 0};
      case 3: return G8Mma{3, 3, 3, 0, 0};
      case 4: return G8Mma{4, 4, 4, 1, 0};
      case 5: return G8Mma{4, 5, 6, 1, 1};
      case 6: return G8Mma{6, 6, 4, 1, 0};
      default: return G8Mma{6, 7, 6, 1, 1};
    }
  }
  // dW (columns in CT units): G = x^T dy per irrep; for E, G[i][j] = sum_k x^[k][i] dy^[k][j]:
  // A = dy^[k][j], B = [x^[k][0] | x^[k][1]] into [G[0][j] | G[1][j]] at 4 + 2j
  static constexpr int kDwBlocks = 8;
  __host__ __device__ static constexpr G8Mma dw(int e) {
    switch (e) {
      case 0: return G8Mma{0, 0, 0, 0, 0};
      case 1: return G8Mma{1, 1, 1, 0, 0};
      case 2: return G8Mma{2, 2, 2, 0, 0};
      case 3: return G8Mma{3, 3, 3, 0, 0};
      case 4: return G8Mma{4, 4, 4, 1, 0};
      case 5: return G8Mma{6, 5, 4, 1, 0};
      case 6: return G8Mma{4, 6, 6, 1, 1};
      default: return G8Mma{6, 7, 6, 1, 1};
    }
  }

  __device__ static void planes(const float (&v)[8], float (&o)[8]) {
    const float Pa = v[0] + v[2], Qa = v[1] + v[3], Ca = v[0] - v[2], Sa = v[1] - v[3];
    const float Pb = v[4] + v[6], Qb = v[5] + v[7], Cb = v[4] - v[6], Sb = v[5] - v[7];
    const float sa = Pa + Qa, da = Pa - Qa, sb = Pb + Qb, db = Pb - Qb;
    o[0] = sa + sb;  // A1
    o[1] = sa - sb;  // A2
    o[2] = da + db;  // B1
    o[3] = da - db;  // B2
    o[4] = Ca + Cb;  // E00
    o[5] = Sb - Sa;  // E01
    o[6] = Sa + Sb;  // E10
    o[7] = Ca - Cb;  // E11
  }

  // Packed fp16 pairs, every plane divided by 8 in the first stage (as for C8).
  __device__ static void planes_h2(const __half2 (&v)[8], __half2 (&o)[8]) {
    const __half2 q = __float2half2_rn(0.125f);
    const __half2 u2 = __hmul2(v[2], q), u3 = __hmul2(v[3], q);
    const __half2 u6 = __hmul2(v[6], q), u7 = __hmul2(v[7], q);
    const __half2 Pa = __hfma2(v[0], q, u2), Qa = __hfma2(v[1], q, u3);
    const __half2 Ca = __hfma2(v[0], q, __hneg2(u2)), Sa = __hfma2(v[1], q, __hneg2(u3));
    const __half2 Pb = __hfma2(v[4], q, u6), Qb = __hfma2(v[5], q, u7);
    const __half2 Cb = __hfma2(v[4], q, __hneg2(u6)), Sb = __hfma2(v[5], q, __hneg2(u7));
    const __half2 sa = __hadd2(Pa, Qa), da = __hsub2(Pa, Qa);
    const __half2 sb = __hadd2(Pb, Qb), db = __hsub2(Pb, Qb);
    o[0] = __hadd2(sa, sb);
    o[1] = __hsub2(sa, sb);
    o[2] = __hadd2(da, db);
    o[3] = __hsub2(da, db);
    o[4] = __hadd2(Ca, Cb);
    o[5] = __hsub2(Sb, Sa);
    o[6] = __hadd2(Sa, Sb);
    o[7] = __hsub2(Ca, Cb);
  }

  // x(r, 0) = (A1 + A2 + (-1)^r (B1 + B2)) / 8 + (c_r (E00 + E11) + s_r (E10 - E01)) / 4
  // x(r, 1) = (A1 - A2 + (-1)^r (B1 - B2)) / 8 + (c_r (E00 - E11) + s_r (E01 + E10)) / 4
  // with (c_r, s_r) = (1, 0), (0, 1), (-1, 0), (0, -1).
  // (times s, as for C8)
  __device__ static void inverse(const float (&F)[8], float (&y)[8], float s) {
    const float s12 = F[0] + F[1], d12 = F[0] - F[1], s34 = F[2] + F[3], d34 = F[2] - F[3];
    const float e = 0.125f * s, h = 0.25f * s;
    const float Pp = e * (s12 + s34), Pm = e * (s12 - s34);
    const float Qp = e * (d12 + d34), Qm = e * (d12 - d34);
    const float c0 = h * (F[4] + F[7]), s0 = h * (F[6] - F[5]);
    const float c1 = h * (F[4] - F[7]), s1 = h * (F[5] + F[6]);
    y[0] = Pp + c0;
    y[1] = Pm + s0;
    y[2] = Pp - c0;
    y[3] = Pm - s0;
    y[4] = Qp + c1;
    y[5] = Qm + s1;
    y[6] = Qp - c1;
    y[7] = Qm - s1;
  }

  // Weight rows of one fibre W[d][c][0..7]: the planes (forward), or for dX
  // (contraction over d) the transposed block of E: W'^(E)[k][j] = W^(E)[j][k].
  __device__ static void weight_rows(const float (&w)[8], int dir, float (&rows)[kWRows]) {
    planes(w, rows);
    if (dir == 1) {
      const float t = rows[5];
      rows[5] = rows[6];
      rows[6] = t;
    }
  }

  __device__ static void dw_planes(const float (&a)[kDwBlocks], float (&G)[8]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) G[k] = a[k];
    G[4] = a[4];  // G[0][0]
    G[5] = a[6];  // G[0][1]
    G[6] = a[5];  // G[1][0]
    G[7] = a[7];  // G[1][1]
  }
};

// ---------------------------------------------------------------------------
// Cyclic group C_6
// ---------------------------------------------------------------------------
// A non-dyadic order (twiddles cos(pi/3) = 1/2 and sin(pi/3) = sqrt(3)/2): the
// real 6-point DFT keeps bins 0..3, bins 0 and 3 real, 1 and 2 complex:
// 2 + 2 * 4 = 10 real N x C x D products instead of 36 (2(T-1)/T^2).
//   a_s = v_s + v_{s+3},  b_s = v_s - v_{s+3}                  (s = 0, 1, 2)
//   V0 = a0 + a1 + a2,  V2 = a0 - (a1 + a2)/2 - i c (a1 - a2),  c = sqrt(3)/2
//   V3 = b0 - b1 + b2,  V1 = b0 + (b1 - b2)/2 - i c (b1 + b2)
// planes V0, V3, Re V1, -Im V1, Re V2, -Im V2; inverse
//   y_t = (Y0 + (-1)^t Y3)/6 + (1/3) sum_{k=1,2} (Re Y_k cos(pi k t/3) - Im Y_k sin(pi k t/3)).
// Fibres are 12 bytes (G8Geo<6>); the layer needs C and D multiples of 4
// (16-byte row strides for the tensor maps).
constexpr float kS6 = 0.86602540378443865f;  // sqrt(3)/2

struct Cyclic6 {
  static constexpr int kT = 6;
  static constexpr int kFwdMmas = 6;
  static constexpr int kDwMmas = 6;
  // Weight rows: What0, What3, then for bins k = 1, 2 at row block r_k = 2 + 3(k-1):
  // Re_k, Im_k, -Re_k (the windows (Re_k ; Im_k) and (Im_k ; -Re_k), as for C_8).
  static constexpr int kWRows = 8;
  __host__ __device__ static constexpr G8Mma fwd(int e) {
    switch (e) {
      case 0: return G8Mma{0, 0, 0, 0, 0};
      case 1: return G8Mma{1, 1, 1, 0, 0};
      case 2: return G8Mma{2, 2, 2, 1, 0};
      case 3: return G8Mma{2, 3, 3, 1, 1};
      case 4: return G8Mma{4, 4, 5, 1, 0};
      default: return G8Mma{4, 5, 6, 1, 1};
    }
  }
  // dW (columns in CT units): G0, G3, then per complex bin a = Re dY_k [Re X_k | -Im X_k]
  // and b = -Im dY_k [Re X_k | -Im X_k]
  static constexpr int kDwBlocks = 10;
  __host__ __device__ static constexpr G8Mma dw(int e) {
    switch (e) {
      case 0: return G8Mma{0, 0, 0, 0, 0};
      case 1: return G8Mma{1, 1, 1, 0, 0};
      case 2: return G8Mma{2, 2, 2, 1, 0};
      case 3: return G8Mma{4, 3, 2, 1, 0};
      case 4: return G8Mma{6, 4, 4, 1, 0};
      default: return G8Mma{8, 5, 4, 1, 0};
    }
  }

  __device__ static void planes(const float (&v)[6], float (&o)[6]) {
    const float a0 = v[0] + v[3], a1 = v[1] + v[4], a2 = v[2] + v[5];
    const float b0 = v[0] - v[3], b1 = v[1] - v[4], b2 = v[2] - v[5];
    o[0] = a0 + a1 + a2;
    o[1] = b0 - b1 + b2;
    o[2] = b0 + 0.5f * (b1 - b2);
    o[3] = kS6 * (b1 + b2);
    o[4] = a0 - 0.5f * (a1 + a2);
    o[5] = kS6 * (a1 - a2);
  }

  // Packed fp16 pairs, every plane divided by 8 (bin 0 sums six values) in the
  // first stage, as for the order-8 groups.
  __device__ static void planes_h2(const __half2 (&v)[6], __half2 (&o)[6]) {
    const __half2 q = __float2half2_rn(0.125f), hf = __float2half2_rn(0.5f);
    const __half2 c = __float2half2_rn(kS6);
    __half2 a[3], b[3];
#pragma unroll
    for (int t = 0; t < 3; ++t) {
      const __half2 u = __hmul2(v[t + 3], q);
      a[t] = __hfma2(v[t], q, u);
      b[t] = __hfma2(v[t], q, __hneg2(u));
    }
    o[0] = __hadd2(__hadd2(a[0], a[1]), a[2]);
    o[1] = __hadd2(__hsub2(b[0], b[1]), b[2]);
    o[2] = __hfma2(hf, __hsub2(b[1], b[2]), b[0]);
    o[3] = __hmul2(c, __hadd2(b[1], b[2]));
    o[4] = __hfma2(__hneg2(hf), __hadd2(a[1], a[2]), a[0]);
    o[5] = __hmul2(c, __hsub2(a[1], a[2]));
  }

  // Group values, times s, from the accumulator blocks Y0, Y3, Re Y1, Im Y1, Re Y2, Im Y2.
  __device__ static void inverse(const float (&F)[6], float (&y)[6], float s) {
    const float e = s * (1.f / 6.f), h = s * (1.f / 3.f);
    const float P = e * (F[0] + F[1]), Q = e * (F[0] - F[1]);
    const float r1 = F[2], i1 = F[3], r2 = F[4], i2 = F[5];
    const float u = 0.5f * (r1 - r2), w = kS6 * (i1 + i2), z = kS6 * (i1 - i2);
    const float v = 0.5f * (r1 + r2);
    y[0] = P + h * (r1 + r2);
    y[1] = Q + h * (u - w);
    y[2] = P - h * (v + z);
    y[3] = Q + h * (r2 - r1);
    y[4] = P + h * (z - v);
    y[5] = Q + h * (u + w);
  }

  __device__ static void weight_rows(const float (&w)[6], int dir, float (&rows)[kWRows]) {
    float pl[6];
    planes(w, pl);  // planes hold -Im; weights want Im (conjugated for dX)
    const float s = dir == 0 ? -1.f : 1.f;
    rows[0] = pl[0];
    rows[1] = pl[1];
#pragma unroll
    for (int bk = 0; bk < 2; ++bk) {
      rows[2 + 3 * bk] = pl[2 + 2 * bk];
      rows[3 + 3 * bk] = s * pl[3 + 2 * bk];
      rows[4 + 3 * bk] = -pl[2 + 2 * bk];
    }
  }

  __device__ static void dw_planes(const float (&a)[kDwBlocks], float (&G)[6]) {
    G[0] = a[0];
    G[1] = a[1];
#pragma unroll
    for (int bk = 0; bk < 2; ++bk) {
      G[2 + 2 * bk] = a[2 + 4 * bk] + a[5 + 4 * bk];
      G[3 + 2 * bk] = a[3 + 4 * bk] - a[4 + 4 * bk];
    }
  }
};

// ---------------------------------------------------------------------------
// Plans and the Fourier-weight layout
// ---------------------------------------------------------------------------
// Per (output tile j, 16-channel chunk kc) a weight chunk of kWRows * BD rows x
// 32 B (K-major, 32-byte swizzle, the image the MMA reads), row block r
// holding the group policy's weight row r of the tile's BD output channels.
struct G8Plan {
  int Ci, Do, BD, nD, nK, chunk_bytes;
  int64_t bytes;
};

__host__ __device__ inline G8Plan make_g8_plan(int Ci, int Do, int wrows) {
  G8Plan p;
  p.Ci = Ci;
  p.Do = Do;
  p.nK = static_cast<int>(cdiv(Ci, kCK));
  p.nD = static_cast<int>(cdiv(Do, 64));  // 8 accumulator blocks of BD columns <= 512
  p.BD = static_cast<int>(align_up(cdiv(Do, p.nD), 16));
  p.chunk_bytes = wrows * p.BD * kCK * 2;
  p.bytes = static_cast<int64_t>(p.nD) * p.nK * p.chunk_bytes;
  return p;
}

struct G8Layout {
  G8Plan fwd, dx;  // forward: contraction over C; dX: over D with the transposed weights
  int64_t off_fwd, off_dx, bytes;
};

__host__ __device__ inline G8Layout make_g8_layout(int C, int D, int wrows) {
  G8Layout L;
  L.fwd = make_g8_plan(C, D, wrows);
  L.dx = make_g8_plan(D, C, wrows);
  L.off_fwd = 0;
  L.off_dx = align_up(L.fwd.bytes, 1024);
  L.bytes = L.off_dx + align_up(L.dx.bytes, 1024);
  return L;
}

// Planes of the four channel pairs of box row r, packed: o[p][k] = plane k of
// channels 2p, 2p+1, low half first.
// (T = 8 loads pair by pair, each pair's two chunks whole; T = 6 loads the row
// once, its fibres straddling the chunks.)
template <class Gp>
__device__ __forceinline__ void g8_planes_row(const uint8_t *row, int r,
                                              uint32_t (&o)[4][Gp::kT]) {
  __half2 v[4][Gp::kT];
  if constexpr (Gp::kT == 6) G8Geo<6>::pairs(row, r, v);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    if constexpr (Gp::kT == 8) G8Geo<8>::pair(row, p, r, v[p]);
    __half2 w[Gp::kT];
    Gp::planes_h2(v[p], w);
#pragma unroll
    for (int k = 0; k < Gp::kT; ++k) o[p][k] = *reinterpret_cast<const uint32_t *>(&w[k]);
  }
}

// One thread per fp16 element of the tiled weight buffer (both directions).
// Direction 0 reads W[o][i][:], direction 1 W[i][o][:] (o: output channel of the pass).
template <class Gp>
__global__ void wfft_g8_kernel(const __half *__restrict__ W, uint8_t *__restrict__ What,
                               G8Layout L, int C) {
  const int64_t n_fwd = L.fwd.bytes / 2, n_dx = L.dx.bytes / 2;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n_fwd + n_dx;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int dir = e < n_fwd ? 0 : 1;
    const G8Plan &P = dir == 0 ? L.fwd : L.dx;
    const int64_t le = dir == 0 ? e : e - n_fwd;
    const int rows = Gp::kWRows * P.BD;
    const int64_t chunk = le / (rows * kCK);
    const int rem = static_cast<int>(le % (rows * kCK));
    const int row = rem / kCK, k = rem % kCK;
    const int j = static_cast<int>(chunk / P.nK), kc = static_cast<int>(chunk % P.nK);
    const int sub = row / P.BD;
    const int o = j * P.BD + row % P.BD;
    const int i = kc * kCK + k;
    float v = 0.f;
    if (o < P.Do && i < P.Ci) {
      const int d = dir == 0 ? o : i, c = dir == 0 ? i : o;
      const __half *src = W + (static_cast<int64_t>(d) * C + c) * Gp::kT;
      float w[Gp::kT], wr[Gp::kWRows];
#pragma unroll
      for (int t = 0; t < Gp::kT; ++t) w[t] = __half2float(src[t]);
      Gp::weight_rows(w, dir, wr);
#pragma unroll
      for (int r = 0; r < Gp::kWRows; ++r)
        if (r == sub) v = wr[r];
    }
    const int64_t base = (dir == 0 ? L.off_fwd : L.off_dx) + chunk * P.chunk_bytes;
    // every weight plane divided by 8 (as the operand planes): no fp16 overflow for any
    // finite W (a bin sums at most 8 values)
    *reinterpret_cast<__half *>(What + base + sw32_offset(row, k)) = __float2half_rn(0.125f * v);
  }
}

// ---------------------------------------------------------------------------
// Forward / dX kernel
// ---------------------------------------------------------------------------
// Persistent, one CTA per SM, 14 warps; a unit is (128-token tile m, output
// tile j) and a chunk is 16 input channels of it:
//   warp 0       TMA: the chunk's two 16 KB boxes of the input (8 channels x 8
//                group elements per row, 128-byte swizzle) and the unit's
//                weight chunk (bulk copy) into a ring of stages
//   warp 1       TMEM allocator + MMA issuer: per chunk eight M=128, K=16 MMAs,
//                N = BD for bins 0 and 4, two N = 2 BD for each complex bin,
//                into 8 BD accumulator columns (double-buffered when BD <= 32)
//   warps 2..9   transform: thread = (token row, box); the 8-point rDFT of its
//                8 channel fibres on packed fp16 pairs, then, after a team barrier, the
//                chunk rewritten in place as eight K-major planes of 4 KB
//   warps 10..17 epilogue, two teams of four taking alternate 8-channel groups
//                of every unit: warp q reads TMEM lane quadrant q (32 token
//                rows), four columns of each accumulator block at a time;
//                inverse rDFT + bias in fp32; per 8 output channels each lane
//                writes its row (128 B) into a 128-byte-swizzled staging box
//                and the warp issues one 4 KB TMA store (two boxes per warp)
constexpr int kG8EpiWarps = 8;
constexpr int kG8Threads = 64 + (8 + kG8EpiWarps) * 32;
// input chunk: 128 tokens x 16 channels x T (4 KB x T: two boxes of 8 channels),
// rewritten in place as T planes of 128 tokens x 32 B
template <int T>
constexpr int g8_xchunk() { return kBM * kCK * T * 2; }
constexpr int kG8Plane = kBM * kCK * 2;         // 4 KB: 128 tokens x 32 B
constexpr int kG8MaxOut = 2;                    // staging boxes per epilogue warp (at most)

struct G8FwdParams {
  const uint8_t *wt;   // weight chunks of this direction, [j][kc]
  const __half *bias;  // [Do] or nullptr
  __half *out;         // [N][Do][T]
  int64_t N;
  int Ci, Do, BD, nD, nK, chunk_bytes;
  int nM, n_units;
  int nacc, acc_stride;
  int stages, stage_bytes, bias_floats;
  int out_box;         // one staging box: 32 rows x 8 channels x T fp16
  int nout;            // staging boxes per epilogue warp: 2, or 1 when that leaves room for a third stage
};

struct G8Smem {
  int stage0, out0, bias, bars, total;
};

__host__ __device__ inline G8Smem g8_fwd_smem(const G8FwdParams &p) {
  G8Smem s;
  s.stage0 = 0;
  s.out0 = p.stages * p.stage_bytes;
  s.bias = s.out0 + kG8EpiWarps * p.nout * p.out_box;
  s.bars = s.bias + static_cast<int>(align_up(p.bias_floats * 4, 16));
  // full, tready, empty per stage; acc_full, acc_empty x2; final; tmem slot
  s.total = s.bars + (3 * p.stages + 4 + 1) * 8 + 16;
  return s;
}

// This CTA's work units u = blockIdx.x + k * gridDim.x as (token tile m,
// output tile j), stepped without divisions (see TcUnits in tc_fwd.cuh).
struct G8Units {
  int m, j, dm, dj, nD, nM;
  bool valid;
  __device__ __forceinline__ explicit G8Units(const G8FwdParams &p) : nD(p.nD), nM(p.nM) {
    m = static_cast<int>(blockIdx.x) / p.nD;
    j = static_cast<int>(blockIdx.x) % p.nD;
    dm = static_cast<int>(gridDim.x) / p.nD;
    dj = static_cast<int>(gridDim.x) % p.nD;
    valid = m < nM;
  }
  __device__ __forceinline__ void next() {
    m += dm;
    j += dj;
    if (j >= nD) {
      j -= nD;
      ++m;
    }
    valid = m < nM;
  }
};

// 18 warps over the 4 SM sub-partitions put 5 warps on two 16K-register slices:
// 5 x 32 x 96 = 15,360 registers fit, 104 would not.
template <class Gp>
__global__ void __maxnreg__(96)
tc_g8_fwd_kernel(const __grid_constant__ CUtensorMap tm_in, const __grid_constant__ CUtensorMap tm_out,
                  const G8FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  constexpr int T = Gp::kT;
  using Geo = G8Geo<T>;
  constexpr int kChunk = g8_xchunk<T>(), kBox = kChunk / 2;
  const G8Smem L = g8_fwd_smem(p);
  float *sbias = reinterpret_cast<float *>(smem + L.bias);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
  uint64_t *full = bars;
  uint64_t *tready = bars + p.stages;
  uint64_t *empty = bars + 2 * p.stages;
  uint64_t *acc_full = bars + 3 * p.stages;
  uint64_t *acc_empty = acc_full + 2;
  uint64_t *final_bar = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(final_bar + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&tready[s], 8);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], kG8EpiWarps);
    }
    mbar_init(final_bar, 1);
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < p.bias_floats; i += blockDim.x)
    sbias[i] = (p.bias != nullptr && i < p.Do) ? __half2float(p.bias[i]) : 0.f;
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      tma_prefetch_desc(&tm_in);
      tma_prefetch_desc(&tm_out);
      int s = 0;
      uint32_t ph = 0;
      for (G8Units U(p); U.valid; U.next()) {
        const int m = U.m, j = U.j;
        for (int kc = 0; kc < p.nK; ++kc) {
          if (ok) ok = mbar_wait(&empty[s], ph ^ 1);
          if (ok) {
            uint8_t *st = smem + L.stage0 + s * p.stage_bytes;
            mbar_arrive_expect_tx(&full[s], kChunk + p.chunk_bytes);
            tma_load_2d(st, &tm_in, kc * (kCK * T), m * kBM, &full[s]);
            tma_load_2d(st + kBox, &tm_in, kc * (kCK * T) + 8 * T, m * kBM, &full[s]);
            bulk_load(st + kChunk,
                      p.wt + (static_cast<int64_t>(j) * p.nK + kc) * p.chunk_bytes,
                      p.chunk_bytes, &full[s]);
          }
          if (++s == p.stages) { s = 0; ph ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id_bd = instr_desc(kBM, p.BD, 0, 0);
      const uint32_t id_2bd = instr_desc(kBM, 2 * p.BD, 0, 0);
      const uint64_t dsw32 = smem_desc(0, 16, 256, kSw32);  // K-major, 32-byte swizzle
      const uint32_t dhi = desc_hi(dsw32);
      const uint32_t x0 = desc_lo(desc_at(dsw32, smem_u32(smem + L.stage0)));
      const uint32_t stage16 = p.stage_bytes >> 4, pl16 = kG8Plane >> 4;
      const uint32_t w16 = 2 * p.BD;  // BD rows of 32 B, in 16-byte units
      int s = 0, a = 0;
      uint32_t ph = 0, aph = 0;
      for (G8Units U(p); U.valid; U.next()) {
        if (ok) ok = mbar_wait(&acc_empty[a], aph ^ 1);
        tc_fence_after();
        const uint32_t acc = tmem_base + a * p.acc_stride;
        for (int kc = 0; kc < p.nK; ++kc) {
          // tready implies full (the transform waited for the TMA bytes first)
          if (ok) ok = mbar_wait(&tready[s], ph);
          tc_fence_after();
          if (ok) {
            const uint32_t xd = x0 + s * stage16, wd = xd + (kChunk >> 4);
#pragma unroll
            for (int e = 0; e < Gp::kFwdMmas; ++e) {  // the group's table: compile-time offsets
              const G8Mma t = Gp::fwd(e);
              mma_f16_lo(acc + t.acc * p.BD, xd + t.a * pl16, wd + t.b * w16, dhi,
                         t.wide ? id_2bd : id_bd, (kc > 0 || t.chained) ? 1u : 0u);
            }
            mma_commit(&empty[s]);
          }
          if (++s == p.stages) { s = 0; ph ^= 1; }
        }
        if (ok) mma_commit(&acc_full[a]);
        if (++a == p.nacc) { a = 0; aph ^= 1; }
      }
      mma_commit(final_bar);
      mbar_wait(final_bar, 0);
    }
  } else if (warp < 10) {
    // ---------------------------------------------------------- transform
    const int t = threadIdx.x - 64;
    const int r = t % kBM, bx = t / kBM;  // token row, box (channels 8 bx .. 8 bx + 7)
    int s = 0;
    uint32_t ph = 0;
    for (G8Units U(p); U.valid; U.next()) {
      for (int kc = 0; kc < p.nK; ++kc) {
        if (ok) ok = mbar_wait(&full[s], ph);
        uint8_t *st = smem + L.stage0 + s * p.stage_bytes;
        const uint8_t *src = st + bx * kBox + r * Geo::kRow;
        uint32_t pw[4][T];  // [channel pair][plane], packed fp16
        g8_planes_row<Gp>(src, r, pw);
        named_bar_sync(2, 256);  // every row read before the planes overwrite it
#pragma unroll
        for (int pp = 0; pp < T; ++pp)
          *reinterpret_cast<uint4 *>(st + pp * kG8Plane + r * 32 + (((bx ^ (r >> 2)) & 1) << 4)) =
              make_uint4(pw[0][pp], pw[1][pp], pw[2][pp], pw[3][pp]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&tready[s]);
        if (++s == p.stages) { s = 0; ph ^= 1; }
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int ew = warp - 10, team = ew / 4;
    const int quad = warp & 3;
    const int groups = p.BD / 8;
    int last_g = -1;  // this team's last 8-channel group of a unit
    for (int g = team; g < groups; g += 2) last_g = g;
    uint8_t *obase = smem + L.out0 + ew * p.nout * p.out_box;
    int a = 0, oi = 0;
    uint32_t aph = 0;
    for (G8Units U(p); U.valid; U.next()) {
      const int m = U.m, j = U.j;
      if (ok) ok = mbar_wait(&acc_full[a], aph);
      tc_fence_after();
      if (last_g < 0) {  // this team reads nothing of the unit
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&acc_empty[a]);
      }
      const uint32_t tl = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + a * p.acc_stride;
      for (int g = team; g < groups; g += 2) {
        const int d0 = j * p.BD + g * 8;
        uint8_t *ob = obase + (p.nout == 2 ? (oi & 1) : 0) * p.out_box;
        if (d0 < p.Do) {
          if (lane == 0) {  // this box's last store has read it
            if (p.nout == 2)
              bulk_wait_read<1>();
            else
              bulk_wait_read<0>();
          }
          __syncwarp();
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // four output channels at a time
          uint32_t Y[T][4];  // [accumulator block][column], in the group's plane order
          __syncwarp();      // the TMEM loads are warp-collective
#pragma unroll
          for (int bk = 0; bk < T; ++bk) tmem_ld4(tl + g * 8 + h * 4 + bk * p.BD, Y[bk]);
          tmem_ld_wait();
          if (h == 1 && g == last_g) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && ok) mbar_arrive(&acc_empty[a]);
          }
          if (d0 >= p.Do) continue;  // whole group is padding
          uint32_t hv[4][T / 2];  // fibres of channels d0 + 4h .. d0 + 4h + 3, packed fp16
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float F[T], y[T];
#pragma unroll
            for (int bk = 0; bk < T; ++bk) F[bk] = __uint_as_float(Y[bk][i]);
            Gp::inverse(F, y, 64.f);  // planes and weights both carry 1/8
            const float bv = sbias[d0 + 4 * h + i];
#pragma unroll
            for (int e = 0; e < T / 2; ++e) hv[i][e] = pack_half2(y[2 * e] + bv, y[2 * e + 1] + bv);
          }
          Geo::put4(ob + lane * Geo::kRow, h, lane, hv);
        }
        if (d0 >= p.Do) continue;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {  // the store clips rows past N and channels past Do
          tma_store_2d(&tm_out, d0 * T, m * kBM + quad * 32, ob);
          bulk_commit();
        }
        ++oi;
      }
      if (++a == p.nacc) { a = 0; aph ^= 1; }
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------------------------
// dW / db kernel
// ---------------------------------------------------------------------------
// G_k[d,c] = sum_n dY_k[n,d] conj(X_k[n,c]) for bins k = 0..4, dW = irDFT_8(G)
// (cross-correlation theorem; the same inverse as the forward), db = sum dY_0
// (from the fp16 bin-0 planes, which carry dY_0 / 8).
// One CTA per (128-row d tile, c tile of CT <= 32 columns, token split),
// 10 warps: TMA, MMA, 8 transform warps that also read the accumulators at the
// end.  Per chunk of 32 tokens the TMA warp loads the tile's dy boxes into box
// slots 0..15 and its x boxes into slots 16.. (8 channels x 8 group elements per
// row, zero-filled past the tensor).  The transform turns every pair of boxes
// (16 channels) into eight MN-major planes in place: dy pair g keeps its planes
// in its own 8 KB (plane p at p x 1 KB), so the M = 128 operand of plane p has
// its 16-channel atoms 8 KB apart; the x planes are laid out plane-major, so
// Re X_k and -Im X_k of all pairs are adjacent and one N = 2 CT operand covers
// [Re X_k | -Im X_k].  Per 16 tokens: G0, G4 (N = CT) and for each complex bin
// acc_a = Re dY_k [Re X_k | -Im X_k], acc_b = -Im dY_k [Re X_k | -Im X_k]
// (N = 2 CT), i.e. Re G_k = a[c] + b[CT + c], Im G_k = a[CT + c] - b[c]:
// 8 MMAs and 14 CT TMEM columns.
constexpr int kG8DwTB = 32;                     // tokens per chunk (2 MMA K-steps)
// one box: 32 tokens x 8 channels x T (4 KB for T = 8); a pair of boxes holds
// the same bytes as the pair's T planes of 32 tokens x 32 B
template <int T>
constexpr int g8_dw_box() { return kG8DwTB * 16 * T; }
constexpr int kG8DwDySlots = 16;                // box slots for dy (the M = 128 operand spans 8 pairs)
constexpr int kG8DwThreads = 64 + 8 * 32;
constexpr int kG8DwMaxPer = 3;                  // (box, token) items per transform thread

struct G8DwParams {
  int64_t N;
  int C, D, Cs;        // Cs: workspace row stride (C rounded up to 16)
  int CT;              // c columns per tile (16 or 32)
  int tiles_d, tiles_c, splits;
  int64_t split_len;   // tokens per split, multiple of kG8DwTB
  int stages;
  int slot_boxes;      // kG8DwDySlots + 2 * CT / 16
  int stack_dy, stack_x;  // 1: one 3-D load brings all of a chunk's dy (x) boxes
  int nqd_stack;       // boxes in the dy stack (those of the largest d tile)
  int box_bytes;       // g8_dw_box<T>()
  float *ws;           // [splits][T][D][Cs]: the T bin planes (C_8: G0, G4, Re G1, Im G1, ..., Im G3)
  float *ws_db;        // [splits][D]
};

struct G8DwSmem {
  int stage0, bars, total;
};

__host__ __device__ inline G8DwSmem g8_dw_smem(const G8DwParams &p) {
  G8DwSmem s;
  s.stage0 = 0;
  s.bars = p.stages * p.slot_boxes * p.box_bytes;
  // full, tready, empty per stage; acc_full; tmem slot
  s.total = s.bars + (3 * p.stages + 1) * 8 + 16;
  return s;
}

template <class Gp>
__global__ void __launch_bounds__(kG8DwThreads, 1)
tc_g8_dw_kernel(const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_x,
                 const G8DwParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  constexpr int T = Gp::kT;
  using Geo = G8Geo<T>;
  constexpr int kBox = g8_dw_box<T>();
  const G8DwSmem L = g8_dw_smem(p);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
  uint64_t *full = bars;
  uint64_t *tready = bars + p.stages;
  uint64_t *empty = bars + 2 * p.stages;
  uint64_t *acc_full = bars + 3 * p.stages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // this CTA's (d tile, c tile, split)
  const int tile = blockIdx.x % (p.tiles_d * p.tiles_c);
  const int split = blockIdx.x / (p.tiles_d * p.tiles_c);
  const int ti = tile / p.tiles_c, tj = tile % p.tiles_c;
  const int d0 = ti * 128, c0 = tj * p.CT;
  const int dt = p.D - d0 < 128 ? p.D - d0 : 128;
  const int nqd = 2 * static_cast<int>(cdiv(dt, 16));  // dy boxes (whole pairs)
  const int npc = p.CT / 16, nqc = 2 * npc;             // x pairs, boxes
  const int nbox = nqd + nqc;
  const int64_t t_begin = static_cast<int64_t>(split) * p.split_len;
  int64_t t_end = t_begin + p.split_len;
  if (t_end > p.N) t_end = p.N;
  const int nch = t_begin < t_end ? static_cast<int>(cdiv(t_end - t_begin, kG8DwTB)) : 0;
  const int xoff = kG8DwDySlots * kBox;  // x region of a stage
  const int ncols = Gp::kDwBlocks * p.CT;
  const uint32_t tmem_cols = ncols <= 256 ? 256u : 512u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&tready[s], 8);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      tma_prefetch_desc(&tm_dy);
      tma_prefetch_desc(&tm_x);
      int s = 0;
      uint32_t ph = 0;
      for (int ch = 0; ch < nch; ++ch) {
        if (ok) ok = mbar_wait(&empty[s], ph ^ 1);
        if (ok) {
          uint8_t *st = smem + L.stage0 + s * p.slot_boxes * kBox;
          const int32_t row = static_cast<int32_t>(t_begin + static_cast<int64_t>(ch) * kG8DwTB);
          // a stack lands whole (boxes past the last channel read as zeros)
          const int bd = p.stack_dy ? p.nqd_stack : nqd;
          mbar_arrive_expect_tx(&full[s], (bd + nqc) * kBox);
          if (p.stack_dy) {
            tma_load_3d(st, &tm_dy, 0, row, d0 / 8, &full[s]);
          } else {
            for (int q = 0; q < nqd; ++q)
              tma_load_2d(st + q * kBox, &tm_dy, (d0 + 8 * q) * T, row, &full[s]);
          }
          if (p.stack_x) {
            tma_load_3d(st + xoff, &tm_x, 0, row, c0 / 8, &full[s]);
          } else {
            for (int q = 0; q < nqc; ++q)
              tma_load_2d(st + xoff + q * kBox, &tm_x, (c0 + 8 * q) * T, row, &full[s]);
          }
        }
        if (++s == p.stages) { s = 0; ph ^= 1; }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id1 = instr_desc(128, p.CT, 0, 0, 1, 1);
      const uint32_t id2 = instr_desc(128, 2 * p.CT, 0, 0, 1, 1);
      const uint64_t da = smem_desc(0, 2 * kBox, 256, kSw32);  // dy: pairs 2 boxes apart
      const uint64_t db = smem_desc(0, kG8DwTB * 32, 256, kSw32);  // x: pairs 1 KB apart
      const uint32_t dhi = desc_hi(da);
      const uint32_t a0 = desc_lo(desc_at(da, smem_u32(smem + L.stage0)));
      const uint32_t b0 = desc_lo(desc_at(db, smem_u32(smem + L.stage0 + xoff)));
      const uint32_t stage16 = (p.slot_boxes * kBox) >> 4;
      const uint32_t apl = (kG8DwTB * 32) >> 4, bpl = (npc * kG8DwTB * 32) >> 4;  // one plane
      int s = 0;
      uint32_t ph = 0;
      for (int ch = 0; ch < nch; ++ch) {
        // tready implies full (the transform waited for the TMA bytes first)
        if (ok) ok = mbar_wait(&tready[s], ph);
        tc_fence_after();
        if (ok) {
          const uint32_t sa = a0 + s * stage16, sb = b0 + s * stage16;
#pragma unroll
          for (int k = 0; k < kG8DwTB / 16; ++k) {  // 16 tokens = 512 B = 32 units
            const uint32_t A = sa + k * 32, B = sb + k * 32;
            const bool first = ch == 0 && k == 0;
#pragma unroll
            for (int e = 0; e < Gp::kDwMmas; ++e) {  // the group's table: compile-time offsets
              const G8Mma t = Gp::dw(e);
              mma_f16_lo(tmem_base + t.acc * p.CT, A + t.a * apl, B + t.b * bpl, dhi,
                         t.wide ? id2 : id1, (first && !t.chained) ? 0u : 1u);
            }
          }
          mma_commit(&empty[s]);
        }
        if (++s == p.stages) { s = 0; ph ^= 1; }
      }
      mma_commit(acc_full);
    }
  } else {
    // ---------------------------------------------------------- transform
    const int t = threadIdx.x - 64;
    const bool do_db = tj == 0;  // the tiles of the first c column produce db
    float db_acc[kG8DwMaxPer][8];
#pragma unroll
    for (int k = 0; k < kG8DwMaxPer; ++k)
#pragma unroll
      for (int q = 0; q < 8; ++q) db_acc[k][q] = 0.f;
    int s = 0;
    uint32_t ph = 0;
    for (int ch = 0; ch < nch; ++ch) {
      if (ok) ok = mbar_wait(&full[s], ph);
      uint8_t *st = smem + L.stage0 + s * p.slot_boxes * kBox;
      uint32_t pw[kG8DwMaxPer][4][T];  // [item][channel pair][plane], packed fp16
#pragma unroll
      for (int k = 0; k < kG8DwMaxPer; ++k) {
        const int e = t + k * 256;
        const int bi = e / kG8DwTB, r = e % kG8DwTB;
        if (bi < nbox) {
          const uint8_t *src = st + (bi < nqd ? bi * kBox : xoff + (bi - nqd) * kBox) +
                               r * Geo::kRow;
          g8_planes_row<Gp>(src, r, pw[k]);
          if (do_db && bi < nqd) {  // bin 0 of the dy planes, as the MMAs see it
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // channels 2q, 2q + 1 of the box
              const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&pw[k][q][0]));
              db_acc[k][2 * q] += f.x;
              db_acc[k][2 * q + 1] += f.y;
            }
          }
        }
      }
      named_bar_sync(2, 256);  // every row read before the planes overwrite it
#pragma unroll
      for (int k = 0; k < kG8DwMaxPer; ++k) {
        const int e = t + k * 256;
        const int bi = e / kG8DwTB, r = e % kG8DwTB;
        if (bi < nbox) {
          const bool is_dy = bi < nqd;
          const int q2 = is_dy ? bi : bi - nqd;
          const int g = q2 / 2, hh = q2 % 2;
          // dy pair g: plane pp at g x 2 boxes + pp x 1 KB; x: plane-major (pp x npc + g) x 1 KB
          uint8_t *pbase = is_dy ? st + g * 2 * kBox : st + xoff + g * kG8DwTB * 32;
          const int pstride = is_dy ? kG8DwTB * 32 : npc * kG8DwTB * 32;
#pragma unroll
          for (int pp = 0; pp < T; ++pp)
            *reinterpret_cast<uint4 *>(pbase + pp * pstride + r * 32 + (((hh ^ (r >> 2)) & 1) << 4)) =
                make_uint4(pw[k][0][pp], pw[k][1][pp], pw[k][2][pp], pw[k][3][pp]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&tready[s]);
      if (++s == p.stages) { s = 0; ph ^= 1; }
    }

    // ---------------------------------------------- dW partials -> workspace
    if (ok) ok = mbar_wait(acc_full, 0);
    tc_fence_after();
    const int quad = warp & 3, half = (warp - 2) / 4;
    const int d = quad * 32 + lane;  // row of the tile
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    const int64_t plane = static_cast<int64_t>(p.D) * p.Cs;
    float *dst = p.ws + static_cast<int64_t>(split) * T * plane + static_cast<int64_t>(d0 + d) * p.Cs + c0;
    for (int g = half; g < p.CT / 8; g += 2) {  // 8-column steps
      uint32_t blk[Gp::kDwBlocks][8];  // accumulator block k, 8 columns of this step
      __syncwarp();  // the TMEM loads are warp-collective
#pragma unroll
      for (int k = 0; k < Gp::kDwBlocks; ++k) tmem_ld8(tl + k * p.CT + g * 8, blk[k]);
      tmem_ld_wait();
      if (d0 + d < p.D && c0 + g * 8 < p.C) {
        float G[T][8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float a[Gp::kDwBlocks], Gi[T];
#pragma unroll
          for (int k = 0; k < Gp::kDwBlocks; ++k) a[k] = __uint_as_float(blk[k][i]);
          Gp::dw_planes(a, Gi);
#pragma unroll
          for (int bin = 0; bin < T; ++bin) G[bin][i] = Gi[bin];
        }
#pragma unroll
        for (int bin = 0; bin < T; ++bin) {
          float4 *o = reinterpret_cast<float4 *>(dst + bin * plane + g * 8);
          o[0] = make_float4(G[bin][0], G[bin][1], G[bin][2], G[bin][3]);
          o[1] = make_float4(G[bin][4], G[bin][5], G[bin][6], G[bin][7]);
        }
      }
    }
    tc_fence_before();
    // db (tiles of the first c column only): fixed-order reduction through shared memory
    if (do_db) {
      named_bar_sync(3, 256);  // the stages are free: every chunk has been consumed
      float *sdb = reinterpret_cast<float *>(smem + L.stage0);  // [kG8DwMaxPer * 256][8]
#pragma unroll
      for (int k = 0; k < kG8DwMaxPer; ++k)
#pragma unroll
        for (int q = 0; q < 8; ++q) sdb[(t + k * 256) * 8 + q] = db_acc[k][q];
      named_bar_sync(3, 256);
      if (t < nqd * 8) {
        const int bi = t / 8, q = t % 8;  // dy box bi, channel q: rows bi*TB .. of the items
        float sum = 0.f;
        for (int rr = 0; rr < kG8DwTB; ++rr) sum += sdb[(bi * kG8DwTB + rr) * 8 + q];
        const int dd = d0 + bi * 8 + q;
        if (dd < p.D && dd < d0 + 128) p.ws_db[static_cast<int64_t>(split) * p.D + dd] = sum;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// Sum of the split partials in a fixed order, then dW[d][c][0..7] = irDFT_8 of
// the eight bin planes, and db[d].  A block takes 16 consecutive (d, c) outputs
// (the last blocks take db); its 32 warps each sum every 32nd split (the loads
// of a warp's splits are independent, so they overlap), then warp 0 adds the
// 32 partial sums in warp order: the same grouping on every run.
constexpr int kRed8Out = 16, kRed8Groups = 32;

__host__ __device__ inline int64_t g8_reduce_blocks(int C, int D) {
  return cdiv(static_cast<int64_t>(D) * C, kRed8Out) + cdiv(D, kRed8Out);
}

template <class Gp>
__global__ void __launch_bounds__(kRed8Out * kRed8Groups)
g8_dw_reduce_kernel(const float *__restrict__ ws, const float *__restrict__ ws_db,
                     __half *__restrict__ dW, __half *__restrict__ db, int splits, int C, int D,
                     int Cs) {
  constexpr int T = Gp::kT;
  __shared__ float part[kRed8Groups][T][kRed8Out];
  const int64_t n = static_cast<int64_t>(D) * C;
  const int64_t plane = static_cast<int64_t>(D) * Cs;
  const int64_t nblk_w = cdiv(n, kRed8Out);
  const int lo = threadIdx.x % kRed8Out, grp = threadIdx.x / kRed8Out;
  if (blockIdx.x < nblk_w) {
    const int64_t e = blockIdx.x * static_cast<int64_t>(kRed8Out) + lo;
    float G[T];
#pragma unroll
    for (int k = 0; k < T; ++k) G[k] = 0.f;
    if (e < n) {
      const float *src = ws + (e / C) * Cs + (e % C);
      for (int s = grp; s < splits; s += kRed8Groups) {
        const float *q = src + static_cast<int64_t>(s) * T * plane;
#pragma unroll
        for (int k = 0; k < T; ++k) G[k] += q[k * plane];
      }
    }
#pragma unroll
    for (int k = 0; k < T; ++k) part[grp][k][lo] = G[k];
    __syncthreads();
    if (grp == 0 && e < n) {
      float t[T];
#pragma unroll
      for (int k = 0; k < T; ++k) t[k] = 0.f;
      for (int q = 0; q < kRed8Groups; ++q)
#pragma unroll
        for (int k = 0; k < T; ++k) t[k] += part[q][k][lo];
      float y[T];
      Gp::inverse(t, y, 64.f);  // x and dy planes both carry 1/8
      uint32_t hv[T / 2];
#pragma unroll
      for (int k = 0; k < T / 2; ++k) hv[k] = pack_half2(y[2 * k], y[2 * k + 1]);
      G8Geo<T>::store(dW + e * T, hv);
    }
  } else if (db != nullptr) {
    const int64_t d = (blockIdx.x - nblk_w) * kRed8Out + lo;
    float sdb = 0.f;
    if (d < D)
      for (int s = grp; s < splits; s += kRed8Groups) sdb += ws_db[static_cast<int64_t>(s) * D + d];
    part[grp][0][lo] = sdb;
    __syncthreads();
    if (grp == 0 && d < D) {
      float t = 0.f;
      for (int q = 0; q < kRed8Groups; ++q) t += part[q][0][lo];
      db[d] = __float2half_rn(8.f * t);  // bin 0 of the dy planes carries 1/8
    }
  }
}

}  // namespace feql
