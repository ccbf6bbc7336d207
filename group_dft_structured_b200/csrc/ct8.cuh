// ct8.cuh — the EQ-Linear layer of the cyclic group C_8 (T = 8) on the sm_100a
// tensor cores, fp16 data with fp32 accumulation.
//
// Flash EQ-Linear states the method for a cyclic group of any order T (arXiv
// abstract: cost 2(T-1)/T^2 of the dense layer) and builds kernels for p4;
// this file is the same dataflow for T = 8.  Along the group axis the real
// 8-point DFT keeps bins 0..4: bins 0 and 4 are real, bins 1, 2, 3 complex,
// so a layer is 2 + 3*4 = 14 real N x C x D products instead of the 64 of
// the unrolled group-circulant matrix.
//
// Transform of one fibre v[0..7] (radix-2 split, c = sqrt(2)/2):
//   a_s = v_s + v_{s+4},  b_s = v_s - v_{s+4}                   (s = 0..3)
//   V0 = a0+a1+a2+a3,  V4 = a0-a1+a2-a3,  V2 = (a0-a2) + i(a3-a1)
//   h = c(b1-b3),  g = c(b1+b3)
//   V1 = (b0+h) - i(b2+g),  V3 = (b0-h) + i(b2-g)
// The planes store V0, V4 and, per complex bin, Re V_k and -Im V_k.
// Inverse (real output, bins 5..7 = conj of 3..1):
//   y_t = (Y0 + (-1)^t Y4)/8 + (1/4) sum_{k=1..3} (Re Y_k cos(pi k t/4) - Im Y_k sin(pi k t/4))
#pragma once

#include <cuda_fp16.h>

#include "plan.cuh"
#include "sm100.cuh"

namespace feql {

constexpr int kT8 = 8;
constexpr float kC8 = 0.70710678118654752f;  // sqrt(2)/2

// ---------------------------------------------------------------------------
// Plans and the Fourier-weight layout for T = 8
// ---------------------------------------------------------------------------
// Per (output tile j, 16-channel chunk kc) a weight chunk of 11*BD rows x 32 B
// (K-major, 32-byte swizzle, the image the MMA reads):
//   [0,BD) What0 | [BD,2BD) What4 | for k = 1,2,3 at r_k = (2 + 3(k-1)) BD:
//   [r_k, r_k+BD) Re_k | [r_k+BD, r_k+2BD) Im_k | [r_k+2BD, r_k+3BD) -Re_k
// so that rows [r_k, r_k+2BD) = (Re_k ; Im_k) multiply Re X_k and the window
// [r_k+BD, r_k+3BD) = (Im_k ; -Re_k) multiplies the stored -Im X_k plane.
constexpr int kCt8Rows = 11;  // weight rows per output channel of a tile

struct Ct8Plan {
  int Ci, Do, BD, nD, nK, chunk_bytes;
  int64_t bytes;
};

__host__ __device__ inline Ct8Plan make_ct8_plan(int Ci, int Do) {
  Ct8Plan p;
  p.Ci = Ci;
  p.Do = Do;
  p.nK = static_cast<int>(cdiv(Ci, kCK));
  p.nD = static_cast<int>(cdiv(Do, 64));  // 8 accumulator blocks of BD columns <= 512
  p.BD = static_cast<int>(align_up(cdiv(Do, p.nD), 16));
  p.chunk_bytes = kCt8Rows * p.BD * kCK * 2;
  p.bytes = static_cast<int64_t>(p.nD) * p.nK * p.chunk_bytes;
  return p;
}

struct Ct8Layout {
  Ct8Plan fwd, dx;  // forward: contraction over C; dX: over D with conj(What)^T
  int64_t off_fwd, off_dx, bytes;
};

__host__ __device__ inline Ct8Layout make_ct8_layout(int C, int D) {
  Ct8Layout L;
  L.fwd = make_ct8_plan(C, D);
  L.dx = make_ct8_plan(D, C);
  L.off_fwd = 0;
  L.off_dx = align_up(L.fwd.bytes, 1024);
  L.bytes = L.off_dx + align_up(L.dx.bytes, 1024);
  return L;
}

// The eight plane values of one real fibre v[0..7] (fp32), in plane order
// V0, V4, Re V1, -Im V1, Re V2, -Im V2, Re V3, -Im V3.
__device__ __forceinline__ void rdft8(const float (&v)[8], float (&o)[8]) {
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

// The same transform for two channels at once on packed fp16 pairs (like the
// p4 butterflies): w0, w1 are the 16-byte rows (8 group elements) of channels
// q and q+1; o[p] packs plane p of (q, q+1), low half first.  Each add or
// multiply rounds to fp16 (three to four roundings per output).
__device__ __forceinline__ void rdft8_pair(const uint4 &w0, const uint4 &w1, uint32_t (&o)[8]) {
  const uint32_t a[4] = {w0.x, w0.y, w0.z, w0.w}, b[4] = {w1.x, w1.y, w1.z, w1.w};
  __half2 v[8];  // v[t] = (channel q, channel q+1) at group element t
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t lo = __byte_perm(a[e], b[e], 0x5410), hi = __byte_perm(a[e], b[e], 0x7632);
    v[2 * e] = *reinterpret_cast<const __half2 *>(&lo);
    v[2 * e + 1] = *reinterpret_cast<const __half2 *>(&hi);
  }
  const __half2 c = __float2half2_rn(kC8);
  const __half2 a0 = __hadd2(v[0], v[4]), a1 = __hadd2(v[1], v[5]);
  const __half2 a2 = __hadd2(v[2], v[6]), a3 = __hadd2(v[3], v[7]);
  const __half2 b0 = __hsub2(v[0], v[4]), b1 = __hsub2(v[1], v[5]);
  const __half2 b2 = __hsub2(v[2], v[6]), b3 = __hsub2(v[3], v[7]);
  const __half2 e02 = __hadd2(a0, a2), e13 = __hadd2(a1, a3);
  const __half2 h = __hmul2(c, __hsub2(b1, b3)), g = __hmul2(c, __hadd2(b1, b3));
  const __half2 r[8] = {__hadd2(e02, e13), __hsub2(e02, e13), __hadd2(b0, h), __hadd2(b2, g),
                        __hsub2(a0, a2),   __hsub2(a1, a3),   __hsub2(b0, h), __hsub2(g, b2)};
#pragma unroll
  for (int p = 0; p < 8; ++p) o[p] = *reinterpret_cast<const uint32_t *>(&r[p]);
}

// Inverse: y[0..7] from Y0, Y4 and (Re, Im) of bins 1..3.
__device__ __forceinline__ void irdft8(float Y0, float Y4, float r1, float i1, float r2, float i2,
                                       float r3, float i3, float (&y)[8]) {
  const float P = 0.125f * (Y0 + Y4), Q = 0.125f * (Y0 - Y4);
  const float u = kC8 * (r1 - r3), w = kC8 * (i1 + i3);  // the +-c terms of bins 1 and 3
  y[0] = P + 0.25f * (r1 + r2 + r3);
  y[1] = Q + 0.25f * (u - w - i2);
  y[2] = P + 0.25f * (i3 - i1 - r2);
  y[3] = Q + 0.25f * (i2 - u - w);
  y[4] = P + 0.25f * (r2 - r1 - r3);
  y[5] = Q + 0.25f * (w - u - i2);
  y[6] = P + 0.25f * (i1 - r2 - i3);
  y[7] = Q + 0.25f * (u + w + i2);
}

// Fourier bins of one weight fibre W[o][i][0..7] for pass direction dir
// (0: forward, What_k[d][c]; 1: dX, conj(What_k)[c][d], i.e. Im negated).
// bins: What0, What4, Re1, Im1, Re2, Im2, Re3, Im3.
__device__ __forceinline__ void weight_bins8(const __half *W, int C, int dir, int o, int i,
                                             float (&bins)[8]) {
  const int d = dir == 0 ? o : i;
  const int c = dir == 0 ? i : o;
  const __half *w = W + (static_cast<int64_t>(d) * C + c) * kT8;
  float v[8], pl[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) v[t] = __half2float(w[t]);
  rdft8(v, pl);  // planes hold -Im; weights want Im (conjugated for dX)
  const float s = dir == 0 ? -1.f : 1.f;
  bins[0] = pl[0];
  bins[1] = pl[1];
  bins[2] = pl[2];
  bins[3] = s * pl[3];
  bins[4] = pl[4];
  bins[5] = s * pl[5];
  bins[6] = pl[6];
  bins[7] = s * pl[7];
}

// One thread per fp16 element of the tiled weight buffer (both directions).
__global__ void wfft_ct8_kernel(const __half *__restrict__ W, uint8_t *__restrict__ What,
                                Ct8Layout L, int C) {
  const int64_t n_fwd = L.fwd.bytes / 2, n_dx = L.dx.bytes / 2;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n_fwd + n_dx;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int dir = e < n_fwd ? 0 : 1;
    const Ct8Plan &P = dir == 0 ? L.fwd : L.dx;
    const int64_t le = dir == 0 ? e : e - n_fwd;
    const int rows = kCt8Rows * P.BD;
    const int64_t chunk = le / (rows * kCK);
    const int rem = static_cast<int>(le % (rows * kCK));
    const int row = rem / kCK, k = rem % kCK;
    const int j = static_cast<int>(chunk / P.nK), kc = static_cast<int>(chunk % P.nK);
    const int sub = row / P.BD;  // 0: What0, 1: What4, then (Re, Im, -Re) for bins 1..3
    const int o = j * P.BD + row % P.BD;
    const int i = kc * kCK + k;
    float v = 0.f;
    if (o < P.Do && i < P.Ci) {
      float bins[8];
      weight_bins8(W, C, dir, o, i, bins);
      if (sub < 2) {
        v = bins[sub];
      } else {
        const int bk = (sub - 2) / 3, part = (sub - 2) % 3;  // bin 1 + bk
        v = part == 0 ? bins[2 + 2 * bk] : part == 1 ? bins[3 + 2 * bk] : -bins[2 + 2 * bk];
      }
    }
    const int64_t base = (dir == 0 ? L.off_fwd : L.off_dx) + chunk * P.chunk_bytes;
    *reinterpret_cast<__half *>(What + base + sw32_offset(row, k)) = __float2half_rn(v);
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
//   warps 10..13 epilogue: warp q reads TMEM lane quadrant q (32 token rows);
//                inverse rDFT + bias in fp32; per 8 output channels each lane
//                writes its row (128 B) into a 128-byte-swizzled staging box
//                and the warp issues one 4 KB TMA store (two boxes per warp)
constexpr int kCt8Threads = 64 + 12 * 32;
constexpr int kCt8XChunk = kBM * kCK * kT8 * 2;  // 32 KB: 128 tokens x 16 channels x 8
constexpr int kCt8Box = kCt8XChunk / 2;          // 16 KB: 8 channels
constexpr int kCt8Plane = kBM * kCK * 2;         // 4 KB: 128 tokens x 32 B
constexpr int kCt8OutBox = 32 * 128;             // 4 KB: 32 rows x 8 channels x 8
constexpr int kCt8NumOut = 2;                    // staging boxes per epilogue warp

struct Ct8FwdParams {
  const uint8_t *wt;   // weight chunks of this direction, [j][kc]
  const __half *bias;  // [Do] or nullptr
  __half *out;         // [N][Do][8]
  int64_t N;
  int Ci, Do, BD, nD, nK, chunk_bytes;
  int nM, n_units;
  int nacc, acc_stride;
  int stages, stage_bytes, bias_floats;
};

struct Ct8Smem {
  int stage0, out0, bias, bars, total;
};

__host__ __device__ inline Ct8Smem ct8_fwd_smem(const Ct8FwdParams &p) {
  Ct8Smem s;
  s.stage0 = 0;
  s.out0 = p.stages * p.stage_bytes;
  s.bias = s.out0 + 4 * kCt8NumOut * kCt8OutBox;
  s.bars = s.bias + static_cast<int>(align_up(p.bias_floats * 4, 16));
  // full, tready, empty per stage; acc_full, acc_empty x2; final; tmem slot
  s.total = s.bars + (3 * p.stages + 4 + 1) * 8 + 16;
  return s;
}

__device__ __forceinline__ bool ct8_unit(const Ct8FwdParams &p, int k, int &m, int &j) {
  const int u = blockIdx.x + k * gridDim.x;
  if (u >= p.n_units) return false;
  m = u / p.nD;
  j = u % p.nD;
  return true;
}

// 14 warps over the 4 SM sub-partitions put 4 warps on one 16K-register slice.
__global__ void __maxnreg__(128)
tc_ct8_fwd_kernel(const __grid_constant__ CUtensorMap tm_in, const __grid_constant__ CUtensorMap tm_out,
                  const Ct8FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const Ct8Smem L = ct8_fwd_smem(p);
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
      mbar_init(&acc_empty[a], 4);
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
      int s = 0, m, j;
      uint32_t ph = 0;
      for (int k = 0; ct8_unit(p, k, m, j); ++k) {
        for (int kc = 0; kc < p.nK; ++kc) {
          if (ok) ok = mbar_wait(&empty[s], ph ^ 1);
          if (ok) {
            uint8_t *st = smem + L.stage0 + s * p.stage_bytes;
            mbar_arrive_expect_tx(&full[s], kCt8XChunk + p.chunk_bytes);
            tma_load_2d(st, &tm_in, kc * (kCK * kT8), m * kBM, &full[s]);
            tma_load_2d(st + kCt8Box, &tm_in, kc * (kCK * kT8) + 64, m * kBM, &full[s]);
            bulk_load(st + kCt8XChunk,
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
      const uint32_t stage16 = p.stage_bytes >> 4, pl16 = kCt8Plane >> 4;
      const uint32_t w16 = 2 * p.BD;  // BD rows of 32 B, in 16-byte units
      int s = 0, a = 0, m, j;
      uint32_t ph = 0, aph = 0;
      for (int it = 0; ct8_unit(p, it, m, j); ++it) {
        if (ok) ok = mbar_wait(&acc_empty[a], aph ^ 1);
        tc_fence_after();
        const uint32_t acc = tmem_base + a * p.acc_stride;
        for (int kc = 0; kc < p.nK; ++kc) {
          if (ok) ok = mbar_wait(&full[s], ph);
          if (ok) ok = mbar_wait(&tready[s], ph);
          tc_fence_after();
          if (ok) {
            const uint32_t xd = x0 + s * stage16, wd = xd + (kCt8XChunk >> 4);
            const uint32_t in = kc > 0 ? 1u : 0u;
            mma_f16_lo(acc, xd, wd, dhi, id_bd, in);                        // Y0
            mma_f16_lo(acc + p.BD, xd + pl16, wd + w16, dhi, id_bd, in);    // Y4
#pragma unroll
            for (int k = 1; k <= 3; ++k) {                                  // Y1, Y2, Y3
              const uint32_t col = acc + 2 * k * p.BD;
              const uint32_t rk = (2 + 3 * (k - 1)) * w16;
              mma_f16_lo(col, xd + 2 * k * pl16, wd + rk, dhi, id_2bd, in);
              mma_f16_lo(col, xd + (2 * k + 1) * pl16, wd + rk + w16, dhi, id_2bd, 1u);
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
    int s = 0, m, j;
    uint32_t ph = 0;
    for (int k = 0; ct8_unit(p, k, m, j); ++k) {
      for (int kc = 0; kc < p.nK; ++kc) {
        if (ok) ok = mbar_wait(&full[s], ph);
        uint8_t *st = smem + L.stage0 + s * p.stage_bytes;
        const uint8_t *src = st + bx * kCt8Box + r * 128;
        uint32_t pw[8][4];  // [plane][channel pair], packed fp16
#pragma unroll
        for (int q = 0; q < 8; q += 2) {  // 16-byte chunk q = channel 8 bx + q, its 8 group elements
          const uint4 r0 = *reinterpret_cast<const uint4 *>(src + ((q ^ (r & 7)) << 4));
          const uint4 r1 = *reinterpret_cast<const uint4 *>(src + (((q + 1) ^ (r & 7)) << 4));
          uint32_t o[8];
          rdft8_pair(r0, r1, o);
#pragma unroll
          for (int pp = 0; pp < 8; ++pp) pw[pp][q / 2] = o[pp];
        }
        named_bar_sync(2, 256);  // every row read before the planes overwrite it
#pragma unroll
        for (int pp = 0; pp < 8; ++pp)
          *reinterpret_cast<uint4 *>(st + pp * kCt8Plane + r * 32 + (((bx ^ (r >> 2)) & 1) << 4)) =
              make_uint4(pw[pp][0], pw[pp][1], pw[pp][2], pw[pp][3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&tready[s]);
        if (++s == p.stages) { s = 0; ph ^= 1; }
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int groups = p.BD / 8;
    uint8_t *obase = smem + L.out0 + (warp - 10) * kCt8NumOut * kCt8OutBox;
    int a = 0, oi = 0, m, j;
    uint32_t aph = 0;
    for (int it = 0; ct8_unit(p, it, m, j); ++it) {
      if (ok) ok = mbar_wait(&acc_full[a], aph);
      tc_fence_after();
      const uint32_t tl = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + a * p.acc_stride;
      for (int g = 0; g < groups; ++g) {
        uint32_t Y[8][8];  // [accumulator block][column]: Y0, Y4, Re1, Im1, Re2, Im2, Re3, Im3
        __syncwarp();      // the TMEM loads are warp-collective
#pragma unroll
        for (int bk = 0; bk < 8; ++bk) tmem_ld8(tl + g * 8 + bk * p.BD, Y[bk]);
        tmem_ld_wait();
        if (g == groups - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0 && ok) mbar_arrive(&acc_empty[a]);
        }
        const int d0 = j * p.BD + g * 8;
        if (d0 >= p.Do) continue;  // whole group is padding
        uint8_t *ob = obase + (oi % kCt8NumOut) * kCt8OutBox;
        if (lane == 0) bulk_wait_read<kCt8NumOut - 1>();  // this box's last store has read it
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {  // 16-byte chunk i of the row = output channel d0 + i
          float y[8];
          irdft8(__uint_as_float(Y[0][i]), __uint_as_float(Y[1][i]), __uint_as_float(Y[2][i]),
                 __uint_as_float(Y[3][i]), __uint_as_float(Y[4][i]), __uint_as_float(Y[5][i]),
                 __uint_as_float(Y[6][i]), __uint_as_float(Y[7][i]), y);
          const float bv = sbias[d0 + i];
          *reinterpret_cast<uint4 *>(ob + lane * 128 + ((i ^ (lane & 7)) << 4)) =
              make_uint4(pack_half2(y[0] + bv, y[1] + bv), pack_half2(y[2] + bv, y[3] + bv),
                         pack_half2(y[4] + bv, y[5] + bv), pack_half2(y[6] + bv, y[7] + bv));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {  // the store clips rows past N and channels past Do
          tma_store_2d(&tm_out, d0 * kT8, m * kBM + quad * 32, ob);
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
// (cross-correlation theorem; the same inverse as the forward), db = sum dY_0.
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
constexpr int kCt8DwTB = 32;                     // tokens per chunk (2 MMA K-steps)
constexpr int kCt8DwBox = kCt8DwTB * 128;        // 4 KB: 32 tokens x 8 channels x 8
constexpr int kCt8DwDySlots = 16;                // box slots for dy (the M = 128 operand spans 8 pairs)
constexpr int kCt8DwThreads = 64 + 8 * 32;
constexpr int kCt8DwMaxPer = 3;                  // (box, token) items per transform thread

struct Ct8DwParams {
  int64_t N;
  int C, D, Cs;        // Cs: workspace row stride (C rounded up to 16)
  int CT;              // c columns per tile (16 or 32)
  int tiles_d, tiles_c, splits;
  int64_t split_len;   // tokens per split, multiple of kCt8DwTB
  int stages;
  int slot_boxes;      // kCt8DwDySlots + 2 * CT / 16
  float *ws;           // [splits][8][D][Cs]: G0, G4, Re G1, Im G1, Re G2, Im G2, Re G3, Im G3
  float *ws_db;        // [splits][D]
};

struct Ct8DwSmem {
  int stage0, bars, total;
};

__host__ __device__ inline Ct8DwSmem ct8_dw_smem(const Ct8DwParams &p) {
  Ct8DwSmem s;
  s.stage0 = 0;
  s.bars = p.stages * p.slot_boxes * kCt8DwBox;
  // full, tready, empty per stage; acc_full; tmem slot
  s.total = s.bars + (3 * p.stages + 1) * 8 + 16;
  return s;
}

__global__ void __launch_bounds__(kCt8DwThreads, 1)
tc_ct8_dw_kernel(const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_x,
                 const Ct8DwParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const Ct8DwSmem L = ct8_dw_smem(p);
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
  const int nch = t_begin < t_end ? static_cast<int>(cdiv(t_end - t_begin, kCt8DwTB)) : 0;
  const int xoff = kCt8DwDySlots * kCt8DwBox;  // x region of a stage
  const int ncols = 14 * p.CT;
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
          uint8_t *st = smem + L.stage0 + s * p.slot_boxes * kCt8DwBox;
          const int32_t row = static_cast<int32_t>(t_begin + static_cast<int64_t>(ch) * kCt8DwTB);
          mbar_arrive_expect_tx(&full[s], nbox * kCt8DwBox);
          for (int q = 0; q < nqd; ++q)
            tma_load_2d(st + q * kCt8DwBox, &tm_dy, (d0 + 8 * q) * kT8, row, &full[s]);
          for (int q = 0; q < nqc; ++q)
            tma_load_2d(st + xoff + q * kCt8DwBox, &tm_x, (c0 + 8 * q) * kT8, row, &full[s]);
        }
        if (++s == p.stages) { s = 0; ph ^= 1; }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id1 = instr_desc(128, p.CT, 0, 0, 1, 1);
      const uint32_t id2 = instr_desc(128, 2 * p.CT, 0, 0, 1, 1);
      const uint64_t da = smem_desc(0, 2 * kCt8DwBox, 256, kSw32);  // dy: pairs 8 KB apart
      const uint64_t db = smem_desc(0, kCt8DwTB * 32, 256, kSw32);  // x: pairs 1 KB apart
      const uint32_t dhi = desc_hi(da);
      const uint32_t a0 = desc_lo(desc_at(da, smem_u32(smem + L.stage0)));
      const uint32_t b0 = desc_lo(desc_at(db, smem_u32(smem + L.stage0 + xoff)));
      const uint32_t stage16 = (p.slot_boxes * kCt8DwBox) >> 4;
      const uint32_t apl = (kCt8DwTB * 32) >> 4, bpl = (npc * kCt8DwTB * 32) >> 4;  // one plane
      int s = 0;
      uint32_t ph = 0;
      for (int ch = 0; ch < nch; ++ch) {
        if (ok) ok = mbar_wait(&full[s], ph);
        if (ok) ok = mbar_wait(&tready[s], ph);
        tc_fence_after();
        if (ok) {
          const uint32_t sa = a0 + s * stage16, sb = b0 + s * stage16;
#pragma unroll
          for (int k = 0; k < kCt8DwTB / 16; ++k) {  // 16 tokens = 512 B = 32 units
            const uint32_t A = sa + k * 32, B = sb + k * 32;
            const uint32_t first = (ch == 0 && k == 0) ? 0u : 1u;
            mma_f16_lo(tmem_base, A, B, dhi, id1, first);                  // G0
            mma_f16_lo(tmem_base + p.CT, A + apl, B + bpl, dhi, id1, first);  // G4
#pragma unroll
            for (int bk = 1; bk <= 3; ++bk) {
              const uint32_t ca = tmem_base + 2 * p.CT + 4 * (bk - 1) * p.CT;
              mma_f16_lo(ca, A + 2 * bk * apl, B + 2 * bk * bpl, dhi, id2, first);
              mma_f16_lo(ca + 2 * p.CT, A + (2 * bk + 1) * apl, B + 2 * bk * bpl, dhi, id2, first);
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
    float db_acc[kCt8DwMaxPer][8];
#pragma unroll
    for (int k = 0; k < kCt8DwMaxPer; ++k)
#pragma unroll
      for (int q = 0; q < 8; ++q) db_acc[k][q] = 0.f;
    int s = 0;
    uint32_t ph = 0;
    for (int ch = 0; ch < nch; ++ch) {
      if (ok) ok = mbar_wait(&full[s], ph);
      uint8_t *st = smem + L.stage0 + s * p.slot_boxes * kCt8DwBox;
      uint32_t pw[kCt8DwMaxPer][8][4];
#pragma unroll
      for (int k = 0; k < kCt8DwMaxPer; ++k) {
        const int e = t + k * 256;
        const int bi = e / kCt8DwTB, r = e % kCt8DwTB;
        if (bi < nbox) {
          const uint8_t *src = st + (bi < nqd ? bi * kCt8DwBox : xoff + (bi - nqd) * kCt8DwBox) +
                               r * 128;
#pragma unroll
          for (int q = 0; q < 8; q += 2) {
            const uint4 r0 = *reinterpret_cast<const uint4 *>(src + ((q ^ (r & 7)) << 4));
            const uint4 r1 = *reinterpret_cast<const uint4 *>(src + (((q + 1) ^ (r & 7)) << 4));
            uint32_t o[8];
            rdft8_pair(r0, r1, o);
            if (bi < nqd) {
              const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&o[0]));
              db_acc[k][q] += f.x;
              db_acc[k][q + 1] += f.y;
            }
#pragma unroll
            for (int pp = 0; pp < 8; ++pp) pw[k][pp][q / 2] = o[pp];
          }
        }
      }
      named_bar_sync(2, 256);  // every row read before the planes overwrite it
#pragma unroll
      for (int k = 0; k < kCt8DwMaxPer; ++k) {
        const int e = t + k * 256;
        const int bi = e / kCt8DwTB, r = e % kCt8DwTB;
        if (bi < nbox) {
          const bool is_dy = bi < nqd;
          const int q2 = is_dy ? bi : bi - nqd;
          const int g = q2 / 2, hh = q2 % 2;
          // dy pair g: plane pp at g x 8 KB + pp x 1 KB; x: plane-major (pp x npc + g) x 1 KB
          uint8_t *pbase = is_dy ? st + g * 2 * kCt8DwBox : st + xoff + g * kCt8DwTB * 32;
          const int pstride = is_dy ? kCt8DwTB * 32 : npc * kCt8DwTB * 32;
#pragma unroll
          for (int pp = 0; pp < 8; ++pp)
            *reinterpret_cast<uint4 *>(pbase + pp * pstride + r * 32 + (((hh ^ (r >> 2)) & 1) << 4)) =
                make_uint4(pw[k][pp][0], pw[k][pp][1], pw[k][pp][2], pw[k][pp][3]);
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
    float *dst = p.ws + static_cast<int64_t>(split) * 8 * plane + static_cast<int64_t>(d0 + d) * p.Cs + c0;
    for (int g = half; g < p.CT / 8; g += 2) {  // 8-column steps
      uint32_t v0[8], v4[8], ra[3][8], rb[3][8], ia[3][8], ib[3][8];
      __syncwarp();  // the TMEM loads are warp-collective
      tmem_ld8(tl + g * 8, v0);
      tmem_ld8(tl + p.CT + g * 8, v4);
#pragma unroll
      for (int bk = 0; bk < 3; ++bk) {
        const uint32_t ca = tl + 2 * p.CT + 4 * bk * p.CT + g * 8;
        tmem_ld8(ca, ra[bk]);                 // a[c]
        tmem_ld8(ca + p.CT, ia[bk]);          // a[CT + c]
        tmem_ld8(ca + 2 * p.CT, rb[bk]);      // b[c]
        tmem_ld8(ca + 3 * p.CT, ib[bk]);      // b[CT + c]
      }
      tmem_ld_wait();
      if (d0 + d < p.D && c0 + g * 8 < p.C) {
        float G[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          G[0][i] = __uint_as_float(v0[i]);
          G[1][i] = __uint_as_float(v4[i]);
#pragma unroll
          for (int bk = 0; bk < 3; ++bk) {
            G[2 + 2 * bk][i] = __uint_as_float(ra[bk][i]) + __uint_as_float(ib[bk][i]);
            G[3 + 2 * bk][i] = __uint_as_float(ia[bk][i]) - __uint_as_float(rb[bk][i]);
          }
        }
#pragma unroll
        for (int bin = 0; bin < 8; ++bin) {
          float4 *o = reinterpret_cast<float4 *>(dst + bin * plane + g * 8);
          o[0] = make_float4(G[bin][0], G[bin][1], G[bin][2], G[bin][3]);
          o[1] = make_float4(G[bin][4], G[bin][5], G[bin][6], G[bin][7]);
        }
      }
    }
    tc_fence_before();
    // db (tiles of the first c column only): fixed-order reduction through shared memory
    if (tj == 0) {
      named_bar_sync(3, 256);  // the stages are free: every chunk has been consumed
      float *sdb = reinterpret_cast<float *>(smem + L.stage0);  // [kCt8DwMaxPer * 256][8]
#pragma unroll
      for (int k = 0; k < kCt8DwMaxPer; ++k)
#pragma unroll
        for (int q = 0; q < 8; ++q) sdb[(t + k * 256) * 8 + q] = db_acc[k][q];
      named_bar_sync(3, 256);
      if (t < nqd * 8) {
        const int bi = t / 8, q = t % 8;  // dy box bi, channel q: rows bi*TB .. of the items
        float sum = 0.f;
        for (int rr = 0; rr < kCt8DwTB; ++rr) sum += sdb[(bi * kCt8DwTB + rr) * 8 + q];
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

__host__ __device__ inline int64_t ct8_reduce_blocks(int C, int D) {
  return cdiv(static_cast<int64_t>(D) * C, kRed8Out) + cdiv(D, kRed8Out);
}

__global__ void __launch_bounds__(kRed8Out * kRed8Groups)
ct8_dw_reduce_kernel(const float *__restrict__ ws, const float *__restrict__ ws_db,
                     __half *__restrict__ dW, __half *__restrict__ db, int splits, int C, int D,
                     int Cs) {
  __shared__ float part[kRed8Groups][kT8][kRed8Out];
  const int64_t n = static_cast<int64_t>(D) * C;
  const int64_t plane = static_cast<int64_t>(D) * Cs;
  const int64_t nblk_w = cdiv(n, kRed8Out);
  const int lo = threadIdx.x % kRed8Out, grp = threadIdx.x / kRed8Out;
  if (blockIdx.x < nblk_w) {
    const int64_t e = blockIdx.x * static_cast<int64_t>(kRed8Out) + lo;
    float G[kT8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (e < n) {
      const float *src = ws + (e / C) * Cs + (e % C);
      for (int s = grp; s < splits; s += kRed8Groups) {
        const float *q = src + static_cast<int64_t>(s) * kT8 * plane;
#pragma unroll
        for (int k = 0; k < kT8; ++k) G[k] += q[k * plane];
      }
    }
#pragma unroll
    for (int k = 0; k < kT8; ++k) part[grp][k][lo] = G[k];
    __syncthreads();
    if (grp == 0 && e < n) {
      float t[kT8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int q = 0; q < kRed8Groups; ++q)
#pragma unroll
        for (int k = 0; k < kT8; ++k) t[k] += part[q][k][lo];
      float y[kT8];
      irdft8(t[0], t[1], t[2], t[3], t[4], t[5], t[6], t[7], y);
      *reinterpret_cast<uint4 *>(dW + e * kT8) =
          make_uint4(pack_half2(y[0], y[1]), pack_half2(y[2], y[3]), pack_half2(y[4], y[5]),
                     pack_half2(y[6], y[7]));
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
      db[d] = __float2half_rn(t);
    }
  }
}

}  // namespace feql
