// tc_fwd.cuh — fused forward / dX kernel on the sm_100a tensor cores (fp16).
//
// Flash EQ-Linear (technical summary "Approccio Algoritmico",
// "Specializzazione per il Gruppo di Rotazione p4", "Implementazione"):
//   out[n, :, :] = irDFT_4( per-bin  X_k[n, :] . What_k^T ) (+ bias)
// with X = rDFT_4(in) along the group axis.  Bins 0 and 2 are real
// contractions, bin 1 is one complex contraction; the Fourier tiles live only
// in shared memory / tensor memory (no intermediate global writes).
//
// One persistent CTA per SM, warp-specialised (320 threads):
//   warp 0      TMA producer: input chunk [128 tokens x 16 channels x 4] and
//               the matching weight chunk into a ring of `stages` slots
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2..5  transform: 4-point rDFT of the chunk, in place, into four
//               K-major fp16 operand planes (X0, X2, Re X1, Im X1)
//   warps 6..9  epilogue: tcgen05.ld of the four fp32 accumulators, inverse
//               rDFT + bias, fp16 pack, swizzled smem staging, TMA store
// Per chunk the MMA warp issues four M=128 x K=16 MMAs:
//   acc[0, BD)    += X0  * What0^T                (N = BD)
//   acc[BD, 2BD)  += X2  * What2^T                (N = BD)
//   acc[2BD, 4BD) += ReX1 * (Re1 ; Im1)^T + ImX1 * (-Im1 ; Re1)^T   (N = 2 BD)
// so columns [2BD, 3BD) hold Re Y1 and [3BD, 4BD) hold Im Y1.
// Every wait is bounded (mbar_wait); a timed-out thread stops issuing work but
// keeps the loop structure so named barriers stay matched.
#pragma once

#include <cuda_fp16.h>

#include "plan.cuh"
#include "sm100.cuh"

namespace feql {

constexpr int kTcThreads = 320;
constexpr int kXChunkBytes = kBM * kCK * kT * 2;  // 16 KB: 128 rows x 128 B
constexpr int kPlaneBytes = kBM * kCK * 2;        // 4 KB: 128 rows x 32 B
constexpr int kOutBoxBytes = kBM * 64 * 2;        // 16 KB: 128 rows x (16 ch x 4) fp16
constexpr int kNumOut = 2;
constexpr int kTmemCols = 512;

struct TcFwdParams {
  const uint8_t *wt;    // weight chunks of this direction
  const __half *bias;   // [Do] or nullptr
  int64_t N;
  int Ci, Do, BD, nD, nK, chunk_bytes;
  int n_units;          // ceil(N/128) * nD
  int nacc, acc_stride; // accumulator buffers in TMEM and their column stride
  int stages;
  int stage_bytes;      // 16 KB input chunk + weight chunk (1 KB aligned)
  int bias_floats;      // nD * BD
};

struct TcSmem {
  // offsets (bytes) from the 1024-aligned dynamic smem base
  int stage0, out0, bias, bars, total;
};

__host__ __device__ inline TcSmem tc_fwd_smem(const TcFwdParams &p) {
  TcSmem s;
  s.stage0 = 0;
  s.out0 = p.stages * p.stage_bytes;
  s.bias = s.out0 + kNumOut * kOutBoxBytes;
  s.bars = s.bias + static_cast<int>(align_up(p.bias_floats * 4, 16));
  // full, tready, empty per stage; acc_full, acc_empty per acc buffer; final; tmem slot
  s.total = s.bars + (3 * p.stages + 2 * 2 + 1) * 8 + 16;
  return s;
}

__global__ void __launch_bounds__(kTcThreads, 1)
tc_fourier_gemm_kernel(const __grid_constant__ CUtensorMap tm_in,
                       const __grid_constant__ CUtensorMap tm_out, const TcFwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const TcSmem L = tc_fwd_smem(p);
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
      mbar_init(&tready[s], 4);
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
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int first = blockIdx.x, step = gridDim.x;
  bool ok = true;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      tma_prefetch_desc(&tm_in);
      tma_prefetch_desc(&tm_out);
      int s = 0;
      uint32_t ph = 0;
      for (int u = first; u < p.n_units; u += step) {
        const int m = u / p.nD, j = u % p.nD;
        for (int kc = 0; kc < p.nK; ++kc) {
          if (ok) ok = mbar_wait(&empty[s], ph ^ 1);
          if (ok) {
            uint8_t *st = smem + L.stage0 + s * p.stage_bytes;
            mbar_arrive_expect_tx(&full[s], kXChunkBytes + p.chunk_bytes);
            tma_load_2d(st, &tm_in, kc * (kCK * kT), m * kBM, &full[s]);
            bulk_load(st + kXChunkBytes,
                      p.wt + (static_cast<int64_t>(j) * p.nK + kc) * p.chunk_bytes,
                      p.chunk_bytes, &full[s]);
          }
          if (++s == p.stages) { s = 0; ph ^= 1; }
        }
      }
      // drain: the last loads must land before the CTA may exit
      for (int i = 0; i < p.stages; ++i) {
        if (ok) ok = mbar_wait(&empty[s], ph ^ 1);
        if (++s == p.stages) { s = 0; ph ^= 1; }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id_bd = instr_desc(kBM, p.BD, 0, 0);
      const uint32_t id_2bd = instr_desc(kBM, 2 * p.BD, 0, 0);
      const uint32_t wrow = 32;  // bytes per weight row (16 fp16)
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int u = first; u < p.n_units; u += step, ++it) {
        const int a = it % p.nacc;
        const uint32_t aph = (it / p.nacc) & 1;
        if (ok) ok = mbar_wait(&acc_empty[a], aph ^ 1);
        tc_fence_after();
        const uint32_t acc = tmem_base + a * p.acc_stride;
        for (int kc = 0; kc < p.nK; ++kc) {
          if (ok) ok = mbar_wait(&full[s], ph);
          if (ok) ok = mbar_wait(&tready[s], ph);
          tc_fence_after();
          if (ok) {
            const uint32_t xs = smem_u32(smem + L.stage0 + s * p.stage_bytes);
            const uint32_t ws = xs + kXChunkBytes;
            const uint32_t acc_in = kc > 0 ? 1u : 0u;
            mma_f16_ss(acc, smem_desc(xs + 0 * kPlaneBytes, 16, 256, kSw32),
                       smem_desc(ws, 16, 256, kSw32), id_bd, acc_in);
            mma_f16_ss(acc + p.BD, smem_desc(xs + 1 * kPlaneBytes, 16, 256, kSw32),
                       smem_desc(ws + p.BD * wrow, 16, 256, kSw32), id_bd, acc_in);
            mma_f16_ss(acc + 2 * p.BD, smem_desc(xs + 2 * kPlaneBytes, 16, 256, kSw32),
                       smem_desc(ws + 2 * p.BD * wrow, 16, 256, kSw32), id_2bd, acc_in);
            mma_f16_ss(acc + 2 * p.BD, smem_desc(xs + 3 * kPlaneBytes, 16, 256, kSw32),
                       smem_desc(ws + 4 * p.BD * wrow, 16, 256, kSw32), id_2bd, 1u);
            mma_commit(&empty[s]);
          }
          if (++s == p.stages) { s = 0; ph ^= 1; }
        }
        if (ok) mma_commit(&acc_full[a]);
      }
      // all MMAs must be complete before TMEM is released
      mma_commit(final_bar);
      mbar_wait(final_bar, 0);
    }
  } else if (warp < 6) {
    // ---------------------------------------------------------- transform
    const int r = threadIdx.x - 64;  // row of the chunk (token within the tile)
    int s = 0;
    uint32_t ph = 0;
    for (int u = first; u < p.n_units; u += step) {
      for (int kc = 0; kc < p.nK; ++kc) {
        if (ok) ok = mbar_wait(&full[s], ph);
        uint8_t *st = smem + L.stage0 + s * p.stage_bytes;
        // row r: 8 x 16 B, logical chunk q = channels 2q, 2q+1 (x 4 group elements)
        uint4 raw[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          raw[q] = *reinterpret_cast<const uint4 *>(st + r * 128 + ((q ^ (r & 7)) << 4));
        uint32_t pl[4][8];  // [plane][channel pair] packed half2
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const __half2 *h = reinterpret_cast<const __half2 *>(&raw[q]);
          float f[2][4];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const float2 lo = __half22float2(h[2 * c]), hi = __half22float2(h[2 * c + 1]);
            const float v0 = lo.x, v1 = lo.y, v2 = hi.x, v3 = hi.y;
            const float a = v0 + v2, b = v1 + v3;
            f[c][0] = a + b;
            f[c][1] = a - b;
            f[c][2] = v0 - v2;
            f[c][3] = v3 - v1;
          }
#pragma unroll
          for (int pp = 0; pp < 4; ++pp) pl[pp][q] = pack_half2(f[0][pp], f[1][pp]);
        }
        named_bar_sync(2, 128);  // every row read before the planes overwrite it
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          uint8_t *plane = st + pp * kPlaneBytes + r * 32;
#pragma unroll
          for (int h = 0; h < 2; ++h)
            *reinterpret_cast<uint4 *>(plane + (((h ^ (r >> 2)) & 1) << 4)) =
                make_uint4(pl[pp][4 * h + 0], pl[pp][4 * h + 1], pl[pp][4 * h + 2],
                           pl[pp][4 * h + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&tready[s]);
        if (++s == p.stages) { s = 0; ph ^= 1; }
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int quad = warp & 3;              // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;       // token within the tile
    const int et = threadIdx.x - 192;       // 0..127 among epilogue threads
    int it = 0, oi = 0;
    for (int u = first; u < p.n_units; u += step, ++it) {
      const int m = u / p.nD, j = u % p.nD;
      const int a = it % p.nacc;
      const uint32_t aph = (it / p.nacc) & 1;
      if (ok) ok = mbar_wait(&acc_full[a], aph);
      tc_fence_after();
      const uint32_t tl = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + a * p.acc_stride;
      const int groups = p.BD / 16;
      for (int g = 0; g < groups; ++g) {
        uint32_t y0[16], y2[16], y1r[16], y1i[16];
        tmem_ld16(tl + g * 16, y0);
        tmem_ld16(tl + p.BD + g * 16, y2);
        tmem_ld16(tl + 2 * p.BD + g * 16, y1r);
        tmem_ld16(tl + 3 * p.BD + g * 16, y1i);
        tmem_ld_wait();
        if (g == groups - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0 && ok) mbar_arrive(&acc_empty[a]);
        }
        const int d0 = j * p.BD + g * 16;
        uint32_t packed[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float Y0 = __uint_as_float(y0[i]), Y2 = __uint_as_float(y2[i]);
          const float Yr = __uint_as_float(y1r[i]), Yi = __uint_as_float(y1i[i]);
          const float bv = sbias[d0 + i];
          const float e = fmaf(0.25f, Y0 + Y2, bv), o = fmaf(0.25f, Y0 - Y2, bv);
          packed[2 * i] = pack_half2(fmaf(0.5f, Yr, e), fmaf(-0.5f, Yi, o));
          packed[2 * i + 1] = pack_half2(fmaf(-0.5f, Yr, e), fmaf(0.5f, Yi, o));
        }
        if (d0 >= p.Do) continue;  // uniform across the epilogue warps
        uint8_t *ob = smem + L.out0 + (oi % kNumOut) * kOutBoxBytes;
        if (et == 0) bulk_wait_read<kNumOut - 1>();
        named_bar_sync(1, 128);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<uint4 *>(ob + row * 128 + ((q ^ (row & 7)) << 4)) =
              make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (et == 0) {
          tma_store_2d(&tm_out, d0 * kT, m * kBM, ob);
          bulk_commit();
        }
        ++oi;
      }
    }
    if (et == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace feql
