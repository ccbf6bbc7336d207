// tc_mlp.cuh — the p4-equivariant MLP block (fc1 -> GELU -> fc2) as one
// kernel on the sm_100a tensor cores, fp16 data with fp32 accumulation.
//
// Flash EQ-Linear builds its networks (technical summary "Livello di Rete":
// Flash EQ-ViT, Flash EQ-Swin) from EQ-Linear layers; a transformer MLP is two
// of them with a pointwise GELU between.  Both layers run the Fourier method
// (rDFT along the group axis, six real products per 16 channels, inverse),
// and the hidden activation never leaves the SM: fc1's accumulators are read
// from TMEM, inverse-transformed, biased, passed through GELU, transformed
// again and written to shared memory as fc2's A operand.
//
//   h[n,j,t] = b1[j] + sum_c sum_s W1[j,c,(t-s) mod 4] x[n,c,s]
//   y[n,o,t] = b2[o] + sum_j sum_s W2[o,j,(t-s) mod 4] GELU(h[n,j,s])
//
// GELU is evaluated in its tanh form, 0.5 z (1 + tanh(sqrt(2/pi)(z + 0.044715 z^3)))
// (Hendrycks and Gimpel), on packed fp16 pairs with the hardware tanh; it is
// within 5e-4 of the exact z*Phi(z) for every z.
//
// One persistent CTA per SM, 128-token tiles, 22 warps:
//   warp 0        TMA: the Fourier weights of both layers, resident (loaded
//                 once) or, when they do not fit, streamed per hidden slice
//                 through a ring of slots; each tile's x chunks [128 tokens x 16
//                 channels x 4] into one of `nx` tile buffers
//   warp 1        TMEM allocator + single-thread MMA issuer
//   warps 2..5    transform: rDFT of the x tile in place into four K-major
//                 planes per chunk (V0, V2, Re V1, -Im V1)
//   warps 6..17   GELU: per hidden slice of HS channels (three warps per TMEM
//                 lane quadrant, every third 8-channel group each) inverse
//                 rDFT + b1 -> GELU -> rDFT -> fp16 planes in one of two
//                 hidden buffers
//   warps 18..21  fc2 epilogue: inverse rDFT + b2, TMA stores of y
// TMEM: fc1 accumulators 2 x 4*HS columns (Y0 | Y2 | Re Y1 | Im Y1 of a
// slice), fc2 accumulators (one or two, by tile) of 4*BD2 columns from 8*HS.
// Issue order over the CTA's hidden slices gs (tile-major, across tiles):
// fc1(0), fc1(1), fc2(0), fc1(2), fc2(1), ..., so the GELU of one slice
// overlaps the fc1 MMAs of the next, also at tile boundaries.
// Every wait is bounded (mbar_wait); a timed-out thread stops issuing work but
// keeps the loop structure so named barriers stay matched.
#pragma once

#include <cuda_fp16.h>

#include "plan.cuh"
#include "rdft4.cuh"
#include "sm100.cuh"
#include "wfft.cuh"

namespace feql {

constexpr int kMlpGeluParts = 3;                         // GELU warps per TMEM lane quadrant
constexpr int kMlpGeluWarps = 4 * kMlpGeluParts;
constexpr int kMlpEpiWarp0 = 6 + kMlpGeluWarps;           // first fc2 epilogue warp
constexpr int kMlpThreads = (kMlpEpiWarp0 + 4) * 32;      // 22 warps
// registers per thread: the busiest SM sub-partition holds ceil(warps / 4)
// warps in its 16K-register slice
constexpr int kMlpMaxRegs = (16384 / (((kMlpThreads / 32 + 3) / 4) * 32)) / 8 * 8;  // 80
constexpr int kMlpYBoxes = 2;                    // output staging boxes per epilogue warp
constexpr int kMlpChunkBytes = kBM * kCK * kT * 2;  // 16 KB: 128 tokens x 16 channels x 4
constexpr int kMlpPlaneBytes = kBM * kCK * 2;       // 4 KB: one plane of a chunk

// Plan of the block: shapes, hidden slicing and the Fourier-weight layout.
//   fc1 weights: [slice j][x chunk kc] blocks of 5*HS rows x 32 B
//   fc2 weights: [hidden chunk kh] blocks of 5*BD2 rows x 32 B
// each block laid out like the single layer's (planes What0, What2, Re1, Im1,
// -Re1 of BD rows, K-major, 32-byte swizzle).
struct MlpPlan {
  int C, H, Co;
  int nK1;             // x chunks of 16 channels
  int HS, nS;          // hidden slice width (multiple of 16) and count
  int nKh;             // hidden chunks of 16 channels: nS * HS / 16
  int BD2;             // fc2 output channels, padded to 16 (<= 64)
  int w1_chunk, w2_chunk;
  int64_t w1_bytes, w2_bytes, off_w2, bytes;
};

__host__ __device__ inline MlpPlan make_mlp_plan(int C, int H, int Co, int hs_max) {
  MlpPlan p;
  p.C = C;
  p.H = H;
  p.Co = Co;
  p.nK1 = static_cast<int>(cdiv(C, kCK));
  p.BD2 = static_cast<int>(align_up(Co, 16));
  p.nS = static_cast<int>(cdiv(H, hs_max));
  p.HS = static_cast<int>(align_up(cdiv(H, p.nS), 16));
  p.nKh = p.nS * p.HS / kCK;
  p.w1_chunk = 5 * p.HS * kCK * 2;
  p.w2_chunk = 5 * p.BD2 * kCK * 2;
  p.w1_bytes = static_cast<int64_t>(p.nS) * p.nK1 * p.w1_chunk;
  p.w2_bytes = static_cast<int64_t>(p.nKh) * p.w2_chunk;
  p.off_w2 = align_up(p.w1_bytes, 1024);
  p.bytes = p.off_w2 + align_up(p.w2_bytes, 1024);
  return p;
}

// Weight transform of both layers: one thread per fp16 element of the buffer.
// fc1's bins carry the inverse transform's scales: bins 0 and 2 are stored
// times 1/8, bin 1 times 1/4 (powers of two: exact); with x's planes divided by
// 4 its accumulators give v_t = h_t / 8 with sums and differences alone.  fc2's
// bins are divided by 4, like the hidden planes (GELU / 4) they multiply, so no
// fp16 plane overflows for any finite x, W1, W2 or hidden activation.
__global__ void wfft_mlp_kernel(const __half *__restrict__ W1, const __half *__restrict__ W2,
                                uint8_t *__restrict__ What, MlpPlan P) {
  const int64_t n1 = P.w1_bytes / 2, n2 = P.w2_bytes / 2;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n1 + n2;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const bool first = e < n1;
    const int64_t le = first ? e : e - n1;
    const int BD = first ? P.HS : P.BD2;
    const int rows = 5 * BD;
    const int64_t chunk = le / (rows * kCK);
    const int rem = static_cast<int>(le % (rows * kCK));
    const int row = rem / kCK, k = rem % kCK;
    const int sub = row / BD;
    int o, i, Do, Ci;
    if (first) {  // chunk = slice j * nK1 + kc
      o = static_cast<int>(chunk / P.nK1) * BD + row % BD;
      i = static_cast<int>(chunk % P.nK1) * kCK + k;
      Do = P.H;
      Ci = P.C;
    } else {  // chunk = hidden chunk kh
      o = row % BD;
      i = static_cast<int>(chunk) * kCK + k;
      Do = P.Co;
      Ci = P.H;
    }
    float v = 0.f;
    if (o < Do && i < Ci) {
      float b0, b2, b1r, b1i;
      weight_bins(first ? W1 : W2, Ci, 0, o, i, b0, b2, b1r, b1i);
      v = sub == 0 ? b0 : sub == 1 ? b2 : sub == 2 ? b1r : sub == 3 ? b1i : -b1r;
      v *= first ? (sub < 2 ? 0.125f : 0.25f) : 0.25f;
    }
    const int64_t base = first ? chunk * P.w1_chunk : P.off_w2 + chunk * P.w2_chunk;
    *reinterpret_cast<__half *>(What + base + sw32_offset(row, k)) = __float2half_rn(v);
  }
}

constexpr int kMlpMaxWSlots = 4;  // weight ring slots (streaming mode)

struct TcMlpParams {
  MlpPlan P;
  const uint8_t *wt;   // Fourier weights (MlpPlan layout)
  const __half *b1;    // [H] or nullptr
  const __half *b2;    // [Co] or nullptr
  int64_t N;
  int nM;              // token tiles
  int nx;              // x tile buffers (1 or 2)
  int wslots;          // 0: both layers' weights resident; else a ring of this many
                       // slots, each holding one hidden slice's fc1 and fc2 weights
};

struct MlpSmem {
  int w1, w2, x0, h0, y0, b1, b2, bars, total;
  int xtile, htile;    // bytes of one x tile buffer / one hidden buffer
  int w1s, w2s, wslot; // streaming: a slice's fc1 / fc2 weight bytes, one ring slot
};

__host__ __device__ inline MlpSmem mlp_smem(const TcMlpParams &p) {
  MlpSmem s;
  s.xtile = p.P.nK1 * kMlpChunkBytes;
  s.htile = (p.P.HS / kCK) * kMlpChunkBytes;
  s.w1s = p.P.nK1 * p.P.w1_chunk;
  s.w2s = (p.P.HS / kCK) * p.P.w2_chunk;
  s.wslot = static_cast<int>(align_up(s.w1s, 1024) + align_up(s.w2s, 1024));
  s.w1 = 0;
  if (p.wslots == 0) {
    s.w2 = static_cast<int>(align_up(p.P.w1_bytes, 1024));
    s.x0 = s.w2 + static_cast<int>(align_up(p.P.w2_bytes, 1024));
  } else {  // slot k: fc1 part at k * wslot, fc2 part after it
    s.w2 = static_cast<int>(align_up(s.w1s, 1024));
    s.x0 = p.wslots * s.wslot;
  }
  s.h0 = s.x0 + p.nx * s.xtile;
  s.y0 = s.h0 + 2 * s.htile;
  s.b1 = s.y0 + 4 * kMlpYBoxes * 4096;
  s.b2 = s.b1 + p.P.nS * p.P.HS * 4;
  s.bars = s.b2 + static_cast<int>(align_up(p.P.BD2 * 4, 16));
  s.total = s.bars + 32 * 8 + 16;
  return s;
}

// TMEM columns the block needs: two fc1 accumulators and one fc2 accumulator;
// a second fc2 accumulator is used when it fits.
__host__ __device__ inline int mlp_tmem_cols(const MlpPlan &P) { return 8 * P.HS + 4 * P.BD2; }
__host__ __device__ inline int mlp_acc2_buffers(const MlpPlan &P) {
  return 8 * P.HS + 8 * P.BD2 <= 512 ? 2 : 1;
}

__device__ __forceinline__ uint32_t tanh_h2(uint32_t x) {
  uint32_t y;
  asm("tanh.approx.f16x2 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// A quarter of the GELU (tanh form) of z = 8v for a packed fp16 pair v:
//   GELU(8v) / 4 = v (1 + tanh(8 k0 v + 512 k1 v^3)),  k0 = sqrt(2/pi), k1 = 0.044715 k0.
// (z / 8 and GELU / 4 keep the fp16 operand planes around it in range; the
// powers of two leave the rounding of every step as for z itself.  Where v^2
// overflows, the tanh argument is +-inf and the result v (1 +- 1) is exact.)
__device__ __forceinline__ uint32_t gelu_eighth_arg_h2(uint32_t vv) {
  const __half2 v = as_h2(vv);
  const __half2 c0 = __float2half2_rn(6.3830764864229232f);  // 8 sqrt(2/pi)
  const __half2 c1 = __float2half2_rn(18.266832965785664f);  // 512 * 0.044715 sqrt(2/pi)
  const __half2 t = as_h2(tanh_h2(as_u32(__hmul2(v, __hfma2(c1, __hmul2(v, v), c0)))));
  return as_u32(__hfma2(v, t, v));
}

// 22 warps: six on the busiest 16K-register sub-partition, 80 registers each.
// kStream: weights streamed per hidden slice (p.wslots > 0) or resident.
template <bool kStream>
__global__ void __maxnreg__(kMlpMaxRegs)
tc_mlp_kernel(const __grid_constant__ CUtensorMap tm_in, const __grid_constant__ CUtensorMap tm_out,
              const TcMlpParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const MlpPlan &P = p.P;
  const MlpSmem L = mlp_smem(p);
  uint32_t *sb1 = reinterpret_cast<uint32_t *>(smem + L.b1);  // b1 / 2, fp16 channel pairs
  float *sb2 = reinterpret_cast<float *>(smem + L.b2);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
  uint64_t *wfull = bars;
  uint64_t *xfull = bars + 1, *xready = bars + 3, *xempty = bars + 5;
  uint64_t *a1full = bars + 7, *a1empty = bars + 9;
  uint64_t *hready = bars + 11, *hempty = bars + 13;
  uint64_t *a2full = bars + 15, *a2empty = bars + 17, *final_bar = bars + 19;
  uint64_t *wsfull = bars + 20, *wsempty = bars + 24;  // weight ring (streaming mode)
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 28);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int hs = P.HS, nS = P.nS;

  if (threadIdx.x == 0) {
    mbar_init(wfull, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&xfull[b], 1);
      mbar_init(&xready[b], 4);
      mbar_init(&xempty[b], 1);
      mbar_init(&a1full[b], 1);
      mbar_init(&a1empty[b], kMlpGeluWarps);
      mbar_init(&hready[b], kMlpGeluWarps);
      mbar_init(&hempty[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&a2full[b], 1);
      mbar_init(&a2empty[b], 4);
    }
    mbar_init(final_bar, 1);
    for (int k = 0; k < kMlpMaxWSlots; ++k) {
      mbar_init(&wsfull[k], 1);
      mbar_init(&wsempty[k], 1);
    }
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < nS * hs / 2; i += blockDim.x) {  // b1 / 8, like fc1's accumulators
    const int j = 2 * i;
    const float v0 = (p.b1 != nullptr && j < P.H) ? 0.125f * __half2float(p.b1[j]) : 0.f;
    const float v1 = (p.b1 != nullptr && j + 1 < P.H) ? 0.125f * __half2float(p.b1[j + 1]) : 0.f;
    sb1[i] = pack_half2(v0, v1);
  }
  for (int i = threadIdx.x; i < P.BD2; i += blockDim.x)
    sb2[i] = (p.b2 != nullptr && i < P.Co) ? __half2float(p.b2[i]) : 0.f;
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t acc2_col = 8 * hs;  // fc2 accumulator buffer a at acc2_col + a * 4 * BD2
  const int nacc2 = mlp_acc2_buffers(P);
  // this CTA's tiles m = blockIdx.x + i * gridDim.x, i < n_my; hidden slices gs = i * nS + s
  const int n_my = static_cast<int>(blockIdx.x) < p.nM
                       ? (p.nM - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                       : 0;
  bool ok = true;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      tma_prefetch_desc(&tm_in);
      tma_prefetch_desc(&tm_out);
      if (!kStream && static_cast<int>(blockIdx.x) < p.nM) {
        mbar_arrive_expect_tx(wfull, static_cast<uint32_t>(P.w1_bytes + P.w2_bytes));
        bulk_load(smem + L.w1, p.wt, static_cast<uint32_t>(P.w1_bytes), wfull);
        bulk_load(smem + L.w2, p.wt + P.off_w2, static_cast<uint32_t>(P.w2_bytes), wfull);
      }
      // in the order the MMA warp consumes them: a tile's x, then (streaming) the
      // weights of each of its hidden slices
      int xb = 0, ws = 0;
      uint32_t xph = 0, wph = 0;
      for (int m = blockIdx.x; m < p.nM; m += gridDim.x) {
        if (ok) ok = mbar_wait(&xempty[xb], xph ^ 1);
        if (ok) {
          uint8_t *xt = smem + L.x0 + xb * L.xtile;
          mbar_arrive_expect_tx(&xfull[xb], L.xtile);
          for (int kc = 0; kc < P.nK1; ++kc)
            tma_load_2d(xt + kc * kMlpChunkBytes, &tm_in, kc * (kCK * kT), m * kBM, &xfull[xb]);
        }
        if (++xb == p.nx) { xb = 0; xph ^= 1; }
        for (int sl = 0; kStream && sl < nS; ++sl) {
          if (ok) ok = mbar_wait(&wsempty[ws], wph ^ 1);
          if (ok) {
            uint8_t *dst = smem + ws * L.wslot;
            mbar_arrive_expect_tx(&wsfull[ws], static_cast<uint32_t>(L.w1s + L.w2s));
            bulk_load(dst, p.wt + static_cast<int64_t>(sl) * L.w1s, static_cast<uint32_t>(L.w1s),
                      &wsfull[ws]);
            bulk_load(dst + L.w2, p.wt + P.off_w2 + static_cast<int64_t>(sl) * L.w2s,
                      static_cast<uint32_t>(L.w2s), &wsfull[ws]);
          }
          if (++ws == p.wslots) { ws = 0; wph ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    // The whole warp runs the issue loop (its descriptors stay warp-uniform);
    // one elected lane issues each MMA and commit.
    {
      const uint32_t id1a = instr_desc(kBM, hs, 0, 0), id1b = instr_desc(kBM, 2 * hs, 0, 0);
      const uint32_t id2a = instr_desc(kBM, P.BD2, 0, 0);
      const uint32_t id2b = instr_desc(kBM, 2 * P.BD2, 0, 0);
      const uint64_t dsw32 = smem_desc(0, 16, 256, kSw32);  // K-major, 32-byte swizzle
      const uint32_t dhi = desc_hi(dsw32);
      const uint32_t x0 = desc_lo(desc_at(dsw32, smem_u32(smem + L.x0)));
      const uint32_t h0 = desc_lo(desc_at(dsw32, smem_u32(smem + L.h0)));
      const uint32_t w1_0 = desc_lo(desc_at(dsw32, smem_u32(smem + L.w1)));
      const uint32_t w2_0 = desc_lo(desc_at(dsw32, smem_u32(smem + L.w2)));
      const uint32_t pl16 = kMlpPlaneBytes >> 4, ch16 = kMlpChunkBytes >> 4;
      const uint32_t xt16 = L.xtile >> 4, ht16 = L.htile >> 4;
      const uint32_t w1r16 = (hs * 32) >> 4, w1c16 = P.w1_chunk >> 4;
      const uint32_t w2r16 = (P.BD2 * 32) >> 4, w2c16 = P.w2_chunk >> 4;
      const int kh_per = hs / kCK;
      if (!kStream && static_cast<int>(blockIdx.x) < p.nM)
        ok = __all_sync(0xffffffffu, mbar_wait(wfull, 0));
      const uint32_t wslot16 = L.wslot >> 4, w2off16 = L.w2 >> 4;
      // The issuing thread's scalar work adds to every MMA, so the two cursors
      // below advance by increments (no divisions).
      int s1 = 0, xb = 0;      // fc1 cursor: slice s1 of the tile in x buffer xb
      uint32_t xph = 0;
      int s2 = 0, ab = 0;      // fc2 cursor: slice s2 of the tile in fc2 accumulator ab
      uint32_t abph = 0;
      int w1s = 0, w2s = 0;    // streaming: weight ring slots of fc1's and fc2's slice
      uint32_t w1ph = 0;
      // fc1 of hidden slice gs: its x tile (ready once per tile), fc1 accumulator gs % 2
      auto fc1 = [&](int gs) {
        const int b = gs & 1, s = s1, x = xb, wsl = w1s;
        if (s == 0 && ok) ok = mbar_wait(&xready[x], xph);
        if (ok) ok = mbar_wait(&a1empty[b], ((gs >> 1) & 1) ^ 1);
        if (kStream && ok) ok = mbar_wait(&wsfull[wsl], w1ph);
        ok = __all_sync(0xffffffffu, ok);
        if (++s1 == nS) {
          s1 = 0;
          if (++xb == p.nx) { xb = 0; xph ^= 1; }
        }
        if (kStream && ++w1s == p.wslots) { w1s = 0; w1ph ^= 1; }
        tc_fence_after();
        if (!ok) return;
        const uint32_t acc = tmem_base + b * 4 * hs;
        uint32_t xd = x0 + x * xt16;
        uint32_t wd = kStream ? w1_0 + wsl * wslot16 : w1_0 + s * P.nK1 * w1c16;
        if (elect_one()) {
          for (int kc = 0; kc < P.nK1; ++kc, xd += ch16, wd += w1c16) {
            const uint32_t acc_in = kc > 0 ? 1u : 0u;
            mma_f16_lo(acc, xd, wd, dhi, id1a, acc_in);
            mma_f16_lo(acc + hs, xd + pl16, wd + w1r16, dhi, id1a, acc_in);
            mma_f16_lo(acc + 2 * hs, xd + 2 * pl16, wd + 2 * w1r16, dhi, id1b, acc_in);
            mma_f16_lo(acc + 2 * hs, xd + 3 * pl16, wd + 3 * w1r16, dhi, id1b, 1u);
          }
          mma_commit(&a1full[b]);
          if (s == nS - 1) mma_commit(&xempty[x]);
        }
        __syncwarp();
      };
      // fc2 over the activations of slice gs into fc2 accumulator (tile % nacc2)
      auto fc2 = [&](int gs) {
        const int b = gs & 1, s = s2, a = ab, wsl = w2s;
        if (s == 0 && ok) ok = mbar_wait(&a2empty[a], abph ^ 1);
        if (ok) ok = mbar_wait(&hready[b], (gs >> 1) & 1);
        ok = __all_sync(0xffffffffu, ok);
        if (++s2 == nS) {
          s2 = 0;
          if (++ab == nacc2) { ab = 0; abph ^= 1; }
        }
        if (kStream && ++w2s == p.wslots) w2s = 0;
        tc_fence_after();
        if (!ok) return;
        const uint32_t acc2 = tmem_base + acc2_col + a * 4 * P.BD2;
        uint32_t hd = h0 + b * ht16;
        // (streaming: the slot's fc1 part was waited for by fc1 of the same slice)
        uint32_t wd = kStream ? w1_0 + wsl * wslot16 + w2off16 : w2_0 + s * kh_per * w2c16;
        if (elect_one()) {
          for (int kh = 0; kh < kh_per; ++kh, hd += ch16, wd += w2c16) {
            const uint32_t acc_in = (s == 0 && kh == 0) ? 0u : 1u;
            mma_f16_lo(acc2, hd, wd, dhi, id2a, acc_in);
            mma_f16_lo(acc2 + P.BD2, hd + pl16, wd + w2r16, dhi, id2a, acc_in);
            mma_f16_lo(acc2 + 2 * P.BD2, hd + 2 * pl16, wd + 2 * w2r16, dhi, id2b, acc_in);
            mma_f16_lo(acc2 + 2 * P.BD2, hd + 3 * pl16, wd + 3 * w2r16, dhi, id2b, 1u);
          }
          mma_commit(&hempty[b]);
          if (s == nS - 1) mma_commit(&a2full[a]);
          if (kStream) mma_commit(&wsempty[wsl]);  // the slice's weights are consumed
        }
        __syncwarp();
      };
      // fc1 runs one slice ahead of fc2, across tile boundaries, so the GELU of
      // slice gs overlaps the fc1 MMAs of slice gs + 1
      const int total = n_my * nS;
      if (total > 0) fc1(0);
      for (int gs = 0; gs < total; ++gs) {
        if (gs + 1 < total) fc1(gs + 1);
        fc2(gs);
      }
      // all MMAs (and hence all loads they consumed) complete before exit
      if (elect_one()) mma_commit(final_bar);
      __syncwarp();
      mbar_wait(final_bar, 0);
    }
  } else if (warp < 6) {
    // ---------------------------------------------------------- transform
    const int r = threadIdx.x - 64;  // token row of the tile
    int xb = 0;
    uint32_t xph = 0;
    for (int m = blockIdx.x; m < p.nM; m += gridDim.x) {
      if (ok) ok = mbar_wait(&xfull[xb], xph);
      uint8_t *xt = smem + L.x0 + xb * L.xtile;
      for (int kc = 0; kc < P.nK1; ++kc) {
        uint8_t *st = xt + kc * kMlpChunkBytes;
        uint4 raw[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          raw[q] = *reinterpret_cast<const uint4 *>(st + r * 128 + ((q ^ (r & 7)) << 4));
        uint32_t pl[4][8];  // [plane][channel pair]: V0, V2, Re V1, -Im V1
#pragma unroll
        for (int q = 0; q < 8; ++q) rdft4_pair_q(raw[q], pl[0][q], pl[1][q], pl[2][q], pl[3][q]);
        named_bar_sync(2, 128);  // every row read before the planes overwrite it
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          uint8_t *plane = st + pp * kMlpPlaneBytes + r * 32;
#pragma unroll
          for (int h = 0; h < 2; ++h)
            *reinterpret_cast<uint4 *>(plane + (((h ^ (r >> 2)) & 1) << 4)) =
                make_uint4(pl[pp][4 * h + 0], pl[pp][4 * h + 1], pl[pp][4 * h + 2],
                           pl[pp][4 * h + 3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&xready[xb]);
      if (++xb == p.nx) { xb = 0; xph ^= 1; }
    }
  } else if (warp < kMlpEpiWarp0) {
    // --------------------------------------------------------------- GELU
    // All GELU warps take every hidden slice gs (fc1 accumulator and hidden
    // buffer gs % 2): warp quadrant q = warp % 4 reads TMEM lanes 32q..32q+31,
    // i.e. token rows row = 32q + lane, and the kMlpGeluParts warps of a
    // quadrant take every kMlpGeluParts-th 8-channel group of the slice.
    const int part = (warp - 6) / 4;
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int groups = hs / 8;  // 8 hidden channels per step
    // this warp's last group (-1: none; it still arrives on both barriers)
    const int c8_last =
        part < groups ? part + (groups - 1 - part) / kMlpGeluParts * kMlpGeluParts : -1;
    int g = 0;
    for (int m = blockIdx.x; m < p.nM; m += gridDim.x, g += nS) {
      for (int s = 0; s < nS; ++s) {
        const int gs = g + s, b = gs & 1;
        const uint32_t bph = (gs >> 1) & 1;
        if (ok) ok = mbar_wait(&a1full[b], bph);
        if (ok) ok = mbar_wait(&hempty[b], bph ^ 1);
        tc_fence_after();
        const uint32_t tl = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * 4 * hs;
        uint8_t *hb = smem + L.h0 + b * L.htile + row * 32;
        const uint32_t *bias = sb1 + s * hs / 2;
        if (c8_last < 0) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0 && ok) mbar_arrive(&a1empty[b]);
        }
        for (int c8 = part; c8 < groups; c8 += kMlpGeluParts) {
          uint32_t y0[8], y2[8], yr[8], yi[8];
          __syncwarp();
          tmem_ld8(tl + c8 * 8, y0);
          tmem_ld8(tl + hs + c8 * 8, y2);
          tmem_ld8(tl + 2 * hs + c8 * 8, yr);
          tmem_ld8(tl + 3 * hs + c8 * 8, yi);
          tmem_ld_wait();
          if (c8 == c8_last) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && ok) mbar_arrive(&a1empty[b]);
          }
          // Per channel pair (c, c+1), packed as fp16 pairs: an eighth of the
          // group values, v_t = h_t / 8 (inverse rDFT + b1 / 8, the scales
          // folded into the weights and x's planes), GELU / 4, and the rDFT of
          // those, whose four bins are fc2's operand planes (a quarter of the
          // activations' bins; channel pairs are the planes' word layout).
          uint32_t pl[4][4];
#pragma unroll
          for (int i2 = 0; i2 < 4; ++i2) {
            const __half2 a0 = as_h2(pack_half2(__uint_as_float(y0[2 * i2]), __uint_as_float(y0[2 * i2 + 1])));
            const __half2 a2 = as_h2(pack_half2(__uint_as_float(y2[2 * i2]), __uint_as_float(y2[2 * i2 + 1])));
            const __half2 ar = as_h2(pack_half2(__uint_as_float(yr[2 * i2]), __uint_as_float(yr[2 * i2 + 1])));
            const __half2 ai = as_h2(pack_half2(__uint_as_float(yi[2 * i2]), __uint_as_float(yi[2 * i2 + 1])));
            const __half2 pb = __hadd2(a0, as_h2(bias[c8 * 4 + i2]));
            const __half2 e = __hadd2(pb, a2), o = __hsub2(pb, a2);
            const __half2 g0 = as_h2(gelu_eighth_arg_h2(as_u32(__hadd2(e, ar))));
            const __half2 g1 = as_h2(gelu_eighth_arg_h2(as_u32(__hsub2(o, ai))));
            const __half2 g2 = as_h2(gelu_eighth_arg_h2(as_u32(__hsub2(e, ar))));
            const __half2 g3 = as_h2(gelu_eighth_arg_h2(as_u32(__hadd2(o, ai))));
            const __half2 s02 = __hadd2(g0, g2), s13 = __hadd2(g1, g3);
            pl[0][i2] = as_u32(__hadd2(s02, s13));   // V0
            pl[1][i2] = as_u32(__hsub2(s02, s13));   // V2
            pl[2][i2] = as_u32(__hsub2(g0, g2));     // Re V1
            pl[3][i2] = as_u32(__hsub2(g1, g3));     // -Im V1
          }
          uint8_t *dst = hb + (c8 >> 1) * kMlpChunkBytes + ((((c8 & 1) ^ (row >> 2)) & 1) << 4);
#pragma unroll
          for (int pp = 0; pp < 4; ++pp)
            *reinterpret_cast<uint4 *>(dst + pp * kMlpPlaneBytes) =
                make_uint4(pl[pp][0], pl[pp][1], pl[pp][2], pl[pp][3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&hready[b]);
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int ew = warp - kMlpEpiWarp0;
    uint8_t *obase = smem + L.y0 + ew * kMlpYBoxes * 4096;
    const int groups = P.BD2 / 16;
    int oi = 0, it = 0;
    for (int m = blockIdx.x; m < p.nM; m += gridDim.x, ++it) {
      const int a = it % nacc2;
      if (ok) ok = mbar_wait(&a2full[a], (it / nacc2) & 1);
      tc_fence_after();
      const uint32_t tl =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc2_col + a * 4 * P.BD2;
      for (int grp = 0; grp < groups; ++grp) {
        const int d0 = grp * 16;
        uint32_t packed[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t y0[8], y2[8], yr[8], yi[8];
          const uint32_t col = tl + d0 + h * 8;
          __syncwarp();
          tmem_ld8(col, y0);
          tmem_ld8(col + P.BD2, y2);
          tmem_ld8(col + 2 * P.BD2, yr);
          tmem_ld8(col + 3 * P.BD2, yi);
          tmem_ld_wait();
          if (h == 1 && grp == groups - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && ok) mbar_arrive(&a2empty[a]);
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float Y0 = __uint_as_float(y0[i]), Y2 = __uint_as_float(y2[i]);
            const float Yr = __uint_as_float(yr[i]), Yi = __uint_as_float(yi[i]);
            const float bv = sb2[d0 + h * 8 + i];
            // the planes and fc2's weights each carry 1/4: the inverse's 1/4 and 1/2 times 16
            const float e = fmaf(4.f, Y0 + Y2, bv), o = fmaf(4.f, Y0 - Y2, bv);
            packed[16 * h + 2 * i] = pack_half2(fmaf(8.f, Yr, e), fmaf(-8.f, Yi, o));
            packed[16 * h + 2 * i + 1] = pack_half2(fmaf(-8.f, Yr, e), fmaf(8.f, Yi, o));
          }
        }
        if (d0 >= P.Co) continue;  // whole group is padding
        uint8_t *ob = obase + (oi % kMlpYBoxes) * 4096;
        if (lane == 0) bulk_wait_read<kMlpYBoxes - 1>();  // this box's last store has read it
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k)
          *reinterpret_cast<uint4 *>(ob + lane * 128 + ((k ^ (lane & 7)) << 4)) =
              make_uint4(packed[4 * k], packed[4 * k + 1], packed[4 * k + 2], packed[4 * k + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_out, d0 * kT, m * kBM + q * 32, ob);
          bulk_commit();
        }
        ++oi;
      }
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

}  // namespace feql
