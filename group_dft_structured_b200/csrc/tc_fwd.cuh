// tc_fwd.cuh — fused forward / dX kernel on the sm_100a tensor cores (fp16).
//
// Flash EQ-Linear (technical summary "Approccio Algoritmico",
// "Specializzazione per il Gruppo di Rotazione p4", "Implementazione"):
//   out[n, :, :] = irDFT_4( per-bin  X_k[n, :] . What_k^T ) (+ bias)
// with X = rDFT_4(in) along the group axis.  Bins 0 and 2 are real
// contractions, bin 1 is one complex contraction; the Fourier tiles live only
// in shared memory / tensor memory (no intermediate global writes).
//
// One persistent CTA per SM, warp-specialised (640 threads, warps 5 and 9 idle):
//   warp 0       TMA producer: input chunks [128 tokens x 16 channels x 4] into
//                a ring of `stages` slots; the weight chunks either ride along
//                in each slot or, when the CTA's whole weight slice fits, are
//                loaded once into a resident buffer
//   warp 1       TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2-4, 6-8, 10, 11
//                transform, two 4-warp teams taking alternate chunks: 4-point
//                rDFT of the chunk (packed fp16 pairs), in place, into four
//                K-major operand planes (X0, X2, Re X1, -Im X1), each divided
//                by 4 so that any finite fp16 input has finite bins
//   warps 12..19 epilogue, two 4-warp teams: tcgen05.ld of the four fp32
//                accumulators, inverse rDFT + bias, fp16 pack, direct 16-byte
//                global stores (each four lanes write one token row's 64
//                contiguous bytes of an 8-channel block)
// Per chunk the MMA warp issues four M=128 x K=16 MMAs:
//   acc[0, BD)    += X0  * What0^T                (N = BD)
//   acc[BD, 2BD)  += X2  * What2^T                (N = BD)
//   acc[2BD, 4BD) += ReX1 * (Re1 ; Im1)^T + (-ImX1) * (Im1 ; -Re1)^T   (N = 2 BD)
// (the weight chunk stores What0, What2, Re1, Im1, -Re1; the two N = 2 BD
// operands are overlapping windows of its last three planes)
// so columns [2BD, 3BD) hold Re Y1 and [3BD, 4BD) hold Im Y1.  When 4*BD <= 256
// the accumulators are double-buffered in TMEM so the epilogue of one tile
// overlaps the MMAs of the next.
// Every wait is bounded (mbar_wait); a timed-out thread stops issuing work but
// keeps the loop structure so named barriers stay matched.
#pragma once

#include <cuda_fp16.h>

#include "plan.cuh"
#include "rdft4.cuh"
#include "sm100.cuh"

namespace feql {

constexpr int kTeams = 2;                         // transform teams and epilogue teams

// Failure-detection test builds (FEQL_TEST_SKIP_FIRST_RELEASE, compiled into a
// separate library with a short FEQL_WAIT_LIMIT_NS) leave out one arrive: the
// first epilogue warp never releases the first accumulator it drains.  The MMA
// thread's bounded wait for that buffer then runs out, the kernel winds down
// (every role stops waiting once its own wait has run out; loads already
// issued are still awaited, TMEM is freed) and FEQL_ERR_TIMEOUT is reported.
#ifdef FEQL_TEST_SKIP_FIRST_RELEASE
constexpr bool kSkipFirstRelease = true;
#else
constexpr bool kSkipFirstRelease = false;
#endif
// Warp w runs on SM sub-partition w % 4.  Sub-partition 1 holds the MMA issuer
// (warp 1), so warps 5 and 9 stay idle and the transform warps sit on the other
// three sub-partitions: warps 2-4, 6-8, 10-11 transform, 12-19 epilogue.
constexpr int kTcWarps = 20;
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kTcEpi0 = 12;                       // first epilogue warp

// Transform ordinal (0..4*kTeams-1) of warp w, or -1 when w is not a transform warp.
__device__ __forceinline__ int tc_xf_ordinal(int w) {
  if (w < 2 || w >= kTcEpi0 || w == 5 || w == 9) return -1;
  return w - 2 - (w > 5) - (w > 9);
}
constexpr int kXChunkBytes = kBM * kCK * kT * 2;  // 16 KB: 128 rows x 128 B
constexpr int kPlaneBytes = kBM * kCK * 2;        // 4 KB: 128 rows x 32 B
constexpr int kTmemCols = 512;

struct TcFwdParams {
  const uint8_t *wt;    // weight chunks of this direction
  const void *bias;     // [Do] (fp16, or fp32 in split-TF32 mode) or nullptr
  int64_t N;
  int Ci, Do, BD, nD, nK, chunk_bytes;
  int nM;               // token tiles: ceil(N / 128)
  int n_units;          // nM * nD
  int nacc, acc_stride; // accumulator buffers in TMEM and their column stride
  int resident;         // 1: the CTA's weight slice is loaded once (fixed D tile per CTA)
  int wres_bytes;       // resident weight buffer: nK * chunk_bytes (1 KB aligned)
  int stages;
  int stage_bytes;      // input chunk slot (16 KB; 32 KB of planes in split-TF32 mode)
                        // + weight chunk unless resident, 1 KB aligned
  int bias_floats;      // nD * BD
  void *out;            // [N][Do][4], fp16 (fp32 in split-TF32 mode)
};

struct TcSmem {
  // offsets (bytes) from the 1024-aligned dynamic smem base
  int wres, stage0, bias, bars, total;
};

__host__ __device__ inline TcSmem tc_fwd_smem(const TcFwdParams &p) {
  TcSmem s;
  s.wres = 0;
  s.stage0 = p.resident ? p.wres_bytes : 0;
  s.bias = s.stage0 + p.stages * p.stage_bytes;
  s.bars = s.bias + static_cast<int>(align_up(p.bias_floats * 4, 16));
  // full, tready, empty per stage; acc_full, acc_empty per acc buffer; final; wfull; tmem slot
  s.total = s.bars + (3 * p.stages + 2 * 2 + 2) * 8 + 16;
  return s;
}

// The work units of this CTA in order: token tile m and output-channel tile j.
// With resident weights every CTA keeps one j (neighbouring CTAs share a token
// tile, so its second read comes from L2); otherwise units are dealt
// round-robin.  The divisions happen once: the issuing threads share their SM
// sub-partition with busy warps, so a per-unit division chain (several hundred
// cycles there) would stall the tensor pipe.
struct TcUnits {
  int m, j;
  int dm, dj, nD, nM;
  bool valid;
  __device__ __forceinline__ explicit TcUnits(const TcFwdParams &p) : nD(p.nD), nM(p.nM) {
    m = static_cast<int>(blockIdx.x) / p.nD;
    j = static_cast<int>(blockIdx.x) % p.nD;
    if (p.resident) {
      const int g = static_cast<int>(gridDim.x) / p.nD;
      dm = g;
      dj = 0;
      valid = static_cast<int>(blockIdx.x) < g * p.nD && m < nM;
    } else {
      dm = static_cast<int>(gridDim.x) / p.nD;
      dj = static_cast<int>(gridDim.x) % p.nD;
      valid = m < nM;
    }
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

// 20 warps over the 4 SM sub-partitions put 5 warps on each 16K-register
// slice: 5 x 32 x 96 = 15,360 registers fits, 104 would not.
//
// kTF32: the split-TF32 mode of fp32 data (FEQL_FP32_3XTF32).  A chunk is 8
// channels (the same 16 KB TMA box: 128 rows x 128 bytes of fp32), transformed
// in fp32 into eight 4 KB planes (the four bins rounded to tf32, hi, and the
// tf32-rounded remainders, lo) that overwrite the 32 KB slot; per chunk the
// MMA thread issues three kind::tf32 MMAs (K = 8) per bin product,
// A_hi B_hi + A_hi B_lo + A_lo B_hi (the lo x lo term, ~2^-22 of the product,
// is dropped: Ootomo and Yokota's split-TF32 scheme), and the epilogue stores
// fp32 rows.  Bins are not scaled (fp32 has the range).
template <bool kTF32>
__global__ void __maxnreg__(96)
tc_fourier_gemm_kernel(const __grid_constant__ CUtensorMap tm_in, const TcFwdParams p) {
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
  uint64_t *wfull = final_bar + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(wfull + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&tready[s], 4);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], p.nacc == 1 ? 4 * kTeams : 4);  // single buffer: all teams release
    }
    mbar_init(final_bar, 1);
    mbar_init(wfull, 1);
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < p.bias_floats; i += blockDim.x) {
    float bv = 0.f;
    if (p.bias != nullptr && i < p.Do)
      bv = kTF32 ? static_cast<const float *>(p.bias)[i]
                 : __half2float(static_cast<const __half *>(p.bias)[i]);
    sbias[i] = bv;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
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
      TcUnits U(p);
      if (p.resident && U.valid) {
        mbar_arrive_expect_tx(wfull, p.nK * p.chunk_bytes);
        bulk_load(smem + L.wres, p.wt + static_cast<int64_t>(U.j) * p.nK * p.chunk_bytes,
                  p.nK * p.chunk_bytes, wfull);
      }
      int s = 0;
      uint32_t ph = 0;
      for (; U.valid; U.next()) {
        const int m = U.m, j = U.j;
        for (int kc = 0; kc < p.nK; ++kc) {
          if (ok) ok = mbar_wait(&empty[s], ph ^ 1);
          if (ok) {
            uint8_t *st = smem + L.stage0 + s * p.stage_bytes;
            if (p.resident) {
              mbar_arrive_expect_tx(&full[s], kXChunkBytes);
              tma_load_2d(st, &tm_in, kc * (kTF32 ? kCK32 * kT : kCK * kT), m * kBM, &full[s]);
            } else {
              mbar_arrive_expect_tx(&full[s], kXChunkBytes + p.chunk_bytes);
              tma_load_2d(st, &tm_in, kc * (kTF32 ? kCK32 * kT : kCK * kT), m * kBM, &full[s]);
              bulk_load(st + (kTF32 ? 2 * kXChunkBytes : kXChunkBytes),
                        p.wt + (static_cast<int64_t>(j) * p.nK + kc) * p.chunk_bytes,
                        p.chunk_bytes, &full[s]);
            }
          }
          if (++s == p.stages) { s = 0; ph ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t fmt = kTF32 ? 2u : 0u;  // operand format: tf32 or f16
      const uint32_t id_bd = instr_desc(kBM, p.BD, fmt, fmt);
      const uint32_t id_2bd = instr_desc(kBM, 2 * p.BD, fmt, fmt);
      const uint32_t wrow = 32;  // bytes per weight row (16 fp16)
      const uint64_t dsw32 = smem_desc(0, 16, 256, kSw32);  // K-major, 32-byte swizzle
      const uint32_t stage_base = smem_u32(smem + L.stage0), wres_base = smem_u32(smem + L.wres);
      TcUnits U(p);
      if (p.resident && U.valid) ok = mbar_wait(wfull, 0);
      int s = 0;
      uint32_t ph = 0;
      // every operand is the low descriptor word of a chunk's base plus a 16-byte-unit
      // offset; the high word is common
      const uint32_t dhi = desc_hi(dsw32);
      const uint32_t pl16 = kPlaneBytes >> 4, w16 = (p.BD * wrow) >> 4;
      const uint32_t stage16 = p.stage_bytes >> 4, chunk16 = p.chunk_bytes >> 4;
      const uint32_t x0 = desc_lo(desc_at(dsw32, stage_base));
      const uint32_t wr0 = desc_lo(desc_at(dsw32, wres_base));
      int a = 0;        // accumulator buffer of this unit
      uint32_t aph = 0;  // its phase
      for (; U.valid; U.next()) {
        if (ok) ok = mbar_wait(&acc_empty[a], aph ^ 1);
        tc_fence_after();
        const uint32_t acc = tmem_base + a * p.acc_stride;
        uint32_t wr = wr0;
        for (int kc = 0; kc < p.nK; ++kc, wr += chunk16) {
          // tready implies full: every transform thread waited for the slot's
          // TMA bytes before its release-arrive, so one acquire covers both
          if (ok) ok = mbar_wait(&tready[s], ph);
          tc_fence_after();
          if (ok) {
            const uint32_t xd = x0 + s * stage16;
            const uint32_t wd =
                p.resident ? wr : xd + ((kTF32 ? 2 * kXChunkBytes : kXChunkBytes) >> 4);
            const uint32_t acc_in = kc > 0 ? 1u : 0u;
            if constexpr (kTF32) {
              // planes 0..3 hi, 4..7 lo; the lo weight tile 5 BD rows after the hi one
              const uint32_t lo_x = 4 * pl16, lo_w = 5 * w16;
#pragma unroll
              for (int b = 0; b < 4; ++b) {
                const uint32_t dcol = acc + (b < 2 ? b : 2) * p.BD;
                const uint32_t id = b < 2 ? id_bd : id_2bd;
                const uint32_t in = (b == 3) ? 1u : acc_in;  // window b adds onto window a
                mma_tf32_lo(dcol, xd + b * pl16, wd + b * w16, dhi, id, in);
                mma_tf32_lo(dcol, xd + b * pl16, wd + b * w16 + lo_w, dhi, id, 1u);
                mma_tf32_lo(dcol, xd + b * pl16 + lo_x, wd + b * w16, dhi, id, 1u);
              }
            } else {
              mma_f16_lo(acc, xd, wd, dhi, id_bd, acc_in);
              mma_f16_lo(acc + p.BD, xd + pl16, wd + w16, dhi, id_bd, acc_in);
              mma_f16_lo(acc + 2 * p.BD, xd + 2 * pl16, wd + 2 * w16, dhi, id_2bd, acc_in);
              mma_f16_lo(acc + 2 * p.BD, xd + 3 * pl16, wd + 3 * w16, dhi, id_2bd, 1u);
            }
            mma_commit(&empty[s]);
          }
          if (++s == p.stages) { s = 0; ph ^= 1; }
        }
        if (ok) mma_commit(&acc_full[a]);
        if (++a == p.nacc) { a = 0; aph ^= 1; }
      }
      // all MMAs (and hence all loads they consumed) complete before exit
      mma_commit(final_bar);
      mbar_wait(final_bar, 0);
    }
  } else if (tc_xf_ordinal(warp) >= 0) {
    // ---------------------------------------------------------- transform
    // kTeams teams of 4 warps take alternate chunks of the ring.
    const int xo = tc_xf_ordinal(warp);
    const int team = xo / 4;
    const int r = (xo % 4) * 32 + lane;  // row of the chunk (token within the tile)
    int s = 0, c = 0;
    uint32_t ph = 0;
    for (TcUnits U(p); U.valid; U.next()) {
      for (int kc = 0; kc < p.nK; ++kc, ++c) {
        if (c % kTeams != team) {
          if (++s == p.stages) { s = 0; ph ^= 1; }
          continue;
        }
        if (ok) ok = mbar_wait(&full[s], ph);
        uint8_t *st = smem + L.stage0 + s * p.stage_bytes;
        // row r: 8 x 16 B; fp16: logical chunk q = channels 2q, 2q+1 (x 4 group
        // elements); fp32: chunk q = channel q's four group elements
        uint4 raw[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          raw[q] = *reinterpret_cast<const uint4 *>(st + r * 128 + ((q ^ (r & 7)) << 4));
        if constexpr (kTF32) {
          named_bar_sync(2 + team, 128);  // every row read before the planes overwrite it
          // per half row (channels 4h..4h+3): the four bins in fp32, each split into
          // its tf32 rounding (planes 0..3) and the rounded remainder (planes 4..7)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t pl[8][4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 u = raw[4 * h + q];
              const float v0 = __uint_as_float(u.x), v1 = __uint_as_float(u.y);
              const float v2 = __uint_as_float(u.z), v3 = __uint_as_float(u.w);
              const float a = v0 + v2, b = v1 + v3;
              const float bins[4] = {a + b, a - b, v0 - v2, v1 - v3};  // V0, V2, Re V1, -Im V1
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                pl[k][q] = tf32_rna(bins[k]);
                pl[4 + k][q] = tf32_rna(bins[k] - __uint_as_float(pl[k][q]));
              }
            }
#pragma unroll
            for (int pp = 0; pp < 8; ++pp)
              *reinterpret_cast<uint4 *>(st + pp * kPlaneBytes + r * 32 +
                                         (((h ^ (r >> 2)) & 1) << 4)) =
                  make_uint4(pl[pp][0], pl[pp][1], pl[pp][2], pl[pp][3]);
          }
        } else {
          uint32_t pl[4][8];  // [plane][channel pair] packed half2: V0, V2, Re V1, -Im V1
#pragma unroll
          for (int q = 0; q < 8; ++q) rdft4_pair_q(raw[q], pl[0][q], pl[1][q], pl[2][q], pl[3][q]);
          named_bar_sync(2 + team, 128);  // every row read before the planes overwrite it
#pragma unroll
          for (int pp = 0; pp < 4; ++pp) {
            uint8_t *plane = st + pp * kPlaneBytes + r * 32;
#pragma unroll
            for (int h = 0; h < 2; ++h)
              *reinterpret_cast<uint4 *>(plane + (((h ^ (r >> 2)) & 1) << 4)) =
                  make_uint4(pl[pp][4 * h + 0], pl[pp][4 * h + 1], pl[pp][4 * h + 2],
                             pl[pp][4 * h + 3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&tready[s]);
        if (++s == p.stages) { s = 0; ph ^= 1; }
      }
    }
  } else if (warp >= kTcEpi0) {
    // ----------------------------------------------------------- epilogue
    // kTeams teams of 4 warps.  With double-buffered accumulators each team
    // owns one TMEM buffer (alternate tiles); with a single buffer the teams
    // split each tile's 16-column groups.  Each warp owns one TMEM lane
    // quadrant (32 token rows).  It reads them with 16x256b loads (four lanes
    // per token row, two channels each) and stores each row's 64-byte channel
    // blocks straight to global memory: every store instruction writes 8 rows
    // x 64 contiguous bytes, and no shared memory goes to output staging.
    const int ew = warp - kTcEpi0;           // epilogue warp index
    const int eteam = ew / 4;
    const int quad = warp & 3;              // TMEM lane quadrant this warp may access
    const int groups = p.BD / 16;
    const bool split = p.nacc == 1;
    const int g0 = split ? eteam : 0, gstep = split ? kTeams : 1;
    int last_g = -1;
    for (int g = g0; g < groups; g += gstep) last_g = g;
    int it = 0;
    for (TcUnits U(p); U.valid; U.next(), ++it) {
      const int m = U.m, j = U.j;
      if (!split && it % kTeams != eteam) continue;
      // accumulator buffer and phase of unit `it` (nacc is 1 or 2)
      const int a = p.nacc == 2 ? (it & 1) : 0;
      const uint32_t aph = (p.nacc == 2 ? it >> 1 : it) & 1;
      if (ok) ok = mbar_wait(&acc_full[a], aph);
      tc_fence_after();
      if (last_g < 0) {  // this team reads nothing of the tile
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&acc_empty[a]);
      }
      const uint32_t tl = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + a * p.acc_stride;
      // thread t: rows r0 = 32 quad + 16 half + t/4 (and r0 + 8), channels
      // c + 2(t%4) and c + 2(t%4) + 1 of each 8-channel block c
      const int tcp = 2 * (lane & 3);
      const int64_t row0 = static_cast<int64_t>(m) * kBM + quad * 32 + (lane >> 2);
      const int64_t row_elems = static_cast<int64_t>(p.Do) * kT;
      for (int g = g0; g < groups; g += gstep) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int c = g * 16 + h * 8;
          uint32_t y0[2][4], y2[2][4], yr[2][4], yi[2][4];
          __syncwarp();  // the TMEM loads are warp-collective
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const uint32_t col = tl + (static_cast<uint32_t>(16 * hf) << 16) + c;
            tmem_ld16x256(col, y0[hf]);
            tmem_ld16x256(col + p.BD, y2[hf]);
            tmem_ld16x256(col + 2 * p.BD, yr[hf]);
            tmem_ld16x256(col + 3 * p.BD, yi[hf]);
          }
          tmem_ld_wait();
          if (h == 1 && g == last_g) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && ok && !(kSkipFirstRelease && ew == 0 && it == 0))
              mbar_arrive(&acc_empty[a]);
          }
          const int d = j * p.BD + c + tcp;  // this thread's first output channel
          if constexpr (kTF32) {
            // fp32 rows: channel d and d + 1 (each checked: Do may be odd), 16 bytes each
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
              for (int rr = 0; rr < 2; ++rr) {
                const int64_t row = row0 + 16 * hf + 8 * rr;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                  const int i = 2 * rr + cc;
                  const float Y0 = __uint_as_float(y0[hf][i]), Y2 = __uint_as_float(y2[hf][i]);
                  const float Yr = __uint_as_float(yr[hf][i]), Yi = __uint_as_float(yi[hf][i]);
                  const float bv = d + cc < p.Do ? sbias[d + cc] : 0.f;
                  const float e = fmaf(0.25f, Y0 + Y2, bv), o = fmaf(0.25f, Y0 - Y2, bv);
                  if (row < p.N && d + cc < p.Do)
                    *reinterpret_cast<float4 *>(static_cast<float *>(p.out) + row * row_elems +
                                                static_cast<int64_t>(d + cc) * kT) =
                        make_float4(fmaf(0.5f, Yr, e), fmaf(-0.5f, Yi, o), fmaf(-0.5f, Yr, e),
                                    fmaf(0.5f, Yi, o));
                }
              }
            }
            continue;
          }
          if (d + 2 > p.Do) continue;        // Do is even: the pair is whole or padding
          const float b0 = sbias[d], b1 = sbias[d + 1];
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {  // rows r0 and r0 + 8
              uint32_t w[4];
#pragma unroll
              for (int cc = 0; cc < 2; ++cc) {
                const int i = 2 * rr + cc;
                const float Y0 = __uint_as_float(y0[hf][i]), Y2 = __uint_as_float(y2[hf][i]);
                const float Yr = __uint_as_float(yr[hf][i]), Yi = __uint_as_float(yi[hf][i]);
                const float bv = cc ? b1 : b0;
                // planes and weights are both stored divided by 4 (Y = 16 * acc)
                const float e = fmaf(4.f, Y0 + Y2, bv), o = fmaf(4.f, Y0 - Y2, bv);
                w[2 * cc] = pack_half2(fmaf(8.f, Yr, e), fmaf(-8.f, Yi, o));
                w[2 * cc + 1] = pack_half2(fmaf(-8.f, Yr, e), fmaf(8.f, Yi, o));
              }
              const int64_t row = row0 + 16 * hf + 8 * rr;
              if (row < p.N)
                *reinterpret_cast<uint4 *>(static_cast<__half *>(p.out) + row * row_elems +
                                           static_cast<int64_t>(d) * kT) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace feql
