// tc_dw.cuh — weight gradient on the sm_100a tensor cores (fp16 data).
//
// The loss <dy, y> has dW[d,c,u] = sum_n sum_t dy[n,d,t] x[n,c,(t-u) mod 4], a
// circular cross-correlation along the group axis, so per frequency bin
// (convolution theorem, Flash EQ-Linear technical summary "Approccio
// Algoritmico"):
//   G_k[d,c] = sum_n dY_k[n,d] conj(X_k[n,c])
//   G0 = sum dY0 X0,  G2 = sum dY2 X2,
//   Re G1 = sum dY1r X1r + dY1i X1i,  Im G1 = sum dY1i X1r - dY1r X1i
// — six real N-contractions — and dW = irDFT_4(G) (applied by the reduce).
// db[d] = sum_n dY0[n,d] comes out of the same rDFT.
//
// Work unit (one per CTA): a 128-row d tile x a CT-column c tile x a token
// split.  Per chunk of TB tokens:
//   warp 0      TMA: the d-tile's dy boxes and the c-tile's x boxes (16
//               channels x 4 group elements x TB tokens each) into a raw ring
//   warps 2..9  4-point rDFT (packed fp16 pairs) of every (token, channel)
//               fibre into planes X0, X2, Re X1, -Im X1 (each divided by 4,
//               as in tc_fwd.cuh) laid out MN-major
//               (channel contiguous, token = K), 32-byte swizzle; one
//               (16-channel box, token) item per thread; db partial sums
//   warp 1      TMEM allocator + MMA issuer: per 16 tokens six M=128 x N=CT
//               MMAs, one of them through the B-negate bit
// After the last chunk warps 2..9 read the four fp32 accumulators out of
// TMEM and write them to the workspace; the split reduce (below: a scalar
// kernel for small outputs, a vectorised one for large) sums the splits in a
// fixed order (bit-identical run to run) and applies the inverse rDFT.
// TMA: one 2-D load per 16-channel box, or with 16-token chunks one 3-D
// "box stack" load per operand (see make_tmap_f16_boxes).
#pragma once

#include <cuda_fp16.h>

#include "plan.cuh"
#include "rdft4.cuh"
#include "sm100.cuh"

namespace feql {

constexpr int kDwXfWarps = 8;     // transform (then epilogue) warps
constexpr int kDwThreads = 64 + kDwXfWarps * 32;
constexpr int kDwMT = 128;       // d rows per tile (MMA M)
constexpr int kDwMaxCT = 128;    // c columns per tile (MMA N; 4 accumulators <= 512 TMEM cols)
constexpr int kDwItems = kDwXfWarps * 32;  // (box, token) items per chunk: nbox * TB

struct TcDwParams {
  int64_t N;
  int C, D, Cs;          // Cs: workspace row stride (C rounded up to 16)
  int CT;                // c columns per tile
  int nqd_max, nqc_max;  // 16-channel boxes per tile (dy, x) in the plane layout
  int tiles_d, tiles_c, splits;
  int64_t split_len;     // tokens per split (multiple of TB)
  int TB;                // tokens per chunk
  int stages;            // raw ring depth
  int raw_bytes;         // (nqd_max + nqc_max) * TB * 128
  int plane_bytes;       // 4 * (8 + nqc_max) * TB * 32
  int tmem_cols;
  int merged;            // 1: bin-1 products as two N = 2*CT MMAs (needs 6*CT TMEM columns)
  int stack_dy, stack_x; // 1: the tensor map loads all of a tile's boxes at once (3-D box stack)
  float *ws;             // [splits][4][D][Cs]
  float *ws_db;          // [splits][D]
};

struct DwSmem {
  int raw0, plane0, bars, total;
};

// This thread's TMEM row of the dW accumulators, 8 columns from c0, as the four
// bins (G0, G2, Re G1, Im G1).  Column layout: [0,CT) G0, [CT,2CT) G2, then
// either Re G1, Im G1 (CT each) or, merged, acc_a and acc_b (2*CT each) with
// Re G1 = a[c] + b[CT+c] and Im G1 = a[CT+c] - b[c].  Whole warp: the TMEM
// loads are warp-collective (.sync.aligned), so the warp reconverges first.
__device__ __forceinline__ void dw_acc_read8(uint32_t tl, int CT, int c0, bool merged,
                                             float (&G)[4][8]) {
  uint32_t v0[8], v2[8], r0[8], r1[8];
  __syncwarp();
  tmem_ld8(tl + c0, v0);
  tmem_ld8(tl + CT + c0, v2);
  tmem_ld8(tl + 2 * CT + c0, r0);
  tmem_ld8(tl + 3 * CT + c0, r1);
  if (merged) {
    uint32_t b0[8], b1[8];
    tmem_ld8(tl + 4 * CT + c0, b0);
    tmem_ld8(tl + 5 * CT + c0, b1);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      G[2][i] = __uint_as_float(r0[i]) + __uint_as_float(b1[i]);
      G[3][i] = __uint_as_float(r1[i]) - __uint_as_float(b0[i]);
    }
  } else {
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      G[2][i] = __uint_as_float(r0[i]);
      G[3][i] = __uint_as_float(r1[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    G[0][i] = __uint_as_float(v0[i]);
    G[1][i] = __uint_as_float(v2[i]);
  }
}

__host__ __device__ inline DwSmem tc_dw_smem(const TcDwParams &p) {
  DwSmem s;
  s.raw0 = 0;
  s.plane0 = p.stages * p.raw_bytes;
  s.bars = s.plane0 + 2 * p.plane_bytes;
  s.total = s.bars + (2 * p.stages + 2 * 2 + 1) * 8 + 16;
  return s;
}

__global__ void __launch_bounds__(kDwThreads, 1)
tc_dw_kernel(const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_x,
             const TcDwParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const DwSmem L = tc_dw_smem(p);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
  uint64_t *full = bars;                 // raw slot landed (TMA tx)
  uint64_t *empty = bars + p.stages;     // raw slot read by the transform warps
  uint64_t *pfull = bars + 2 * p.stages; // plane buffer written by the transform warps
  uint64_t *pempty = pfull + 2;          // plane buffer consumed (MMA commit)
  uint64_t *acc_full = pempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int u = blockIdx.x;
  const int tiles = p.tiles_d * p.tiles_c;
  const int split = u / tiles, ti = (u % tiles) / p.tiles_c, tj = u % p.tiles_c;
  const int64_t t_begin = static_cast<int64_t>(split) * p.split_len;
  int64_t t_end = t_begin + p.split_len;
  if (t_end > p.N) t_end = p.N;
  const int nchunks = t_begin < t_end ? static_cast<int>(cdiv(t_end - t_begin, p.TB)) : 0;
  int nqd = static_cast<int>(cdiv(p.D - ti * kDwMT, 16));
  if (nqd > p.nqd_max) nqd = p.nqd_max;
  int nqc = static_cast<int>(cdiv(p.C - tj * p.CT, 16));
  if (nqc > p.nqc_max) nqc = p.nqc_max;
  const int nbox = nqd + nqc;
  const int chunk_plane = p.TB * 32;  // bytes of one 16-channel plane chunk
  const int x_off = 4 * 8 * chunk_plane;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDwXfWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&pfull[b], kDwXfWarps);
      mbar_init(&pempty[b], 1);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
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
      for (int ch = 0; ch < nchunks; ++ch) {
        if (ok) ok = mbar_wait(&empty[s], ph ^ 1);
        if (ok) {
          uint8_t *raw = smem + L.raw0 + s * p.raw_bytes;
          const int32_t row = static_cast<int32_t>(t_begin + static_cast<int64_t>(ch) * p.TB);
          uint8_t *rawx = raw + p.nqd_max * p.TB * 128;
          // a box stack always lands whole (boxes past the last channel read as zeros)
          const int bd = p.stack_dy ? p.nqd_max : nqd, bc = p.stack_x ? p.nqc_max : nqc;
          mbar_arrive_expect_tx(&full[s], (bd + bc) * p.TB * 128);
          if (p.stack_dy) {
            tma_load_3d(raw, &tm_dy, 0, row, ti * (kDwMT / 16), &full[s]);
          } else {
            for (int q = 0; q < nqd; ++q)
              tma_load_2d(raw + q * p.TB * 128, &tm_dy, (ti * kDwMT + q * 16) * kT, row, &full[s]);
          }
          if (p.stack_x) {
            tma_load_3d(rawx, &tm_x, 0, row, tj * (p.CT / 16), &full[s]);
          } else {
            for (int q = 0; q < nqc; ++q)
              tma_load_2d(rawx + q * p.TB * 128, &tm_x, (tj * p.CT + q * 16) * kT, row, &full[s]);
          }
        }
        if (++s == p.stages) { s = 0; ph ^= 1; }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    // The planes hold -Im of bin 1 (for dy and x alike), so
    //   Re G1 = dY1r X1r + (-dY1i)(-X1i),   Im G1 = -(-dY1i) X1r + dY1r (-X1i),
    // the first Im term through the B-negate bit.
    // Merged form (6*CT TMEM columns): the x planes Re X1 and -Im X1 are
    // adjacent, so one N = 2*CT MMA per dy plane gives both products:
    //   acc_a = [dY1r X1r | -dY1r X1i],  acc_b = [-dY1i X1r | dY1i X1i]
    // and the epilogue forms Re G1 = a0 + b1, Im G1 = a1 - b0 (4 MMAs, not 6).
    if (lane == 0) {
      const uint32_t id = instr_desc(kDwMT, p.CT, 0, 0, 1, 1);
      const uint32_t id_neg = instr_desc(kDwMT, p.CT, 0, 0, 1, 1, 1);
      const uint32_t id2 = instr_desc(kDwMT, 2 * p.CT, 0, 0, 1, 1);
      const uint64_t dmn = smem_desc(0, chunk_plane, 256, kSw32);  // MN-major planes
      const uint32_t dhi = desc_hi(dmn);
      const uint32_t acc0 = tmem_base, acc2 = tmem_base + p.CT;
      const uint32_t acc1r = tmem_base + 2 * p.CT, acc1i = tmem_base + 3 * p.CT;
      const uint32_t acca = tmem_base + 2 * p.CT, accb = tmem_base + 4 * p.CT;
      const uint32_t plane_base = smem_u32(smem + L.plane0);
      const uint32_t a_bin = 8 * chunk_plane, b_bin = p.nqc_max * chunk_plane;
      for (int ch = 0; ch < nchunks; ++ch) {
        const int pb = ch & 1;
        if (ok) ok = mbar_wait(&pfull[pb], (ch >> 1) & 1);
        tc_fence_after();
        if (ok) {
          const uint32_t pl = plane_base + pb * p.plane_bytes;
          // every operand is the low descriptor word of one of two bases plus a
          // 16-byte-unit offset; the high word is common
          const uint32_t ba = desc_lo(desc_at(dmn, pl)), bb = desc_lo(desc_at(dmn, pl + x_off));
          const uint32_t a16 = a_bin >> 4, b16 = b_bin >> 4;
          for (int k = 0; k < p.TB / 16; ++k) {
            const uint32_t A0 = ba + k * 32, A1 = A0 + a16;  // 16 tokens x 32 B = 512 B
            const uint32_t A2 = A1 + a16, A3 = A2 + a16;
            const uint32_t B0 = bb + k * 32, B1 = B0 + b16;
            const uint32_t B2 = B1 + b16, B3 = B2 + b16;
            const uint32_t first = (ch == 0 && k == 0) ? 0u : 1u;
            mma_f16_lo(acc0, A0, B0, dhi, id, first);
            mma_f16_lo(acc2, A1, B1, dhi, id, first);
            if (p.merged) {
              mma_f16_lo(acca, A2, B2, dhi, id2, first);
              mma_f16_lo(accb, A3, B2, dhi, id2, first);
            } else {
              mma_f16_lo(acc1r, A2, B2, dhi, id, first);
              mma_f16_lo(acc1r, A3, B3, dhi, id, 1u);
              mma_f16_lo(acc1i, A3, B2, dhi, id_neg, first);
              mma_f16_lo(acc1i, A2, B3, dhi, id, 1u);
            }
          }
          mma_commit(&pempty[pb]);
        }
      }
      mma_commit(acc_full);
    }
  } else {
    // ---------------------------------------------------------- transform
    // one (box, token) item per thread and chunk
    const int t = threadIdx.x - 64;
    const int b = t / p.TB, r = t % p.TB;
    const bool active = b < nbox;
    const bool is_dy = b < nqd;
    const bool do_db = tj == 0 && is_dy;
    float db_acc[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) db_acc[c] = 0.f;
    int s = 0;
    uint32_t ph = 0;
    for (int ch = 0; ch < nchunks; ++ch) {
      const int pb = ch & 1;
      if (ok) ok = mbar_wait(&full[s], ph);
      if (ok) ok = mbar_wait(&pempty[pb], ((ch >> 1) & 1) ^ 1);
      if (active) {
        // dy boxes from the start of the slot, x boxes after nqd_max dy boxes
        const int slot_box = is_dy ? b : p.nqd_max + (b - nqd);
        const uint8_t *src = smem + L.raw0 + s * p.raw_bytes + slot_box * p.TB * 128 + r * 128;
        uint8_t *planes = smem + L.plane0 + pb * p.plane_bytes;
        uint32_t pl[4][8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 v = *reinterpret_cast<const uint4 *>(src + ((q ^ (r & 7)) << 4));
          rdft4_pair_q(v, pl[0][q], pl[1][q], pl[2][q], pl[3][q]);
        }
        uint8_t *dst = is_dy ? planes + b * chunk_plane : planes + x_off + (b - nqd) * chunk_plane;
        const int pstride = is_dy ? 8 * chunk_plane : p.nqc_max * chunk_plane;
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          uint8_t *row = dst + pp * pstride + r * 32;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
            *reinterpret_cast<uint4 *>(row + (((hh ^ (r >> 2)) & 1) << 4)) =
                make_uint4(pl[pp][4 * hh + 0], pl[pp][4 * hh + 1], pl[pp][4 * hh + 2],
                           pl[pp][4 * hh + 3]);
        }
        if (do_db) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float2 f = __half22float2(as_h2(pl[0][q]));
            db_acc[2 * q] += f.x;
            db_acc[2 * q + 1] += f.y;
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && ok) {
        mbar_arrive(&empty[s]);
        mbar_arrive(&pfull[pb]);
      }
      if (++s == p.stages) { s = 0; ph ^= 1; }
    }

    // ------------------------------------------------------------ epilogue
    // two warps per TMEM lane quadrant, alternating 16-column groups
    if (ok) ok = mbar_wait(acc_full, 0);
    tc_fence_after();
    const int quad = warp & 3, half = (warp - 2) / 4;
    const int d = ti * kDwMT + quad * 32 + lane;
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    const int ncol = p.CT / 16;
    float *dst = p.ws + (static_cast<int64_t>(split) * 4 * p.D + d) * p.Cs +
                 static_cast<int64_t>(tj) * p.CT;
    const int64_t bin_stride = static_cast<int64_t>(p.D) * p.Cs;
    for (int g = half; g < 2 * ncol; g += 2) {  // 8-column steps
      float G[4][8];
      dw_acc_read8(tl, p.CT, g * 8, p.merged, G);
      if (d < p.D && tj * p.CT + g * 8 < p.C) {
#pragma unroll
        for (int bin = 0; bin < 4; ++bin) {
          float4 *o = reinterpret_cast<float4 *>(dst + bin * bin_stride + g * 8);
          o[0] = make_float4(G[bin][0], G[bin][1], G[bin][2], G[bin][3]);
          o[1] = make_float4(G[bin][4], G[bin][5], G[bin][6], G[bin][7]);
        }
      }
    }
    tc_fence_before();

    // db: fixed-order reduction of the per-thread partials through shared memory
    if (tj == 0) {
      named_bar_sync(3, kDwXfWarps * 32);  // raw ring is free: every chunk has been consumed
      float *sdb = reinterpret_cast<float *>(smem + L.raw0);  // [kDwItems][16]
#pragma unroll
      for (int c = 0; c < 16; ++c) sdb[t * 16 + c] = db_acc[c];
      named_bar_sync(3, kDwXfWarps * 32);
      if (t < nqd * 16) {
        const int bb = t / 16, c = t % 16;
        float sum = 0.f;
        for (int rr = 0; rr < p.TB; ++rr) sum += sdb[(bb * p.TB + rr) * 16 + c];
        const int dd = ti * kDwMT + bb * 16 + c;
        if (dd < p.D) p.ws_db[static_cast<int64_t>(split) * p.D + dd] = sum;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // the partial sums are written: the split reduce (launched as this grid's
  // programmatic dependent) may be scheduled as the CTAs exit
  if (threadIdx.x == 0) pdl_launch_dependents();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

// Small outputs (a few thousand (d, c) pairs, where the vector kernel below
// has too few blocks): a block takes 16 consecutive (d, c) outputs (the last
// blocks take db); its 32 thread groups each sum every 32nd split, then the
// first group adds the 32 partial sums in group order — the same grouping on
// every run.  Both reduce kernels may be launched as programmatic dependents
// of the kernel that writes the partials (pdl_wait before the first read).
constexpr int kRedOut = 16, kRedGroups = 32;
constexpr int64_t kRedScalarMaxOut = 8192;  // D * C up to which the scalar kernel runs

__global__ void __launch_bounds__(kRedOut * kRedGroups)
dw_tc_reduce_scalar_kernel(const float *__restrict__ ws, const float *__restrict__ ws_db,
                    __half *__restrict__ dW, __half *__restrict__ db, int splits, int C, int D,
                    int Cs) {
  __shared__ float part[kRedGroups][4][kRedOut];
  pdl_wait();
  const int64_t plane = static_cast<int64_t>(D) * Cs;
  const int64_t n = static_cast<int64_t>(D) * C;
  const int64_t nblk_w = cdiv(n, kRedOut);
  const int lo = threadIdx.x % kRedOut, grp = threadIdx.x / kRedOut;
  if (blockIdx.x < nblk_w) {
    const int64_t e = blockIdx.x * static_cast<int64_t>(kRedOut) + lo;
    float g[4] = {0.f, 0.f, 0.f, 0.f};
    if (e < n) {
      const float *src = ws + (e / C) * Cs + (e % C);
#pragma unroll 4
      for (int s = grp; s < splits; s += kRedGroups) {
        const float *q = src + static_cast<int64_t>(s) * 4 * plane;
#pragma unroll
        for (int k = 0; k < 4; ++k) g[k] += q[k * plane];
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) part[grp][k][lo] = g[k];
    __syncthreads();
    if (grp == 0 && e < n) {
      float t[4] = {0.f, 0.f, 0.f, 0.f};
      for (int q = 0; q < kRedGroups; ++q)
#pragma unroll
        for (int k = 0; k < 4; ++k) t[k] += part[q][k][lo];
      const float ev = 4.f * (t[0] + t[1]), od = 4.f * (t[0] - t[1]);
      uint2 pk;
      pk.x = pack_half2(ev + 8.f * t[2], od - 8.f * t[3]);
      pk.y = pack_half2(ev - 8.f * t[2], od + 8.f * t[3]);
      *reinterpret_cast<uint2 *>(dW + e * kT) = pk;
    }
  } else if (db != nullptr) {
    const int64_t d = (blockIdx.x - nblk_w) * kRedOut + lo;
    float sdb = 0.f;
    if (d < D)
#pragma unroll 4
      for (int s = grp; s < splits; s += kRedGroups) sdb += ws_db[static_cast<int64_t>(s) * D + d];
    part[grp][0][lo] = sdb;
    __syncthreads();
    if (grp == 0 && d < D) {
      float t = 0.f;
      for (int q = 0; q < kRedGroups; ++q) t += part[q][0][lo];
      db[d] = __float2half_rn(4.f * t);
    }
  }
}

// Blocks for dw_tc_reduce_scalar_kernel: the dW outputs, then the db outputs.
__host__ __device__ inline int64_t dw_reduce_scalar_blocks(int C, int D) {
  return cdiv(static_cast<int64_t>(D) * C, kRedOut) + cdiv(D, kRedOut);
}

// Sum of the split partials in a fixed order, inverse rDFT, fp16 cast:
//   dW[d][c][u] = (G0 + (-1)^u G2)/4 + Re(G1 i^u)/2,   db[d] = sum of partials.
// The partials come from planes divided by 4 on both sides (G/16, and db/4),
// so the constants applied are 4, 8 and 4.
// A dW block owns `q` quads (one d, four consecutive c, all four bins: 16
// floats) and 256/q split groups; thread (group g, quad) adds splits g, g +
// groups, ... with 16-byte loads, then the groups are folded pairwise in a fixed
// tree through shared memory — the same order on every run, so the result is
// bit-stable.  db blocks do the same for 32 scalars with 8 groups.  Many
// independent loads per thread keep the partials (mostly still in L2) streaming.
constexpr int kRedThreads = 256;
constexpr int kRedDbItems = 32;

struct RedPlan {
  int q;            // quads per dW block (4..32, a power of two)
  int64_t wblocks;  // dW blocks, followed by the db blocks
  int64_t blocks;
};

__host__ __device__ inline RedPlan make_red_plan(int C, int D, int sms) {
  RedPlan r;
  const int64_t nq = static_cast<int64_t>(D) * (align_up(C, 16) / 4);
  r.q = 32;
  while (r.q > 4 && cdiv(nq, r.q) < 2 * static_cast<int64_t>(sms)) r.q /= 2;
  r.wblocks = cdiv(nq, r.q);
  r.blocks = r.wblocks + cdiv(D, kRedDbItems);
  return r;
}

__global__ void __launch_bounds__(kRedThreads)
dw_tc_reduce_kernel(const float *__restrict__ ws, const float *__restrict__ ws_db,
                    __half *__restrict__ dW, __half *__restrict__ db, int splits, int C, int D,
                    int Cs, int q, int64_t wblocks) {
  __shared__ float red[16][kRedThreads];
  pdl_wait();
  const int t = threadIdx.x;
  if (blockIdx.x < wblocks) {
    const int groups = kRedThreads / q;
    const int quad = t % q, grp = t / q;
    const int64_t plane = static_cast<int64_t>(D) * Cs;
    const int nqr = Cs / 4;  // quads per d row
    const int64_t item = blockIdx.x * static_cast<int64_t>(q) + quad;
    const bool live = item < static_cast<int64_t>(D) * nqr;
    float acc[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) acc[k] = 0.f;
    if (live) {
      const float *src = ws + item * 4;  // d * Cs + 4 * cq
#pragma unroll 2
      for (int sp = grp; sp < splits; sp += groups) {
        const float *b0 = src + static_cast<int64_t>(sp) * 4 * plane;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 v = *reinterpret_cast<const float4 *>(b0 + k * plane);
          acc[4 * k + 0] += v.x;
          acc[4 * k + 1] += v.y;
          acc[4 * k + 2] += v.z;
          acc[4 * k + 3] += v.w;
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) red[k][t] = acc[k];
    for (int h = groups / 2; h >= 1; h /= 2) {
      __syncthreads();
      if (grp < h)
#pragma unroll
        for (int k = 0; k < 16; ++k) red[k][t] += red[k][t + h * q];
    }
    __syncthreads();
    if (grp == 0 && live) {
      const int d = static_cast<int>(item / nqr), c0 = static_cast<int>(item % nqr) * 4;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = c0 + i;
        if (c >= C) break;
        const float g0 = red[i][t], g2 = red[4 + i][t], gr = red[8 + i][t], gi = red[12 + i][t];
        const float ev = 4.f * (g0 + g2), od = 4.f * (g0 - g2);
        uint2 pk;
        pk.x = pack_half2(ev + 8.f * gr, od - 8.f * gi);
        pk.y = pack_half2(ev - 8.f * gr, od + 8.f * gi);
        *reinterpret_cast<uint2 *>(dW + (static_cast<int64_t>(d) * C + c) * kT) = pk;
      }
    }
  } else if (db != nullptr) {
    constexpr int kGroups = kRedThreads / kRedDbItems;
    const int di = t % kRedDbItems, grp = t / kRedDbItems;
    const int64_t d = (blockIdx.x - wblocks) * kRedDbItems + di;
    float sdb = 0.f;
    if (d < D)
#pragma unroll 4
      for (int sp = grp; sp < splits; sp += kGroups) sdb += ws_db[static_cast<int64_t>(sp) * D + d];
    red[0][t] = sdb;
    for (int h = kGroups / 2; h >= 1; h /= 2) {
      __syncthreads();
      if (grp < h) red[0][t] += red[0][t + h * kRedDbItems];
    }
    __syncthreads();
    if (grp == 0 && d < D) db[d] = __float2half_rn(4.f * red[0][t]);
  }
}

// Launches the split reduce that suits the output size (both sum the splits in
// a fixed order) as a programmatic dependent of the kernel before it on the
// stream: its blocks take the SMs as that kernel's CTAs exit and wait there
// (pdl_wait) for its partial sums, so no launch gap separates the two.
inline int launch_dw_tc_reduce(const float *ws, const float *ws_db, __half *dW, __half *db,
                               int splits, int C, int D, int Cs, int sms, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.stream = stream;
  cfg.dynamicSmemBytes = 0;
  cudaError_t e;
  if (static_cast<int64_t>(D) * C <= kRedScalarMaxOut) {
    cfg.gridDim = dim3(static_cast<unsigned>(dw_reduce_scalar_blocks(C, D)));
    cfg.blockDim = dim3(kRedOut * kRedGroups);
    e = cudaLaunchKernelEx(&cfg, dw_tc_reduce_scalar_kernel, ws, ws_db, dW, db, splits, C, D, Cs);
  } else {
    const RedPlan rp = make_red_plan(C, D, sms);
    if (rp.blocks > 0x7fffffff) return 1;
    cfg.gridDim = dim3(static_cast<unsigned>(rp.blocks));
    cfg.blockDim = dim3(kRedThreads);
    e = cudaLaunchKernelEx(&cfg, dw_tc_reduce_kernel, ws, ws_db, dW, db, splits, C, D, Cs, rp.q,
                           rp.wblocks);
  }
  return e == cudaSuccess ? 0 : 2;
}

}  // namespace feql
