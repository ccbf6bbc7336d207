// tc_bwd.cuh — fused backward: dX and the dW/db partial sums from one pass
// over dy (sm_100a tensor cores, fp16 data).
//
// Both gradients need the rDFT of the same dy tile (Flash EQ-Linear,
// technical summary "Implementazione": fused dataflow), so one kernel reads
// x and dy once and produces
//   dX[n,:] = irDFT_4( per-bin dY_k[n,:] . conj(What_k) )          (forward of conj(What)^T)
//   G_k[d,c] += sum_{n in split} dY_k[n,d] conj(X_k[n,c])          (split-K partials of dW)
//   db[d]    += sum_{n in split} dY_0[n,d]
// and the split reduce of tc_dw.cuh finishes dW/db as for feql_backward_dw.
//
// One CTA per token split (a multiple of 64 tokens); shapes with C <= 64 and
// D <= 128 (one dW tile, one dX output tile).  Per stage of 64 tokens:
//   warp 0      TMA: every 16-channel box of dy and x for the 64 tokens
//   warps 2..17 4-point rDFT of every (token, channel) fibre, in place, one
//               fibre row per thread: each 8 KB box becomes four 2 KB planes
//               (V0, V2, Re V1, -Im V1, each divided by 4 as in tc_fwd.cuh),
//               rows = tokens, 32-byte swizzle; in a dy box the first 4 KB
//               hold V0 and V2 interleaved in blocks of 16 token rows (V0 of
//               tokens 16j.., then V2 of the same tokens) and the second 4 KB
//               Re V1 and -Im V1 the same way; db sums in registers
//   warp 1      TMEM allocator + MMA issuer:
//                 dW: per 16 tokens six M=128 (d) x N=CT (c) MMAs, both
//                     operands MN-major (the planes read column-wise)
//                 dX: per 16-channel d chunk, against the resident
//                     conj(What)^T tiles, K-major (the same planes read
//                     row-wise), into a double-buffered accumulator, two
//                     M=128 MMAs: bins 0 and 2 over the interleaved V0/V2
//                     rows with N = 2 BD (What0 | What2; the cross products
//                     in the other halves are not read), and bin 1 over the
//                     interleaved Re V1 / -Im V1 rows against the window
//                     (Re1 ; Im1), whose four products the epilogue combines
//   warps 18..21 dX epilogue: warp q's TMEM lane quadrant holds tokens
//               16q..16q+15 in lanes 0..15 (V0 and Re V1 rows) and 16..31
//               (V2 and -Im V1 rows); 16x256b TMEM loads give each thread two
//               channels of two tokens from both halves, so the inverse rDFT
//               needs no shuffle and each four lanes store one token's 64
//               contiguous bytes (fp16, direct stores), which leaves the
//               shared memory to the stages (three fit for C = 24, D = 96)
// After the last stage warps 2..17 write the dW partials and db to the
// workspace; the split reduce of tc_dw.cuh, launched as this kernel's
// programmatic dependent, finishes dW and db.  Every wait is bounded.
#pragma once

#include <cuda_fp16.h>

#include "plan.cuh"
#include "rdft4.cuh"
#include "sm100.cuh"
#include "tc_dw.cuh"

namespace feql {

constexpr int kBwTB = 64;                    // tokens per stage (dX MMA M)
constexpr int kBwBox = kBwTB * 128;          // 8 KB: 64 tokens x 16 channels x 4 fp16
constexpr int kBwPlane = kBwTB * 32;         // 2 KB: one bin of one box
constexpr int kBwXfWarps = 16;               // one (box, token) item per thread and stage
constexpr int kBwEpWarps = 4;
constexpr int kBwThreads = 64 + (kBwXfWarps + kBwEpWarps) * 32;
constexpr int kBwMaxItems = kBwXfWarps * 32;  // (box, token) items a stage may hold

struct TcBwdParams {
  const uint8_t *wt;   // conj(What)^T tiles of the dX direction (one output tile)
  __half *dx;          // [N][C][4]
  int64_t N;
  int C, D, Cs;        // Cs: workspace row stride
  int nqd, nqc;        // 16-channel boxes of dy and of x
  int slots;           // box slots per stage: max(8, nqd + nqc) (dW operand reads 8 d boxes)
  int CT;              // dW columns: 16 * nqc
  int BD;              // dX output tile (>= C)
  int chunk_bytes;     // one dX weight chunk: 5 * BD rows x 32 B
  int wres_bytes;      // nqd * chunk_bytes, 1 KB aligned
  int stages;
  int splits;
  int64_t split_len;   // tokens per CTA, multiple of 64
  int ndx;             // dX accumulator buffers (1 or 2)
  int merged;          // dW bin 1 as two N = 2*CT MMAs (6*CT TMEM columns), see tc_dw.cuh
  int stack_dy, stack_x;  // 1: one 3-D load brings all of a stage's dy (x) boxes
  float *ws;           // [splits][4][D][Cs]
  float *ws_db;        // [splits][D]
};

// Byte offset of token row r of plane pp (0..3) inside a transformed dy box:
// V0 and V2 interleaved in 16-row blocks in the first 4 KB, Re V1 and -Im V1
// the same way in the second (each half a 128-row K-major operand for one
// merged dX MMA; one 512-byte block per plane and 16-token dW step).
__device__ __forceinline__ int bw_dy_row(int pp, int r) {
  return ((pp >> 1) << 12) + ((r >> 4) << 10) + ((pp & 1) << 9) + ((r & 15) << 5);
}

struct BwSmem {
  int wres, stage0, bars, total;
};

__host__ __device__ inline BwSmem tc_bwd_smem(const TcBwdParams &p) {
  BwSmem s;
  s.wres = 0;
  s.stage0 = p.wres_bytes;
  s.bars = s.stage0 + p.stages * p.slots * kBwBox;
  // full, tready, empty per stage; dxfull, dxempty x2; dwfull; wfull; tmem slot
  s.total = s.bars + (3 * p.stages + 4 + 2) * 8 + 16;
  return s;
}

// 22 warps over the 4 SM sub-partitions put 6 warps on one 16K-register slice:
// 6 x 32 x 80 = 15,360 (88 would not fit).  The transform is latency-bound, so
// it gets many warps with one item each rather than few with several.
// kDbCol: C is not a multiple of 16, so the last x box has a padding channel
// (p.C itself, zero in the loaded data).  The transform sets that channel's
// bin-0 plane value to 1/4, so the dW bin-0 MMA produces
//   G0[d][C] = sum_n (dY0[n,d] / 4) * (1/4) = db[d] / 16
// in the padding column and db needs no accumulation in registers.
template <bool kDbCol>
__global__ void __maxnreg__(80)
tc_bwd_kernel(const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_x,
              const TcBwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const BwSmem L = tc_bwd_smem(p);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
  uint64_t *full = bars;
  uint64_t *tready = bars + p.stages;
  uint64_t *empty = bars + 2 * p.stages;
  uint64_t *dxfull = bars + 3 * p.stages;
  uint64_t *dxempty = dxfull + 2;
  uint64_t *dwfull = dxempty + 2;
  uint64_t *wfull = dwfull + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(wfull + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int split = blockIdx.x;
  const int64_t t_begin = static_cast<int64_t>(split) * p.split_len;
  int64_t t_end = t_begin + p.split_len;
  if (t_end > p.N) t_end = p.N;
  const int nst = t_begin < t_end ? static_cast<int>(cdiv(t_end - t_begin, kBwTB)) : 0;
  const int nbox = p.nqd + p.nqc;
  const int dx0 = (p.merged ? 6 : 4) * p.CT;  // first TMEM column of the dX accumulators

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&tready[s], kBwXfWarps);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&dxfull[b], 1);
      mbar_init(&dxempty[b], kBwEpWarps);
    }
    mbar_init(dwfull, 1);
    mbar_init(wfull, 1);
    fence_mbar_init();
  }
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
      tma_prefetch_desc(&tm_dy);
      tma_prefetch_desc(&tm_x);
      if (nst > 0) {
        mbar_arrive_expect_tx(wfull, p.nqd * p.chunk_bytes);
        bulk_load(smem + L.wres, p.wt, p.nqd * p.chunk_bytes, wfull);
      }
      int s = 0;
      uint32_t ph = 0;
      for (int ch = 0; ch < nst; ++ch) {
        if (ok) ok = mbar_wait(&empty[s], ph ^ 1);
        if (ok) {
          uint8_t *st = smem + L.stage0 + s * p.slots * kBwBox;
          const int32_t row = static_cast<int32_t>(t_begin + static_cast<int64_t>(ch) * kBwTB);
          mbar_arrive_expect_tx(&full[s], nbox * kBwBox);
          if (p.stack_dy) {
            tma_load_3d(st, &tm_dy, 0, row, 0, &full[s]);
          } else {
            for (int q = 0; q < p.nqd; ++q)
              tma_load_2d(st + q * kBwBox, &tm_dy, q * 16 * kT, row, &full[s]);
          }
          if (p.stack_x) {
            tma_load_3d(st + p.nqd * kBwBox, &tm_x, 0, row, 0, &full[s]);
          } else {
            for (int q = 0; q < p.nqc; ++q)
              tma_load_2d(st + (p.nqd + q) * kBwBox, &tm_x, q * 16 * kT, row, &full[s]);
          }
        }
        if (++s == p.stages) { s = 0; ph ^= 1; }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      // dW: planes hold -Im of bin 1 for dy and x alike (see tc_dw.cuh)
      const uint32_t id_w = instr_desc(128, p.CT, 0, 0, 1, 1);
      const uint32_t id_wneg = instr_desc(128, p.CT, 0, 0, 1, 1, 1);
      // dX: K-major operands, M = 128 interleaved rows (bins 0 and 2, or Re and
      // -Im of bin 1, of 64 tokens)
      const uint32_t id_x = instr_desc(128, 2 * p.BD, 0, 0);
      const uint32_t acc0 = tmem_base, acc2 = tmem_base + p.CT;
      const uint32_t acc1r = tmem_base + 2 * p.CT, acc1i = tmem_base + 3 * p.CT;
      const uint32_t acca = tmem_base + 2 * p.CT, accb = tmem_base + 4 * p.CT;
      const uint32_t id_w2 = instr_desc(128, 2 * p.CT, 0, 0, 1, 1);
      if (nst > 0 && ok) ok = mbar_wait(wfull, 0);
      const uint32_t wres = smem_u32(smem + L.wres);
      const uint32_t stage_base = smem_u32(smem + L.stage0);
      const uint64_t dmn = smem_desc(0, kBwBox, 256, kSw32);    // dy planes read column-wise (dW)
      const uint64_t dmx = smem_desc(0, kBwPlane, 256, kSw32);  // x planes read column-wise (dW)
      const uint64_t dk = smem_desc(0, 16, 256, kSw32);       // K-major rows (dX, weights)
      const uint32_t dhi = desc_hi(dk);  // same for dmn and dmx: only the low words differ
      const uint32_t xb16 = (p.nqc * kBwPlane) >> 4;  // one x bin
      const uint32_t wl = desc_lo(desc_at(dk, wres)), chunk16 = p.chunk_bytes >> 4;
      const uint32_t w1 = (p.BD * 32) >> 4;
      int s = 0, b = 0;         // ring slot; dX accumulator buffer (stepped, no divisions)
      uint32_t ph = 0, bph = 0;
      for (int ch = 0; ch < nst; ++ch) {
        // tready implies full (the transform waited for the slot's TMA bytes
        // before its release-arrive); the dX accumulator buffer of this stage
        // is tested in the same round trip
        if (ok) ok = mbar_wait2(&tready[s], ph, &dxempty[b], bph ^ 1);
        tc_fence_after();
        const uint32_t st = stage_base + s * p.slots * kBwBox;
        // every operand below is the low descriptor word of one of these bases plus a
        // 16-byte-unit offset (the high words are all dhi)
        const uint32_t mn = desc_lo(desc_at(dmn, st)), mx = desc_lo(desc_at(dmx, st + p.nqd * kBwBox));
        const uint32_t kl = desc_lo(desc_at(dk, st));
        if (ok) {
#pragma unroll
          for (int k = 0; k < kBwTB / 16; ++k) {
            // dy planes: d chunks 8 KB apart, V0/V2 and Re/-Im V1 blocks of 16
            // tokens interleaved (1 KB per step, the bin-1 pair 4 KB in); x
            // planes: plane-major, c chunks 2 KB apart; 16 tokens = 512 B
            const uint32_t A0 = mn + k * 64, A1 = A0 + 32;
            const uint32_t A2 = A0 + 256, A3 = A2 + 32;
            const uint32_t B0 = mx + k * 32, B1 = B0 + xb16;
            const uint32_t B2 = B1 + xb16, B3 = B2 + xb16;
            const uint32_t first = (ch == 0 && k == 0) ? 0u : 1u;
            mma_f16_lo(acc0, A0, B0, dhi, id_w, first);
            mma_f16_lo(acc2, A1, B1, dhi, id_w, first);
            if (p.merged) {  // see tc_dw.cuh: acc_a, acc_b over [Re X1 | -Im X1]
              mma_f16_lo(acca, A2, B2, dhi, id_w2, first);
              mma_f16_lo(accb, A3, B2, dhi, id_w2, first);
            } else {
              mma_f16_lo(acc1r, A2, B2, dhi, id_w, first);
              mma_f16_lo(acc1r, A3, B3, dhi, id_w, 1u);
              mma_f16_lo(acc1i, A3, B2, dhi, id_wneg, first);
              mma_f16_lo(acc1i, A2, B3, dhi, id_w, 1u);
            }
          }
        }
        if (ok) {
          const uint32_t acc = tmem_base + dx0 + b * 4 * p.BD;
          uint32_t ab = kl, wb = wl;  // running box and weight-chunk descriptor words
          for (int q = 0; q < p.nqd; ++q, ab += kBwBox >> 4, wb += chunk16) {
            const uint32_t in = q > 0 ? 1u : 0u;
            mma_f16_lo(acc, ab, wb, dhi, id_x, in);
            mma_f16_lo(acc + 2 * p.BD, ab + 256, wb + 2 * w1, dhi, id_x, in);
          }
          mma_commit(&dxfull[b]);
          mma_commit(&empty[s]);
        }
        if (++s == p.stages) { s = 0; ph ^= 1; }
        if (++b == p.ndx) { b = 0; bph ^= 1; }
      }
      mma_commit(dwfull);
    }
  } else if (warp < 2 + kBwXfWarps) {
    // ---------------------------------------------------------- transform
    const int t = threadIdx.x - 64;
    constexpr int kPer = kBwMaxItems / (kBwXfWarps * 32);  // items per thread (1)
    constexpr int kDbRegs = kDbCol ? 1 : 16;                 // db accumulators per item
    float db_acc[kPer][kDbRegs];
#pragma unroll
    for (int k = 0; k < kPer; ++k)
#pragma unroll
      for (int c = 0; c < kDbRegs; ++c) db_acc[k][c] = 0.f;
    int s = 0;
    uint32_t ph = 0;
    for (int ch = 0; ch < nst; ++ch) {
      if (ok) ok = mbar_wait(&full[s], ph);
      uint8_t *st = smem + L.stage0 + s * p.slots * kBwBox;
      uint32_t pl[kPer][4][8];
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int e = t + k * kBwXfWarps * 32;
        const int b = e / kBwTB, r = e % kBwTB;
        if (b < nbox) {
          const uint8_t *src = st + b * kBwBox + r * 128;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint4 v = *reinterpret_cast<const uint4 *>(src + ((q ^ (r & 7)) << 4));
            rdft4_pair_q(v, pl[k][0][q], pl[k][1][q], pl[k][2][q], pl[k][3][q]);
          }
        }
      }
      named_bar_sync(2, kBwXfWarps * 32);  // all rows read before the planes overwrite them
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int e = t + k * kBwXfWarps * 32;
        const int b = e / kBwTB, r = e % kBwTB;
        if (b < nbox) {
          // dy box: its four planes in place (bw_dy_row); x box q: plane pp at
          // x + (pp * nqc + q) planes
          const bool is_dy = b < p.nqd;
          if (kDbCol && b == p.nqd + p.C / 16) {
            // the padding channel C of this x box: bin 0 = 1 (stored as 1/4)
            const int cq = (p.C % 16) >> 1;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              if (q == cq) pl[k][0][q] = (p.C & 1) ? (pl[k][0][q] & 0xFFFFu) | 0x34000000u
                                                  : (pl[k][0][q] & 0xFFFF0000u) | 0x3400u;
          }
          uint8_t *base = is_dy ? st + b * kBwBox : st + p.nqd * kBwBox + (b - p.nqd) * kBwPlane;
          // planes 0, 1 and 2, 3 are each one stride apart
          const int o01 = is_dy ? bw_dy_row(0, r) : r * 32;
          const int s01 = is_dy ? 512 : p.nqc * kBwPlane;
          const int o23 = is_dy ? bw_dy_row(2, r) : 2 * p.nqc * kBwPlane + r * 32;
          const int s23 = s01;
#pragma unroll
          for (int pp = 0; pp < 4; ++pp) {
            uint8_t *row = base + (pp < 2 ? o01 + pp * s01 : o23 + (pp - 2) * s23);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
              *reinterpret_cast<uint4 *>(row + (((hh ^ (r >> 2)) & 1) << 4)) =
                  make_uint4(pl[k][pp][4 * hh + 0], pl[k][pp][4 * hh + 1], pl[k][pp][4 * hh + 2],
                             pl[k][pp][4 * hh + 3]);
          }
          if (!kDbCol && b < p.nqd) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float2 f = __half22float2(as_h2(pl[k][0][q]));
              db_acc[k][2 * q % kDbRegs] += f.x;
              db_acc[k][(2 * q + 1) % kDbRegs] += f.y;
            }
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&tready[s]);
      if (++s == p.stages) { s = 0; ph ^= 1; }
    }

    // ---------------------------------------------- dW partials -> workspace
    if (ok) ok = mbar_wait(dwfull, 0);
    tc_fence_after();
    const int quad = warp & 3, part = (warp - 2) / 4;  // kBwXfWarps / 4 warps per quadrant
    const int d = quad * 32 + lane;
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    float *dst = p.ws + (static_cast<int64_t>(split) * 4 * p.D + d) * p.Cs;
    const int64_t bin_stride = static_cast<int64_t>(p.D) * p.Cs;
    for (int g = part; g < p.CT / 8; g += kBwXfWarps / 4) {  // 8-column steps
      float G[4][8];
      dw_acc_read8(tl, p.CT, g * 8, p.merged, G);
      if (d < p.D && g * 8 < p.C) {
#pragma unroll
        for (int bin = 0; bin < 4; ++bin) {
          float4 *o = reinterpret_cast<float4 *>(dst + bin * bin_stride + g * 8);
          o[0] = make_float4(G[bin][0], G[bin][1], G[bin][2], G[bin][3]);
          o[1] = make_float4(G[bin][4], G[bin][5], G[bin][6], G[bin][7]);
        }
      }
      if (kDbCol && d < p.D && g == p.C / 8) {
        // db partial in the padding column; the reduce expects sum of dY0 / 4
        const int j = p.C % 8;
        float v = G[0][0];
#pragma unroll
        for (int i = 1; i < 8; ++i)
          if (i == j) v = G[0][i];
        p.ws_db[static_cast<int64_t>(split) * p.D + d] = 4.f * v;
      }
    }
    tc_fence_before();
    if (!kDbCol) {
    // db: fixed-order reduction of the per-thread partials through shared memory
    named_bar_sync(3, kBwXfWarps * 32);  // stages are free: every chunk has been consumed
    float *sdb = reinterpret_cast<float *>(smem + L.stage0);  // [kBwMaxItems][16]
#pragma unroll
    for (int k = 0; k < kPer; ++k)
#pragma unroll
      for (int c = 0; c < 16; ++c) sdb[(t + k * kBwXfWarps * 32) * 16 + c] = db_acc[k][c];
    named_bar_sync(3, kBwXfWarps * 32);
    if (t < p.nqd * 16) {
      const int bb = t / 16, c = t % 16;
      float sum = 0.f;
      for (int rr = 0; rr < kBwTB; ++rr) sum += sdb[(bb * kBwTB + rr) * 16 + c];
      const int dd = bb * 16 + c;
      if (dd < p.D) p.ws_db[static_cast<int64_t>(split) * p.D + dd] = sum;
    }
    }
  } else {
    // ------------------------------------------------------- dX epilogue
    // Per 8-channel block six 16x256b loads: thread t holds channels
    // c0 + 2(t%4) and c0 + 2(t%4) + 1 of tokens 16q + t/4 and 16q + t/4 + 8:
    //   bin 0 (lanes 0..15, columns [0, BD)), bin 2 (lanes 16..31, [BD, 2BD)),
    //   bin 1: Re rows (lanes 0..15) and -Im rows (16..31) against (Re1 ; Im1)
    //   (columns [2BD, 4BD)): Re Y1 = a_r + b_i, Im Y1 = a_i - b_r.
    const int quad = warp & 3;
    const int64_t row_elems = static_cast<int64_t>(p.C) * kT;
    const int nblk = (p.C + 7) / 8;    // 8-channel blocks holding real channels
    const int tc = 2 * (lane & 3);     // first channel of this thread's pair in a block
    int b = 0;
    uint32_t bph = 0;
    for (int ch = 0; ch < nst; ++ch, b = b + 1 == p.ndx ? 0 : b + 1, bph ^= (b == 0)) {
      if (ok) ok = mbar_wait(&dxfull[b], bph);
      tc_fence_after();
      const uint32_t lo = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + dx0 + b * 4 * p.BD;
      const uint32_t hi = lo + (16u << 16);
      const int64_t n0 = t_begin + static_cast<int64_t>(ch) * kBwTB + quad * 16 + (lane >> 2);
      __half *row0 = p.dx + n0 * row_elems, *row1 = row0 + 8 * row_elems;
      for (int g = 0; g < nblk; ++g) {
        const int c0 = 8 * g;
        uint32_t y0[4], y2[4], ar[4], ai[4], br[4], bi[4];
        // the TMEM loads are warp-collective: reconverge after the wait and the
        // per-lane stores of the previous block
        __syncwarp();
        tmem_ld16x256(lo + c0, y0);
        tmem_ld16x256(hi + p.BD + c0, y2);
        tmem_ld16x256(lo + 2 * p.BD + c0, ar);
        tmem_ld16x256(lo + 3 * p.BD + c0, ai);
        tmem_ld16x256(hi + 2 * p.BD + c0, br);
        tmem_ld16x256(hi + 3 * p.BD + c0, bi);
        tmem_ld_wait();
        if (g == nblk - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0 && ok) mbar_arrive(&dxempty[b]);
        }
        // dy planes and weights are both stored divided by 4 (Y = 16 * acc);
        // out[i] = (u0, u1) and (u2, u3) of register i's (token, channel)
        uint32_t out[4][2];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float Y0 = __uint_as_float(y0[i]), Y2 = __uint_as_float(y2[i]);
          const float Yr = __uint_as_float(ar[i]) + __uint_as_float(bi[i]);
          const float Yi = __uint_as_float(ai[i]) - __uint_as_float(br[i]);
          const float e = 4.f * (Y0 + Y2), o = 4.f * (Y0 - Y2);
          out[i][0] = pack_half2(fmaf(8.f, Yr, e), fmaf(-8.f, Yi, o));
          out[i][1] = pack_half2(fmaf(-8.f, Yr, e), fmaf(8.f, Yi, o));
        }
        // C is even: a thread's channel pair is either whole or past the end
        if (c0 + tc + 2 <= p.C) {
          if (n0 < t_end)
            *reinterpret_cast<uint4 *>(row0 + (c0 + tc) * kT) =
                make_uint4(out[0][0], out[0][1], out[1][0], out[1][1]);
          if (n0 + 8 < t_end)
            *reinterpret_cast<uint4 *>(row1 + (c0 + tc) * kT) =
                make_uint4(out[2][0], out[2][1], out[3][0], out[3][1]);
        }
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
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace feql
