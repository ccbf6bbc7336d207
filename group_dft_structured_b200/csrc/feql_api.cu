// feql_api.cu — the C ABI of libfeql.so (declared in include/feql.h).
//
// Host side only: argument validation, per-shape plans, TMA tensor maps and
// kernel launches.  Every arithmetic step runs in the kernels included below.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "../../include/feql.h"
#include "plan.cuh"
#include "simt.cuh"
#include "simt_ct.cuh"
#include "sm100.cuh"
#include "tc_bwd.cuh"
#include "tc_dw.cuh"
#include "tc_fwd.cuh"
#include "group8.cuh"
#include "tc_mlp.cuh"
#include "wfft.cuh"

using namespace feql;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxChannels = 1 << 16;   // per group element
constexpr int64_t kMaxTokens = (1ll << 31) - 1;  // TMA coordinates are int32

struct DeviceInfo {
  int sms = 0;
  int smem_optin = 0;
  int cc_major = 0, cc_minor = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
bool g_dev_ok[kMaxDevices];

int device_info(DeviceInfo *out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FEQL_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_dev_ok[dev]) {
    DeviceInfo d;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return FEQL_ERR_CUDA;
    g_dev[dev] = d;
    g_dev_ok[dev] = true;
  }
  *out = g_dev[dev];
  return FEQL_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major fp16 matrix [rows][cols] viewed as a 2-D tensor; box = 64 cols x box_rows
// rows, 128-byte swizzle, zero fill out of range.
// Box of box_cols x box_rows, 128-byte swizzle (64 columns: 128-byte rows), or
// without swizzle for other widths (the 96-byte rows of 8 channels x 6).
int make_tmap_f16(CUtensorMap *m, const void *base, int64_t rows, int64_t cols,
                  int box_rows = kBM, int box_cols = 64) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return FEQL_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FEQL_OK : FEQL_ERR_CUDA;
}

// A [rows][row_elems] fp16 tensor seen as a stack of 64-element (128-byte)
// column boxes: dims (64 elements, rows, boxes), strides (row_elems*2 B, 128 B).
// One load of a (64, box_rows, box_count) box writes box_count boxes of
// box_rows 128-byte rows one after the other, the shared-memory image of
// box_count 2-D loads.  Needs row_elems % 64 == 0 (else a box would run into
// the next row).
int make_tmap_f16_boxes(CUtensorMap *m, const void *base, int64_t rows, int64_t row_elems,
                        int box_rows, int box_count, int box_cols = 64) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || row_elems % box_cols != 0) return FEQL_ERR_CUDA;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(box_cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(row_elems / box_cols)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_elems) * 2,
                           static_cast<cuuint64_t>(box_cols) * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows),
                       static_cast<cuuint32_t>(box_count)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FEQL_OK : FEQL_ERR_CUDA;
}

// Row-major fp32 matrix [rows][cols] viewed as a 2-D tensor; box = 32 cols (128
// bytes) x box_rows rows, 128-byte swizzle, zero fill out of range: the same
// shared-memory image as make_tmap_f16's box, with 8 channels x 4 group
// elements of fp32 per row.
int make_tmap_f32(CUtensorMap *m, const void *base, int64_t rows, int64_t cols,
                  int box_rows = kBM) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return FEQL_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 4};
  cuuint32_t box[2] = {32, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FEQL_OK : FEQL_ERR_CUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_dtype(int dt) { return dt >= FEQL_FP16 && dt <= FEQL_FP16_SIMT; }

// Resolves FEQL_FP32 to the library's fp32 algorithm.
int resolve(int dt) { return dt == FEQL_FP32 ? FEQL_FP32_SIMT : dt; }

// The p4 layer's FEQL_FP32: split TF32 on the tensor cores up to 512 channels on
// either side (measured within the fp32 bound at that contraction depth per
// bin), fp32 FMA on CUDA cores beyond.  Depends on (C, D) only, so the weight
// transform and the passes agree on the Fourier buffer's layout.
constexpr int kTf32MaxChannels = 512;
int resolve(int dt, int C, int D) {
  if (dt != FEQL_FP32) return dt;
  return (C <= kTf32MaxChannels && D <= kTf32MaxChannels) ? FEQL_FP32_3XTF32 : FEQL_FP32_SIMT;
}

bool is_tc(int dt) { return dt == FEQL_FP16; }
bool is_tf32(int dt) { return dt == FEQL_FP32_3XTF32; }
// Layout kind of the Fourier-weight buffer of a (resolved) mode.
int what_kind(int dt) { return is_tc(dt) ? kWhatF16 : (is_tf32(dt) ? kWhatTF32 : kWhatSimt); }
bool is_half(int dt) { return dt == FEQL_FP16 || dt == FEQL_FP16_SIMT; }

int check_shape(int C, int D) {
  if (C <= 0 || D <= 0 || C > kMaxChannels || D > kMaxChannels) return FEQL_ERR_INVALID_ARG;
  return FEQL_OK;
}

int launch_status() {
  return cudaGetLastError() == cudaSuccess ? FEQL_OK : FEQL_ERR_CUDA;
}

int grid_for(int64_t work, int threads, int sms) {
  int64_t g = cdiv(work, threads);
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

// ---------------------------------------------------------------- tc launch
// tf32: fp32 data in the split-TF32 mode (FEQL_FP32_3XTF32), else fp16.
int launch_tc_gemm(const void *in, const uint8_t *wt, const TcPlan &P, const void *bias,
                   void *out, int64_t N, cudaStream_t stream, bool tf32 = false) {
  DeviceInfo dev;
  int st = device_info(&dev);
  if (st != FEQL_OK) return st;
  if (dev.cc_major != 10) return FEQL_ERR_UNSUPPORTED;
  TcFwdParams p;
  p.wt = wt;
  p.bias = bias;
  p.N = N;
  p.Ci = P.Ci;
  p.Do = P.Do;
  p.BD = P.BD;
  p.nD = P.nD;
  p.nK = P.nK;
  p.chunk_bytes = P.chunk_bytes;
  const int64_t nM = cdiv(N, kBM);
  if (nM * P.nD > INT32_MAX) return FEQL_ERR_UNSUPPORTED;
  p.nM = static_cast<int>(nM);
  p.n_units = static_cast<int>(nM * P.nD);
  p.nacc = (4 * P.BD <= 256) ? 2 : 1;
  p.acc_stride = p.nacc == 2 ? 256 : 0;
  p.bias_floats = P.nD * P.BD;
  p.out = out;
  const int slot = tf32 ? 2 * kXChunkBytes : kXChunkBytes;  // input chunk / its planes
  const int budget = dev.smem_optin - 1024;  // 1 KB for aligning the base
  // Resident weights when the CTA's slice fits beside >= 4 input stages and
  // there are enough CTAs for one fixed output tile each.
  p.resident = 1;
  p.wres_bytes = static_cast<int>(align_up(static_cast<int64_t>(P.nK) * P.chunk_bytes, 1024));
  p.stage_bytes = slot;
  p.stages = 8;
  while (p.stages > 4 && tc_fwd_smem(p).total > budget) --p.stages;
  if (tc_fwd_smem(p).total > budget || dev.sms < P.nD) {
    p.resident = 0;
    p.wres_bytes = 0;
    p.stage_bytes = slot + static_cast<int>(align_up(P.chunk_bytes, 1024));
    p.stages = 8;
    while (p.stages > 2 && tc_fwd_smem(p).total > budget) --p.stages;
    if (tc_fwd_smem(p).total > budget) return FEQL_ERR_UNSUPPORTED;
  }
  const int smem = tc_fwd_smem(p).total + 1024;
  int grid;
  if (p.resident) {
    const int64_t per_tile = nM < dev.sms / P.nD ? nM : dev.sms / P.nD;  // CTAs per output tile
    grid = static_cast<int>(per_tile * P.nD);
  } else {
    grid = p.n_units < dev.sms ? p.n_units : dev.sms;
  }

  CUtensorMap tm_in;
  st = tf32 ? make_tmap_f32(&tm_in, in, N, static_cast<int64_t>(P.Ci) * kT)
            : make_tmap_f16(&tm_in, in, N, static_cast<int64_t>(P.Ci) * kT);
  if (st != FEQL_OK) return st;
  auto kernel = tf32 ? tc_fourier_gemm_kernel<true> : tc_fourier_gemm_kernel<false>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return FEQL_ERR_CUDA;
  kernel<<<grid, kTcThreads, smem, stream>>>(tm_in, p);
  return launch_status();
}

template <typename T>
int launch_simt_fwd(const void *in, const float *Wp, const void *bias, void *out, int64_t N,
                    int Ci, int Do, cudaStream_t stream) {
  const int64_t gx = cdiv(N, kSimtTile);
  if (gx > INT32_MAX) return FEQL_ERR_UNSUPPORTED;
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(cdiv(Do, kSimtTile)));
  if (grid.y > 65535) return FEQL_ERR_UNSUPPORTED;
  simt_fwd_kernel<T><<<grid, kSimtThreads, 0, stream>>>(
      static_cast<const T *>(in), Wp, static_cast<const T *>(bias), static_cast<T *>(out), N, Ci,
      Do);
  return launch_status();
}

// ---------------------------------------------------------------- dW plan
struct DwPlan {
  int splits;
  int64_t split_len;
  int64_t ws_floats;
};

DwPlan make_dw_plan(int64_t N, int C, int D, int sms) {
  DwPlan q;
  const int64_t tiles = cdiv(D, kSimtTile) * cdiv(C, kSimtTile);
  int64_t s = cdiv(2ll * sms, tiles);
  const int64_t max_s = cdiv(N, kSimtK) > 0 ? cdiv(N, kSimtK) : 1;
  if (s > max_s) s = max_s;
  if (s > 1024) s = 1024;
  if (s < 1) s = 1;
  q.split_len = align_up(cdiv(N > 0 ? N : 1, s), kSimtK);
  q.splits = static_cast<int>(cdiv(N > 0 ? N : 1, q.split_len));
  q.ws_floats = static_cast<int64_t>(q.splits) * (4ll * C * D + D);
  return q;
}

// Tensor-core dW plan: d tiles of 128 rows, c tiles of CT <= 128 columns, the
// token axis split so that tiles x splits fills the SMs once.
TcDwParams make_tc_dw_plan(int64_t N, int C, int D, int sms) {
  TcDwParams p;
  p.N = N;
  p.C = C;
  p.D = D;
  p.Cs = static_cast<int>(align_up(C, 16));
  const int nct = static_cast<int>(cdiv(C, kDwMaxCT));
  p.CT = static_cast<int>(align_up(cdiv(C, nct), 16));
  p.tiles_c = static_cast<int>(cdiv(C, p.CT));
  p.tiles_d = static_cast<int>(cdiv(D, kDwMT));
  p.nqd_max = static_cast<int>(cdiv(D, 16) < 8 ? cdiv(D, 16) : 8);
  p.nqc_max = p.CT / 16;
  const int nbox = p.nqd_max + p.nqc_max;
  // tokens per chunk: every (box, token) item of a chunk has one transform
  // thread slot (kDwItems), and the plane buffer (8 dy chunks per bin for the
  // M = 128 operand) stays within ~40 KB
  p.TB = 32;
  while (p.TB * nbox > kDwItems) p.TB /= 2;
  const int64_t tiles = static_cast<int64_t>(p.tiles_d) * p.tiles_c;
  int64_t s = sms / tiles;
  if (s < 1) s = 1;
  const int64_t max_s = cdiv(N > 0 ? N : 1, p.TB);
  if (s > max_s) s = max_s;
  p.split_len = align_up(cdiv(N > 0 ? N : 1, s), p.TB);
  p.splits = static_cast<int>(cdiv(N > 0 ? N : 1, p.split_len));
  p.raw_bytes = nbox * p.TB * 128;
  p.plane_bytes = 4 * (8 + p.nqc_max) * p.TB * 32;
  p.merged = 6 * p.CT <= 512 ? 1 : 0;
  int cols = 32;
  while (cols < (p.merged ? 6 : 4) * p.CT) cols *= 2;
  p.tmem_cols = cols;
  p.stages = 0;
  p.stack_dy = 0;
  p.stack_x = 0;
  p.ws = nullptr;
  p.ws_db = nullptr;
  return p;
}

int64_t tc_dw_ws_floats(const TcDwParams &p) {
  return static_cast<int64_t>(p.splits) * (4ll * p.D * p.Cs + p.D);
}

int launch_tc_dw(TcDwParams p, const void *x, const void *dy, __half *dW, __half *db, float *ws,
                 const DeviceInfo &dev, cudaStream_t stream) {
  if (dev.cc_major != 10) return FEQL_ERR_UNSUPPORTED;
  p.ws = ws;
  p.ws_db = ws + static_cast<int64_t>(p.splits) * 4 * p.D * p.Cs;
  if (p.N > 0) {
    const int budget = dev.smem_optin - 1024;
    p.stages = 8;
    while (p.stages > 2 && tc_dw_smem(p).total > budget) --p.stages;
    if (tc_dw_smem(p).total > budget) return FEQL_ERR_UNSUPPORTED;
    const int smem = tc_dw_smem(p).total + 1024;
    // Chunks of 16 tokens make 2 KB boxes, and issuing one TMA load per box
    // then limits the kernel: such chunks take one load per operand when the
    // channels form whole boxes.  Larger chunks keep one 2-D load per box
    // (measured faster there).
    CUtensorMap tm_dy, tm_x;
    const bool small = p.TB <= 16;
    p.stack_dy = small && make_tmap_f16_boxes(&tm_dy, dy, p.N, static_cast<int64_t>(p.D) * kT,
                                              p.TB, p.nqd_max) == FEQL_OK;
    int st = FEQL_OK;
    if (!p.stack_dy) st = make_tmap_f16(&tm_dy, dy, p.N, static_cast<int64_t>(p.D) * kT, p.TB);
    if (st != FEQL_OK) return st;
    p.stack_x = small && make_tmap_f16_boxes(&tm_x, x, p.N, static_cast<int64_t>(p.C) * kT, p.TB,
                                             p.nqc_max) == FEQL_OK;
    if (!p.stack_x) st = make_tmap_f16(&tm_x, x, p.N, static_cast<int64_t>(p.C) * kT, p.TB);
    if (st != FEQL_OK) return st;
    if (cudaFuncSetAttribute(tc_dw_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return FEQL_ERR_CUDA;
    const int grid = p.tiles_d * p.tiles_c * p.splits;
    tc_dw_kernel<<<grid, kDwThreads, smem, stream>>>(tm_dy, tm_x, p);
  }
  {
    const int r = launch_dw_tc_reduce(p.ws, p.ws_db, dW, db, p.N > 0 ? p.splits : 0, p.C, p.D,
                                      p.Cs, dev.sms, stream);
    if (r != 0) return r == 1 ? FEQL_ERR_UNSUPPORTED : FEQL_ERR_CUDA;
  }
  return launch_status();
}

// Fused backward plan; false when the shape is outside the fused kernel's
// range (then feql_backward runs the dX and dW kernels one after the other).
bool make_tc_bwd_plan(int64_t N, int C, int D, const WhatLayout &L, const DeviceInfo &dev,
                      TcBwdParams &p) {
  if (N <= 0 || L.dx.nD != 1) return false;
  p.N = N;
  p.C = C;
  p.D = D;
  p.Cs = static_cast<int>(align_up(C, 16));
  p.nqd = static_cast<int>(cdiv(D, 16));
  p.nqc = static_cast<int>(cdiv(C, 16));
  if (p.nqd + p.nqc > kBwMaxItems / kBwTB) return false;
  p.slots = p.nqd + p.nqc > 8 ? p.nqd + p.nqc : 8;
  p.CT = 16 * p.nqc;
  p.BD = L.dx.BD;
  p.chunk_bytes = L.dx.chunk_bytes;
  // TMEM columns: dW (6*CT merged, else 4*CT) + dX buffers (4*BD each)
  if (4 * p.CT + 4 * p.BD > 512) return false;
  p.merged = (6 * p.CT + 4 * p.BD <= 512) ? 1 : 0;
  p.ndx = ((p.merged ? 6 : 4) * p.CT + 8 * p.BD <= 512) ? 2 : 1;
  p.wres_bytes = static_cast<int>(align_up(static_cast<int64_t>(p.nqd) * p.chunk_bytes, 1024));
  int64_t s = dev.sms;
  if (s > cdiv(N, kBwTB)) s = cdiv(N, kBwTB);
  p.split_len = align_up(cdiv(N, s), kBwTB);
  p.splits = static_cast<int>(cdiv(N, p.split_len));
  const int budget = dev.smem_optin - 1024;
  p.stages = 4;
  while (p.stages > 2 && tc_bwd_smem(p).total > budget) --p.stages;
  if (tc_bwd_smem(p).total > budget) return false;
  p.dx = nullptr;
  p.ws = nullptr;
  p.ws_db = nullptr;
  p.stack_dy = 0;
  p.stack_x = 0;
  return true;
}

int launch_tc_bwd(TcBwdParams p, const void *x, const void *dy, const uint8_t *wt, __half *dx,
                  __half *dW, __half *db, float *ws, const DeviceInfo &dev, cudaStream_t stream) {
  if (dev.cc_major != 10) return FEQL_ERR_UNSUPPORTED;
  p.wt = wt;
  p.dx = dx;
  p.ws = ws;
  p.ws_db = ws + static_cast<int64_t>(p.splits) * 4 * p.D * p.Cs;
  const int smem = tc_bwd_smem(p).total + 1024;
  // one load per operand and stage when the channels form whole boxes
  CUtensorMap tm_dy, tm_x;
  int st = FEQL_OK;
  p.stack_dy = make_tmap_f16_boxes(&tm_dy, dy, p.N, static_cast<int64_t>(p.D) * kT, kBwTB,
                                   p.nqd) == FEQL_OK;
  if (!p.stack_dy) st = make_tmap_f16(&tm_dy, dy, p.N, static_cast<int64_t>(p.D) * kT, kBwTB);
  if (st != FEQL_OK) return st;
  p.stack_x = make_tmap_f16_boxes(&tm_x, x, p.N, static_cast<int64_t>(p.C) * kT, kBwTB,
                                  p.nqc) == FEQL_OK;
  if (!p.stack_x) st = make_tmap_f16(&tm_x, x, p.N, static_cast<int64_t>(p.C) * kT, kBwTB);
  if (st != FEQL_OK) return st;
  // db from the dW bin-0 MMA when the last x box has a padding channel
  auto kernel = (p.C % 16) != 0 ? tc_bwd_kernel<true> : tc_bwd_kernel<false>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return FEQL_ERR_CUDA;
  kernel<<<p.splits, kBwThreads, smem, stream>>>(tm_dy, tm_x, p);
  if (cudaGetLastError() != cudaSuccess) return FEQL_ERR_CUDA;
  // the split reduce as the kernel's programmatic dependent (see tc_dw.cuh)
  {
    const int r =
        launch_dw_tc_reduce(p.ws, p.ws_db, dW, db, p.splits, p.C, p.D, p.Cs, dev.sms, stream);
    if (r != 0) return r == 1 ? FEQL_ERR_UNSUPPORTED : FEQL_ERR_CUDA;
  }
  return launch_status();
}

// ---------------------------------------------------------------------------
// Groups of order 8: C_8 and the point group D4 of p4m (fp16, tensor cores)
// ---------------------------------------------------------------------------
template <class Gp>
int launch_g8_fwd(const void *in, const uint8_t *wt, const G8Plan &P, const __half *bias,
                   void *out, int64_t N, cudaStream_t stream) {
  DeviceInfo dev;
  int st = device_info(&dev);
  if (st != FEQL_OK) return st;
  if (dev.cc_major != 10) return FEQL_ERR_UNSUPPORTED;
  G8FwdParams p;
  p.wt = wt;
  p.bias = bias;
  p.out = static_cast<__half *>(out);
  p.N = N;
  p.Ci = P.Ci;
  p.Do = P.Do;
  p.BD = P.BD;
  p.nD = P.nD;
  p.nK = P.nK;
  p.chunk_bytes = P.chunk_bytes;
  p.nM = static_cast<int>(cdiv(N, kBM));
  p.n_units = p.nM * p.nD;
  constexpr int T = Gp::kT;
  p.nacc = 2 * T * p.BD <= 512 ? 2 : 1;
  p.acc_stride = T * p.BD;
  p.stage_bytes = g8_xchunk<T>() + static_cast<int>(align_up(p.chunk_bytes, 1024));
  p.out_box = 32 * 16 * T;
  p.bias_floats = p.nD * p.BD;
  const int budget = dev.smem_optin - 1024;
  // two staging boxes per epilogue warp when a unit has few input chunks (its
  // time goes to the epilogue) or when they cost no input stage; otherwise one
  // box if that leaves room for more stages while two would leave fewer than four
  int fit[3] = {0, 0, 0};
  for (int nout = 1; nout <= kG8MaxOut; ++nout) {
    p.nout = nout;
    p.stages = 6;
    while (p.stages > 2 && g8_fwd_smem(p).total > budget) --p.stages;
    fit[nout] = g8_fwd_smem(p).total > budget ? 0 : p.stages;
  }
  p.nout = ((p.nK <= 2 && fit[2] >= 3) || fit[2] >= 4 || fit[2] >= fit[1]) ? 2 : 1;
  p.stages = fit[p.nout];
  if (p.stages == 0) return FEQL_ERR_UNSUPPORTED;
  CUtensorMap tm, tm_out;
  st = make_tmap_f16(&tm, in, N, static_cast<int64_t>(P.Ci) * T, kBM, 8 * T);
  if (st != FEQL_OK) return st;
  st = make_tmap_f16(&tm_out, out, N, static_cast<int64_t>(P.Do) * T, 32, 8 * T);
  if (st != FEQL_OK) return st;
  const int smem = g8_fwd_smem(p).total + 1024;
  if (cudaFuncSetAttribute(tc_g8_fwd_kernel<Gp>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return FEQL_ERR_CUDA;
  const int grid = p.n_units < dev.sms ? p.n_units : dev.sms;
  tc_g8_fwd_kernel<Gp><<<grid, kG8Threads, smem, stream>>>(tm, tm_out, p);
  return launch_status();
}

G8DwParams make_g8_dw_plan(int64_t N, int C, int D, int sms, int T) {
  G8DwParams p;
  p.N = N;
  p.C = C;
  p.D = D;
  p.Cs = static_cast<int>(align_up(C, 16));
  p.CT = C <= 16 ? 16 : 32;
  p.tiles_d = static_cast<int>(cdiv(D, 128));
  p.tiles_c = static_cast<int>(cdiv(C, p.CT));
  const int tiles = p.tiles_d * p.tiles_c;
  int64_t s = sms / tiles > 1 ? sms / tiles : 1;
  const int64_t chunks = cdiv(N, kG8DwTB);
  if (s > chunks) s = chunks;
  p.split_len = N > 0 ? align_up(cdiv(N, s), kG8DwTB) : kG8DwTB;
  p.splits = N > 0 ? static_cast<int>(cdiv(N, p.split_len)) : 0;
  p.slot_boxes = kG8DwDySlots + 2 * (p.CT / 16);
  p.box_bytes = kG8DwTB * 16 * T;
  p.stages = 1;
  p.stack_dy = 0;
  p.stack_x = 0;
  p.nqd_stack = 0;
  p.ws = nullptr;
  p.ws_db = nullptr;
  return p;
}

int64_t g8_dw_ws_floats(const G8DwParams &p, int T) {
  return static_cast<int64_t>(p.splits) * (static_cast<int64_t>(T) * p.D * p.Cs + p.D);
}

template <class Gp>
int launch_g8_dw(const void *x, const void *dy, __half *dW, __half *db, float *ws,
                  size_t ws_bytes, int64_t N, int C, int D, cudaStream_t stream) {
  DeviceInfo dev;
  int st = device_info(&dev);
  if (st != FEQL_OK) return st;
  if (dev.cc_major != 10) return FEQL_ERR_UNSUPPORTED;
  constexpr int T = Gp::kT;
  G8DwParams p = make_g8_dw_plan(N, C, D, dev.sms, T);
  if (ws_bytes < static_cast<size_t>(g8_dw_ws_floats(p, T)) * 4) return FEQL_ERR_INVALID_ARG;
  p.ws = ws;
  p.ws_db = ws + static_cast<int64_t>(p.splits) * T * p.D * p.Cs;
  const int budget = dev.smem_optin - 1024;
  p.stages = 4;
  while (p.stages > 1 && g8_dw_smem(p).total > budget) --p.stages;
  if (g8_dw_smem(p).total > budget) return FEQL_ERR_UNSUPPORTED;
  if (p.splits > 0) {
    CUtensorMap tm_dy, tm_x;
    // one load per operand and chunk when the channels form whole 8-channel
    // boxes (the dy stack spans the largest tile's boxes), else one per box
    const int dt0 = D < 128 ? D : 128;
    p.nqd_stack = 2 * static_cast<int>(cdiv(dt0, 16));
    p.stack_dy = make_tmap_f16_boxes(&tm_dy, dy, N, static_cast<int64_t>(D) * T, kG8DwTB,
                                     p.nqd_stack, 8 * T) == FEQL_OK;
    if (!p.stack_dy)
      st = make_tmap_f16(&tm_dy, dy, N, static_cast<int64_t>(D) * T, kG8DwTB, 8 * T);
    if (st != FEQL_OK) return st;
    p.stack_x = make_tmap_f16_boxes(&tm_x, x, N, static_cast<int64_t>(C) * T, kG8DwTB,
                                    2 * (p.CT / 16), 8 * T) == FEQL_OK;
    if (!p.stack_x) st = make_tmap_f16(&tm_x, x, N, static_cast<int64_t>(C) * T, kG8DwTB, 8 * T);
    if (st != FEQL_OK) return st;
    const int smem = g8_dw_smem(p).total + 1024;
    if (cudaFuncSetAttribute(tc_g8_dw_kernel<Gp>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return FEQL_ERR_CUDA;
    const int64_t grid = static_cast<int64_t>(p.splits) * p.tiles_d * p.tiles_c;
    if (grid > INT32_MAX) return FEQL_ERR_UNSUPPORTED;
    tc_g8_dw_kernel<Gp><<<static_cast<unsigned>(grid), kG8DwThreads, smem, stream>>>(tm_dy, tm_x, p);
  }
  const int64_t rblocks = g8_reduce_blocks(C, D);
  if (rblocks > INT32_MAX) return FEQL_ERR_UNSUPPORTED;
  g8_dw_reduce_kernel<Gp><<<static_cast<unsigned>(rblocks), kRed8Out * kRed8Groups, 0, stream>>>(
      p.ws, p.ws_db, dW, db, p.splits, C, D, p.Cs);
  return launch_status();
}

// ---------------------------------------------------------------- MLP block
// Shared memory a block may use on sm_100 (227 KB), less the base alignment.
constexpr int kMlpSmemBudget = 227 * 1024 - 1024;

// The plan depends only on (C, H, Co), so the weight buffer's layout does too.
// The widest hidden slice (fewest fc1 MMAs: the kernel is bound by its MMA
// issue) whose two fc1 accumulators and the fc2 accumulator fit 512 TMEM
// columns; for it, both layers' weights resident if they fit beside the
// buffers, else streamed per hidden slice through a ring of 3 or 2 slots; two
// x tile buffers if they fit, else one.
int plan_mlp(int C, int H, int Co, TcMlpParams *out) {
  if (align_up(Co, 16) > 96) return FEQL_ERR_UNSUPPORTED;  // fc2 accumulator: 4 * 96 columns
  const int hs_opts[4] = {64, 48, 32, 16};
  const int slot_opts[3] = {0, 3, 2};  // 0: resident
  for (int hs_max : hs_opts) {
    for (int wslots : slot_opts) {
      for (int nx = 2; nx >= 1; --nx) {
        TcMlpParams p;
        p.P = make_mlp_plan(C, H, Co, hs_max);
        p.nx = nx;
        p.wslots = wslots;
        if (mlp_tmem_cols(p.P) > 512 || mlp_smem(p).total > kMlpSmemBudget) continue;
        *out = p;
        return FEQL_OK;
      }
    }
  }
  return FEQL_ERR_UNSUPPORTED;
}

int mlp_check(int C, int H, int Co, int dtype) {
  if (!valid_dtype(dtype) || check_shape(C, H) != FEQL_OK || check_shape(H, Co) != FEQL_OK)
    return FEQL_ERR_INVALID_ARG;
  if (resolve(dtype) != FEQL_FP16) return FEQL_ERR_UNSUPPORTED;
  if ((C | Co) & 1) return FEQL_ERR_UNSUPPORTED;  // TMA rows of 8C and 8Co bytes
  return FEQL_OK;
}

int launch_mlp(const void *x, const uint8_t *wt, const __half *b1, const __half *b2, void *y,
               int64_t N, const TcMlpParams &plan, cudaStream_t stream) {
  DeviceInfo dev;
  int st = device_info(&dev);
  if (st != FEQL_OK) return st;
  if (dev.cc_major != 10) return FEQL_ERR_UNSUPPORTED;
  TcMlpParams p = plan;
  p.wt = wt;
  p.b1 = b1;
  p.b2 = b2;
  p.N = N;
  const int64_t nM = cdiv(N, kBM);
  if (nM > INT32_MAX) return FEQL_ERR_UNSUPPORTED;
  p.nM = static_cast<int>(nM);
  const int smem = mlp_smem(p).total + 1024;
  if (smem > dev.smem_optin) return FEQL_ERR_UNSUPPORTED;
  CUtensorMap tm_in, tm_out;
  st = make_tmap_f16(&tm_in, x, N, static_cast<int64_t>(p.P.C) * kT, kBM);
  if (st != FEQL_OK) return st;
  st = make_tmap_f16(&tm_out, y, N, static_cast<int64_t>(p.P.Co) * kT, 32);
  if (st != FEQL_OK) return st;
  auto kernel = p.wslots > 0 ? tc_mlp_kernel<true> : tc_mlp_kernel<false>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return FEQL_ERR_CUDA;
  const int grid = p.nM < dev.sms ? p.nM : dev.sms;
  kernel<<<grid, kMlpThreads, smem, stream>>>(tm_in, tm_out, p);
  return launch_status();
}

// Checks shared by the C_T entry points: a supported group order and mode, and
// the kernel family that serves them (T = 4 is forwarded before this).  In
// FEQL_FP16 the tensor-core kernels serve T = 8, and T = 6 when C and D are
// multiples of 4 (16-byte row strides for the tensor maps of 12-byte fibres);
// the CUDA-core kernels every order 2..16 otherwise.
enum CtPath { kCtTensor8 = 1, kCtSimt = 2, kCtTensor6 = 3 };

int ct_route(int T, int C, int D, int dtype, int *path) {
  if (!valid_dtype(dtype)) return FEQL_ERR_INVALID_ARG;
  if (T < 2 || T > kCtMaxT) return FEQL_ERR_UNSUPPORTED;
  const int dt = resolve(dtype);
  if (dt == FEQL_FP32_3XTF32) return FEQL_ERR_UNSUPPORTED;
  *path = kCtSimt;
  if (dt == FEQL_FP16 && T == 8) *path = kCtTensor8;
  if (dt == FEQL_FP16 && T == 6 && C % 4 == 0 && D % 4 == 0) *path = kCtTensor6;
  return FEQL_OK;
}

// ---------------------------------------------------------- C_T on CUDA cores
#define FEQL_CT_ORDERS(X) X(2) X(3) X(5) X(6) X(7) X(8) X(9) X(10) X(11) X(12) X(13) X(14) X(15) X(16)

template <int T, typename Ty>
int ct_simt_wfft_launch(const void *W, void *What, int C, int D, cudaStream_t s, int sms) {
  ct_simt_wfft_kernel<T, Ty><<<grid_for(static_cast<int64_t>(C) * D, 256, sms), 256, 0, s>>>(
      static_cast<const Ty *>(W), static_cast<float *>(What), C, D);
  return launch_status();
}

template <int T, typename Ty>
int ct_simt_pass_launch(const void *in, const float *Wp, const void *bias, void *out, int64_t N,
                        int Ci, int Do, cudaStream_t s) {
  const int64_t gx = cdiv(N, kCtTile);
  if (gx > INT32_MAX) return FEQL_ERR_UNSUPPORTED;
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(cdiv(Do, kCtTile)));
  if (grid.y > 65535) return FEQL_ERR_UNSUPPORTED;
  ct_simt_fwd_kernel<T, Ty><<<grid, kCtThreads, 0, s>>>(
      static_cast<const Ty *>(in), Wp, static_cast<const Ty *>(bias), static_cast<Ty *>(out), N,
      Ci, Do);
  return launch_status();
}

struct CtDwPlan {
  int tiles_d, tiles_c, splits;
  int64_t split_len;
};

// Token splits: about two blocks per SM over all (d, c) tiles, at most 64 (the
// reduce sums them serially per output).
CtDwPlan make_ct_dw_plan(int64_t N, int C, int D, int sms) {
  CtDwPlan p;
  p.tiles_d = static_cast<int>(cdiv(D, kCtTile));
  p.tiles_c = static_cast<int>(cdiv(C, kCtTile));
  int64_t s = 2 * static_cast<int64_t>(sms) / (p.tiles_d * p.tiles_c);
  if (s < 1) s = 1;
  if (s > 64) s = 64;
  const int64_t chunks = cdiv(N, kCtK);
  if (s > chunks) s = chunks;
  p.split_len = N > 0 ? align_up(cdiv(N, s), kCtK) : kCtK;
  p.splits = N > 0 ? static_cast<int>(cdiv(N, p.split_len)) : 0;
  return p;
}

int64_t ct_dw_ws_floats(const CtDwPlan &p, int T, int C, int D) {
  return static_cast<int64_t>(p.splits) * (static_cast<int64_t>(T) * D * C + D);
}

template <int T, typename Ty>
int ct_simt_dw_launch(const void *x, const void *dy, void *dW, void *db, float *ws, size_t ws_bytes,
                      int64_t N, int C, int D, cudaStream_t s, int sms) {
  const CtDwPlan p = make_ct_dw_plan(N, C, D, sms);
  if (ws_bytes < static_cast<size_t>(ct_dw_ws_floats(p, T, C, D)) * 4) return FEQL_ERR_INVALID_ARG;
  float *ws_db = ws + static_cast<int64_t>(p.splits) * T * D * C;
  if (p.splits > 0) {
    const int64_t grid = static_cast<int64_t>(p.splits) * p.tiles_d * p.tiles_c;
    if (grid > INT32_MAX) return FEQL_ERR_UNSUPPORTED;
    ct_simt_dw_kernel<T, Ty><<<static_cast<unsigned>(grid), kCtThreads, 0, s>>>(
        static_cast<const Ty *>(x), static_cast<const Ty *>(dy), ws, ws_db, N, C, D, p.split_len,
        p.tiles_d, p.tiles_c);
  }
  ct_simt_dw_reduce_kernel<T, Ty><<<grid_for(static_cast<int64_t>(D) * C + D, 256, sms), 256, 0, s>>>(
      ws, ws_db, static_cast<Ty *>(dW), static_cast<Ty *>(db), p.splits, C, D);
  return launch_status();
}

template <typename Ty>
int ct_simt_wfft(int T, const void *W, void *What, int C, int D, cudaStream_t s, int sms) {
  switch (T) {
#define FEQL_CASE(t) case t: return ct_simt_wfft_launch<t, Ty>(W, What, C, D, s, sms);
    FEQL_CT_ORDERS(FEQL_CASE)
#undef FEQL_CASE
    default: return FEQL_ERR_UNSUPPORTED;
  }
}

template <typename Ty>
int ct_simt_pass(int T, const void *in, const float *Wp, const void *bias, void *out, int64_t N,
                 int Ci, int Do, cudaStream_t s) {
  switch (T) {
#define FEQL_CASE(t) case t: return ct_simt_pass_launch<t, Ty>(in, Wp, bias, out, N, Ci, Do, s);
    FEQL_CT_ORDERS(FEQL_CASE)
#undef FEQL_CASE
    default: return FEQL_ERR_UNSUPPORTED;
  }
}

template <typename Ty>
int ct_simt_dw(int T, const void *x, const void *dy, void *dW, void *db, float *ws, size_t ws_bytes,
               int64_t N, int C, int D, cudaStream_t s, int sms) {
  switch (T) {
#define FEQL_CASE(t) \
  case t: return ct_simt_dw_launch<t, Ty>(x, dy, dW, db, ws, ws_bytes, N, C, D, s, sms);
    FEQL_CT_ORDERS(FEQL_CASE)
#undef FEQL_CASE
    default: return FEQL_ERR_UNSUPPORTED;
  }
}


// FEQL_FP16 is the one mode of the p4m kernels.
int p4m_check(int dtype) {
  if (!valid_dtype(dtype)) return FEQL_ERR_INVALID_ARG;
  if (resolve(dtype) != FEQL_FP16) return FEQL_ERR_UNSUPPORTED;
  return FEQL_OK;
}

// The order-8 entry points after their group/mode check: argument checks,
// then the templated launches.
template <class Gp>
size_t g8_weight_fft_bytes(int C, int D) {
  if (check_shape(C, D) != FEQL_OK) return 0;
  return static_cast<size_t>(make_g8_layout(C, D, Gp::kWRows).bytes);
}

template <class Gp>
int g8_weight_fft(const void *W, void *What, int C, int D, feql_stream stream) {
  if (W == nullptr || What == nullptr || check_shape(C, D) != FEQL_OK) return FEQL_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(What)) return FEQL_ERR_INVALID_ARG;
  DeviceInfo dev;
  const int st = device_info(&dev);
  if (st != FEQL_OK) return st;
  const G8Layout L = make_g8_layout(C, D, Gp::kWRows);
  wfft_g8_kernel<Gp><<<grid_for((L.fwd.bytes + L.dx.bytes) / 2, 256, dev.sms), 256, 0,
                       reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const __half *>(W), static_cast<uint8_t *>(What), L, C);
  return launch_status();
}

template <class Gp>
int g8_pass(const void *in, const void *What, const void *bias, void *out, int64_t N, int C, int D,
            feql_stream stream, int dir) {
  if (N < 0 || N > kMaxTokens || check_shape(C, D) != FEQL_OK) return FEQL_ERR_INVALID_ARG;
  if (N > 0 && (in == nullptr || What == nullptr || out == nullptr)) return FEQL_ERR_INVALID_ARG;
  if (!aligned16(in) || !aligned16(What) || !aligned16(out)) return FEQL_ERR_INVALID_ARG;
  if (bias != nullptr && !aligned16(bias)) return FEQL_ERR_INVALID_ARG;
  if (N == 0) return FEQL_OK;
  const G8Layout L = make_g8_layout(C, D, Gp::kWRows);
  const uint8_t *wt = static_cast<const uint8_t *>(What) + (dir == 0 ? L.off_fwd : L.off_dx);
  return launch_g8_fwd<Gp>(in, wt, dir == 0 ? L.fwd : L.dx, static_cast<const __half *>(bias),
                           out, N, reinterpret_cast<cudaStream_t>(stream));
}

size_t g8_dw_workspace_bytes(int64_t N, int C, int D, int T) {
  if (N < 0 || N > kMaxTokens || check_shape(C, D) != FEQL_OK) return 0;
  DeviceInfo dev;
  if (device_info(&dev) != FEQL_OK) return 0;
  return static_cast<size_t>(g8_dw_ws_floats(make_g8_dw_plan(N, C, D, dev.sms, T), T)) * 4;
}

template <class Gp>
int g8_dw(const void *x, const void *dy, void *dW, void *db, void *ws, size_t ws_bytes, int64_t N,
          int C, int D, feql_stream stream) {
  if (dW == nullptr || ws == nullptr || N < 0 || N > kMaxTokens || check_shape(C, D) != FEQL_OK)
    return FEQL_ERR_INVALID_ARG;
  if (N > 0 && (x == nullptr || dy == nullptr)) return FEQL_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(dy) || !aligned16(dW) || !aligned16(ws) ||
      (db != nullptr && !aligned16(db)))
    return FEQL_ERR_INVALID_ARG;
  return launch_g8_dw<Gp>(x, dy, static_cast<__half *>(dW), static_cast<__half *>(db),
                          static_cast<float *>(ws), ws_bytes, N, C, D,
                          reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace

// =============================================================================
extern "C" {

size_t feql_weight_fft_bytes(int C, int D, int dtype) {
  if (!valid_dtype(dtype) || check_shape(C, D) != FEQL_OK) return 0;
  return static_cast<size_t>(make_what_layout(C, D, what_kind(resolve(dtype, C, D))).bytes);
}

int feql_weight_fft(const void *W, void *What, int C, int D, int dtype, feql_stream stream) {
  if (!valid_dtype(dtype) || W == nullptr || What == nullptr) return FEQL_ERR_INVALID_ARG;
  if (check_shape(C, D) != FEQL_OK) return FEQL_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(What)) return FEQL_ERR_INVALID_ARG;
  const int dt = resolve(dtype, C, D);
  if (is_tc(dt) && ((C | D) & 1)) return FEQL_ERR_UNSUPPORTED;
  DeviceInfo dev;
  int st = device_info(&dev);
  if (st != FEQL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WhatLayout L = make_what_layout(C, D, what_kind(dt));
  if (is_tf32(dt)) {
    const int64_t words = (L.fwd.bytes + L.dx.bytes) / 4;
    wfft_tf32_kernel<<<grid_for(words, 256, dev.sms), 256, 0, s>>>(
        static_cast<const float *>(W), static_cast<uint8_t *>(What), L, C);
  } else if (is_tc(dt)) {
    const int64_t elems = (L.fwd.bytes + L.dx.bytes) / 2;
    wfft_tc_kernel<<<grid_for(elems, 256, dev.sms), 256, 0, s>>>(
        static_cast<const __half *>(W), static_cast<uint8_t *>(What), L, C);
  } else if (is_half(dt)) {
    wfft_simt_kernel<__half><<<grid_for(2ll * C * D, 256, dev.sms), 256, 0, s>>>(
        static_cast<const __half *>(W), static_cast<float *>(What), C, D);
  } else {
    wfft_simt_kernel<float><<<grid_for(2ll * C * D, 256, dev.sms), 256, 0, s>>>(
        static_cast<const float *>(W), static_cast<float *>(What), C, D);
  }
  return launch_status();
}

static int pass_common(const void *in, const void *What, const void *bias, void *out, int64_t N,
                       int C, int D, int dtype, feql_stream stream, int dir) {
  if (!valid_dtype(dtype) || N < 0 || N > kMaxTokens || check_shape(C, D) != FEQL_OK)
    return FEQL_ERR_INVALID_ARG;
  if (N > 0 && (in == nullptr || What == nullptr || out == nullptr)) return FEQL_ERR_INVALID_ARG;
  if (!aligned16(in) || !aligned16(What) || !aligned16(out)) return FEQL_ERR_INVALID_ARG;
  if (bias != nullptr && !aligned16(bias)) return FEQL_ERR_INVALID_ARG;
  const int dt = resolve(dtype, C, D);
  if (is_tc(dt) && ((C | D) & 1)) return FEQL_ERR_UNSUPPORTED;
  if (N == 0) return FEQL_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WhatLayout L = make_what_layout(C, D, what_kind(dt));
  const int Ci = dir == 0 ? C : D, Do = dir == 0 ? D : C;
  if (is_tf32(dt)) {
    const uint8_t *wt = static_cast<const uint8_t *>(What) + (dir == 0 ? L.off_fwd : L.off_dx);
    return launch_tc_gemm(in, wt, dir == 0 ? L.fwd : L.dx, bias, out, N, s, true);
  }
  if (is_tc(dt)) {
    const uint8_t *wt = static_cast<const uint8_t *>(What) + (dir == 0 ? L.off_fwd : L.off_dx);
    return launch_tc_gemm(in, wt, dir == 0 ? L.fwd : L.dx, bias, out, N, s);
  }
  const float *Wp = static_cast<const float *>(What) + (dir == 0 ? L.off_fwd : L.off_dx) / 4;
  if (is_half(dt)) return launch_simt_fwd<__half>(in, Wp, bias, out, N, Ci, Do, s);
  return launch_simt_fwd<float>(in, Wp, bias, out, N, Ci, Do, s);
}

int feql_forward(const void *x, const void *What, const void *b, void *y, int64_t N, int C, int D,
                 int dtype, feql_stream stream) {
  return pass_common(x, What, b, y, N, C, D, dtype, stream, 0);
}

int feql_backward_dx(const void *dy, const void *What, void *dx, int64_t N, int C, int D,
                     int dtype, feql_stream stream) {
  return pass_common(dy, What, nullptr, dx, N, C, D, dtype, stream, 1);
}

size_t feql_backward_dw_workspace_bytes(int64_t N, int C, int D, int dtype) {
  if (!valid_dtype(dtype) || N < 0 || N > kMaxTokens || check_shape(C, D) != FEQL_OK) return 0;
  DeviceInfo dev;
  if (device_info(&dev) != FEQL_OK) return 0;
  if (is_tc(resolve(dtype, C, D)))
    return static_cast<size_t>(tc_dw_ws_floats(make_tc_dw_plan(N, C, D, dev.sms))) * 4;
  return static_cast<size_t>(make_dw_plan(N, C, D, dev.sms).ws_floats) * 4;
}

int feql_backward(const void *x, const void *dy, const void *What, void *dx, void *dW, void *db,
                  void *ws, size_t ws_bytes, int64_t N, int C, int D, int dtype,
                  feql_stream stream) {
  if (!valid_dtype(dtype) || dW == nullptr || ws == nullptr) return FEQL_ERR_INVALID_ARG;
  if (N < 0 || N > kMaxTokens || check_shape(C, D) != FEQL_OK) return FEQL_ERR_INVALID_ARG;
  if (N > 0 && (x == nullptr || dy == nullptr || What == nullptr || dx == nullptr))
    return FEQL_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(dy) || !aligned16(What) || !aligned16(dx) || !aligned16(dW) ||
      !aligned16(ws) || (db != nullptr && !aligned16(db)))
    return FEQL_ERR_INVALID_ARG;
  const int dt = resolve(dtype, C, D);
  if (is_tc(dt) && ((C | D) & 1)) return FEQL_ERR_UNSUPPORTED;
  DeviceInfo dev;
  int st = device_info(&dev);
  if (st != FEQL_OK) return st;
  if (is_tc(dt) && N > 0) {
    const WhatLayout L = make_what_layout(C, D, true);
    TcBwdParams p;
    if (make_tc_bwd_plan(N, C, D, L, dev, p)) {
      // the regular dW workspace always covers the fused plan (no more splits)
      if (ws_bytes < static_cast<size_t>(p.splits) * (4ull * p.D * p.Cs + p.D) * 4)
        return FEQL_ERR_INVALID_ARG;
      return launch_tc_bwd(p, x, dy, static_cast<const uint8_t *>(What) + L.off_dx,
                           static_cast<__half *>(dx), static_cast<__half *>(dW),
                           static_cast<__half *>(db), static_cast<float *>(ws), dev,
                           reinterpret_cast<cudaStream_t>(stream));
    }
  }
  st = feql_backward_dx(dy, What, dx, N, C, D, dtype, stream);
  if (st != FEQL_OK) return st;
  return feql_backward_dw(x, dy, dW, db, ws, ws_bytes, N, C, D, dtype, stream);
}

int feql_backward_dw(const void *x, const void *dy, void *dW, void *db, void *ws, size_t ws_bytes,
                     int64_t N, int C, int D, int dtype, feql_stream stream) {
  if (!valid_dtype(dtype) || dW == nullptr || ws == nullptr) return FEQL_ERR_INVALID_ARG;
  if (N < 0 || N > kMaxTokens || check_shape(C, D) != FEQL_OK) return FEQL_ERR_INVALID_ARG;
  if (N > 0 && (x == nullptr || dy == nullptr)) return FEQL_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(dy) || !aligned16(dW) || !aligned16(ws))
    return FEQL_ERR_INVALID_ARG;
  if (db != nullptr && !aligned16(db)) return FEQL_ERR_INVALID_ARG;
  // split-TF32 mode: the weight gradient runs on the fp32 CUDA-core kernels
  const int dt = resolve(dtype, C, D);
  if (is_tc(dt) && ((C | D) & 1)) return FEQL_ERR_UNSUPPORTED;
  DeviceInfo dev;
  int st = device_info(&dev);
  if (st != FEQL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (is_tc(dt)) {
    TcDwParams p = make_tc_dw_plan(N, C, D, dev.sms);
    if (ws_bytes < static_cast<size_t>(tc_dw_ws_floats(p)) * 4) return FEQL_ERR_INVALID_ARG;
    return launch_tc_dw(p, x, dy, static_cast<__half *>(dW), static_cast<__half *>(db),
                        static_cast<float *>(ws), dev, s);
  }
  const DwPlan q = make_dw_plan(N, C, D, dev.sms);
  if (ws_bytes < static_cast<size_t>(q.ws_floats) * 4) return FEQL_ERR_INVALID_ARG;
  float *wsf = static_cast<float *>(ws);
  float *wsdb = wsf + static_cast<int64_t>(q.splits) * 4 * C * D;
  dim3 grid(static_cast<unsigned>(cdiv(D, kSimtTile)), static_cast<unsigned>(cdiv(C, kSimtTile)),
            static_cast<unsigned>(q.splits));
  if (grid.y > 65535) return FEQL_ERR_UNSUPPORTED;
  const int64_t red = static_cast<int64_t>(C) * D + D;
  if (is_half(dt)) {
    simt_dw_partial_kernel<__half><<<grid, kSimtThreads, 0, s>>>(
        static_cast<const __half *>(x), static_cast<const __half *>(dy), wsf, wsdb, N, C, D,
        q.split_len);
    dw_reduce_kernel<__half><<<grid_for(red, 256, dev.sms), 256, 0, s>>>(
        wsf, wsdb, static_cast<__half *>(dW), static_cast<__half *>(db), q.splits, C, D);
  } else {
    simt_dw_partial_kernel<float><<<grid, kSimtThreads, 0, s>>>(
        static_cast<const float *>(x), static_cast<const float *>(dy), wsf, wsdb, N, C, D,
        q.split_len);
    dw_reduce_kernel<float><<<grid_for(red, 256, dev.sms), 256, 0, s>>>(
        wsf, wsdb, static_cast<float *>(dW), static_cast<float *>(db), q.splits, C, D);
  }
  return launch_status();
}

// ---------------------------------------------------------------------------
// Cyclic group C_T
// ---------------------------------------------------------------------------
size_t feql_ct_weight_fft_bytes(int T, int C, int D, int dtype) {
  if (T == 4) return feql_weight_fft_bytes(C, D, dtype);
  int path = 0;
  if (ct_route(T, C, D, dtype, &path) != FEQL_OK || check_shape(C, D) != FEQL_OK) return 0;
  if (path == kCtTensor8) return g8_weight_fft_bytes<Cyclic8>(C, D);
  if (path == kCtTensor6) return g8_weight_fft_bytes<Cyclic6>(C, D);
  return static_cast<size_t>(2) * T * C * D * 4;  // fp32 planes [dir][plane][Do][Ci]
}

int feql_ct_weight_fft(int T, const void *W, void *What, int C, int D, int dtype,
                       feql_stream stream) {
  if (T == 4) return feql_weight_fft(W, What, C, D, dtype, stream);
  int path = 0;
  int st = ct_route(T, C, D, dtype, &path);
  if (st != FEQL_OK) return st;
  if (path == kCtTensor8) return g8_weight_fft<Cyclic8>(W, What, C, D, stream);
  if (path == kCtTensor6) return g8_weight_fft<Cyclic6>(W, What, C, D, stream);
  if (W == nullptr || What == nullptr || check_shape(C, D) != FEQL_OK) return FEQL_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(What)) return FEQL_ERR_INVALID_ARG;
  DeviceInfo dev;
  st = device_info(&dev);
  if (st != FEQL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return is_half(resolve(dtype)) ? ct_simt_wfft<__half>(T, W, What, C, D, s, dev.sms)
                                 : ct_simt_wfft<float>(T, W, What, C, D, s, dev.sms);
}

static int ct_pass(int T, const void *in, const void *What, const void *bias, void *out, int64_t N,
                   int C, int D, int dtype, feql_stream stream, int dir) {
  int path = 0;
  const int st = ct_route(T, C, D, dtype, &path);
  if (st != FEQL_OK) return st;
  if (path == kCtTensor8) return g8_pass<Cyclic8>(in, What, bias, out, N, C, D, stream, dir);
  if (path == kCtTensor6) return g8_pass<Cyclic6>(in, What, bias, out, N, C, D, stream, dir);
  if (N < 0 || N > kMaxTokens || check_shape(C, D) != FEQL_OK) return FEQL_ERR_INVALID_ARG;
  if (N > 0 && (in == nullptr || What == nullptr || out == nullptr)) return FEQL_ERR_INVALID_ARG;
  if (!aligned16(in) || !aligned16(What) || !aligned16(out)) return FEQL_ERR_INVALID_ARG;
  if (bias != nullptr && !aligned16(bias)) return FEQL_ERR_INVALID_ARG;
  if (N == 0) return FEQL_OK;
  const float *Wp = static_cast<const float *>(What) + (dir == 0 ? 0 : static_cast<int64_t>(T) * C * D);
  const int Ci = dir == 0 ? C : D, Do = dir == 0 ? D : C;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return is_half(resolve(dtype)) ? ct_simt_pass<__half>(T, in, Wp, bias, out, N, Ci, Do, s)
                                 : ct_simt_pass<float>(T, in, Wp, bias, out, N, Ci, Do, s);
}

int feql_ct_forward(int T, const void *x, const void *What, const void *b, void *y, int64_t N,
                    int C, int D, int dtype, feql_stream stream) {
  if (T == 4) return feql_forward(x, What, b, y, N, C, D, dtype, stream);
  return ct_pass(T, x, What, b, y, N, C, D, dtype, stream, 0);
}

int feql_ct_backward_dx(int T, const void *dy, const void *What, void *dx, int64_t N, int C, int D,
                        int dtype, feql_stream stream) {
  if (T == 4) return feql_backward_dx(dy, What, dx, N, C, D, dtype, stream);
  return ct_pass(T, dy, What, nullptr, dx, N, C, D, dtype, stream, 1);
}

size_t feql_ct_backward_dw_workspace_bytes(int T, int64_t N, int C, int D, int dtype) {
  if (T == 4) return feql_backward_dw_workspace_bytes(N, C, D, dtype);
  int path = 0;
  if (ct_route(T, C, D, dtype, &path) != FEQL_OK) return 0;
  if (path == kCtTensor8) return g8_dw_workspace_bytes(N, C, D, 8);
  if (path == kCtTensor6) return g8_dw_workspace_bytes(N, C, D, 6);
  if (N < 0 || N > kMaxTokens || check_shape(C, D) != FEQL_OK) return 0;
  DeviceInfo dev;
  if (device_info(&dev) != FEQL_OK) return 0;
  return static_cast<size_t>(ct_dw_ws_floats(make_ct_dw_plan(N, C, D, dev.sms), T, C, D)) * 4;
}

int feql_ct_backward_dw(int T, const void *x, const void *dy, void *dW, void *db, void *ws,
                        size_t ws_bytes, int64_t N, int C, int D, int dtype, feql_stream stream) {
  if (T == 4) return feql_backward_dw(x, dy, dW, db, ws, ws_bytes, N, C, D, dtype, stream);
  int path = 0;
  int st = ct_route(T, C, D, dtype, &path);
  if (st != FEQL_OK) return st;
  if (path == kCtTensor8) return g8_dw<Cyclic8>(x, dy, dW, db, ws, ws_bytes, N, C, D, stream);
  if (path == kCtTensor6) return g8_dw<Cyclic6>(x, dy, dW, db, ws, ws_bytes, N, C, D, stream);
  if (dW == nullptr || ws == nullptr || N < 0 || N > kMaxTokens || check_shape(C, D) != FEQL_OK)
    return FEQL_ERR_INVALID_ARG;
  if (N > 0 && (x == nullptr || dy == nullptr)) return FEQL_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(dy) || !aligned16(dW) || !aligned16(ws) ||
      (db != nullptr && !aligned16(db)))
    return FEQL_ERR_INVALID_ARG;
  DeviceInfo dev;
  st = device_info(&dev);
  if (st != FEQL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float *w = static_cast<float *>(ws);
  return is_half(resolve(dtype))
             ? ct_simt_dw<__half>(T, x, dy, dW, db, w, ws_bytes, N, C, D, s, dev.sms)
             : ct_simt_dw<float>(T, x, dy, dW, db, w, ws_bytes, N, C, D, s, dev.sms);
}

// ---------------------------------------------------------------------------
// p4m (point group D4)
// ---------------------------------------------------------------------------
size_t feql_p4m_weight_fft_bytes(int C, int D, int dtype) {
  if (p4m_check(dtype) != FEQL_OK) return 0;
  return g8_weight_fft_bytes<Dihedral4>(C, D);
}

int feql_p4m_weight_fft(const void *W, void *What, int C, int D, int dtype, feql_stream stream) {
  const int st = p4m_check(dtype);
  if (st != FEQL_OK) return st;
  return g8_weight_fft<Dihedral4>(W, What, C, D, stream);
}

int feql_p4m_forward(const void *x, const void *What, const void *b, void *y, int64_t N, int C,
                     int D, int dtype, feql_stream stream) {
  const int st = p4m_check(dtype);
  if (st != FEQL_OK) return st;
  return g8_pass<Dihedral4>(x, What, b, y, N, C, D, stream, 0);
}

int feql_p4m_backward_dx(const void *dy, const void *What, void *dx, int64_t N, int C, int D,
                         int dtype, feql_stream stream) {
  const int st = p4m_check(dtype);
  if (st != FEQL_OK) return st;
  return g8_pass<Dihedral4>(dy, What, nullptr, dx, N, C, D, stream, 1);
}

size_t feql_p4m_backward_dw_workspace_bytes(int64_t N, int C, int D, int dtype) {
  if (p4m_check(dtype) != FEQL_OK) return 0;
  return g8_dw_workspace_bytes(N, C, D, 8);
}

int feql_p4m_backward_dw(const void *x, const void *dy, void *dW, void *db, void *ws,
                         size_t ws_bytes, int64_t N, int C, int D, int dtype, feql_stream stream) {
  const int st = p4m_check(dtype);
  if (st != FEQL_OK) return st;
  return g8_dw<Dihedral4>(x, dy, dW, db, ws, ws_bytes, N, C, D, stream);
}

size_t feql_mlp_weight_fft_bytes(int C, int H, int Co, int dtype) {
  TcMlpParams p;
  if (mlp_check(C, H, Co, dtype) != FEQL_OK || plan_mlp(C, H, Co, &p) != FEQL_OK) return 0;
  return static_cast<size_t>(p.P.bytes);
}

int feql_mlp_weight_fft(const void *W1, const void *W2, void *What, int C, int H, int Co,
                        int dtype, feql_stream stream) {
  int st = mlp_check(C, H, Co, dtype);
  if (st != FEQL_OK) return st;
  if (W1 == nullptr || W2 == nullptr || What == nullptr) return FEQL_ERR_INVALID_ARG;
  if (!aligned16(W1) || !aligned16(W2) || !aligned16(What)) return FEQL_ERR_INVALID_ARG;
  TcMlpParams p;
  st = plan_mlp(C, H, Co, &p);
  if (st != FEQL_OK) return st;
  DeviceInfo dev;
  st = device_info(&dev);
  if (st != FEQL_OK) return st;
  wfft_mlp_kernel<<<grid_for((p.P.w1_bytes + p.P.w2_bytes) / 2, 256, dev.sms), 256, 0,
                    reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const __half *>(W1), static_cast<const __half *>(W2),
      static_cast<uint8_t *>(What), p.P);
  return launch_status();
}

int feql_mlp_forward(const void *x, const void *What, const void *b1, const void *b2, void *y,
                     int64_t N, int C, int H, int Co, int dtype, feql_stream stream) {
  int st = mlp_check(C, H, Co, dtype);
  if (st != FEQL_OK) return st;
  if (N < 0 || N > kMaxTokens) return FEQL_ERR_INVALID_ARG;
  if (N > 0 && (x == nullptr || What == nullptr || y == nullptr)) return FEQL_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(What) || !aligned16(y) || (b1 != nullptr && !aligned16(b1)) ||
      (b2 != nullptr && !aligned16(b2)))
    return FEQL_ERR_INVALID_ARG;
  TcMlpParams p;
  st = plan_mlp(C, H, Co, &p);
  if (st != FEQL_OK) return st;
  if (N == 0) return FEQL_OK;
  return launch_mlp(x, static_cast<const uint8_t *>(What), static_cast<const __half *>(b1),
                    static_cast<const __half *>(b2), y, N, p,
                    reinterpret_cast<cudaStream_t>(stream));
}

int feql_device_status(feql_stream stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return FEQL_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, feql::g_status, sizeof(v)) != cudaSuccess) return FEQL_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(feql::g_status, &zero, sizeof(zero)) != cudaSuccess)
    return FEQL_ERR_CUDA;
  return (v & kStatusTimeout) ? FEQL_ERR_TIMEOUT : FEQL_OK;
}

const char *feql_status_string(int status) {
  switch (status) {
    case FEQL_OK: return "ok";
    case FEQL_ERR_INVALID_ARG: return "invalid argument";
    case FEQL_ERR_UNSUPPORTED: return "unsupported shape or mode";
    case FEQL_ERR_CUDA: return "CUDA error";
    case FEQL_ERR_TIMEOUT: return "device-side bounded wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"

// =============================================================================
// Weight gradient without caller-provided scratch.
//
// Some callers cannot allocate device memory at the point where they need the
// weight gradient: code running inside a framework that owns every allocation
// (a custom allocator or a memory pool that must not grow), plug-ins whose
// host can only hand over the input and output tensors, or runtimes that
// forbid allocation after start-up.  feql_backward_dw needs a split-K
// workspace; this variant takes it from a fixed array that lives in the
// library's device image instead.
//
// The array is a file-scope __device__ object of kNoAllocScratchBytes.  Every
// GPU that loads the library holds it until the process exits.  In host code
// its name is only a host-side stand-in, so the device address is looked up
// with cudaGetSymbolAddress, once per device, by the first call made with that
// device current (make that first call before any stream capture).  The array
// is shared by all calls: calls that overlap on the GPU (different streams,
// threads) race on it and must be serialised by the caller.  Nothing in it
// needs clearing between calls — every element the reduction reads is written
// earlier in the same call — so it simply keeps the last call's partial sums.
// No cudaMalloc, cudaFree or other allocating routine is called.
// =============================================================================
namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(16) << 20;  // 16 MiB

std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices];

}  // namespace

static __device__ __align__(256) unsigned char g_dw_scratch[kNoAllocScratchBytes];

namespace {

// Device address of g_dw_scratch on the current device (looked up once per device).
int noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FEQL_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dw_scratch) != cudaSuccess || p == nullptr) return FEQL_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return FEQL_OK;
}

}  // namespace

extern "C" int feql_backward_dw_noalloc(const void *x, const void *dy, void *dW, void *db,
                                        int64_t N, int C, int D, int dtype, feql_stream stream) {
  if (!valid_dtype(dtype) || dW == nullptr) return FEQL_ERR_INVALID_ARG;
  if (N < 0 || N > kMaxTokens || check_shape(C, D) != FEQL_OK) return FEQL_ERR_INVALID_ARG;
  if (N > 0 && (x == nullptr || dy == nullptr)) return FEQL_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(dy) || !aligned16(dW)) return FEQL_ERR_INVALID_ARG;
  if (db != nullptr && !aligned16(db)) return FEQL_ERR_INVALID_ARG;
  if (resolve(dtype) != FEQL_FP16) return FEQL_ERR_UNSUPPORTED;  // tensor-core fp16 path only
  if ((C | D) & 1) return FEQL_ERR_UNSUPPORTED;
  DeviceInfo dev;
  int st = device_info(&dev);
  if (st != FEQL_OK) return st;
  TcDwParams p = make_tc_dw_plan(N, C, D, dev.sms);
  // One token split needs 4*D*Cs + D floats of partial sums; if even one does
  // not fit, the shape is rejected.  Otherwise use as many splits as fit (the
  // regular plan's count when it fits, fewer — slower, and summed in a
  // different grouping — if not).
  const int64_t cap = static_cast<int64_t>(kNoAllocScratchBytes / 4);
  const int64_t per_split = 4ll * p.D * p.Cs + p.D;
  if (per_split > cap) return FEQL_ERR_UNSUPPORTED;
  if (tc_dw_ws_floats(p) > cap) {
    const int64_t max_splits = cap / per_split;
    p.split_len = align_up(cdiv(N > 0 ? N : 1, max_splits), p.TB);
    p.splits = static_cast<int>(cdiv(N > 0 ? N : 1, p.split_len));
  }
  // the kernels index the array by split: never launch a plan that outgrows it
  if (tc_dw_ws_floats(p) > cap) return FEQL_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != FEQL_OK) return st;
  return launch_tc_dw(p, x, dy, static_cast<__half *>(dW), static_cast<__half *>(db),
                      static_cast<float *>(scratch), dev, reinterpret_cast<cudaStream_t>(stream));
}
