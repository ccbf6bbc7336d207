/*
 * feql.h — C ABI of the B200 (sm_100a) p4 Flash EQ-Linear library (libfeql.so).
 *
 * The layer (Flash EQ-Linear, technical summary "Intuizione Centrale"; arXiv
 * abstract): the p4 equivariant linear layer is a circular convolution along
 * the group axis (T = 4) composed with a linear map along the channels,
 *
 *     y[n,d,t] = b[d] + sum_c sum_s W[d,c,(t-s) mod 4] * x[n,c,s],
 *
 * computed exactly through a real DFT along the group axis: bins 0 and 2 are
 * real channel contractions and bin 1 is one complex contraction (bin 3 is its
 * conjugate), six real GEMMs of N x C x D instead of sixteen (technical
 * summary "Specializzazione per il Gruppo di Rotazione p4"; abstract, cost
 * 2(T-1)/T^2 of the dense form).
 *
 * Layouts (all row-major, contiguous, group index innermost):
 *     x  [N][C][4]     y  [N][D][4]     W  [D][C][4]     b [D]
 *     dy [N][D][4]     dx [N][C][4]     dW [D][C][4]     db [D]
 * C and D count channels per group element (the unrolled widths are 4C, 4D).
 *
 * Conventions shared by every entry point:
 *  - Every data pointer is a DEVICE pointer on the current CUDA device,
 *    owned by the caller; the library allocates no device memory and keeps no
 *    per-call state (it caches only per-device properties).
 *  - Calls only enqueue work on `stream` (NULL = legacy default stream) and
 *    never synchronise, except feql_device_status.
 *  - Element type of x, y, W, b, dy, dx, dW, db follows `dtype`:
 *    FEQL_FP16* -> IEEE binary16, FEQL_FP32* -> binary32.  Accumulation is
 *    fp32 in every mode.
 *  - Pointers must be 16-byte aligned.  Inputs and outputs must not overlap.
 *  - Return value: FEQL_OK, or an feql_status code; on an error nothing is
 *    enqueued (FEQL_ERR_CUDA: a launch failed; see feql_status_string).
 *  - N == 0 is a valid no-op (for feql_backward_dw it zeroes dW and db); the
 *    token-indexed pointers (x, y, dy, dx) may then be NULL.
 *  - Value range (FEQL_FP16): every finite fp16 x, dy and W is accepted.  The
 *    group-axis sums of the transform reach |G| max|v| (G the group: 4 for p4,
 *    6 for C_6, 8 for C_8 and p4m), so the fp16 operand planes and Fourier
 *    weights hold every bin divided by 4 (p4) or 8 (the others: an exact power
 *    of two that the fp32 epilogues undo); results are within the fp16 mode's
 *    tolerance whenever the outputs y, dx, dW and db themselves are finite in
 *    fp16 (an output beyond 65504 becomes inf, as in any fp16 layer).  The MLP
 *    block likewise accepts every finite x, W1, W2, b1, b2 whose hidden
 *    activation h and output y are finite in fp16 (its hidden planes hold
 *    GELU(h) / 4).  Where a scaled value falls among the fp16 subnormals (below
 *    2^-14) it is rounded to the subnormal spacing 2^-24, at most twice per
 *    butterfly stage: an absolute error per bin of at most 2^-21 for p4 and
 *    2^-19 for the order-6 and -8 groups.
 */
#ifndef FEQL_H
#define FEQL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *feql_stream;

/* Arithmetic mode. */
typedef enum {
  FEQL_FP16 = 0,        /* fp16 data, fp32 accumulate, tcgen05 tensor cores */
  FEQL_FP32 = 1,        /* fp32 data; the p4 layer takes FEQL_FP32_3XTF32 when C, D <= 512,
                           else FEQL_FP32_SIMT (every other entry point: FEQL_FP32_SIMT) */
  FEQL_FP32_SIMT = 2,   /* fp32 data, fp32 FMA on CUDA cores */
  FEQL_FP32_3XTF32 = 3, /* fp32 data, split TF32 on the tensor cores: each operand is its
                           tf32 rounding (hi) plus the rounded remainder (lo), three tf32
                           products hi*hi + hi*lo + lo*hi per product (Ootomo and Yokota),
                           fp32 accumulation; forward and dX of the p4 layer (dW and db run
                           on the fp32 CUDA-core kernels) */
  FEQL_FP16_SIMT = 4    /* fp16 data, fp32 FMA on CUDA cores (cross-check path) */
} feql_dtype;

typedef enum {
  FEQL_OK = 0,
  FEQL_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad dtype, misaligned, workspace too small */
  FEQL_ERR_UNSUPPORTED = 2, /* shape/mode the kernels do not cover (e.g. odd C or D in fp16) */
  FEQL_ERR_CUDA = 3,        /* a CUDA runtime/driver call or a launch failed */
  FEQL_ERR_TIMEOUT = 4      /* a kernel's bounded wait expired (reported by feql_device_status) */
} feql_status;

/* Size in bytes of the opaque Fourier-weight buffer What for (C, D, dtype);
 * 0 on invalid arguments.  The layout is private to the library and depends
 * only on (C, D, dtype). */
size_t feql_weight_fft_bytes(int C, int D, int dtype);

/* a1 — weight transform, run once per weight update (technical summary
 * "Approccio Algoritmico": the convolution theorem needs W in the Fourier
 * domain).  Computes the non-redundant bins of the 4-point real DFT of W
 * along the group axis,
 *     What0 = W0+W1+W2+W3,  What2 = W0-W1+W2-W3,  What1 = (W0-W2) + i(W3-W1),
 * and stores them, for both the forward and the dX pass (conjugated and
 * transposed), in the kernels' tile layout.
 *   W    : device, [D][C][4] of dtype (read only)
 *   What : device, feql_weight_fft_bytes(C, D, dtype) bytes (written)
 */
int feql_weight_fft(const void *W, void *What, int C, int D, int dtype, feql_stream stream);

/* a2–a4 — forward: 4-point rDFT of x along the group axis, the six real
 * per-frequency channel contractions, inverse rDFT, + bias; the Fourier
 * intermediates never leave the chip (technical summary "Implementazione":
 * fused dataflow without intermediate global writes).
 *   x    : device [N][C][4]           What : from feql_weight_fft (same C, D, dtype)
 *   b    : device [D] or NULL (no bias)
 *   y    : device [N][D][4] (written)
 */
int feql_forward(const void *x, const void *What, const void *b, void *y,
                 int64_t N, int C, int D, int dtype, feql_stream stream);

/* a5 — backward input gradient: dx[n,c,s] = sum_{d,t} W[d,c,(t-s) mod 4] dy[n,d,t],
 * the same structure as the forward with conj(What)^T (contraction over D),
 * no bias.
 *   dy : device [N][D][4]   dx : device [N][C][4] (written) */
int feql_backward_dx(const void *dy, const void *What, void *dx,
                     int64_t N, int C, int D, int dtype, feql_stream stream);

/* Workspace (bytes) feql_backward_dw needs for these sizes on the current device. */
size_t feql_backward_dw_workspace_bytes(int64_t N, int C, int D, int dtype);

/* a6 — backward weight gradient of the loss <dy, y>:
 *     dW[d,c,u] = sum_n sum_t dy[n,d,t] x[n,c,(t-u) mod 4],   db[d] = sum_{n,t} dy[n,d,t].
 * Per frequency bin G_k[d,c] = sum_n dY_k[n,d] conj(X_k[n,c]) is accumulated
 * over N in a split-K reduction, reduced in a fixed order (bit-identical run
 * to run), then inverse-transformed.
 *   x  : device [N][C][4]    dy : device [N][D][4]
 *   dW : device [D][C][4] (written)    db : device [D] or NULL (written)
 *   ws : device scratch of ws_bytes >= feql_backward_dw_workspace_bytes(...) */
int feql_backward_dw(const void *x, const void *dy, void *dW, void *db,
                     void *ws, size_t ws_bytes,
                     int64_t N, int C, int D, int dtype, feql_stream stream);

/* a5 + a6 fused — both gradients from one pass over dy (technical summary
 * "Implementazione": fused dataflow; dX and dW share the rDFT of dy):
 * the results of feql_backward_dx followed by feql_backward_dw, reading x and
 * dy once instead of dy twice.  Fused for FEQL_FP16 with C <= 64, D <= 128
 * (one dW tile, one dX output tile: the bench's Swin-like layer); any other
 * shape or mode runs the two separate passes and returns their result.
 *   x, dy, What : as for feql_backward_dx / feql_backward_dw
 *   dx  : device [N][C][4] (written)   dW : [D][C][4]   db : [D] or NULL
 *   ws  : ws_bytes >= feql_backward_dw_workspace_bytes(N, C, D, dtype) */
int feql_backward(const void *x, const void *dy, const void *What, void *dx, void *dW, void *db,
                  void *ws, size_t ws_bytes, int64_t N, int C, int D, int dtype,
                  feql_stream stream);

/* Weight gradient for callers that cannot allocate device memory (code inside
 * a framework that owns every allocation, plug-ins that are handed only their
 * input and output tensors, runtimes that forbid allocation after start-up).
 * The paper has no counterpart: this is a library convenience.
 * Same arguments and results as feql_backward_dw in FEQL_FP16 mode, minus the
 * workspace: the split-K partial sums go to a fixed 16 MiB array inside the
 * library's device image, which every GPU that loads the library keeps until
 * the process exits.  Allocates nothing.
 *  - Limit: one token split needs (4*D*roundup(C,16) + D) * 4 bytes of
 *    partial sums; shapes where that exceeds 16 MiB (e.g. C = D = 1024) get
 *    FEQL_ERR_UNSUPPORTED without anything launched, as do modes other than
 *    FEQL_FP16 and odd C or D.  When the regular split count does not fit,
 *    fewer splits are used: less parallelism, and the fp32 partial sums are
 *    grouped differently (results agree to rounding, not bit for bit).
 *  - The first call on a device looks up the array's device address (make it
 *    before any stream capture).
 *  - All calls share the one array: calls that overlap on the GPU race and
 *    must be serialised by the caller.  No state carries over between calls. */
int feql_backward_dw_noalloc(const void *x, const void *dy, void *dW, void *db,
                             int64_t N, int C, int D, int dtype, feql_stream stream);

/* ---------------------------------------------------------------------------
 * Cyclic group C_T of order T (Flash EQ-Linear, arXiv abstract: the method for
 * a group of size T costs 2(T-1)/T^2 of the dense layer; the paper's kernels
 * are for p4).  Tensors as above with the group axis of length T:
 * x[N][C][T], y[N][D][T], W[D][C][T], dW[D][C][T]; b, db [D].
 *   y[n,d,t] = b[d] + sum_c sum_s W[d,c,(t-s) mod T] x[n,c,s]
 * T = 4 is the p4 layer: every call forwards to the function above with the
 * same arguments (all modes).  T = 8 in FEQL_FP16: tensor-core kernels (bins 0
 * and 4 real, 1..3 complex, 14 real products instead of 64).  T = 6 in
 * FEQL_FP16 with C and D multiples of 4: the same tensor-core kernels with the
 * order-6 twiddles (bins 0 and 3 real, 1 and 2 complex, 10 real products
 * instead of 36; the 12-byte fibres need 16-byte row strides).  Every order
 * 2 <= T <= 16 in FEQL_FP32 / FEQL_FP32_SIMT / FEQL_FP16_SIMT, and in
 * FEQL_FP16 for the other orders and shapes: CUDA-core kernels of the same method
 * with the DFT twiddles of order T (non-dyadic for T = 3, 5, 6, 7, 12 ...;
 * (2T-2)/T^2 or, for odd T, (2T-1)/T^2 of the dense products), fp32
 * arithmetic on fp32 or fp16 data.  FEQL_FP32_3XTF32 and orders outside 2..16
 * return FEQL_ERR_UNSUPPORTED.  Any C, D >= 1.  Argument checks, N == 0,
 * ownership, streams and errors are as for the p4 functions; the Fourier
 * buffer has its own layout and size per (T, dtype) (feql_ct_weight_fft_bytes). */
size_t feql_ct_weight_fft_bytes(int T, int C, int D, int dtype);
int feql_ct_weight_fft(int T, const void *W, void *What, int C, int D, int dtype,
                       feql_stream stream);
int feql_ct_forward(int T, const void *x, const void *What, const void *b, void *y, int64_t N,
                    int C, int D, int dtype, feql_stream stream);
int feql_ct_backward_dx(int T, const void *dy, const void *What, void *dx, int64_t N, int C,
                        int D, int dtype, feql_stream stream);
size_t feql_ct_backward_dw_workspace_bytes(int T, int64_t N, int C, int D, int dtype);
int feql_ct_backward_dw(int T, const void *x, const void *dy, void *dW, void *db, void *ws,
                        size_t ws_bytes, int64_t N, int C, int D, int dtype, feql_stream stream);

/* ---------------------------------------------------------------------------
 * The wallpaper group p4m: rotations by 90 degrees and reflections, point group
 * D4 of order 8 (Flash EQ-Linear, technical summary "Limitazioni e Lavoro
 * Futuro": reflection groups are the named next step).  Group element
 * g = (r, m), rotation by r * 90 degrees after the reflection m, stored at index
 * 4 m + r of the group axis: x[N][C][8], y[N][D][8], W[D][C][8], dW[D][C][8].
 * The layer is the group convolution
 *   y[n,d,g] = b[d] + sum_c sum_h W[d,c,h^-1 g] x[n,c,h],
 *   (r1, m1)(r2, m2) = (r1 + (-1)^m1 r2 mod 4, m1 xor m2),
 * which on the rotations alone is the p4 layer.  D4 is not abelian: its Fourier
 * transform has four 1-dim irreps and one 2-dim irrep E, so per token the layer
 * is four scalar channel contractions and one 2 x 2 block contraction, 12 real
 * products of N x C x D instead of the 64 of the unrolled matrix (forward:
 * y^ = x^ W^; dX: dx^ = dy^ W^^T; dW: dW^ = x^^T dy^ summed over tokens).
 * FEQL_FP16 only (other modes FEQL_ERR_UNSUPPORTED); any C, D >= 1.  Argument
 * checks, N == 0, ownership, streams and errors are as for the p4 functions;
 * the Fourier buffer has its own layout (feql_p4m_weight_fft_bytes). */
size_t feql_p4m_weight_fft_bytes(int C, int D, int dtype);
int feql_p4m_weight_fft(const void *W, void *What, int C, int D, int dtype, feql_stream stream);
int feql_p4m_forward(const void *x, const void *What, const void *b, void *y, int64_t N, int C,
                     int D, int dtype, feql_stream stream);
int feql_p4m_backward_dx(const void *dy, const void *What, void *dx, int64_t N, int C, int D,
                         int dtype, feql_stream stream);
size_t feql_p4m_backward_dw_workspace_bytes(int64_t N, int C, int D, int dtype);
int feql_p4m_backward_dw(const void *x, const void *dy, void *dW, void *db, void *ws,
                         size_t ws_bytes, int64_t N, int C, int D, int dtype, feql_stream stream);

/* ---------------------------------------------------------------------------
 * p4-equivariant MLP block, forward (Flash EQ-Linear, technical summary
 * "Livello di Rete": the EQ-ViT / EQ-Swin networks built from the layer; their
 * MLP is two EQ-Linear layers around a pointwise GELU):
 *   h[n,j,t] = b1[j] + sum_c sum_s W1[j,c,(t-s) mod 4] x[n,c,s]        fc1: C -> H
 *   y[n,o,t] = b2[o] + sum_j sum_s W2[o,j,(t-s) mod 4] GELU(h[n,j,s])   fc2: H -> Co
 * in one kernel: the hidden activation h never goes to device memory.  GELU is
 * evaluated in its tanh form (within 5e-4 of the exact z*Phi(z)) on fp16 values.
 *   x  : device [N][C][4]     y : device [N][Co][4] (written)
 *   W1 : device [H][C][4]     b1: device [H] or NULL
 *   W2 : device [Co][H][4]    b2: device [Co] or NULL
 * FEQL_FP16 only (other modes FEQL_ERR_UNSUPPORTED).  C and Co even; Co <= 96;
 * one 128-token tile of x (C rounded up to 16 channels, 2 KB per channel) must
 * fit in shared memory beside the other buffers (C <= 96).  The Fourier weights
 * of both layers stay resident in shared memory when they fit (e.g. the Swin
 * stage-1 block, C = 24, H = 96, Co = 24) and are otherwise streamed per hidden
 * slice (e.g. the ViT-Ti block 48 -> 192 -> 48 or ViT-S 96 -> 384 -> 96); other
 * shapes return FEQL_ERR_UNSUPPORTED (feql_mlp_weight_fft_bytes returns 0 for
 * them).  Conventions otherwise as above (device pointers, 16-byte alignment,
 * stream-ordered, N == 0 is a no-op). */
size_t feql_mlp_weight_fft_bytes(int C, int H, int Co, int dtype);
/* Fourier weights of both layers in the kernel's tile layout (opaque; depends
 * only on C, H, Co): What must hold feql_mlp_weight_fft_bytes(C, H, Co, dtype) bytes. */
int feql_mlp_weight_fft(const void *W1, const void *W2, void *What, int C, int H, int Co,
                        int dtype, feql_stream stream);
int feql_mlp_forward(const void *x, const void *What, const void *b1, const void *b2, void *y,
                     int64_t N, int C, int H, int Co, int dtype, feql_stream stream);

/* Synchronises `stream`, then returns and clears the device-side status word
 * of the current device: FEQL_OK, or FEQL_ERR_TIMEOUT when some kernel gave up
 * on a bounded wait since the last call (its outputs are then undefined). */
int feql_device_status(feql_stream stream);

/* Static description of a status code. */
const char *feql_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* FEQL_H */
