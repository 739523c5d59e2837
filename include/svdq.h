/*
 * svdq.h -- C ABI of the B200 (sm_100a) SVDQuant-style W4A4 + low-rank linear layer.
 *
 * The layer ("Bringing Nunchaku 4-bit diffusion inference to Diffusers", section "SVDQuant deep
 * dive"): a diffusion transformer's main linears run with 4-bit weights and 4-bit activations
 * (W4A4); outliers are absorbed by a 16-bit low-rank branch, W = L1.L2 + R, with only the residual
 * R quantized; the branch's down-projection X.L1 is fused with the activation quantization and its
 * up-projection with the 4-bit GEMM. Post-training: the split happens offline, before this ABI.
 * The 4-bit format is NVFP4 ("FLUX 3 Image Klein on NVIDIA Blackwell", method 1): E2M1 codes, one
 * E4M3 scale per 16 elements along K, one fp32 scale per tensor. The fused QKV and SwiGLU
 * epilogues follow the fused NVFP4 GEMMs of the same section.
 *
 *   y = alpha * sum_k dec(qx) dec(sx) dec(qw) dec(sw)  +  (X L1s) L2  (+ bias)   [then SwiGLU]
 *   alpha = g_x * g_w;  X [M,K] bf16 row-major;  W, R [N,K] (nn.Linear layout)
 *
 * Two kernels run per layer call:
 *   svdq_quantize_act  -- smoothing x_hat = x * inv_lambda, NVFP4 quantization of x_hat, and the
 *                         down-projection U = X L1s on tensor cores, in one pass over X;
 *   svdq_gemm          -- tcgen05 block-scaled FP4 GEMM on clusters of two CTAs sharing each
 *                         256-row tile (TMA-fed shared-memory rings, TMEM accumulators) whose
 *                         epilogue adds the up-projection U L2 (bf16 MMAs into the same
 *                         accumulator), bias and SwiGLU before one store.
 * Further down: the row-wise FP8 (W8A8) variant of the same layer (svdq_fp8r_*), and the MLP
 * chain's call that fuses the down layer's activation quantization into the gate/up GEMM's
 * SwiGLU epilogue (svdq_gemm_swiglu_quant).
 *
 * Conventions for every entry point:
 *   - Pointers named as device memory must be device pointers on the current device; the library
 *     never allocates device memory and never frees what it is given. Callers size buffers with
 *     svdq_weight_bytes / svdq_act_bytes.
 *   - Work is enqueued on `stream` (a cudaStream_t / CUstream; NULL = legacy default stream) and is
 *     asynchronous; argument checks happen on the host before anything is enqueued, and on a
 *     failed check nothing is enqueued.
 *   - The per-call kernels are launched with programmatic stream serialization: one may start its
 *     set-up (barriers, tensor memory) while the kernel before it on the stream is finishing, but
 *     it reads or writes no global memory until that kernel has completed. Stream order is kept.
 *   - Shapes: K % 256 == 0; N % n_tile == 0 for the n_tile chosen at pack time (384 for a weight
 *     without SwiGLU where 768 divides N, else 256 where it divides N, else 192, else 128; SwiGLU
 *     needs N even); r in {0, 16, 32, 64}; 1 <= M < 2^24.
 *     Device pointers 16-byte aligned.
 *     Other shapes return SVDQ_ERR_UNSUPPORTED.
 *   - A device that is not sm_100 returns SVDQ_ERR_UNSUPPORTED. There is no CPU fallback.
 *   - Every device-side wait is bounded; a wait that runs out sets a bit in the library's device
 *     status word (read with svdq_device_status) and the kernel returns instead of hanging.
 *   - svdq_last_error() returns a human-readable message for the calling thread's last failure.
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SVDQ_ABI_VERSION 1

#if defined(__GNUC__)
#define SVDQ_API __attribute__((visibility("default")))
#else
#define SVDQ_API
#endif

typedef void* svdq_stream_t; /* cudaStream_t */

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1, /* null pointer, buffer too small, negative size, or a          */
                            /*   descriptor no svdq_pack_weight / svdq_act_bind call makes */
  SVDQ_ERR_UNSUPPORTED = 2, /* shape / alignment / device architecture not supported       */
  SVDQ_ERR_CUDA = 3,        /* a CUDA runtime call failed (message in svdq_last_error)     */
  SVDQ_ERR_TIMEOUT = 4      /* a bounded device-side wait ran out (svdq_device_status)     */
} svdq_status;

typedef enum {
  SVDQ_EPI_NONE = 0,        /* y = alpha acc + U L2                                  */
  SVDQ_EPI_BIAS = 1,        /* ... + bias[n]                                         */
  SVDQ_EPI_SWIGLU = 2,      /* y[:, j] = silu(y[:, j]) * y[:, N/2 + j], j < N/2     */
  SVDQ_EPI_BIAS_SWIGLU = 3  /* bias added to both halves before silu                 */
} svdq_epilogue;

typedef enum { SVDQ_OUT_BF16 = 0, SVDQ_OUT_F32 = 1 } svdq_out_dtype;

/* A packed layer weight. Filled by svdq_pack_weight; every pointer points into the caller's `dst`
 * buffer. Treat as read-only; it may be copied by value. Every call that takes one first checks
 * its sizes, n_tile and buffer pointers (SVDQ_ERR_INVALID_ARG before any CUDA call). */
typedef struct svdq_weight {
  int N, K, r;
  int swiglu_interleaved; /* 1: gate/up rows interleaved per n_tile for the SwiGLU epilogue  */
  int n_tile;             /* GEMM tile width along N chosen at pack time                     */
  int reserved0;
  void* codes;            /* uint8 [N][K/2] E2M1 codes, two per byte (element 2i low nibble), */
                          /*   rows in GEMM order (interleaved when swiglu_interleaved)        */
  void* scales;           /* E4M3 scales in the per-n_tile MMA layout                          */
  float* g_w;             /* device fp32 tensor scale of R                                     */
  float* inv_lambda;      /* device fp32 [K] smoothing reciprocals                             */
  void* L1s_t;            /* bf16 [r][K] = (diag(lambda)^-1 L1)^T                              */
  void* L2_t;             /* bf16 [N][r] = L2^T, rows in GEMM order                            */
  unsigned long long tmap[2][16]; /* opaque: cached TMA descriptors of codes and L2_t          */
} svdq_weight;

/* A quantized activation. Bound to caller memory by svdq_act_bind; written by svdq_quantize_act.
 * Checked like svdq_weight: 1 <= M < 2^24, M_pad as below, K and r valid, buffers non-null. */
typedef struct svdq_act {
  int M, K, r, M_pad;     /* M_pad = M rounded up to 128                                       */
  void* codes;            /* uint8 [M_pad][K/2] E2M1 codes (rows >= M are zero)                */
  void* scales;           /* E4M3, [M_pad/128][K/64] atoms of 512 bytes: byte                  */
                          /*   (m%32)*16 + ((m%128)/32)*4 + (k/16)%4 of atom (m/128, k/64)     */
  void* U;                /* bf16 [2][M_pad][r]: u = fp32(X L1s) / alpha as hi = bf16(u) then  */
                          /*   lo = bf16(u - hi), ~16 significant bits for the up-projection   */
  float* alpha;           /* device fp32: fp32(g_x * g_w)                                      */
} svdq_act;

/* Bytes of device memory a packed weight / a quantized activation needs (0 on bad shapes). */
SVDQ_API size_t svdq_weight_bytes(int N, int K, int r);
SVDQ_API size_t svdq_act_bytes(int M, int K, int r);
/* Bytes of a packed weight blob for an explicit GEMM tile width n_tile (384, 256, 192 or 128; the
 * value a descriptor's n_tile field holds), e.g. to check a checkpoint's blob before re-binding it
 * with svdq_weight_bind. 0 on bad shapes or a tile width that does not divide N (384: 768 must
 * divide N). svdq_weight_bind also refuses n_tile 384 for a SwiGLU weight. */
SVDQ_API size_t svdq_weight_bytes_tiled(int N, int K, int r, int n_tile);

/* Offline pack of one layer's weight (not on the per-step path).
 *   R_nk        device fp32 [N][K]  residual R = W_hat - diag(lambda) L1s L2 (nn.Linear layout)
 *   L1s_kr      device bf16 [K][r]  diag(lambda)^-1 L1 (so the branch consumes raw X); NULL if r==0
 *   L2_rn       device bf16 [r][N]  L2; NULL if r == 0
 *   inv_lambda  device fp32 [K]     smoothing reciprocals 1/lambda_j
 *   swiglu      1 to interleave gate rows [0,N/2) and up rows [N/2,N) for SVDQ_EPI_*SWIGLU
 *   dst         device buffer of at least svdq_weight_bytes(N,K,r) bytes, 256-byte aligned
 *   out         host struct filled with pointers into dst
 * Computes g_w = fp32(amax(R)/2688) (1 if amax < 2^-100), quantizes R per 16-element block along
 * K (scale s = E4M3_rne_sat(fp32(amax_b / fp32(6 g_w))), codes E2M1_rne_sat(fp32(r * fp32(1 /
 * fp32(dec(s) g_w)))), all-zero codes when s == 0), and lays codes, scales, L1s^T, L2^T out for
 * the two kernels. Inputs may be freed once the stream has passed this call. */
SVDQ_API svdq_status svdq_pack_weight(const float* R_nk, const uint16_t* L1s_kr, const uint16_t* L2_rn,
                             const float* inv_lambda, int N, int K, int r, int swiglu,
                             void* dst, size_t dst_bytes, svdq_weight* out, svdq_stream_t stream);

/* Checkpoints: re-bind a packed weight blob without re-packing, e.g. one written by
 * svdq_pack_weight, saved, and copied back to device memory. N, K, r, swiglu and n_tile are the
 * values of the descriptor the blob was packed with (n_tile is not re-derived: an SVDQ_N_TILE
 * override at pack time stays valid). The blob is 256-byte aligned and at least the packed size
 * for those values. Fills `out` with pointers into `blob` and re-encodes its TMA descriptors for
 * this address. */
SVDQ_API svdq_status svdq_weight_bind(int N, int K, int r, int swiglu, int n_tile, void* blob, size_t blob_bytes,
                             svdq_weight* out);

/* Host-only: lay an svdq_act out over `dst` (device, >= svdq_act_bytes(M,K,r), 256-aligned). */
SVDQ_API svdq_status svdq_act_bind(int M, int K, int r, void* dst, size_t dst_bytes, svdq_act* out);

/* Static activation scale from calibration data: g_x = fp32(amax(x * inv_lambda) / 2688)
 * (1 if amax < 2^-100), written to the device fp32 *g_x_out. X: device bf16 [M][K]. */
SVDQ_API svdq_status svdq_calibrate_act(const uint16_t* X, int M, const svdq_weight* w, float* g_x_out,
                               svdq_stream_t stream);

/* Kernel 1 (per layer call). X: device bf16 [M][K] (M == act->M, K == w->K, r == w->r);
 * g_x: device fp32 static activation scale. Writes act->codes, act->scales, act->U, act->alpha. */
SVDQ_API svdq_status svdq_quantize_act(const uint16_t* X, const svdq_weight* w, const float* g_x,
                              const svdq_act* act, svdq_stream_t stream);

/* Kernel 2 (per layer call). Y: device [M][N] (or [M][N/2] with SwiGLU) of `out_dtype`,
 * row-major; bias: device bf16 [N] in the original (un-interleaved) column order, NULL unless the
 * epilogue adds one. Rows >= M are not written. Everything is enqueued on `stream` and nothing is
 * allocated, so the call can be captured in a CUDA graph together with svdq_quantize_act. */
SVDQ_API svdq_status svdq_gemm(const svdq_act* act, const svdq_weight* w, const uint16_t* bias,
                      svdq_epilogue epi, void* Y, svdq_out_dtype out_dtype, svdq_stream_t stream);

/* Debug / parity: the packed codes and scales back in canonical row-major form.
 * codes: device uint8 [rows][K/2] (element 2i low nibble); scales: device uint8 [rows][K/16].
 * Weight rows come back in the original order (SwiGLU interleave undone); act rows are 0..M-1. */
SVDQ_API svdq_status svdq_export_weight(const svdq_weight* w, uint8_t* codes, uint8_t* scales,
                               svdq_stream_t stream);
SVDQ_API svdq_status svdq_export_act(const svdq_act* act, uint8_t* codes, uint8_t* scales,
                            svdq_stream_t stream);

/* Synchronizes the current device and returns SVDQ_ERR_TIMEOUT if any bounded wait of this
 * library's kernels ran out since the last reset (reset != 0 clears the word). */
SVDQ_API svdq_status svdq_device_status(int reset);

/* Runs a one-thread kernel that waits on a barrier nothing arrives on, with a limit of
 * `limit_ns` nanoseconds (1000 .. 10^9); the wait runs out, the kernel records it in the status
 * word and returns. Exercises the same bounded-wait routine the GEMM uses. */
SVDQ_API svdq_status svdq_watchdog_selftest(unsigned long long limit_ns, svdq_stream_t stream);

/* Bounded-wait limit used by the GEMM's barrier waits (default 2 s; 1 ms .. 60 s). */
SVDQ_API svdq_status svdq_set_wait_limit_ns(unsigned long long ns);

/* ---------------------------------------------------------------------------------------------
 * Row-wise FP8 (W8A8) variant. "FLUX 3 Image Klein on NVIDIA Blackwell", method 1, names FP8
 * next to NVFP4, and the Diffusers release notes name row-wise FP8 ("fp8r") weights; no formula
 * is given. Reading: the layer keeps its SVDQuant structure (smoothing, 16-bit low-rank branch,
 * quantized residual R); R and the smoothed activations become E4M3 codes with one fp32 scale per
 * row -- per output row of R, per token of X (from the call's own X):
 *   s = fp32(amax_row / 448) (1 if amax_row < 2^-100),  q = E4M3_rne_sat(fp32(v * fp32(1 / s))),
 *   y = s_x[m] s_w[n] sum_k dec(qx) dec(qw) + (X L1s) L2 (+ bias) (-> SwiGLU).
 * Same conventions as the NVFP4 calls above (caller-owned memory, stream-ordered, no allocation,
 * host checks before any work, SVDQ_ERR_INVALID_ARG for descriptors no pack / bind call makes). */
typedef struct svdq_fp8r_weight {
  int N, K, r;
  int swiglu_interleaved; /* 1: gate/up rows interleaved per n_tile, as for svdq_weight         */
  int n_tile;             /* GEMM tile width along N (256 / 192 / 128: the FP8 GEMM has no 384) */
  int reserved0;
  void* codes;            /* uint8 [N][K] E4M3 codes, rows in GEMM order                         */
  float* row_scale;       /* device fp32 [N] s_w per GEMM row                                    */
  float* inv_lambda;      /* device fp32 [K] smoothing reciprocals                               */
  void* L1s_t;            /* bf16 [r][K] = (diag(lambda)^-1 L1)^T                                */
  void* L2_t;             /* bf16 [2][N][r]: v = fp32(L2^T * fp32(1 / s_w)) per GEMM row, stored */
                          /*   as hi = bf16(v) (rows 0..N-1) then lo = bf16(v - hi)             */
  unsigned long long tmap[2][16]; /* opaque: cached TMA descriptors of codes and L2_t            */
} svdq_fp8r_weight;

typedef struct svdq_fp8r_act {
  int M, K, r, M_pad;     /* M_pad = M rounded up to 128                                         */
  void* codes;            /* uint8 [M_pad][K] E4M3 codes (rows >= M are zero)                    */
  float* row_scale;       /* device fp32 [M_pad] s_x (1 for rows >= M)                           */
  float* row_rscale;      /* device fp32 [M_pad] fp32(1 / s_x)                                   */
  void* U;                /* bf16 [2][M_pad][r]: u = fp32(fp32(X L1s) * fp32(1 / s_x)) as hi =    */
                          /*   bf16(u) then lo = bf16(u - hi)                                    */
} svdq_fp8r_act;

/* Bytes of device memory an FP8 packed weight / quantized activation needs (0 on bad shapes:
 * the same shapes as svdq_weight_bytes / svdq_act_bytes). */
SVDQ_API size_t svdq_fp8r_weight_bytes(int N, int K, int r);
SVDQ_API size_t svdq_fp8r_act_bytes(int M, int K, int r);

/* Offline pack, arguments as svdq_pack_weight. Computes s_w and the E4M3 codes of every row of
 * R, and L2^T / s_w as a bf16 hi/lo pair, in the GEMM's row order. */
SVDQ_API svdq_status svdq_fp8r_pack_weight(const float* R_nk, const uint16_t* L1s_kr, const uint16_t* L2_rn,
                                  const float* inv_lambda, int N, int K, int r, int swiglu, void* dst,
                                  size_t dst_bytes, svdq_fp8r_weight* out, svdq_stream_t stream);

/* Host-only: lay an svdq_fp8r_act out over `dst` (device, >= svdq_fp8r_act_bytes, 256-aligned). */
SVDQ_API svdq_status svdq_fp8r_act_bind(int M, int K, int r, void* dst, size_t dst_bytes, svdq_fp8r_act* out);

/* Per layer call: the row-scale pass over X (s_x, 1/s_x), then the quantizing pass (smoothing,
 * E4M3 codes, U = X L1s on the tensor cores, stored times 1/s_x). X: device bf16 [M][K]. */
SVDQ_API svdq_status svdq_fp8r_quantize_act(const uint16_t* X, const svdq_fp8r_weight* w,
                                   const svdq_fp8r_act* act, svdq_stream_t stream);

/* Per layer call: the FP8 GEMM (tcgen05 kind::f8f6f4) with the branch's up-projection in the
 * same accumulator and y = s_x s_w acc (+ bias) (-> SwiGLU) in the epilogue. Y, bias, epi and
 * out_dtype as for svdq_gemm. */
SVDQ_API svdq_status svdq_fp8r_gemm(const svdq_fp8r_act* act, const svdq_fp8r_weight* w, const uint16_t* bias,
                           svdq_epilogue epi, void* Y, svdq_out_dtype out_dtype, svdq_stream_t stream);

/* Debug / parity: codes [rows][K] (uint8, 16-byte aligned) and row scales [rows] (fp32) in
 * canonical form (weight rows in the original order; act rows 0..M-1). */
SVDQ_API svdq_status svdq_fp8r_export_weight(const svdq_fp8r_weight* w, uint8_t* codes, float* scales,
                                    svdq_stream_t stream);
SVDQ_API svdq_status svdq_fp8r_export_act(const svdq_fp8r_act* act, uint8_t* codes, float* scales,
                                 svdq_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * MLP chain: the down layer's kernel 1 fused into the gate/up GEMM's SwiGLU epilogue. The pages
 * fuse the branch's down-projection with activation quantization ("Bringing Nunchaku 4-bit
 * diffusion inference to Diffusers", "SVDQuant deep dive") and fuse SwiGLU into the NVFP4 GEMM
 * ("FLUX 3 Image Klein on NVIDIA Blackwell", method 1); this call does both for the next layer,
 * so h = SwiGLU(...) need not cross HBM.
 *
 * Scratch bytes for svdq_gemm_swiglu_quant at M tokens and next-layer rank r_next (16/32/64):
 * the column-split partial sums of U' (fp32). 0 on bad arguments. */
SVDQ_API size_t svdq_mlp_scratch_bytes(int M, int r_next);

/* One call in place of svdq_gemm (gate/up, SwiGLU) + svdq_quantize_act (down layer):
 *   act, w, bias  the gate/up layer as for svdq_gemm; w packed with swiglu=1 and n_tile 256
 *   w_next        the down layer's packed weight (K = w->N / 2, rank 16/32/64)
 *   g_x_next      device fp32 static activation scale of the down layer (svdq_calibrate_act)
 *   act_next      the down layer's activation (M = act->M): codes, scales, U and alpha written as
 *                 svdq_quantize_act would write them from h = bf16(SwiGLU(...)); codes and scales
 *                 are bit-identical to that path, U agrees to fp32 summation order
 *   scratch       device, >= svdq_mlp_scratch_bytes(M, r_next), 16-byte aligned
 *   H             optional device bf16 [M][N/2] that also receives h (NULL: h is not stored)
 * GPU tests check the down layer's codes, scales and alpha bit-exactly and its output within 2e-3
 * against the oracle on the h this call produced, and against the unfused two-call chain. */
SVDQ_API svdq_status svdq_gemm_swiglu_quant(const svdq_act* act, const svdq_weight* w, const uint16_t* bias,
                                   const svdq_weight* w_next, const float* g_x_next,
                                   const svdq_act* act_next, void* scratch, size_t scratch_bytes,
                                   uint16_t* H, svdq_stream_t stream);

/* The same call for callers that cannot allocate device memory and have no scratch buffer to lend:
 * a plug-in that runs inside a host framework which owns every device allocation (its enqueue step
 * may not call cudaMalloc), or latency-bound code for which cudaMalloc's implicit device
 * synchronisation is not acceptable. The pages have no counterpart; this is a convenience of this
 * library. Arguments as for svdq_gemm_swiglu_quant without `scratch` / `scratch_bytes`: the
 * partial sums go to a buffer of SVDQ_MLP_BUILTIN_SCRATCH_BYTES (8 MiB) that is part of the
 * library's device image, so every GPU that loads the library holds it until the process exits.
 *   - Limit: svdq_mlp_scratch_bytes(M, r_next) must not exceed that size (at r_next = 32: M <= 8192
 *     tokens; r_next = 16: 16384; r_next = 64: 4096); larger calls return SVDQ_ERR_UNSUPPORTED and
 *     enqueue nothing.
 *   - The first call on a device looks up the buffer's device address (cudaGetSymbolAddress, on the
 *     current device) and sets the kernels up; make that first call before any stream capture.
 *   - Every call on a device uses the same buffer and leaves its contents behind (every entry a call
 *     reads is written by the same call first). Calls whose work overlaps on the GPU -- on two
 *     streams, or on two threads -- race on it; order them on one stream.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine. */
#define SVDQ_MLP_BUILTIN_SCRATCH_BYTES ((size_t)8 << 20)
SVDQ_API svdq_status svdq_gemm_swiglu_quant_noscratch(const svdq_act* act, const svdq_weight* w,
                                                      const uint16_t* bias, const svdq_weight* w_next,
                                                      const float* g_x_next, const svdq_act* act_next,
                                                      uint16_t* H, svdq_stream_t stream);

SVDQ_API const char* svdq_status_str(svdq_status s);
SVDQ_API const char* svdq_last_error(void);
SVDQ_API int svdq_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SVDQ_H_ */
