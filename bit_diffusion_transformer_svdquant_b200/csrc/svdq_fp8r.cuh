// Row-wise FP8 (W8A8) variant of the layer: the SVDQuant structure of the NVFP4 path (smoothing,
// 16-bit low-rank branch, quantized residual R) with R and the smoothed activations as E4M3 codes
// and one fp32 scale per row. The pages name the format ("FLUX 3 Image Klein on NVIDIA Blackwell",
// method 1: NVFP4 / FP8 quantization; the Diffusers release notes list row-wise FP8 "fp8r"
// weights) without a formula. Rounding points (IEEE fp32, round to nearest even):
//   s   = fp32(amax_row / 448)                 (1 if amax_row < 2^-100)
//   q_k = E4M3_sat(fp32(v_k * fp32(1 / s)))     (the sign kept when the magnitude rounds to 0)
//   y   = s_x[m] s_w[n] sum_k dec(qx_mk) dec(qw_nk) + (X L1s) L2 (+ bias) (-> SwiGLU)
// The weight row scale is per output row, the activation row scale per token, computed from the
// call's own smoothed X (a row-amax pass before the quantizing pass).
//
// The branch rides in the FP8 product's TMEM accumulator, as in the NVFP4 GEMM: kernel 1 stores
// U / s_x and the pack stores L2^T / s_w, each as a bf16 hi/lo pair (~16 significant bits), and
// three bf16 MMAs per 16 columns of r (hi.hi, lo.hi, hi.lo) add U L2 / (s_x s_w) before the
// epilogue multiplies every accumulator element by s_x[m] s_w[n].
//
// Kernels: pack_weight_kernel / pack_l2_kernel (offline); per call act_row_scale_kernel, then kernel 1
// (svdq::quant_act_kernel) with the RowAct quantizer policy below (a per-element E4M3 quantizer),
// then the pair GEMM (svdq::pair_gemm_kernel) with the Fp8Gemm format policy below (tcgen05.mma
// kind::f8f6f4, no scale-factor operands, double-buffered accumulators).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "svdq_gemm.cuh"
#include "svdq_ptx.cuh"
#include "svdq_quant.cuh"

namespace svdq {
namespace fp8r {

__device__ __forceinline__ float row_scale_from_amax(float amax) {
  return amax >= tiny_amax() ? __fdiv_rn(amax, 448.0f) : 1.0f;
}

// Two fp32 -> two E4M3 codes (round to nearest even, saturating at +-448), `lo` in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// D[tmem] (+)= A[smem] x B[smem]^T, E4M3 x E4M3 with fp32 accumulation, M = 256 across the CTA
// pair, K = 32 per instruction (warp-wide call; elect.sync picks the issuing lane).
__device__ __forceinline__ void mma_e4m3_pair_warp(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                   uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// Instruction descriptor, kind::f8f6f4: fp32 accumulator (D format 1), A and B E4M3 (format 0),
// both K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3(int m, int n) {
  return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// ------------------------------------------------------------------------------------------------
// Offline weight pack.

// One warp per GEMM row p (original row orig_row_of(p)): the row's amax, s_w[p], and its E4M3
// codes at codes[p][0..K).
__global__ void pack_weight_kernel(const float* __restrict__ R, int N, int K, int n_tile, int swiglu,
                                   uint8_t* __restrict__ codes, float* __restrict__ row_scale) {
  const int lane = threadIdx.x & 31;
  const int warps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
  for (int p = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5); p < N; p += warps) {
    const float* src = R + static_cast<size_t>(orig_row_of(p, N, n_tile, swiglu)) * K;
    float amax = 0.0f;
    for (int k = lane * 4; k < K; k += 128) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(src + k));
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = row_scale_from_amax(amax);
    const float rs = __frcp_rn(s);
    uint8_t* dst = codes + static_cast<size_t>(p) * K;
    for (int k = lane * 4; k < K; k += 128) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(src + k));
      *reinterpret_cast<uint32_t*>(dst + k) = cvt_e4m3x2(__fmul_rn(v.x, rs), __fmul_rn(v.y, rs)) |
                                              (cvt_e4m3x2(__fmul_rn(v.z, rs), __fmul_rn(v.w, rs)) << 16);
    }
    if (lane == 0) row_scale[p] = s;
  }
}

// L2^T / s_w in GEMM row order as a bf16 hi/lo pair: with v = fp32(L2[j][orig_row_of(p)] *
// fp32(1 / s_w[p])), out[p][j] = bf16(v) and out[N + p][j] = bf16(v - bf16(v)).
__global__ void pack_l2_kernel(const __nv_bfloat16* __restrict__ L2, const float* __restrict__ row_scale, int N,
                               int r, int n_tile, int swiglu, __nv_bfloat16* __restrict__ out) {
  const size_t total = static_cast<size_t>(N) * r;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(i / r), j = static_cast<int>(i - static_cast<size_t>(p) * r);
    const float l2 = __bfloat162float(L2[static_cast<size_t>(j) * N + orig_row_of(p, N, n_tile, swiglu)]);
    const float v = __fmul_rn(l2, __frcp_rn(row_scale[p]));
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    out[i] = hi;
    out[total + i] = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(hi)));
  }
}

// Canonical export: codes[n][0..K) and scales[n] of original row n.
__global__ void export_weight_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ row_scale, int N,
                                     int K, int n_tile, int swiglu, uint8_t* __restrict__ out_codes,
                                     float* __restrict__ out_scales) {
  const size_t per_row = static_cast<size_t>(K) >> 4;
  const size_t total = static_cast<size_t>(N) * per_row;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(i / per_row);
    const size_t c = (i - static_cast<size_t>(n) * per_row) << 4;
    const int p = gemm_row_of(n, N, n_tile, swiglu);
    *reinterpret_cast<uint4*>(out_codes + static_cast<size_t>(n) * K + c) =
        *reinterpret_cast<const uint4*>(codes + static_cast<size_t>(p) * K + c);
    if (c == 0) out_scales[n] = row_scale[p];
  }
}

// ------------------------------------------------------------------------------------------------
// Per call: activation row scales, then the quantizing pass.

// Row m: s_x[m] = fp32(amax_k |fp32(x_mk * inv_lambda_k)| / 448) (1 below 2^-100) and
// rs_x[m] = fp32(1 / s_x[m]); pad rows M <= m < M_pad get 1. One warp per row, 16-byte loads.
__global__ void act_row_scale_kernel(const __nv_bfloat16* __restrict__ X, const float* __restrict__ inv_lambda,
                                     int M, int M_pad, int K, float* __restrict__ s_x, float* __restrict__ rs_x) {
  grid_dependency_wait();  // X (and the row scales the previous call's GEMM read) belong to earlier kernels
  grid_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int warps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
  for (int m = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5); m < M_pad; m += warps) {
    float amax = 0.0f;
    if (m < M) {
      const __nv_bfloat16* row = X + static_cast<size_t>(m) * K;
      for (int k = lane * 8; k < K; k += 256) {
        float x[8];
        bf16x8_to_f32(ldg_stream(row + k), x);
        const float4 l0 = __ldg(reinterpret_cast<const float4*>(inv_lambda + k));
        const float4 l1 = __ldg(reinterpret_cast<const float4*>(inv_lambda + k + 4));
        const float l[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(__fmul_rn(x[e], l[e])));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    }
    const float s = row_scale_from_amax(amax);
    if (lane == 0) {
      s_x[m] = s;
      rs_x[m] = __frcp_rn(s);
    }
  }
}

struct ActArgs {
  const float* inv_lambda;
  const float* rs_x;    // [M_pad] fp32(1 / s_x)
  uint8_t* codes;       // [M_pad][K] E4M3
  __nv_bfloat16* U;     // [2][M_pad][r]: hi then lo of fp32(X L1s) * rs_x
  unsigned long long wait_ns;
  int M, K, M_pad, k_per_cta;
};

// Kernel 1 (row-wise FP8) is svdq::quant_act_kernel with this quantizer policy: each thread
// turns its two 16-element blocks of a stage into E4M3 codes q = E4M3_sat(fp32(x_hat * rs_x))
// with its rows' reciprocal scales (written by act_row_scale_kernel before the launch) and stores
// each block's 16 codes as one 16-byte store; U is stored times the row's rs_x.
struct RowAct {
  using Args = ActArgs;
  __device__ static void prologue(const Args&, float*) {}
  struct Thread {
    float rs[2];
    uint8_t* code_ptr[2];
    __device__ Thread(const Args& a, const float*, int m_tile, int rl, int b, int kbeg, int grp) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int row = m_tile * 128 + rl + 64 * i;
        rs[i] = a.rs_x[row];  // M_pad entries; pad rows hold 1
        code_ptr[i] = a.codes + static_cast<size_t>(row) * a.K + kbeg + (b << 4) + (grp << 6);
      }
    }
    __device__ void stage(const float2 (&lam)[8], const uint4 (&x)[2][2]) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float2 r2 = make_float2(rs[i], rs[i]);
        const uint32_t wx[8] = {x[i][0].x, x[i][0].y, x[i][0].z, x[i][0].w, x[i][1].x, x[i][1].y, x[i][1].z, x[i][1].w};
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          const float2 v0 = mul2_rn(make_float2(__uint_as_float(wx[j] << 16), __uint_as_float(wx[j] & 0xFFFF0000u)), lam[j]);
          const float2 v1 =
              mul2_rn(make_float2(__uint_as_float(wx[j + 1] << 16), __uint_as_float(wx[j + 1] & 0xFFFF0000u)), lam[j + 1]);
          const float2 q0 = mul2_rn(v0, r2), q1 = mul2_rn(v1, r2);
          w[j >> 1] = cvt_e4m3x2(q0.x, q0.y) | (cvt_e4m3x2(q1.x, q1.y) << 16);
        }
        *reinterpret_cast<uint4*>(code_ptr[i]) = make_uint4(w[0], w[1], w[2], w[3]);
        code_ptr[i] += 128;  // two K steps: this group's next stage
      }
    }
  };
  __device__ static float u_scale(const Args& a, int row) { return a.rs_x[row]; }
  __device__ static void finish(const Args&) {}
};

// ------------------------------------------------------------------------------------------------
// Kernel 2 (row-wise FP8): the CTA-pair tcgen05 GEMM of svdq_gemm.cuh with kind::f8f6f4.

struct GemmArgs {
  const float* s_x;     // [M_pad] activation row scales
  const float* s_w;     // [N] weight row scales, GEMM order
  const __nv_bfloat16* bias;
  void* Y;
  unsigned long long wait_ns;
  int M, M_pad, N, K, r;
  int m_tiles, m_pairs, n_tiles, k_iters, num_tiles;  // k_iters = K / 128
  int ldy, out_f32, epi;                              // epi bit 0: bias, bit 1: SwiGLU
};

// The row-wise FP8 format of the pair GEMM (a policy of svdq::pair_gemm_kernel): E4M3 x E4M3
// (kind::f8f6f4, K = 32 per MMA, the same 128 bytes per row and K step as NVFP4), no scale-factor
// operands, so the writer warps stay idle and both accumulator buffers fit in TMEM at every tile
// width (the epilogue of one tile overlaps the next tile's MMAs); L2^T / s_w is kept as a bf16
// hi/lo pair, so the branch is U_hi L2_hi + U_lo L2_hi + U_hi L2_lo (three bf16 MMAs per 16
// columns); the epilogue scales accumulator element (m, g) by s_x[m] s_w[g].
struct Fp8Gemm {
  using Args = GemmArgs;
  static constexpr bool kScales = false;
  static constexpr bool kL2HiLo = true;
  // the four MMAs of a 128-element K step (each K = 32, 32 bytes of codes per row)
  template <int N_TILE, int SF_ATOMS_B>
  __device__ static void kstep(uint32_t d, uint32_t la, uint32_t lb, uint32_t hi_ab, uint32_t, uint32_t accumulate) {
    static_assert(N_TILE <= 256, "FP8 tiles are at most 256 wide");
    constexpr uint32_t id = idesc_e4m3(256, N_TILE);
    mma_e4m3_pair_warp(d, desc_join(la, hi_ab), desc_join(lb, hi_ab), id, accumulate);
    mma_e4m3_pair_warp(d, desc_join(la + 2u, hi_ab), desc_join(lb + 2u, hi_ab), id, 1u);
    mma_e4m3_pair_warp(d, desc_join(la + 4u, hi_ab), desc_join(lb + 4u, hi_ab), id, 1u);
    mma_e4m3_pair_warp(d, desc_join(la + 6u, hi_ab), desc_join(lb + 6u, hi_ab), id, 1u);
  }
  struct Epi {
    float sx;
    __device__ Epi(const Args& a, int srow) : sx(__ldg(a.s_x + srow)) {}
    // y = s_x s_w[g] acc (+ bias) for 8 accumulator columns g0.. of v[off..]
    template <bool BIAS, class V>
    __device__ void apply8(const Args& a, V& v, int off, int g0, const __nv_bfloat16* bias8) const {
      const float4 w0 = __ldg(reinterpret_cast<const float4*>(a.s_w + g0));
      const float4 w1 = __ldg(reinterpret_cast<const float4*>(a.s_w + g0 + 4));
      const float w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      if constexpr (BIAS) {
        float b[8];
        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(bias8)), b);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[off + j] = fmaf(__fmul_rn(sx, w[j]), v[off + j], b[j]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[off + j] = __fmul_rn(sx, w[j]) * v[off + j];
      }
    }
  };
};

}  // namespace fp8r
}  // namespace svdq
