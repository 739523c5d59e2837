// NVFP4 quantization kernels: the per-call activation kernel (smoothing + NVFP4 quantization +
// low-rank down-projection in one pass over X), the offline weight pack, the activation-scale
// calibration, and the canonical-layout export used by parity checks.
//
// Method ("Bringing Nunchaku 4-bit diffusion inference to Diffusers", "SVDQuant deep dive"): the
// low-rank branch's down-projection X.L1 is fused with the activation quantization kernel, so X is
// read from HBM once for both. NVFP4 rounding points (all IEEE fp32, round-to-nearest-even):
//   g   = fp32(amax / 2688)           (1 if amax < 2^-100)
//   s_b = E4M3_sat(fp32(amax_b / fp32(6 g)))
//   q_k = E2M1_sat(fp32(v_k * fp32(1 / fp32(dec(s_b) g))))   (all +0 when s_b == 0)
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "svdq_ptx.cuh"

namespace svdq {

constexpr unsigned kStatusProducer = 1u, kStatusMma = 2u, kStatusEpilogue = 4u, kStatusDrain = 8u,
                   kStatusSelftest = 16u;

__device__ unsigned g_svdq_status = 0;

__device__ __forceinline__ float tiny_amax() { return __uint_as_float(27u << 23); }  // 2^-100

__device__ __forceinline__ float tensor_scale_from_amax(float amax) {
  return amax >= tiny_amax() ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

// Byte offset of the E4M3 scale of row m, 16-element block kb, in the activation MMA layout:
// atoms of 128 rows x 4 blocks (512 bytes), atoms ordered K-fastest.
__host__ __device__ __forceinline__ size_t act_sf_offset(int m, int kb, int K) {
  return ((static_cast<size_t>(m >> 7) * (K >> 6) + (kb >> 2)) << 9) + ((m & 31) << 4) + (((m >> 5) & 3) << 2) +
         (kb & 3);
}
// Same for a weight row p in GEMM order: per n_tile, per 64-wide K atom, ceil(n_tile/128) atoms.
__host__ __device__ __forceinline__ size_t wgt_sf_offset(int p, int kb, int K, int n_tile) {
  const int atoms = (n_tile + 127) >> 7;
  const int nb = p / n_tile, pl = p - nb * n_tile;
  const int a = pl >> 7, pr = pl & 127;
  return (((static_cast<size_t>(nb) * (K >> 6) + (kb >> 2)) * atoms + a) << 9) + ((pr & 31) << 4) +
         ((pr >> 5) << 2) + (kb & 3);
}
// GEMM row of original weight row n (gate/up interleave per n_tile for SwiGLU) and its inverse.
__host__ __device__ __forceinline__ int gemm_row_of(int n, int N, int n_tile, int swiglu) {
  if (!swiglu) return n;
  const int half = n_tile >> 1, hN = N >> 1;
  if (n < hN) return (n / half) * n_tile + n % half;
  const int u = n - hN;
  return (u / half) * n_tile + half + u % half;
}
__host__ __device__ __forceinline__ int orig_row_of(int p, int N, int n_tile, int swiglu) {
  if (!swiglu) return p;
  const int half = n_tile >> 1, nb = p / n_tile, pl = p - nb * n_tile;
  return pl < half ? nb * half + pl : (N >> 1) + nb * half + (pl - half);
}

// One thread's 8 consecutive values; lanes l and l^1 hold the two halves of one 16-element block
// (all 32 lanes must call together). Returns the 8 packed E2M1 codes, sets s to the block scale.
__device__ __forceinline__ uint32_t nvfp4_half_block(const float (&v)[8], float g, float d6, uint32_t& s) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
  s = cvt_e4m3(__fdiv_rn(a, d6));
  if (s == 0) return 0u;
  const float rS = __frcp_rn(__fmul_rn(e4m3_value(s), g));
  float q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(v[i], rS);
  return cvt_e2m1x8(q);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------------------------------------
// Kernel 1: smoothing + NVFP4 activation quantization + U = X L1s, one pass over X.
// U is stored divided by alpha = g_x g_w (so the GEMM applies one scale at the end) as a bf16
// hi/lo pair.
// CTA = 16 rows x all of K, 8 warps splitting K in 32-column chunks. Within a warp, lane (g, t)
// (g = lane/4, t = lane%4) loads 8 consecutive bf16 of rows g and g+8 with 128-bit loads; the same
// registers are both the quantizer's input and the A fragments of two m16n8k16 bf16 MMAs (the
// reduction index is permuted consistently in A and B, which leaves the product unchanged).
struct QuantActArgs {
  const __nv_bfloat16* X;
  const float* inv_lambda;
  const __nv_bfloat16* L1s_t;  // [r][K]
  const float* g_x;
  const float* g_w;
  uint8_t* codes;              // [M_pad][K/2]
  uint8_t* sf;                 // activation MMA layout
  __nv_bfloat16* U;            // [2][M_pad][r]: hi then lo
  float* alpha;
  int M, K, M_pad;
};

template <int R>
__global__ void __launch_bounds__(256) quant_act_kernel(const QuantActArgs a) {
  constexpr int NT = R / 8;
  __shared__ float part[R > 0 ? 8 * 16 * R : 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int m0 = blockIdx.x * 16;
  const int rowA = m0 + g, rowB = m0 + g + 8;
  const bool okA = rowA < a.M, okB = rowB < a.M;
  const int K = a.K;
  const float gx = *a.g_x;
  const float d6 = __fmul_rn(6.0f, gx);
  const __nv_bfloat16* xA = a.X + static_cast<size_t>(okA ? rowA : 0) * K;
  const __nv_bfloat16* xB = a.X + static_cast<size_t>(okB ? rowB : 0) * K;
  uint8_t* cA = a.codes + static_cast<size_t>(rowA) * (K >> 1);
  uint8_t* cB = a.codes + static_cast<size_t>(rowB) * (K >> 1);

  float acc[NT > 0 ? NT : 1][4];
#pragma unroll
  for (int j = 0; j < (NT > 0 ? NT : 1); ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;

  const int nchunks = K >> 5;
  const uint4 zero = make_uint4(0, 0, 0, 0);
  int c = warp;
  uint4 xa = zero, xb = zero;
  if (c < nchunks) {
    const int k = (c << 5) + (t << 3);
    if (okA) xa = ldg_stream(xA + k);
    if (okB) xb = ldg_stream(xB + k);
  }
  for (; c < nchunks; c += 8) {
    const int k = (c << 5) + (t << 3);
    // prefetch the next chunk of this warp before working on the current one
    uint4 na = zero, nb = zero;
    if (c + 8 < nchunks) {
      if (okA) na = ldg_stream(xA + k + 256);
      if (okB) nb = ldg_stream(xB + k + 256);
    }
    const float4 l0 = __ldg(reinterpret_cast<const float4*>(a.inv_lambda + k));
    const float4 l1 = __ldg(reinterpret_cast<const float4*>(a.inv_lambda + k + 4));
    const float lam[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
    float va[8], vb[8];
    bf16x8_to_f32(xa, va);
    bf16x8_to_f32(xb, vb);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      va[i] = __fmul_rn(va[i], lam[i]);
      vb[i] = __fmul_rn(vb[i], lam[i]);
    }
    uint32_t sa, sb;
    const uint32_t qa = nvfp4_half_block(va, gx, d6, sa);
    const uint32_t qb = nvfp4_half_block(vb, gx, d6, sb);
    *reinterpret_cast<uint32_t*>(cA + (k >> 1)) = qa;
    *reinterpret_cast<uint32_t*>(cB + (k >> 1)) = qb;
    if ((t & 1) == 0) {
      a.sf[act_sf_offset(rowA, k >> 4, K)] = static_cast<uint8_t>(sa);
      a.sf[act_sf_offset(rowB, k >> 4, K)] = static_cast<uint8_t>(sb);
    }
    if constexpr (R > 0) {
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        const uint4 bq = __ldg(reinterpret_cast<const uint4*>(a.L1s_t + static_cast<size_t>(j * 8 + g) * K + k));
        mma_bf16_16816(acc[j], xa.x, xb.x, xa.y, xb.y, bq.x, bq.y);
        mma_bf16_16816(acc[j], xa.z, xb.z, xa.w, xb.w, bq.z, bq.w);
      }
    }
    xa = na;
    xb = nb;
  }

  const float alpha = __fmul_rn(gx, *a.g_w);
  if constexpr (R > 0) {
    float* pw = part + warp * 16 * R;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int col = j * 8 + 2 * t;
      pw[g * R + col] = acc[j][0];
      pw[g * R + col + 1] = acc[j][1];
      pw[(g + 8) * R + col] = acc[j][2];
      pw[(g + 8) * R + col + 1] = acc[j][3];
    }
    __syncthreads();
    // U / alpha as a bf16 pair: hi = bf16(u), lo = bf16(u - hi) (the difference is exact in fp32),
    // so that two bf16 MMAs against L2 carry about 16 significant bits of the branch.
    const float cinv = __frcp_rn(alpha);
    __nv_bfloat16* u_hi = a.U + static_cast<size_t>(m0) * R;
    __nv_bfloat16* u_lo = u_hi + static_cast<size_t>(a.M_pad) * R;
    for (int i = threadIdx.x; i < 16 * R; i += 256) {
      float s = 0.0f;
#pragma unroll
      for (int w = 0; w < 8; ++w) s += part[w * 16 * R + i];
      const float u = __fmul_rn(s, cinv);
      const __nv_bfloat16 hi = __float2bfloat16_rn(u);
      u_hi[i] = hi;
      u_lo[i] = __float2bfloat16_rn(__fsub_rn(u, __bfloat162float(hi)));
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *a.alpha = alpha;
}

// ------------------------------------------------------------------------------------------------
// Offline pack and calibration helpers.

// atomicMax of |x| (as fp32 bit patterns, valid for non-negative floats) into *out.
__global__ void amax_f32_kernel(const float* __restrict__ x, size_t n4, unsigned* out) {
  float m = 0.0f;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(x) + i);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(out, __float_as_uint(m));
}

// atomicMax of |x * inv_lambda| over X [M][K] bf16 (8 elements per thread).
__global__ void act_amax_kernel(const __nv_bfloat16* __restrict__ X, const float* __restrict__ inv_lambda,
                                size_t n8, int K, unsigned* out) {
  float m = 0.0f;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int k = static_cast<int>((i * 8) % static_cast<size_t>(K));
    float v[8];
    bf16x8_to_f32(ldg_stream(X + i * 8), v);
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(__fmul_rn(v[j], __ldg(inv_lambda + k + j))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(out, __float_as_uint(m));
}

// In place: amax bit pattern -> fp32 tensor scale.
__global__ void finalize_scale_kernel(float* g) {
  *g = tensor_scale_from_amax(__uint_as_float(*reinterpret_cast<unsigned*>(g)));
}

// Quantize R [N][K] fp32 (original row order) into GEMM-order codes and tile-layout scales.
__global__ void pack_quant_kernel(const float* __restrict__ R, int N, int K, int n_tile, int swiglu,
                                  const float* __restrict__ g_w, uint8_t* __restrict__ codes,
                                  uint8_t* __restrict__ sf) {
  const float g = *g_w;
  const float d6 = __fmul_rn(6.0f, g);
  const size_t total = static_cast<size_t>(N) * (K >> 3);  // multiple of 32
  const int per_row = K >> 3;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(i / per_row);
    const int k = static_cast<int>(i - static_cast<size_t>(n) * per_row) * 8;
    const float4 a0 = __ldg(reinterpret_cast<const float4*>(R + static_cast<size_t>(n) * K + k));
    const float4 a1 = __ldg(reinterpret_cast<const float4*>(R + static_cast<size_t>(n) * K + k + 4));
    const float v[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    uint32_t s;
    const uint32_t q = nvfp4_half_block(v, g, d6, s);
    const int p = gemm_row_of(n, N, n_tile, swiglu);
    *reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(p) * (K >> 1) + (k >> 1)) = q;
    if (((k >> 3) & 1) == 0) sf[wgt_sf_offset(p, k >> 4, K, n_tile)] = static_cast<uint8_t>(s);
  }
}

// L1s [K][r] -> L1s_t [r][K]
__global__ void transpose_l1_kernel(const __nv_bfloat16* __restrict__ L1s, int K, int r,
                                    __nv_bfloat16* __restrict__ out) {
  const size_t total = static_cast<size_t>(K) * r;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(i / K), k = static_cast<int>(i % K);
    out[i] = L1s[static_cast<size_t>(k) * r + j];
  }
}

// L2 [r][N] -> L2_t [N][r] with rows in GEMM order
__global__ void pack_l2_kernel(const __nv_bfloat16* __restrict__ L2, int N, int r, int n_tile, int swiglu,
                               __nv_bfloat16* __restrict__ out) {
  const size_t total = static_cast<size_t>(N) * r;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(i / r), j = static_cast<int>(i % r);
    out[i] = L2[static_cast<size_t>(j) * N + orig_row_of(p, N, n_tile, swiglu)];
  }
}

// Canonical export: codes [rows][K/2] and scales [rows][K/16], one thread per 16-element block.
__global__ void export_weight_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf, int N,
                                     int K, int n_tile, int swiglu, uint8_t* __restrict__ out_codes,
                                     uint8_t* __restrict__ out_sf) {
  const size_t total = static_cast<size_t>(N) * (K >> 4);
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(i / (K >> 4)), kb = static_cast<int>(i % (K >> 4));
    const int p = gemm_row_of(n, N, n_tile, swiglu);
    *reinterpret_cast<uint2*>(out_codes + static_cast<size_t>(n) * (K >> 1) + kb * 8) =
        *reinterpret_cast<const uint2*>(codes + static_cast<size_t>(p) * (K >> 1) + kb * 8);
    out_sf[i] = sf[wgt_sf_offset(p, kb, K, n_tile)];
  }
}

__global__ void export_act_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf, int M, int K,
                                  uint8_t* __restrict__ out_codes, uint8_t* __restrict__ out_sf) {
  const size_t total = static_cast<size_t>(M) * (K >> 4);
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(i / (K >> 4)), kb = static_cast<int>(i % (K >> 4));
    *reinterpret_cast<uint2*>(out_codes + static_cast<size_t>(m) * (K >> 1) + kb * 8) =
        *reinterpret_cast<const uint2*>(codes + static_cast<size_t>(m) * (K >> 1) + kb * 8);
    out_sf[i] = sf[act_sf_offset(m, kb, K)];
  }
}

// One thread waits on a barrier that nothing arrives on; the bounded wait must run out.
__global__ void watchdog_selftest_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_addr(&bar);
  mbar_init(b, 1);
  fence_barrier_init();
  (void)mbar_wait_bounded(b, 0, limit_ns, &g_svdq_status, kStatusSelftest, nullptr);
}

}  // namespace svdq
