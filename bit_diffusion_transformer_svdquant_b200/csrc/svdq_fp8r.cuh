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
// Kernels: pack_weight_kernel / pack_l2_kernel (offline), act_row_scale_kernel and
// quant_act_kernel (per call, the latter the NVFP4 kernel 1's TMA + tcgen05 structure with a
// per-element E4M3 quantizer), gemm_kernel (the NVFP4 GEMM's CTA-pair structure with
// tcgen05.mma kind::f8f6f4, no scale-factor operands, double-buffered accumulators).
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
// Kernel 2 (row-wise FP8): CTA-pair tcgen05 GEMM, kind::f8f6f4.

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

template <int N_TILE, int STAGES>
struct GemmLayout {
  static constexpr int kBRows = N_TILE / 2;  // rows of B staged by each CTA of the pair
  static constexpr int kA = 128 * 128;       // 128 rows x 128 E4M3 (one K step)
  static constexpr int kB = kBRows * 128;
  static constexpr int kStage = kA + kB;
  static constexpr int kOffB = kA;
  // low-rank slots: U_hi at 0, U_lo at kOffULo, L2_hi at kOffB, L2_lo at kOffL2Lo (rc <= 32 columns)
  static constexpr int kOffL2Lo = kOffB + kBRows * kLrChunk * 2;
  // relay barriers: the issuer learns through them that both CTAs' copies of a ring slot landed
  static constexpr int kSyncBufs = 4;
  static constexpr int kAccBufs = 2;
  static constexpr int kStageOutWarp = 4096;
  static constexpr int kOutOff = STAGES * kStage;
  static constexpr int kBarOff = kOutOff + 8 * kStageOutWarp;
  // full[STAGES], empty[STAGES], accf[2], acce[2], drain, sync[kSyncBufs]
  static constexpr int kNumBars = 2 * STAGES + 2 * kAccBufs + 1 + kSyncBufs;
  static constexpr int kSmem = kBarOff + kNumBars * 8 + 16 + 1024;
  static_assert(kStage % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(kOffL2Lo % 512 == 0, "64B-swizzled boxes start on 512-byte boundaries");
  static_assert(kOffL2Lo + kBRows * kLrChunk * 2 <= kStage, "low-rank slot fits a ring stage");
  static_assert(kAccBufs * N_TILE <= 512, "TMEM budget");
  static_assert(kSyncBufs <= STAGES, "a relay barrier's previous slot must still own its ring stage");
  static_assert(kSmem <= 232448, "shared memory budget");
};

// Structure as the NVFP4 pair GEMM (warp 0 TMA producer, warp 1 TMEM allocation and, in the even
// CTA, the warp-uniform MMA issuer, warps 2..9 epilogue), with these differences: no scale
// factors; warp 10 of each CTA relays "this CTA's copies of the slot landed" to the issuer's
// barrier in the even CTA (warps 11..13 idle); two accumulator buffers for every tile width (no
// TMEM scale buffers), so the epilogue of one tile overlaps the next tile's MMAs; the low-rank
// slot carries L2's lo half too; the epilogue scales by s_x[row] s_w[column].
template <int N_TILE, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmL2,
                const __grid_constant__ CUtensorMap tmY, const GemmArgs args) {
  using L = GemmLayout<N_TILE, STAGES>;
  constexpr int kSyncBufs = L::kSyncBufs, kAccBufs = L::kAccBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto accf_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto acce_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + kAccBufs + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 2 * kAccBufs);
  auto sync_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 * kAccBufs + 1 + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBarOff + L::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = args.r;
  const uint32_t rank = cluster_ctarank();  // 0: issues the pair's MMAs
  const int pair0 = static_cast<int>(cluster_id_x()), npairs = static_cast<int>(num_clusters_x());

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), 16);  // 8 epilogue warps in each CTA
    }
    mbar_init(drain_bar, 1);
    for (int b = 0; b < kSyncBufs; ++b) mbar_init(sync_bar(b), 2);  // the relay warp of each CTA
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmY);
    if (r > 0) {
      prefetch_tmap(&tmU);
      prefetch_tmap(&tmL2);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_addr(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  // both CTAs' barriers are initialised before any remote arrive
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  unsigned* status = &g_svdq_status;
  const uint64_t wait_ns = args.wait_ns;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      const int rc = r < kLrChunk ? r : kLrChunk;
      const uint32_t lr_bytes = static_cast<uint32_t>((2 * 128 + 2 * L::kBRows) * rc * 2);
      bool ok = true;
      for (int tile = pair0; ok && tile < args.num_tiles; tile += npairs) {
        int m_pair, n_blk;
        tile_coords(tile, args.m_pairs, args.n_tiles, m_pair, n_blk);
        // an odd CTA past the last 128-row block loads zero-filled codes; none of its rows are stored
        const int m_blk = 2 * m_pair + static_cast<int>(rank);
        const int b_row = n_blk * N_TILE + static_cast<int>(rank) * L::kBRows;
        for (int c0 = 0; c0 < r; c0 += kLrChunk) {
          if (!(ok = mbar_wait_bounded(empty_bar(stage), phase ^ 1u, wait_ns, status, kStatusProducer, abort_flag)))
            break;
          const uint32_t sa = sbase + stage * L::kStage;
          mbar_arrive_expect_tx(full_bar(stage), lr_bytes);
          tma_load_2d(sa, &tmU, c0, m_blk * 128, full_bar(stage));
          tma_load_2d(sa + kOffULo, &tmU, c0, args.M_pad + m_blk * 128, full_bar(stage));
          tma_load_2d(sa + L::kOffB, &tmL2, c0, b_row, full_bar(stage));
          tma_load_2d(sa + L::kOffL2Lo, &tmL2, c0, args.N + b_row, full_bar(stage));
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        for (int kt = 0; kt < args.k_iters; ++kt) {
          if (!(ok = mbar_wait_bounded(empty_bar(stage), phase ^ 1u, wait_ns, status, kStatusProducer, abort_flag)))
            break;
          const uint32_t sa = sbase + stage * L::kStage;
          mbar_arrive_expect_tx(full_bar(stage), L::kStage);
          tma_load_2d(sa, &tmA, kt * 128, m_blk * 128, full_bar(stage));
          tma_load_2d(sa + L::kOffB, &tmB, kt * 128, b_row, full_bar(stage));
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Drain: every copy this thread started has landed before the CTA may exit.
      for (int s = 0; s < STAGES; ++s)
        if (armed & (1u << s))
          mbar_wait_bounded(full_bar(s), (armed_parity >> s) & 1u, wait_ns, status, kStatusDrain, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (even CTA)
    if (rank == 0) {
      auto wait_all = [&](uint32_t bar, uint32_t parity, unsigned code, volatile int* abort_ptr) {
        return __all_sync(0xffffffffu, mbar_wait_bounded_cluster(bar, parity, wait_ns, status, code, abort_ptr));
      };
      const int num_tiles = args.num_tiles, k_iters = args.k_iters;
      const int rc = r < kLrChunk ? r : kLrChunk;
      const int nj = rc >> 4;
      const uint32_t idesc_f8 = idesc_e4m3(256, N_TILE);
      const uint32_t idesc_lr = idesc_bf16(256, N_TILE);
      // descriptor halves: low = start address / 16 | LBO (16 B) / 16 << 16; high = SBO / 16 |
      // version 1 | swizzle mode << 29
      const uint32_t lo0 = (sbase >> 4) | (1u << 16);
      const uint32_t hi_ab = (1024u >> 4) | (1u << 14) | (2u << 29);
      const uint32_t hi_lr = ((8u * rc * 2u) >> 4) | (1u << 14) | (lr_swizzle_mode(rc) << 29);
      constexpr uint16_t kBoth = 3;
      int stage = 0, sb = 0, acc = 0;
      uint32_t phase = 0, sb_phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = pair0; ok && tile < num_tiles; tile += npairs) {
        if (!(ok = wait_all(acce_bar(acc), acc_phase ^ 1u, kStatusMma, abort_flag))) break;
        const uint32_t d = tmem + static_cast<uint32_t>(acc * N_TILE);
        uint32_t accumulate = 0;
        for (int c0 = 0; c0 < r; c0 += kLrChunk) {
          if (!(ok = wait_all(sync_bar(sb), sb_phase, kStatusMma, abort_flag))) break;
          tc_fence_after();
          const uint32_t lo = lo0 + stage * (L::kStage >> 4);
          for (int j = 0; j < nj; ++j) {
            const uint64_t u_hi = desc_join(lo + 2u * j, hi_lr);
            const uint64_t u_lo = desc_join(lo + (kOffULo >> 4) + 2u * j, hi_lr);
            const uint64_t l_hi = desc_join(lo + (L::kOffB >> 4) + 2u * j, hi_lr);
            const uint64_t l_lo = desc_join(lo + (L::kOffL2Lo >> 4) + 2u * j, hi_lr);
            mma_bf16_pair_warp(d, u_hi, l_hi, idesc_lr, accumulate);
            mma_bf16_pair_warp(d, u_lo, l_hi, idesc_lr, 1u);
            mma_bf16_pair_warp(d, u_hi, l_lo, idesc_lr, 1u);
            accumulate = 1;
          }
          tc_commit_pair_mc_warp(empty_bar(stage), kBoth);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          if (++sb == kSyncBufs) { sb = 0; sb_phase ^= 1u; }
        }
        if (!ok) break;
        for (int kt = 0; kt < k_iters; ++kt) {
          if (!(ok = wait_all(sync_bar(sb), sb_phase, kStatusMma, abort_flag))) break;
          tc_fence_after();
          const uint32_t la = lo0 + stage * (L::kStage >> 4);
          const uint32_t lb = la + (L::kOffB >> 4);
          mma_e4m3_pair_warp(d, desc_join(la, hi_ab), desc_join(lb, hi_ab), idesc_f8, accumulate);
          mma_e4m3_pair_warp(d, desc_join(la + 2u, hi_ab), desc_join(lb + 2u, hi_ab), idesc_f8, 1u);
          mma_e4m3_pair_warp(d, desc_join(la + 4u, hi_ab), desc_join(lb + 4u, hi_ab), idesc_f8, 1u);
          mma_e4m3_pair_warp(d, desc_join(la + 6u, hi_ab), desc_join(lb + 6u, hi_ab), idesc_f8, 1u);
          accumulate = 1;
          tc_commit_pair_mc_warp(empty_bar(stage), kBoth);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          if (++sb == kSyncBufs) { sb = 0; sb_phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_mc_warp(accf_bar(acc), kBoth);
        if (++acc == kAccBufs) { acc = 0; acc_phase ^= 1u; }
      }
      // Drain: all issued MMAs complete before TMEM may be freed.
      tc_commit_pair_mc_warp(drain_bar, 1);
      __all_sync(0xffffffffu, mbar_wait_bounded(drain_bar, 0, wait_ns, status, kStatusDrain, nullptr));
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------------ relay (warp 10)
    // Per ring slot: wait for this CTA's copies to land, then arrive on the slot's relay barrier in
    // the even CTA. Before that, wait for the release of the slot kSyncBufs back (the previous
    // user of the same relay barrier), so that no CTA arrives for a slot while the barrier's
    // previous phase still waits for the other CTA.
    int stage = 0, sb = 0, slots_done = 0;
    uint32_t phase = 0;
    const int lr_slots = (r + kLrChunk - 1) / kLrChunk;
    bool ok = true;
    for (int tile = pair0; ok && tile < args.num_tiles; tile += npairs) {
      for (int slot = 0; slot < lr_slots + args.k_iters; ++slot) {
        const bool got_data = mbar_wait_bounded(full_bar(stage), phase, wait_ns, status, kStatusEpilogue, abort_flag);
        if (!__all_sync(0xffffffffu, got_data)) { ok = false; break; }
        bool got = true;
        if (slots_done >= kSyncBufs) {
          int ps = stage - kSyncBufs;
          uint32_t pp = phase;
          if (ps < 0) {
            ps += STAGES;
            pp ^= 1u;
          }
          got = mbar_wait_bounded(empty_bar(ps), pp, wait_ns, status, kStatusEpilogue, abort_flag);
        }
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(cluster_map(sync_bar(sb), 0));
        ++slots_done;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        if (++sb == kSyncBufs) sb = 0;
      }
    }
  } else if (warp >= 2 && warp < 10) {
    // ------------------------------------------------------------------ epilogue (warps 2..9)
    // As in the NVFP4 GEMM: warp (q, h) owns TMEM lane quadrant q = warp % 4 and half h of the
    // tile's 32-column output chunks; loads, scaling, SwiGLU, swizzled staging boxes, TMA stores
    // that clip rows >= M. The scale of accumulator element (row, GEMM column g) is s_x[row] s_w[g].
    const int q = warp & 3, h = (warp - 2) >> 2;
    const bool has_bias = (args.epi & 1) != 0;
    const bool swiglu = (args.epi & 2) != 0;
    const bool f32 = args.out_f32 != 0;
    const int hN = args.N >> 1;
    uint8_t* stage_out = smem + L::kOutOff + (warp - 2) * L::kStageOutWarp;
    constexpr int kPlainPerWarp = N_TILE / 64;  // chunks per warp without SwiGLU
    constexpr int kGluChunks = N_TILE / 64;     // output chunks per tile with SwiGLU
    constexpr int kHalf = N_TILE / 2;
    const int glu_beg = h * ((kGluChunks + 1) >> 1);
    const int glu_end = h ? kGluChunks : ((kGluChunks + 1) >> 1);
    int acc = 0;
    uint32_t acc_phase = 0;
    auto store_box = [&](uint8_t* dst, int row0, int col0) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&tmY, smem_addr(dst), col0, row0);
        bulk_commit_group();
      }
    };
    auto boxes_free = [&]() {
      if (lane == 0) bulk_wait_group_read<0>();
      __syncwarp();
    };
    // 32 bf16 values of row `lane` -> staging box b (64-byte rows, 16-byte chunk j at j ^ ((lane / 2) % 4))
    auto write_box_bf16 = [&](const float (&v)[32], int b) {
      uint8_t* dst = stage_out + b * 2048;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * j + 2 * e], v[8 * j + 2 * e + 1]);
          w[e] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        *reinterpret_cast<uint4*>(dst + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    };
    // 32 fp32 values of row `lane` -> the warp's 4 KB box (128-byte rows, chunk j at j ^ (lane % 8))
    auto write_box_f32 = [&](const float (&v)[32]) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float4*>(stage_out + lane * 128 + ((j ^ (lane & 7)) << 4)) =
            make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    };
    auto load8 = [&](const float* p, float (&o)[8]) {
      const float4 a0 = __ldg(reinterpret_cast<const float4*>(p));
      const float4 a1 = __ldg(reinterpret_cast<const float4*>(p + 4));
      o[0] = a0.x; o[1] = a0.y; o[2] = a0.z; o[3] = a0.w;
      o[4] = a1.x; o[5] = a1.y; o[6] = a1.z; o[7] = a1.w;
    };
    // y = s_x s_w[g0 + i] acc (+ bias[n0 + i]) for 32 accumulator columns
    auto affine = [&](float (&v)[32], float sx, int g0, int n0) {
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        float sw[8], b[8];
        load8(args.s_w + g0 + i, sw);
        if (has_bias) {
          bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(args.bias + n0 + i)), b);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) b[j] = 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) v[i + j] = fmaf(__fmul_rn(sx, sw[j]), v[i + j], b[j]);
      }
    };
    auto release_acc = [&]() {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_map(acce_bar(acc), 0));
    };
    for (int tile = pair0; tile < args.num_tiles; tile += npairs) {
      int m_pair, n_blk;
      tile_coords(tile, args.m_pairs, args.n_tiles, m_pair, n_blk);
      const int m_blk = 2 * m_pair + static_cast<int>(rank);
      const bool got = mbar_wait_bounded(accf_bar(acc), acc_phase, wait_ns, status, kStatusEpilogue, abort_flag);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int row0 = m_blk * 128 + q * 32;
      // rows past M_pad (an odd CTA past the last block) are never stored; read a valid scale
      const int srow = row0 + lane < args.M_pad ? row0 + lane : args.M_pad - 1;
      const float sx = __ldg(args.s_x + srow);
      const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * N_TILE);
      if (!swiglu) {
        // one 32-column chunk at a time; with two accumulator buffers the issuer is already on the
        // next tile, so the epilogue's latency is hidden behind its MMAs
        const int c_beg = h * kPlainPerWarp;
#pragma unroll 1
        for (int i = 0; i < kPlainPerWarp; ++i) {
          float v[32];
          tmem_ld_32x32(tb + (c_beg + i) * 32, v);
          tmem_wait_ld();
          if (i + 1 == kPlainPerWarp) release_acc();
          const int g0 = n_blk * N_TILE + (c_beg + i) * 32;
          affine(v, sx, g0, g0);
          boxes_free();
          if (f32) write_box_f32(v);
          else write_box_bf16(v, 0);
          store_box(stage_out, row0, g0);
        }
      } else {
        // output chunk c pairs gate GEMM columns c*32.. with up GEMM columns n_tile/2 + c*32..
        const int n_mine = glu_end - glu_beg;
#pragma unroll 1
        for (int c = 0; c < n_mine; ++c) {
          const int cc = glu_beg + c;
          float gt[32], up[32];
          tmem_ld_32x32(tb + cc * 32, gt);
          tmem_ld_32x32(tb + kHalf + cc * 32, up);
          tmem_wait_ld();
          if (c + 1 == n_mine) release_acc();
          const int j0 = n_blk * kHalf + cc * 32;   // output (and gate bias) column
          const int g0 = n_blk * N_TILE + cc * 32;  // gate GEMM column
          affine(gt, sx, g0, j0);
          affine(up, sx, g0 + kHalf, hN + j0);
#pragma unroll
          for (int i = 0; i < 32; ++i) gt[i] = __fdividef(gt[i], 1.0f + __expf(-gt[i])) * up[i];
          boxes_free();
          if (f32) write_box_f32(gt);
          else write_box_bf16(gt, 0);
          store_box(stage_out, row0, j0);
        }
      }
      if (++acc == kAccBufs) { acc = 0; acc_phase ^= 1u; }
    }
    // every TMA store issued by this warp has completed before the CTA may exit
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  // Neither CTA frees TMEM or exits while the other may still arrive on its barriers or while the
  // pair's MMAs may still read its shared memory.
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace fp8r
}  // namespace svdq
