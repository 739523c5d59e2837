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
// A 384-wide tile runs as two pair MMAs: N = 256 over tile columns 0..255 and N = 128 over
// 256..383, each taking half of its B rows from each CTA of the pair. Each CTA stages its share as
// one contiguous box of 192 rows, so CTA c holds tile columns [128c, 128c + 128) followed by
// [256 + 64c, 256 + 64c + 64). Packed (storage) row q of a tile -> tile column (the MMA's N index,
// which is also the accumulator column) and back; the identity for the narrower tiles.
__host__ __device__ __forceinline__ int tile_col_of_packed(int q, int n_tile) {
  if (n_tile != 384) return q;
  const int c = q >= 192 ? 1 : 0, s = q - 192 * c;
  return s < 128 ? 128 * c + s : 256 + 64 * c + (s - 128);
}
__host__ __device__ __forceinline__ int packed_of_tile_col(int t, int n_tile) {
  if (n_tile != 384) return t;
  if (t < 256) return 192 * (t >> 7) + (t & 127);
  const int u = t - 256;
  return 192 * (u >> 6) + 128 + (u & 63);
}
// Same for a packed weight row p: per n_tile, per 64-wide K atom, ceil(n_tile/128) atoms of 128
// tile columns each (the B scale layout the MMAs read from TMEM).
__host__ __device__ __forceinline__ size_t wgt_sf_offset(int p, int kb, int K, int n_tile) {
  const int atoms = (n_tile + 127) >> 7;
  const int nb = p / n_tile, pl = tile_col_of_packed(p - nb * n_tile, n_tile);
  const int a = pl >> 7, pr = pl & 127;
  return (((static_cast<size_t>(nb) * (K >> 6) + (kb >> 2)) * atoms + a) << 9) + ((pr & 31) << 4) +
         ((pr >> 5) << 2) + (kb & 3);
}
// Packed (GEMM) row of original weight row n and its inverse: the gate/up interleave per n_tile for
// SwiGLU (tile column t < n_tile/2 a gate row, the rest the matching up rows), then the placement of
// tile columns in the CTAs' B boxes above.
__host__ __device__ __forceinline__ int gemm_row_of(int n, int N, int n_tile, int swiglu) {
  int g = n;
  if (swiglu) {
    const int half = n_tile >> 1, hN = N >> 1;
    if (n < hN) {
      g = (n / half) * n_tile + n % half;
    } else {
      const int u = n - hN;
      g = (u / half) * n_tile + half + u % half;
    }
  }
  const int nb = g / n_tile;
  return nb * n_tile + packed_of_tile_col(g - nb * n_tile, n_tile);
}
__host__ __device__ __forceinline__ int orig_row_of(int p, int N, int n_tile, int swiglu) {
  const int nb = p / n_tile, pl = tile_col_of_packed(p - nb * n_tile, n_tile);
  if (!swiglu) return nb * n_tile + pl;
  const int half = n_tile >> 1;
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

// Two IEEE round-to-nearest fp32 products in one instruction (lane-wise, same rounding as __fmul_rn).
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(r)
      : "l"(*reinterpret_cast<const uint64_t*>(&a)), "l"(*reinterpret_cast<const uint64_t*>(&b)));
  return *reinterpret_cast<const float2*>(&r);
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// Every thread of every CTA in the cluster arrives (warp-converged: .aligned).
__device__ __forceinline__ void cluster_sync_all() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Generic address of the same shared-memory location in CTA `rank` of the cluster (plain loads
// through it read that CTA's shared memory).
template <class T>
__device__ __forceinline__ T* cluster_map_generic(T* p, uint32_t rank) {
  uint64_t r;
  asm volatile("mapa.u64 %0, %1, %2;" : "=l"(r) : "l"(reinterpret_cast<uint64_t>(p)), "r"(rank));
  return reinterpret_cast<T*>(r);
}

// Largest magnitude of 16 values, as a balanced tree of 3-input maxima (depth 3 instead of a
// 16-long running max).
__device__ __forceinline__ float max3_abs(float a, float b, float c) {
  float r;
  asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float amax16(const float2 (&v)[8]) {
  const float m0 = max3_abs(v[0].x, v[0].y, v[1].x), m1 = max3_abs(v[1].y, v[2].x, v[2].y);
  const float m2 = max3_abs(v[3].x, v[3].y, v[4].x), m3 = max3_abs(v[4].y, v[5].x, v[5].y);
  const float m4 = max3_abs(v[6].x, v[6].y, v[7].x);
  return fmaxf(max3_abs(m0, m1, m2), max3_abs(m3, m4, v[7].y));
}

// The E4M3 code of a block scale is E4M3_rne_sat(fp32(amax / d6)). Kernel 1 first takes the
// quotient as q = fp32(amax * rd6) with rd6 = fp32(1 / d6): q is within 3 units in the last place
// of the correctly rounded quotient, so both round to the same E4M3 value unless q lies within 4
// units of an E4M3 rounding boundary (a midpoint between E4M3 values: fp32 mantissa bits 19..0
// equal to 0x80000) or below E4M3's normal range (2^-6). This tells whether the exact IEEE
// division must decide.
__device__ __forceinline__ bool scale_needs_division(float q) {
  return q < 0.015625f || (__float_as_uint(q) & 0xFFFFFu) - 0x7FFFCu <= 8u;
}

// ------------------------------------------------------------------------------------------------
// Kernel 1: smoothing + activation quantization + U = X L1s, one pass over X. One kernel body
// serves both formats; a policy class supplies the quantizer (Nvfp4Act here, the row-wise FP8
// RowAct in svdq_fp8r.cuh) and the scale U is stored with.
//
// A CTA (one per SM) owns 128 rows of X and a K range: the whole K, or a share of it when a
// thread-block cluster of 2, 3 or 4 CTAs splits K so that few row tiles still fill the SMs in one
// wave. TMA streams 128 x 64 bf16 stages (128B swizzle; an L2 evict-first policy, since X is read
// once) of X, the stage's 64-column slice of L1s^T and its 64 inverse smoothing factors into an
// 8-deep shared-memory ring (6 at r = 64). Every stage is read twice from shared memory: by one of
// two groups of eight quantizer warps (the groups take alternate stages, so two stages are being
// quantized at any time: smoothing, block amax, E4M3 scale, E2M1 codes, stored straight to global
// memory), and by a single-thread tcgen05 bf16 MMA (M=128, N=r, K=16) that accumulates the
// down-projection in TMEM. X thus crosses HBM once. At the end four warps read U from TMEM; with a
// K split the partial U of every CTA is summed in rank order through distributed shared memory. U
// is stored divided by alpha = g_x g_w (one scale for the whole GEMM) as a bf16 hi/lo pair.
constexpr int kQTile = 128 * 128;  // 128 rows x 64 bf16
constexpr int kQuantWarps = 16;    // two groups of eight
constexpr int kQ1Threads = 64 + 32 * kQuantWarps;  // warp 0 TMA, warp 1 MMA, warps 2..17 quantize (2..5 drain U)

template <int R>
struct Q1Layout {
  static constexpr int kStages = R <= 32 ? 8 : 6;
  static constexpr int kL1 = (R * 128 + 1023) / 1024 * 1024;
  static constexpr int kLamOff = kQTile + kL1;      // the stage's 64 inverse smoothing factors (fp32)
  static constexpr int kStage = kQTile + kL1 + 1024;
  static constexpr int kPartOff = kStages * kStage;
  // a cluster member's partial U: 128 rows padded to R + 4 floats (16-byte rows, conflict-free
  // 16-byte accesses per quarter warp). Up to r = 32 the leader holds one slot per peer (at most 3),
  // which the peers write into; at r = 64 each CTA keeps its own, which the leader reads.
  static constexpr int kPart = (R + 4) * 128 * 4;
  static constexpr int kPartSlots = R <= 32 ? 3 : 1;
  static constexpr int kTabOff = kPartOff + kPartSlots * kPart;  // 128 fp32: 1 / (dec(s) g_x) per scale code
  static constexpr int kBarOff = kTabOff + 128 * 4;
  static constexpr int kNumBars = 2 * kStages + 2;
  static constexpr int kSmem = kBarOff + kNumBars * 8 + 16 + 1024;
  static constexpr int kTmemCols = R <= 32 ? 32 : 64;
  static_assert(kStage % 1024 == 0, "stage alignment");
  static_assert(kStages % 2 == 0, "each quantizer group owns the ring slots of one parity");
  static_assert(kSmem <= 232448, "shared memory budget");
};

struct QuantActArgs {
  const float* inv_lambda;
  const float* g_x;
  const float* g_w;
  uint8_t* codes;              // [M_pad][K/2]
  uint8_t* sf;                 // activation MMA layout
  __nv_bfloat16* U;            // [2][M_pad][r]: hi then lo
  float* alpha;
  unsigned long long wait_ns;
  int M, K, M_pad, k_per_cta;
};

// The NVFP4 quantizer of kernel 1 (a policy of quant_act_kernel). Rounding points as in the
// header of this file; the per-scale-code reciprocals 1 / (dec(s) g_x) live in a 128-entry table
// in shared memory (entry 0, an all-zero block whose codes are forced to +0, holds 0).
struct Nvfp4Act {
  using Args = QuantActArgs;
  __device__ static void prologue(const Args& a, float* tab) {
    const float gx = *a.g_x;
    if (threadIdx.x < 128) tab[threadIdx.x] = threadIdx.x ? __frcp_rn(__fmul_rn(e4m3_value(threadIdx.x), gx)) : 0.0f;
  }
  // One quantizer thread: 16-element block b of local rows rl and rl + 64 of every stage its
  // group takes (every other stage from `grp` on).
  struct Thread {
    float d6, rd6;
    const float* tab;
    uint8_t* code_ptr[2];
    uint8_t* sf_ptr[2];
    __device__ Thread(const Args& a, const float* tab_, int m_tile, int rl, int b, int kbeg, int grp) : tab(tab_) {
      d6 = __fmul_rn(6.0f, *a.g_x);
      rd6 = __frcp_rn(d6);
      // code and scale destinations at the group's first stage; a group step moves 64 code bytes
      // along the row and two 512-byte scale atoms along K
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int row = m_tile * 128 + rl + 64 * i;
        code_ptr[i] = a.codes + static_cast<size_t>(row) * (a.K >> 1) + ((kbeg + (b << 4)) >> 1) + (grp << 5);
        sf_ptr[i] = a.sf + act_sf_offset(row, (kbeg >> 4) + b, a.K) + (grp << 9);
      }
    }
    // the two blocks go through each phase together, so that their dependency chains interleave
    __device__ void stage(const float2 (&lam)[8], const uint4 (&x)[2][2]) {
      float2 v[2][8];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t wx[8] = {x[i][0].x, x[i][0].y, x[i][0].z, x[i][0].w, x[i][1].x, x[i][1].y, x[i][1].z, x[i][1].w};
#pragma unroll
        for (int j = 0; j < 8; ++j)
          v[i][j] = mul2_rn(make_float2(__uint_as_float(wx[j] << 16), __uint_as_float(wx[j] & 0xFFFF0000u)), lam[j]);
      }
      float am[2], qs[2];
      bool exact = false;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        am[i] = amax16(v[i]);
        qs[i] = __fmul_rn(am[i], rd6);
        exact |= scale_needs_division(qs[i]);
      }
      if (exact) {
#pragma unroll
        for (int i = 0; i < 2; ++i)
          if (scale_needs_division(qs[i])) qs[i] = __fdiv_rn(am[i], d6);
      }
      uint32_t sc[2];
      float rr[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        sc[i] = cvt_e4m3(qs[i]);
        rr[i] = tab[sc[i]];  // a zero scale multiplies by 0 and its codes are then forced to +0
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float2 r2 = make_float2(rr[i], rr[i]);
        float q[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 p = mul2_rn(v[i][j], r2);
          q[2 * j] = p.x;
          q[2 * j + 1] = p.y;
        }
        uint2 codes;
        codes.x = cvt_e2m1x8(*reinterpret_cast<const float(*)[8]>(q));
        codes.y = cvt_e2m1x8(*reinterpret_cast<const float(*)[8]>(q + 8));
        if (sc[i] == 0) codes = make_uint2(0u, 0u);
        *reinterpret_cast<uint2*>(code_ptr[i]) = codes;
        *sf_ptr[i] = static_cast<uint8_t>(sc[i]);
        code_ptr[i] += 64;
        sf_ptr[i] += 1024;
      }
    }
  };
  // U is stored divided by alpha = fp32(g_x g_w): one scale for the whole GEMM
  __device__ static float u_scale(const Args& a, int row) {
    (void)row;
    return __frcp_rn(__fmul_rn(*a.g_x, *a.g_w));
  }
  __device__ static void finish(const Args& a) {
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.alpha = __fmul_rn(*a.g_x, *a.g_w);
  }
};

template <int R, class Q>
__global__ void __launch_bounds__(kQ1Threads, 1)
    quant_act_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmL1,
                     const typename Q::Args a) {
  using L = Q1Layout<R>;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  const uint32_t accf_bar = bar0 + 8u * (2 * S);
  const uint32_t drain_bar = accf_bar + 8u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBarOff + L::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t csize = cluster_nctarank(), crank = cluster_ctarank();
  const int m_tile = blockIdx.x / csize;
  const int kbeg = static_cast<int>(crank) * a.k_per_cta;
  const int n_steps = a.k_per_cta >> 6;
  const int K = a.K;
  unsigned* status = &g_svdq_status;
  const uint64_t wait_ns = a.wait_ns;

  // Barrier set-up and the TMEM allocation touch no global memory, so they run before the wait for
  // the previous kernel on the stream (which may still be finishing: programmatic launch). The
  // first ring fill (one load per slot) is then issued by the producer thread at once, so its
  // latency overlaps the table set-up of the other warps.
  const int n_pre = n_steps < S ? n_steps : S;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 8 + (R > 0 ? 1 : 0));  // one quantizer group + the MMA commit
    }
    mbar_init(accf_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (R > 0 && warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  grid_dependency_wait();
  grid_launch_dependents();
  if (threadIdx.x == 0) {
    const uint64_t pol_x = l2_policy_evict_first();
    for (int st = 0; st < n_pre; ++st) {
      const uint32_t sa = sbase + st * L::kStage;
      mbar_arrive_expect_tx(full_bar(st), kQTile + R * 128 + 256);
      const int kx = kbeg + (st << 6);
      tma_load_2d_hint(sa, &tmX, kx, m_tile * 128, full_bar(st), pol_x);
      if (R > 0) tma_load_2d(sa + kQTile, &tmL1, kx, 0, full_bar(st));
      bulk_load(sa + L::kLamOff, a.inv_lambda + kx, 256, full_bar(st));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  float* tab = reinterpret_cast<float*>(smem + L::kTabOff);
  Q::prologue(a, tab);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = R > 0 ? *tmem_slot : 0u;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_x = l2_policy_evict_first();
      // stages 0 .. n_pre - 1 went out with the set-up (phase 0 of their slots)
      int stage = n_pre == S ? 0 : n_pre;
      uint32_t phase = n_pre == S ? 1u : 0u;
      uint32_t armed = (1u << n_pre) - 1u, armed_parity = 0;
      for (int st = n_pre; st < n_steps; ++st) {
        if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, wait_ns, status, kStatusProducer, abort_flag)) break;
        const uint32_t sa = sbase + stage * L::kStage;
        mbar_arrive_expect_tx(full_bar(stage), kQTile + R * 128 + 256);
        const int kx = kbeg + (st << 6);
        tma_load_2d_hint(sa, &tmX, kx, m_tile * 128, full_bar(stage), pol_x);
        if (R > 0) tma_load_2d(sa + kQTile, &tmL1, kx, 0, full_bar(stage));
        bulk_load(sa + L::kLamOff, a.inv_lambda + kx, 256, full_bar(stage));
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      for (int s = 0; s < S; ++s)
        if (armed & (1u << s))
          mbar_wait_bounded(full_bar(s), (armed_parity >> s) & 1u, wait_ns, status, kStatusDrain, nullptr);
    }
  } else if (warp == 1) {
    if (R > 0 && lane == 0) {
      int stage = 0;
      uint32_t phase = 0, accumulate = 0;
      bool ok = true;
      const uint32_t idesc = idesc_bf16(128, R);
      for (int st = 0; st < n_steps; ++st) {
        if (!(ok = mbar_wait_bounded(full_bar(stage), phase, wait_ns, status, kStatusMma, abort_flag))) break;
        tc_fence_after();
        const uint32_t sa = sbase + stage * L::kStage;
        const uint64_t dx = smem_desc(sa, 16, 1024, 2);
        const uint64_t dl = smem_desc(sa + kQTile, 16, 1024, 2);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          mma_bf16(tmem, dx + 2u * j, dl + 2u * j, idesc, accumulate);
          accumulate = 1;
        }
        tc_commit(empty_bar(stage));
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      if (ok) tc_commit(accf_bar);
      tc_commit(drain_bar);
      mbar_wait_bounded(drain_bar, 0, wait_ns, status, kStatusDrain, nullptr);
    }
  } else {
    // quantizers: group g = (warp - 2) / 8 takes stages g, g + 2, ...; within the group, thread t
    // of 256 owns 16-element block b = t % 4 of rows t / 4 and t / 4 + 64 of the stage. The four
    // threads of a row read its 128 swizzled bytes; a warp's 16-byte reads cover 8 rows x 4 blocks
    // and stay conflict-free (chunks 2b and 2b+1 XOR row % 8).
    const int qw = warp - 2;
    const int grp = qw >> 3;
    const int t = ((qw & 7) << 5) + lane;
    const int b = t & 3;
    typename Q::Thread qt(a, tab, m_tile, t >> 2, b, kbeg, grp);
    int stage = grp;
    uint32_t phase = 0;
    for (int st = grp; st < n_steps; st += 2) {
      const bool got = mbar_wait_bounded(full_bar(stage), phase, wait_ns, status, kStatusEpilogue, abort_flag);
      if (!__all_sync(0xffffffffu, got)) break;
      const uint8_t* tile = smem + stage * L::kStage;
      // this thread's 16 inverse smoothing factors travelled with the stage (a broadcast read: the
      // threads of one block index b share them)
      float2 lam[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 l = reinterpret_cast<const float4*>(tile + L::kLamOff)[4 * b + j];
        lam[2 * j] = make_float2(l.x, l.y);
        lam[2 * j + 1] = make_float2(l.z, l.w);
      }
      uint4 x[2][2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int rl = (t >> 2) + 64 * i;
        x[i][0] = *reinterpret_cast<const uint4*>(tile + rl * 128 + (((2 * b) ^ (rl & 7)) << 4));
        x[i][1] = *reinterpret_cast<const uint4*>(tile + rl * 128 + (((2 * b + 1) ^ (rl & 7)) << 4));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(stage));  // the stage's data is in registers
      qt.stage(lam, x);
      stage += 2;
      if (stage >= S) { stage -= S; phase ^= 1u; }
    }
    if constexpr (R > 0) {
      // warps 2..5 (quadrant q = warp % 4) read this CTA's rows of U from TMEM; a lone CTA
      // finishes them at once, a cluster member parks its partial in shared memory for the
      // cluster's first CTA, which adds the partials in rank order.
      const int q = warp & 3;
      const bool mine_rows = warp < 6;
      bool got = true;
      if (mine_rows) got = mbar_wait_bounded(accf_bar, 0, wait_ns, status, kStatusEpilogue, abort_flag);
      got = __all_sync(0xffffffffu, got) && mine_rows;
      float u[R];
#pragma unroll
      for (int j = 0; j < R; ++j) u[j] = 0.0f;
      if (got) {
        tc_fence_after();
        const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16);
        if constexpr (R == 16) {
          uint32_t rr[16];
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
              : "=r"(rr[0]), "=r"(rr[1]), "=r"(rr[2]), "=r"(rr[3]), "=r"(rr[4]), "=r"(rr[5]), "=r"(rr[6]), "=r"(rr[7]),
                "=r"(rr[8]), "=r"(rr[9]), "=r"(rr[10]), "=r"(rr[11]), "=r"(rr[12]), "=r"(rr[13]), "=r"(rr[14]),
                "=r"(rr[15])
              : "r"(ta));
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) u[e] = __uint_as_float(rr[e]);
        } else {
#pragma unroll
          for (int j = 0; j < R; j += 32) {
            float t32[32];
            tmem_ld_32x32(ta + j, t32);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) u[j + e] = t32[e];
          }
        }
        if (csize > 1 && crank != 0) {
          // up to r = 32 straight into the leader's slot for this rank (remote stores do not wait
          // for a reply; the cluster barrier below makes them visible), at r = 64 into this CTA
          float4* part = reinterpret_cast<float4*>(smem + L::kPartOff + (R <= 32 ? (crank - 1) * L::kPart : 0)) +
                         (q * 32 + lane) * ((R + 4) / 4);
          if constexpr (R <= 32) part = cluster_map_generic(part, 0);
#pragma unroll
          for (int j = 0; j < R; j += 4) part[j / 4] = make_float4(u[j], u[j + 1], u[j + 2], u[j + 3]);
        }
      }
      if (csize > 1) cluster_sync_all();
      if (got && crank == 0) {
        const int rl = q * 32 + lane;
        // Up to r = 32 the peers' rows are already in this CTA's slots. At r = 64, whose 64 values per
        // row already take most registers, the leader reads each peer's row with 4-byte remote loads,
        // 16 at a time. (One 4-byte remote load per value at a time took ~7 us on B200 for two peers.)
        for (uint32_t rk = 1; rk < csize; ++rk) {
          if constexpr (R <= 32) {
            const float4* pg =
                reinterpret_cast<const float4*>(smem + L::kPartOff + (rk - 1) * L::kPart) + rl * ((R + 4) / 4);
            float4 pv[R / 4];
#pragma unroll
            for (int e = 0; e < R / 4; ++e) pv[e] = pg[e];
#pragma unroll
            for (int e = 0; e < R / 4; ++e) {
              u[4 * e] += pv[e].x;
              u[4 * e + 1] += pv[e].y;
              u[4 * e + 2] += pv[e].z;
              u[4 * e + 3] += pv[e].w;
            }
          } else {
            const float* pg = cluster_map_generic(reinterpret_cast<const float*>(smem + L::kPartOff) + rl * (R + 4), rk);
#pragma unroll
            for (int j0 = 0; j0 < R; j0 += 16) {
              float pv[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) pv[e] = pg[j0 + e];
#pragma unroll
              for (int e = 0; e < 16; ++e) u[j0 + e] += pv[e];
            }
          }
        }
        const float cinv = Q::u_scale(a, m_tile * 128 + rl);
        __nv_bfloat16* u_hi = a.U + (static_cast<size_t>(m_tile) * 128 + rl) * R;
        __nv_bfloat16* u_lo = u_hi + static_cast<size_t>(a.M_pad) * R;
#pragma unroll
        for (int j = 0; j < R; j += 8) {
          uint32_t wh[4], wl[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float v0 = __fmul_rn(u[j + 2 * e], cinv), v1 = __fmul_rn(u[j + 2 * e + 1], cinv);
            const __nv_bfloat162 hi = __floats2bfloat162_rn(v0, v1);
            const __nv_bfloat162 lo = __floats2bfloat162_rn(__fsub_rn(v0, __low2float(hi)), __fsub_rn(v1, __high2float(hi)));
            wh[e] = *reinterpret_cast<const uint32_t*>(&hi);
            wl[e] = *reinterpret_cast<const uint32_t*>(&lo);
          }
          *reinterpret_cast<uint4*>(u_hi + j) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
          *reinterpret_cast<uint4*>(u_lo + j) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
        }
      }
    }
  }

  if constexpr (R == 0) {
    if (csize > 1) cluster_sync_all();
  } else {
    // warps 0 and 1 take part in the cluster barrier the quantizer warps passed above
    if (csize > 1 && warp < 2) cluster_sync_all();
  }
  Q::finish(a);
  // peers keep their shared memory until the leader has read it
  if (csize > 1) cluster_sync_all();
  tc_fence_before();
  __syncthreads();
  if (R > 0 && warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
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

// atomicMax of |x * inv_lambda| over X [M][K] bf16. Thread (blockIdx.x, threadIdx.x) owns the
// 8-column chunk c of every row blockIdx.y, blockIdx.y + gridDim.y, ...: its 8 inverse smoothing
// factors stay in registers, and a warp reads 32 consecutive 16-byte chunks of a row (four rows in
// flight per thread).
__global__ void act_amax_kernel(const __nv_bfloat16* __restrict__ X, const float* __restrict__ inv_lambda,
                                int M, int K, unsigned* out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int per_row = K >> 3;
  float m = 0.0f;
  if (c < per_row) {
    float lam[8];
    const float4 l0 = __ldg(reinterpret_cast<const float4*>(inv_lambda + 8 * c));
    const float4 l1 = __ldg(reinterpret_cast<const float4*>(inv_lambda + 8 * c) + 1);
    lam[0] = l0.x; lam[1] = l0.y; lam[2] = l0.z; lam[3] = l0.w;
    lam[4] = l1.x; lam[5] = l1.y; lam[6] = l1.z; lam[7] = l1.w;
    const int G = gridDim.y;
    const __nv_bfloat16* col = X + 8 * static_cast<size_t>(c);
    auto take = [&](uint4 raw) {
      float v[8];
      bf16x8_to_f32(raw, v);
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(__fmul_rn(v[j], lam[j])));
    };
    int r = blockIdx.y;
    for (; r + 3 * G < M; r += 4 * G) {
      const uint4 a0 = ldg_stream(col + static_cast<size_t>(r) * K);
      const uint4 a1 = ldg_stream(col + static_cast<size_t>(r + G) * K);
      const uint4 a2 = ldg_stream(col + static_cast<size_t>(r + 2 * G) * K);
      const uint4 a3 = ldg_stream(col + static_cast<size_t>(r + 3 * G) * K);
      take(a0);
      take(a1);
      take(a2);
      take(a3);
    }
    for (; r < M; r += G) take(ldg_stream(col + static_cast<size_t>(r) * K));
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
