// Kernel 2: block-scaled NVFP4 GEMM on the 5th-generation tensor cores (tcgen05), with the
// low-rank up-projection and the bias / SwiGLU epilogue fused in.
//
// Method ("Bringing Nunchaku 4-bit diffusion inference to Diffusers", "SVDQuant deep dive"): the
// branch's up-projection (X L1) L2 is fused with the 4-bit GEMM; here it is one extra bf16 MMA
// (K = r) into the same TMEM accumulator, with U pre-divided by alpha = g_x g_w so that a single
// scale applies at the end. The fused QKV / SwiGLU epilogues follow the fused NVFP4 GEMMs of
// "FLUX 3 Image Klein on NVIDIA Blackwell", method 1.
//
// Structure (one persistent CTA per SM, 6 warps):
//   warp 0      TMA producer: per 256-wide K step, A (128 x 128 B) and B (n_tile x 128 B) codes as
//               128B-swizzled 2-D tiles, plus the matching scale-factor atoms as 1-D bulk copies,
//               into a STAGES-deep shared-memory ring (full/empty mbarriers). Before a tile's K
//               loop, ring slots carry the tile's U_hi, U_lo (128 x r) and L2^T (n_tile x r) in
//               chunks of 32 columns of r.
//   warp 1      TMEM allocator + single-thread MMA issuer:
//               4 x tcgen05.mma kind::mxf4nvf4 (M=128, N=n_tile, K=64) per K step, 2 r/16 x
//               kind::f16 (hi and lo halves of U against the same L2 tile) for the low-rank term; tcgen05.commit frees ring slots and publishes
//               finished accumulators. Accumulators are double-buffered in TMEM when they fit.
//   warps 2..5  epilogue: tcgen05.ld (each warp its 32-lane quadrant), y = alpha acc (+ bias),
//               SwiGLU on interleaved gate/up columns, bf16 or fp32 store.
//   warps 6..9  scale-factor writers: per K step, copy the stage's E4M3 scale atoms from shared
//               memory into a double-buffered TMEM region with tcgen05.st (each warp its lane
//               quadrant). Measured on B200, every tcgen05.cp costs ~64 tensor-pipe cycles whatever
//               its shape, so copying 12 atoms per K step with tcgen05.cp starved the MMAs; stores
//               from four warps run beside the MMAs without slowing them.
// Every mbarrier wait is bounded (global timer); a wait that runs out records a status bit, sets
// a shared abort flag so that the other roles stop too, and the kernel drains its own copies and
// MMAs before freeing TMEM and returning.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "svdq_ptx.cuh"
#include "svdq_quant.cuh"

namespace svdq {

struct GemmArgs {
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* alpha;
  const __nv_bfloat16* bias;
  void* Y;
  unsigned long long wait_ns;
  int M, M_pad, N, K, r;
  int m_tiles, n_tiles, k_iters, num_tiles;
  int ldy, out_f32, epi;  // epi bit 0: bias, bit 1: SwiGLU
};

template <int N_TILE, int STAGES>
struct GemmLayout {
  static constexpr int kA = 128 * 128;
  static constexpr int kB = N_TILE * 128;
  static constexpr int kSfAtomsB = (N_TILE + 127) / 128;
  static constexpr int kSfa = 4 * 512;
  static constexpr int kSfb = 4 * kSfAtomsB * 512;
  static constexpr int kStage = kA + kB + kSfa + kSfb;
  static constexpr int kOffB = kA;
  static constexpr int kOffSfa = kA + kB;
  static constexpr int kOffSfb = kA + kB + kSfa;
  // TMEM scale-factor buffer (one K step): SFA 4 MMAs x 4 columns, then SFB 4 MMAs x 4 x atoms.
  static constexpr int kSfCols = 16 + 16 * kSfAtomsB;
  static constexpr int kAccBufs = (2 * N_TILE + 2 * kSfCols <= 512) ? 2 : 1;
  static constexpr int kColSf = kAccBufs * N_TILE;  // two buffers of kSfCols columns from here
  // epilogue staging: 4 warps x 2 buffers x (32 rows x 32 columns of fp32 at most)
  static constexpr int kStageOut = 32 * 32 * 4;
  static constexpr int kOutOff = STAGES * kStage;
  static constexpr int kBarOff = kOutOff + 4 * 2 * kStageOut;
  static constexpr int kNumBars = 2 * STAGES + 2 * kAccBufs + 1 + 4;
  static constexpr int kSmem = kBarOff + kNumBars * 8 + 16 + 1024;
  static_assert(kStage % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(kColSf + 2 * kSfCols <= 512, "TMEM budget");
  static_assert(kSmem <= 232448, "shared memory budget");
};

// Low-rank operands move in chunks of rc = min(r, 32) columns: U_hi, U_lo (128 x rc each) and
// L2^T (n_tile x rc), all bf16 with rc*2-byte rows (32B or 64B swizzle), one ring slot per chunk.
constexpr int kLrChunk = 32;
constexpr int kOffULo = 128 * kLrChunk * 2;
__device__ __forceinline__ uint32_t lr_swizzle_mode(int rc) { return rc == 16 ? 6u : 4u; }

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint4 (&v)[4]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0].x), "r"(v[0].y), "r"(v[0].z), "r"(v[0].w), "r"(v[1].x), "r"(v[1].y), "r"(v[1].z), "r"(v[1].w),
      "r"(v[2].x), "r"(v[2].y), "r"(v[2].z), "r"(v[2].w), "r"(v[3].x), "r"(v[3].y), "r"(v[3].z), "r"(v[3].w)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

constexpr int kGemmThreads = 320;

template <int N_TILE, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    svdq_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmL2,
                     const __grid_constant__ CUtensorMap tmY, const GemmArgs args) {
  using L = GemmLayout<N_TILE, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto accf_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto acce_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + L::kAccBufs + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 2 * L::kAccBufs);
  auto sf_full_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 * L::kAccBufs + 1 + b); };
  auto sf_free_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 * L::kAccBufs + 3 + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBarOff + L::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = args.r;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < L::kAccBufs; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), 4);
    }
    mbar_init(drain_bar, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(sf_full_bar(b), 4);
      mbar_init(sf_free_bar(b), 1);
    }
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
    tmem_alloc(smem_addr(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
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
      const uint32_t lr_bytes = static_cast<uint32_t>((2 * 128 + N_TILE) * rc * 2);
      const int sf_row_stride = args.K >> 6;  // 64-wide K atoms per 128-row block
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < args.num_tiles; tile += gridDim.x) {
        const int m_blk = tile % args.m_tiles, n_blk = tile / args.m_tiles;
        for (int c0 = 0; c0 < r; c0 += kLrChunk) {
          if (!(ok = mbar_wait_bounded(empty_bar(stage), phase ^ 1u, wait_ns, status, kStatusProducer, abort_flag)))
            break;
          const uint32_t sa = sbase + stage * L::kStage;
          mbar_arrive_expect_tx(full_bar(stage), lr_bytes);
          tma_load_2d(sa, &tmU, c0, m_blk * 128, full_bar(stage));
          tma_load_2d(sa + kOffULo, &tmU, c0, args.M_pad + m_blk * 128, full_bar(stage));
          tma_load_2d(sa + L::kOffB, &tmL2, c0, n_blk * N_TILE, full_bar(stage));
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        const uint8_t* sfa_tile = args.sfa + (static_cast<size_t>(m_blk) * sf_row_stride << 9);
        const uint8_t* sfb_tile = args.sfb + (static_cast<size_t>(n_blk) * sf_row_stride * L::kSfAtomsB << 9);
        for (int kt = 0; kt < args.k_iters; ++kt) {
          if (!(ok = mbar_wait_bounded(empty_bar(stage), phase ^ 1u, wait_ns, status, kStatusProducer, abort_flag)))
            break;
          const uint32_t sa = sbase + stage * L::kStage;
          mbar_arrive_expect_tx(full_bar(stage), L::kStage);
          tma_load_2d(sa, &tmA, kt * 128, m_blk * 128, full_bar(stage));
          tma_load_2d(sa + L::kOffB, &tmB, kt * 128, n_blk * N_TILE, full_bar(stage));
          bulk_load(sa + L::kOffSfa, sfa_tile + (static_cast<size_t>(kt) * 4 << 9), L::kSfa, full_bar(stage));
          bulk_load(sa + L::kOffSfb, sfb_tile + (static_cast<size_t>(kt) * 4 * L::kSfAtomsB << 9), L::kSfb,
                    full_bar(stage));
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
    // ------------------------------------------------------------------ MMA issuer
    // Per K step: wait for the step's scale buffer (the writers arrive there only after they have
    // seen the stage's data land), 4 MMAs, one commit that releases the stage (the writers also take
    // it as the release of the scale buffer used two steps back).
    // The whole warp runs this loop (warp-uniform operands); elect.sync inside the MMA and commit
    // helpers picks the issuing lane, and a wait succeeds only when it succeeds in every lane.
    auto wait_all = [&](uint32_t bar, uint32_t parity, unsigned code, volatile int* abort_ptr) {
      return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, wait_ns, status, code, abort_ptr));
    };
    const int num_tiles = args.num_tiles, k_iters = args.k_iters;
    const int rc = r < kLrChunk ? r : kLrChunk;
    const int nj = rc >> 4;
    const uint32_t idesc_fp4 = idesc_nvfp4(128, N_TILE);
    const uint32_t idesc_lr = idesc_bf16(128, N_TILE);
    // descriptor halves: low = start address / 16 | LBO (16 B) / 16 << 16; high = SBO / 16 |
    // version 1 | swizzle mode << 29
    const uint32_t lo0 = (sbase >> 4) | (1u << 16);
    const uint32_t hi_ab = (1024u >> 4) | (1u << 14) | (2u << 29);
    const uint32_t hi_lr = ((8u * rc * 2u) >> 4) | (1u << 14) | (lr_swizzle_mode(rc) << 29);
    const uint32_t tsf0 = tmem + L::kColSf;
    int stage = 0, sfb = 0, acc = 0;
    uint32_t phase = 0, sf_phase = 0, acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      if (!(ok = wait_all(acce_bar(acc), acc_phase ^ 1u, kStatusMma, abort_flag))) break;
      const uint32_t d = tmem + static_cast<uint32_t>(acc * N_TILE);
      uint32_t accumulate = 0;
      for (int c0 = 0; c0 < r; c0 += kLrChunk) {
        if (!(ok = wait_all(full_bar(stage), phase, kStatusMma, abort_flag))) break;
        tc_fence_after();
        const uint32_t lo = lo0 + stage * (L::kStage >> 4);
        for (int j = 0; j < nj; ++j) {
          const uint64_t bl = desc_join(lo + (L::kOffB >> 4) + 2u * j, hi_lr);
          mma_bf16_warp(d, desc_join(lo + 2u * j, hi_lr), bl, idesc_lr, accumulate);
          mma_bf16_warp(d, desc_join(lo + (kOffULo >> 4) + 2u * j, hi_lr), bl, idesc_lr, 1u);
          accumulate = 1;
        }
        tc_commit_warp(empty_bar(stage));
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      for (int kt = 0; kt < k_iters; ++kt) {
        // The wait sits before the step's first MMA: placed between queued MMAs, a barrier wait
        // measurably stalled the tensor pipe on B200.
        if (!(ok = wait_all(sf_full_bar(sfb), sf_phase, kStatusMma, abort_flag))) break;
        tc_fence_after();
        const uint32_t la = lo0 + stage * (L::kStage >> 4);
        const uint32_t lb = la + (L::kOffB >> 4);
        const uint32_t tsf = tsf0 + sfb * L::kSfCols;
        mma_nvfp4_warp(d, desc_join(la, hi_ab), desc_join(lb, hi_ab), idesc_fp4, tsf, tsf + 16, accumulate);
        mma_nvfp4_warp(d, desc_join(la + 2u, hi_ab), desc_join(lb + 2u, hi_ab), idesc_fp4, tsf + 4,
                       tsf + 16 + 4 * L::kSfAtomsB, 1u);
        mma_nvfp4_warp(d, desc_join(la + 4u, hi_ab), desc_join(lb + 4u, hi_ab), idesc_fp4, tsf + 8,
                       tsf + 16 + 8 * L::kSfAtomsB, 1u);
        mma_nvfp4_warp(d, desc_join(la + 6u, hi_ab), desc_join(lb + 6u, hi_ab), idesc_fp4, tsf + 12,
                       tsf + 16 + 12 * L::kSfAtomsB, 1u);
        accumulate = 1;
        tc_commit_warp(empty_bar(stage));
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        if (++sfb == 2) { sfb = 0; sf_phase ^= 1u; }
      }
      if (!ok) break;
      tc_commit_warp(accf_bar(acc));
      if (++acc == L::kAccBufs) { acc = 0; acc_phase ^= 1u; }
    }
    // Drain: all issued MMAs complete before TMEM is freed.
    tc_commit_warp(drain_bar);
    wait_all(drain_bar, 0, kStatusDrain, nullptr);
  } else if (warp >= 6) {
    // ------------------------------------------------------------------ scale-factor writers (warps 6..9)
    // Each warp owns one TMEM lane quadrant and writes into it the replicated scale-factor layout
    // the block-scaled MMA reads: for a 128-row atom, lane l, column c holds the 4 E4M3 scales of
    // row l + 32 c -- exactly bytes [16 l, 16 l + 16) of the 512-byte atom in shared memory.
    const int q = warp & 3;
    int stage = 0, sfb = 0;
    uint32_t phase = 0, sf_phase = 0;
    // (stage, phase) of the last two K steps: buffer sfb was last read by the K step two back, and
    // the MMA thread's release of that step's stage completes once those MMAs have finished.
    int h_stage0 = -1, h_stage1 = -1;
    uint32_t h_phase0 = 0, h_phase1 = 0;
    const int lr_slots = (r + kLrChunk - 1) / kLrChunk;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < args.num_tiles; tile += gridDim.x) {
      for (int c = 0; c < lr_slots; ++c)
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      for (int kt = 0; kt < args.k_iters; ++kt) {
        const bool got_data = mbar_wait_bounded(full_bar(stage), phase, wait_ns, status, kStatusEpilogue, abort_flag);
        if (!__all_sync(0xffffffffu, got_data)) { ok = false; break; }
        // read the stage's scale atoms now; only the TMEM stores wait for the buffer
        const uint8_t* sfs = smem + stage * L::kStage + L::kOffSfa + lane * 16;
        uint4 fa[4], fb[4 * L::kSfAtomsB];
#pragma unroll
        for (int i = 0; i < 4; ++i) fa[i] = *reinterpret_cast<const uint4*>(sfs + 512 * i);
#pragma unroll
        for (int i = 0; i < 4 * L::kSfAtomsB; ++i)
          fb[i] = *reinterpret_cast<const uint4*>(smem + stage * L::kStage + L::kOffSfb + lane * 16 + 512 * i);
        bool got = true;
        const int hs = sfb ? h_stage1 : h_stage0;
        const uint32_t hp = sfb ? h_phase1 : h_phase0;
        if (hs >= 0) got = mbar_wait_bounded(empty_bar(hs), hp, wait_ns, status, kStatusEpilogue, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tsf = tmem + (static_cast<uint32_t>(q * 32) << 16) + L::kColSf + sfb * L::kSfCols;
        tmem_st_x16(tsf, fa);
#pragma unroll
        for (int h = 0; h < L::kSfAtomsB; ++h) {
          const uint4 v[4] = {fb[4 * h], fb[4 * h + 1], fb[4 * h + 2], fb[4 * h + 3]};
          tmem_st_x16(tsf + 16 + 16 * h, v);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sf_full_bar(sfb));
        if (sfb) {
          h_stage1 = stage;
          h_phase1 = phase;
        } else {
          h_stage0 = stage;
          h_phase0 = phase;
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        if (++sfb == 2) { sfb = 0; sf_phase ^= 1u; }
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    // Each warp drains its 32-lane TMEM quadrant 32 columns at a time, applies alpha / bias /
    // SwiGLU, writes the 32 x 32 block into a swizzled shared-memory buffer (64B swizzle for bf16,
    // 128B for fp32 rows: conflict-free 16-byte writes) and one lane stores it with a TMA tensor
    // store; two buffers per warp let the next block fill while the previous store drains. Rows at
    // or beyond M are clipped by the tensor map.
    const int q = warp & 3;
    const float alpha = *args.alpha;
    const bool has_bias = (args.epi & 1) != 0;
    const bool swiglu = (args.epi & 2) != 0;
    const bool f32 = args.out_f32 != 0;
    const int hN = args.N >> 1;
    uint8_t* stage_out = smem + L::kOutOff + q * 2 * L::kStageOut;
    int buf = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    auto emit = [&](const float (&v)[32], int row0, int col0) {
      // buffer reuse: the store issued from it two blocks ago has finished reading
      if (lane == 0) bulk_wait_group_read<1>();
      __syncwarp();
      uint8_t* dst = stage_out + buf * L::kStageOut;
      if (f32) {
        // 128-byte rows, 8 chunks of 16 bytes; chunk j of row `lane` lives at j ^ (lane % 8)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<float4*>(dst + lane * 128 + ((j ^ (lane & 7)) << 4)) =
              make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      } else {
        // 64-byte rows, 4 chunks; chunk j of row `lane` lives at j ^ ((lane / 2) % 4)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * j + 2 * e], v[8 * j + 2 * e + 1]);
            w[e] = *reinterpret_cast<const uint32_t*>(&h);
          }
          *reinterpret_cast<uint4*>(dst + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&tmY, smem_addr(dst), col0, row0);
        bulk_commit_group();
      }
      buf ^= 1;
    };
    for (int tile = blockIdx.x; tile < args.num_tiles; tile += gridDim.x) {
      const int m_blk = tile % args.m_tiles, n_blk = tile / args.m_tiles;
      // warp-uniform outcome: tcgen05.ld below is a .sync.aligned warp instruction
      const bool got = mbar_wait_bounded(accf_bar(acc), acc_phase, wait_ns, status, kStatusEpilogue, abort_flag);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int row0 = m_blk * 128 + q * 32;
      const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * N_TILE);
      if (!swiglu) {
#pragma unroll 1
        for (int c = 0; c < N_TILE / 32; ++c) {
          float v[32];
          tmem_ld_32x32(tb + c * 32, v);
          tmem_wait_ld();
          if (c == N_TILE / 32 - 1) {
            // all of this accumulator is in registers or already consumed: hand it back early
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce_bar(acc));
          }
          const int n0 = n_blk * N_TILE + c * 32;
          if (has_bias) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              float b[8];
              bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(args.bias + n0 + i)), b);
#pragma unroll
              for (int j = 0; j < 8; ++j) v[i + j] = fmaf(alpha, v[i + j], b[j]);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = alpha * v[i];
          }
          emit(v, row0, n0);
        }
      } else {
        constexpr int kHalf = N_TILE / 2;
#pragma unroll 1
        for (int c = 0; c < kHalf / 32; ++c) {
          float gt[32], up[32];
          tmem_ld_32x32(tb + c * 32, gt);
          tmem_ld_32x32(tb + kHalf + c * 32, up);
          tmem_wait_ld();
          if (c == kHalf / 32 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce_bar(acc));
          }
          const int j0 = n_blk * kHalf + c * 32;
          if (has_bias) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              float bg[8], bu[8];
              bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(args.bias + j0 + i)), bg);
              bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(args.bias + hN + j0 + i)), bu);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                gt[i + j] = fmaf(alpha, gt[i + j], bg[j]);
                up[i + j] = fmaf(alpha, up[i + j], bu[j]);
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              gt[i] = alpha * gt[i];
              up[i] = alpha * up[i];
            }
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) gt[i] = gt[i] / (1.0f + __expf(-gt[i])) * up[i];
          emit(gt, row0, j0);
        }
      }
      if (++acc == L::kAccBufs) { acc = 0; acc_phase ^= 1u; }
    }
    // every TMA store issued by this warp has completed before the CTA may exit
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace svdq
