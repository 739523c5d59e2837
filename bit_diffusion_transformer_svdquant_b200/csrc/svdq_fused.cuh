// The next layer's kernel 1 fused into the SwiGLU epilogue of the gate/up GEMM (the MLP chain).
//
// Method ("Bringing Nunchaku 4-bit diffusion inference to Diffusers", "SVDQuant deep dive": the
// branch's down-projection is fused with activation quantization; "FLUX 3 Image Klein on NVIDIA
// Blackwell", method 1: fused SwiGLU NVFP4 GEMMs). In the unfused chain the gate/up GEMM writes the
// SwiGLU output h (bf16) and the down layer's kernel 1 reads it back to smooth, quantize and
// project it. Here the gate/up GEMM's epilogue does that work on h while it is on chip:
//   * NVFP4 codes and scales of x = fp32(h * inv_lambda') with the down layer's static g_x' (the
//     same arithmetic as kernel 1, so the codes are bit-identical to the unfused chain's);
//   * the down-projection U' = h L1s' as pair MMAs over the tile's 128 columns of h, accumulated in
//     TMEM across the column tiles a CTA pair sweeps; the pair writes its partial sum once per
//     sweep and finalize_u_kernel adds the partials in a fixed order and stores U' / alpha' as the
//     bf16 hi/lo pair kernel 1 writes.
// h itself goes to HBM only if the caller asks for it.
//
// Structure: the NVFP4 CTA-pair GEMM at n_tile 256 (warp 0 producer, warp 1 TMEM + issuer,
// warps 2..9 epilogue, warps 10..13 scale writers) with these changes:
//   schedule   units of (256-row block, column split): a pair sweeps the split's column tiles of one
//              row block in order, so U' accumulates in its TMEM; splits are chosen so that the
//              units about fill the resident pairs;
//   producer   after a tile's K steps, the PREVIOUS tile's L1s'^T slice (r/2 rows per CTA x 128
//              columns, two 128B-swizzled boxes) into the next ring slot, so that no slice buffer
//              takes the shared memory of a fifth ring stage (the writers report that slot like a
//              low-rank slot, and the U' MMAs that read it release it);
//   issuer     after tile t's K loop it issues the U' MMAs of tile t-1 (the epilogue of t-1 ran
//              meanwhile), then the accumulator commit of t; the unit's first U' MMA overwrites
//              the U' accumulator once the previous unit's has been drained;
//   epilogue   h = SwiGLU(alpha acc + bias) is rounded to bf16 and written into the staging area
//              as a 128B-swizzled K-major 128 x 128 tile (the U' MMA's A operand); after the
//              accumulator is released the h tile is read back and quantized for the next layer;
//              at the end of a unit four warps per CTA drain U' into the partials buffer.
// Barriers added to the GEMM's, each completing once per use in an order that no waiter can fall
// two phases behind: h_full (both CTAs' h tiles written; the even CTA's), h_empty (the h tile read),
// u_done (a unit's U' complete), u_free (a unit's U' drained; the even CTA's).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "svdq_gemm.cuh"
#include "svdq_ptx.cuh"
#include "svdq_quant.cuh"

namespace svdq {
namespace fused {

// Arrive with cluster-scope release: the shared-memory writes before it (fenced to the async proxy)
// are read by a pair MMA that the other CTA issues.
__device__ __forceinline__ void mbar_arrive_release_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

struct Args {
  // the gate/up layer
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* alpha;
  const __nv_bfloat16* bias;   // [N] original column order, or null
  unsigned long long wait_ns;
  int M, M_pad, N, K, r;
  int m_tiles, m_pairs, n_tiles, k_iters;
  int splits, num_units;       // units = m_pairs * splits
  int store_h;                 // 1: also store h (bf16 [M][N/2]) through tmH
  // the next layer
  const float* inv_lambda2;    // [K2] smoothing reciprocals
  const float* g_x2;           // static activation scale
  uint8_t* codes2;             // [M_pad][K2/2]
  uint8_t* sf2;                // activation scale atoms
  float* partials;             // [splits][M_pad][r2] fp32
  int K2;                      // = N / 2
};

template <int STAGES, int R2>
struct Layout {
  using G = GemmLayout<256, STAGES>;
  static constexpr int kStage = G::kStage;
  static constexpr int kHTile = 128 * 128 * 2;        // 128 rows x 128 bf16: two 64-column atoms
  static constexpr int kHOff = STAGES * kStage;
  // a tile's L1s'^T slice (r/2 rows x 128 bf16 columns per CTA, two 64-column atoms) travels in a
  // ring slot of its own, right before the U' MMAs that read it
  static constexpr int kSliceAtom = (R2 / 2) * 128;
  static constexpr int kSlice = 2 * kSliceAtom;
  static constexpr int kTabOff = kHOff + kHTile;  // 128 fp32: 1 / (dec(s) g_x') per scale code
  static constexpr int kBarOff = kTabOff + 512;
  // full[S], empty[S], accf, acce, drain, sf_full[4], h_full, h_empty, u_done, u_free
  static constexpr int kNumBars = 2 * STAGES + 3 + G::kSfBufs + 4;
  static constexpr int kSmem = kBarOff + kNumBars * 8 + 16 + 1024;
  static constexpr int kColU = G::kColSf + G::kSfBufs * G::kSfCols;  // U' accumulator columns
  static_assert(G::kAccBufs == 1, "one 256-column accumulator");
  static_assert(kColU + R2 <= 512, "TMEM budget");
  static_assert(kHOff % 1024 == 0 && kSliceAtom % 1024 == 0, "128B-swizzled tiles start on 1024-byte boundaries");
  static_assert(kSlice <= kStage, "a slice fits a ring stage");
  static_assert(G::kSfBufs <= STAGES, "a scale buffer's previous slot must still own its ring stage");
  static_assert(kSmem <= 232448, "shared memory budget");
};

__device__ __forceinline__ void unit_range(int unit, int splits, int n_tiles, int& m_pair, int& split, int& n_beg,
                                           int& n_end) {
  m_pair = unit / splits;
  split = unit - m_pair * splits;
  n_beg = split * n_tiles / splits;
  n_end = (split + 1) * n_tiles / splits;
}

// Byte offset of the 16-byte chunk `chunk` (columns 8 chunk .. 8 chunk + 7 of a 64-column atom) of
// row `row` in a 128B-swizzled K-major tile of 128-byte rows.
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int STAGES, int R2>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_swiglu_quant_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmL2,
                             const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmL1n,
                             const Args args) {
  using L = Layout<STAGES, R2>;
  using G = typename L::G;
  constexpr int N_TILE = 256, kHalf = 128;
  constexpr int kSfBufs = G::kSfBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  const uint32_t accf_bar = bar0 + 8u * (2 * STAGES);
  const uint32_t acce_bar = accf_bar + 8u;
  const uint32_t drain_bar = accf_bar + 16u;
  auto sf_full_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 3 + b); };
  const uint32_t h_full_bar = bar0 + 8u * (2 * STAGES + 3 + kSfBufs);
  const uint32_t h_empty_bar = h_full_bar + 8u;
  const uint32_t u_done_bar = h_full_bar + 16u;
  const uint32_t u_free_bar = h_full_bar + 24u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBarOff + L::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t h_tile = sbase + L::kHOff;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = args.r;
  const uint32_t rank = cluster_ctarank();  // 0: issues the pair's MMAs
  const int pair0 = static_cast<int>(cluster_id_x()), npairs = static_cast<int>(num_clusters_x());

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(accf_bar, 1);
    mbar_init(acce_bar, 16);  // 8 epilogue warps in each CTA
    mbar_init(drain_bar, 1);
    for (int b = 0; b < kSfBufs; ++b) mbar_init(sf_full_bar(b), 8);  // 4 writer warps in each CTA
    mbar_init(h_full_bar, 16);  // 8 epilogue warps in each CTA
    mbar_init(h_empty_bar, 1);
    mbar_init(u_done_bar, 1);
    mbar_init(u_free_bar, 8);   // 4 draining warps in each CTA
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmL1n);
    if (args.store_h) prefetch_tmap(&tmH);
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
  // The set-up above touches no global memory, so it overlaps the end of the previous kernel on the
  // stream (programmatic launch); everything below may read what that kernel wrote.
  grid_dependency_wait();
  grid_launch_dependents();
  // the next layer's reciprocal-scale table, as kernel 1 builds it
  if (threadIdx.x < 128) {
    const float gx2 = *args.g_x2;
    reinterpret_cast<float*>(smem + L::kTabOff)[threadIdx.x] = __frcp_rn(__fmul_rn(e4m3_value(threadIdx.x), gx2));
  }
  __syncthreads();
  const uint32_t tmem = *tmem_slot;
  unsigned* status = &g_svdq_status;
  const uint64_t wait_ns = args.wait_ns;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      const int rc = r < kLrChunk ? r : kLrChunk;
      const uint32_t lr_bytes = static_cast<uint32_t>((2 * 128 + G::kBRows) * rc * 2);
      const int sf_row_stride = args.K >> 6;
      const int y_slice = static_cast<int>(rank) * (R2 / 2);
      int prev_n_blk = -1;  // the tile whose U' MMAs come next (after this tile's K steps)
      bool ok = true;
      // the L1s'^T slice of tile `nb` (next-layer K columns nb*128 .. +127, this CTA's r/2 rows) into
      // the next ring slot, which its U' MMAs read and release
      auto load_slice = [&](int nb) -> bool {
        if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, wait_ns, status, kStatusProducer, abort_flag)) return false;
        const uint32_t sa = sbase + stage * L::kStage;
        mbar_arrive_expect_tx(full_bar(stage), L::kSlice);
        tma_load_2d(sa, &tmL1n, nb * kHalf, y_slice, full_bar(stage));
        tma_load_2d(sa + L::kSliceAtom, &tmL1n, nb * kHalf + 64, y_slice, full_bar(stage));
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        return true;
      };
      for (int unit = pair0; ok && unit < args.num_units; unit += npairs) {
        int m_pair, split, n_beg, n_end;
        unit_range(unit, args.splits, args.n_tiles, m_pair, split, n_beg, n_end);
        const int m_blk = 2 * m_pair + static_cast<int>(rank);
        const int m_sf = m_blk < args.m_tiles ? m_blk : args.m_tiles - 1;
        for (int n_blk = n_beg; ok && n_blk < n_end; ++n_blk) {
          const int b_row = n_blk * N_TILE + static_cast<int>(rank) * G::kBRows;
          for (int c0 = 0; c0 < r; c0 += kLrChunk) {
            if (!(ok = mbar_wait_bounded(empty_bar(stage), phase ^ 1u, wait_ns, status, kStatusProducer, abort_flag)))
              break;
            const uint32_t sa = sbase + stage * L::kStage;
            mbar_arrive_expect_tx(full_bar(stage), lr_bytes);
            tma_load_2d(sa, &tmU, c0, m_blk * 128, full_bar(stage));
            tma_load_2d(sa + kOffULo, &tmU, c0, args.M_pad + m_blk * 128, full_bar(stage));
            tma_load_2d(sa + G::kOffB, &tmL2, c0, b_row, full_bar(stage));
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          const uint8_t* sfa_tile = args.sfa + (static_cast<size_t>(m_sf) * sf_row_stride << 9);
          const uint8_t* sfb_tile = args.sfb + (static_cast<size_t>(n_blk) * sf_row_stride * G::kSfAtomsB << 9);
          for (int kt = 0; kt < args.k_iters; ++kt) {
            if (!(ok = mbar_wait_bounded(empty_bar(stage), phase ^ 1u, wait_ns, status, kStatusProducer, abort_flag)))
              break;
            const uint32_t sa = sbase + stage * L::kStage;
            mbar_arrive_expect_tx(full_bar(stage), L::kStage);
            tma_load_2d(sa, &tmA, kt * 128, m_blk * 128, full_bar(stage));
            tma_load_2d(sa + G::kOffB, &tmB, kt * 128, b_row, full_bar(stage));
            bulk_load(sa + G::kOffSfa, sfa_tile + (static_cast<size_t>(kt) * 4 << 9), G::kSfa, full_bar(stage));
            bulk_load(sa + G::kOffSfb, sfb_tile + (static_cast<size_t>(kt) * 4 * G::kSfAtomsB << 9), G::kSfb,
                      full_bar(stage));
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          // the previous tile's slice, for the U' MMAs the issuer adds after this tile's K steps
          if (prev_n_blk >= 0 && !(ok = load_slice(prev_n_blk))) break;
          prev_n_blk = n_blk;
        }
      }
      if (ok && prev_n_blk >= 0) load_slice(prev_n_blk);
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
      const int k_iters = args.k_iters;
      const int rc = r < kLrChunk ? r : kLrChunk;
      const int nj = rc >> 4;
      const uint32_t idesc_fp4 = idesc_nvfp4(256, N_TILE);
      const uint32_t idesc_lr = idesc_bf16(256, N_TILE);
      const uint32_t idesc_u = idesc_bf16(256, R2);
      const uint32_t lo0 = (sbase >> 4) | (1u << 16);
      const uint32_t hi_ab = (1024u >> 4) | (1u << 14) | (2u << 29);
      const uint32_t hi_lr = ((8u * rc * 2u) >> 4) | (1u << 14) | (lr_swizzle_mode(rc) << 29);
      const uint32_t tsf0 = tmem + G::kColSf;
      const uint32_t d_u = tmem + L::kColU;
      constexpr uint16_t kBoth = 3;
      int stage = 0, sfb = 0, tseq = 0, useq = 0;
      uint32_t phase = 0, sf_phase = 0, acc_phase = 0;
      // the tile whose U' MMAs are still to be issued (its epilogue runs under the next tile's MMAs)
      int pend = -1;
      bool pend_first = false, pend_last = false;
      bool ok = true;
      // U' += h(t) L1s'(t): A = the h tile (two 64-column atoms, 128 rows per CTA), B = tile t's slice
      // in the next ring slot (both CTAs' halves landed once the slot's sf_full completes)
      auto issue_u = [&](int t, bool first, bool last) -> bool {
        if (!wait_all(h_full_bar, static_cast<uint32_t>(t) & 1u, kStatusMma, abort_flag)) return false;
        if (first && useq > 0 && !wait_all(u_free_bar, static_cast<uint32_t>(useq - 1) & 1u, kStatusMma, abort_flag))
          return false;
        if (!wait_all(sf_full_bar(sfb), sf_phase, kStatusMma, abort_flag)) return false;
        tc_fence_after();
        const uint32_t la = (h_tile >> 4) | (1u << 16);
        const uint32_t lb = lo0 + stage * (L::kStage >> 4);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t a_off = static_cast<uint32_t>((j >> 2) * (16384 >> 4) + (j & 3) * 2);
          const uint32_t b_off = static_cast<uint32_t>((j >> 2) * (L::kSliceAtom >> 4) + (j & 3) * 2);
          mma_bf16_pair_warp(d_u, desc_join(la + a_off, hi_ab), desc_join(lb + b_off, hi_ab), idesc_u,
                             (first && j == 0) ? 0u : 1u);
        }
        tc_commit_pair_mc_warp(empty_bar(stage), kBoth);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        if (++sfb == kSfBufs) { sfb = 0; sf_phase ^= 1u; }
        tc_commit_pair_mc_warp(h_empty_bar, kBoth);
        if (last) {
          tc_commit_pair_mc_warp(u_done_bar, kBoth);
          ++useq;
        }
        return true;
      };
      for (int unit = pair0; ok && unit < args.num_units; unit += npairs) {
        int m_pair, split, n_beg, n_end;
        unit_range(unit, args.splits, args.n_tiles, m_pair, split, n_beg, n_end);
        for (int n_blk = n_beg; ok && n_blk < n_end; ++n_blk, ++tseq) {
          if (!(ok = wait_all(acce_bar, acc_phase ^ 1u, kStatusMma, abort_flag))) break;
          const uint32_t d = tmem;
          uint32_t accumulate = 0;
          for (int c0 = 0; c0 < r; c0 += kLrChunk) {
            if (!(ok = wait_all(sf_full_bar(sfb), sf_phase, kStatusMma, abort_flag))) break;
            tc_fence_after();
            const uint32_t lo = lo0 + stage * (L::kStage >> 4);
            for (int j = 0; j < nj; ++j) {
              const uint64_t bl = desc_join(lo + (G::kOffB >> 4) + 2u * j, hi_lr);
              mma_bf16_pair_warp(d, desc_join(lo + 2u * j, hi_lr), bl, idesc_lr, accumulate);
              mma_bf16_pair_warp(d, desc_join(lo + (kOffULo >> 4) + 2u * j, hi_lr), bl, idesc_lr, 1u);
              accumulate = 1;
            }
            tc_commit_pair_mc_warp(empty_bar(stage), kBoth);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            if (++sfb == kSfBufs) { sfb = 0; sf_phase ^= 1u; }
          }
          if (!ok) break;
          for (int kt = 0; kt < k_iters; ++kt) {
            if (!(ok = wait_all(sf_full_bar(sfb), sf_phase, kStatusMma, abort_flag))) break;
            tc_fence_after();
            const uint32_t la = lo0 + stage * (L::kStage >> 4);
            const uint32_t lb = la + (G::kOffB >> 4);
            const uint32_t tsf = tsf0 + sfb * G::kSfCols;
            mma_nvfp4_pair_warp(d, desc_join(la, hi_ab), desc_join(lb, hi_ab), idesc_fp4, tsf, tsf + 16, accumulate);
            mma_nvfp4_pair_warp(d, desc_join(la + 2u, hi_ab), desc_join(lb + 2u, hi_ab), idesc_fp4, tsf + 4,
                                tsf + 16 + 4 * G::kSfAtomsB, 1u);
            mma_nvfp4_pair_warp(d, desc_join(la + 4u, hi_ab), desc_join(lb + 4u, hi_ab), idesc_fp4, tsf + 8,
                                tsf + 16 + 8 * G::kSfAtomsB, 1u);
            mma_nvfp4_pair_warp(d, desc_join(la + 6u, hi_ab), desc_join(lb + 6u, hi_ab), idesc_fp4, tsf + 12,
                                tsf + 16 + 12 * G::kSfAtomsB, 1u);
            accumulate = 1;
            tc_commit_pair_mc_warp(empty_bar(stage), kBoth);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            if (++sfb == kSfBufs) { sfb = 0; sf_phase ^= 1u; }
          }
          if (!ok) break;
          if (pend >= 0 && !(ok = issue_u(pend, pend_first, pend_last))) break;
          tc_commit_pair_mc_warp(accf_bar, kBoth);
          acc_phase ^= 1u;
          pend = tseq;
          pend_first = n_blk == n_beg;
          pend_last = n_blk == n_end - 1;
        }
      }
      if (ok && pend >= 0) issue_u(pend, pend_first, pend_last);
      // Drain: all issued MMAs complete before TMEM may be freed.
      tc_commit_pair_mc_warp(drain_bar, 1);
      __all_sync(0xffffffffu, mbar_wait_bounded(drain_bar, 0, wait_ns, status, kStatusDrain, nullptr));
    }
  } else if (warp >= 10) {
    // ------------------------------------------------------------------ scale-factor writers (warps 10..13)
    // As in the NVFP4 GEMM: per ring slot, the step's scale atoms into one of 4 TMEM scale buffers,
    // then an arrive on the issuer's barrier in the even CTA.
    const int q = warp & 3;
    int stage = 0, sfb = 0, slots_done = 0;
    uint32_t phase = 0;
    const int lr_slots = (r + kLrChunk - 1) / kLrChunk;
    // one ring slot: wait for this CTA's data, store its scale atoms (K-step slots only), report it
    auto slot = [&](bool has_sf) -> bool {
      const bool got_data = mbar_wait_bounded(full_bar(stage), phase, wait_ns, status, kStatusEpilogue, abort_flag);
      if (!__all_sync(0xffffffffu, got_data)) return false;
      uint4 fa[4], fb[4 * G::kSfAtomsB];
      if (has_sf) {
        const uint8_t* sfs = smem + stage * L::kStage + G::kOffSfa + lane * 16;
#pragma unroll
        for (int i = 0; i < 4; ++i) fa[i] = *reinterpret_cast<const uint4*>(sfs + 512 * i);
#pragma unroll
        for (int i = 0; i < 4 * G::kSfAtomsB; ++i)
          fb[i] = *reinterpret_cast<const uint4*>(smem + stage * L::kStage + G::kOffSfb + lane * 16 + 512 * i);
      }
      bool got = true;
      if (slots_done >= kSfBufs) {
        int ps = stage - kSfBufs;
        uint32_t pp = phase;
        if (ps < 0) {
          ps += STAGES;
          pp ^= 1u;
        }
        got = mbar_wait_bounded(empty_bar(ps), pp, wait_ns, status, kStatusEpilogue, abort_flag);
      }
      if (!__all_sync(0xffffffffu, got)) return false;
      if (has_sf) {
        tc_fence_after();
        const uint32_t tsf = tmem + (static_cast<uint32_t>(q * 32) << 16) + G::kColSf + sfb * G::kSfCols;
        tmem_st_x16(tsf, fa);
#pragma unroll
        for (int h = 0; h < G::kSfAtomsB; ++h) {
          const uint4 v[4] = {fb[4 * h], fb[4 * h + 1], fb[4 * h + 2], fb[4 * h + 3]};
          tmem_st_x16(tsf + 16 + 16 * h, v);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_map(sf_full_bar(sfb), 0));
      ++slots_done;
      if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      if (++sfb == kSfBufs) sfb = 0;
      return true;
    };
    // per tile: its low-rank slots, its K steps, then (from the second tile on) the slot that
    // carries the previous tile's L1s' slice; after the last tile, that tile's slice slot
    bool ok = true, any = false;
    for (int unit = pair0; ok && unit < args.num_units; unit += npairs) {
      int m_pair, split, n_beg, n_end;
      unit_range(unit, args.splits, args.n_tiles, m_pair, split, n_beg, n_end);
      for (int n_blk = n_beg; ok && n_blk < n_end; ++n_blk) {
        for (int sl = 0; ok && sl < lr_slots + args.k_iters; ++sl) ok = slot(sl >= lr_slots);
        if (ok && any) ok = slot(false);
        any = true;
      }
    }
    if (ok && any) slot(false);
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..9)
    // Warp (q, h): TMEM lane quadrant q = warp % 4 (rows q*32 .. q*32+31 of this CTA's 128) and
    // half h of the tile's 128 SwiGLU outputs (columns 64h .. 64h+63, atom h of the h tile).
    const int q = warp & 3, h = (warp - 2) >> 2;
    const float alpha = *args.alpha;
    const float gx2 = *args.g_x2;
    const float d6 = __fmul_rn(6.0f, gx2);
    const float rd6 = __frcp_rn(d6);
    const float* rs_tab = reinterpret_cast<const float*>(smem + L::kTabOff);
    const bool has_bias = args.bias != nullptr;
    const int hN = args.N >> 1;
    const int rl = q * 32 + lane;                   // this thread's row of the CTA's 128
    uint8_t* atom = smem + L::kHOff + h * 16384;    // this warp's 64 columns of the h tile
    int tseq = 0, useq = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    // U' of the unit just finished: TMEM -> partials[split][row][0..R2); then release the columns
    auto drain_u = [&](int m_pair, int split) -> bool {
      const bool got = mbar_wait_bounded(u_done_bar, static_cast<uint32_t>(useq - 1) & 1u, wait_ns, status,
                                         kStatusEpilogue, abort_flag);
      if (!__all_sync(0xffffffffu, got)) return false;
      tc_fence_after();
      const uint32_t tu = tmem + (static_cast<uint32_t>(q * 32) << 16) + L::kColU;
      float u[R2];
      if constexpr (R2 == 16) {
        tmem_ld_32x16(tu, u);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < R2; j += 32) {
          float t32[32];
          tmem_ld_32x32(tu + j, t32);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) u[j + e] = t32[e];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_map(u_free_bar, 0));
      const int row = (2 * m_pair + static_cast<int>(rank)) * 128 + rl;
      if (row < args.M_pad) {
        float4* dst = reinterpret_cast<float4*>(args.partials + (static_cast<size_t>(split) * args.M_pad + row) * R2);
#pragma unroll
        for (int j = 0; j < R2; j += 4) dst[j >> 2] = make_float4(u[j], u[j + 1], u[j + 2], u[j + 3]);
      }
      return true;
    };
    int prev_m_pair = 0, prev_split = 0;
    for (int unit = pair0; ok && unit < args.num_units; unit += npairs) {
      int m_pair, split, n_beg, n_end;
      unit_range(unit, args.splits, args.n_tiles, m_pair, split, n_beg, n_end);
      const int m_blk = 2 * m_pair + static_cast<int>(rank);
      const int row = m_blk * 128 + rl;
      for (int n_blk = n_beg; ok && n_blk < n_end; ++n_blk, ++tseq) {
        const bool got = mbar_wait_bounded(accf_bar, acc_phase, wait_ns, status, kStatusEpilogue, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tc_fence_after();
        // the previous unit's U' completed with this tile's accumulator: drain it first
        if (n_blk == n_beg && useq > 0 && h == 0 && !(ok = drain_u(prev_m_pair, prev_split))) break;
        // the h tile is free once the previous tile's U' MMAs (committed before this tile's
        // accumulator) have read it; and any store of it has finished reading
        if (tseq > 0) {
          const bool free_h = mbar_wait_bounded(h_empty_bar, static_cast<uint32_t>(tseq - 1) & 1u, wait_ns, status,
                                                kStatusEpilogue, abort_flag);
          if (!__all_sync(0xffffffffu, free_h)) { ok = false; break; }
        }
        if (args.store_h) {
          if (lane == 0) bulk_wait_group_read<0>();
          __syncwarp();
        }
        const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16);
        // pass 1: 16-column halves of this warp's 64 outputs: gate/up loads of the next half in
        // flight while one is activated; bf16 h into the h tile; accumulator released after the
        // last load (the same arithmetic as the NVFP4 GEMM's SwiGLU epilogue)
        {
          float g[2][16], u[2][16];
          auto load_half = [&](int hc, float (&gg)[16], float (&uu)[16]) {
            const int col = h * 64 + 16 * hc;
            tmem_ld_32x16(tb + col, gg);
            tmem_ld_32x16(tb + kHalf + col, uu);
          };
          load_half(0, g[0], u[0]);
          tmem_wait_ld();
#pragma unroll
          for (int hc = 0; hc < 4; ++hc) {
            if (hc + 1 < 4) load_half(hc + 1, g[(hc + 1) & 1], u[(hc + 1) & 1]);
            else {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive_cluster(cluster_map(acce_bar, 0));
            }
            const int j0 = n_blk * kHalf + h * 64 + 16 * hc;  // output (and gate bias) column
            float (&gg)[16] = g[hc & 1];
            float (&uu)[16] = u[hc & 1];
#pragma unroll
            for (int i = 0; i < 16; i += 8) {
              float bg[8], bu[8];
              if (has_bias) {
                bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(args.bias + j0 + i)), bg);
                bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(args.bias + hN + j0 + i)), bu);
              } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) bg[e] = bu[e] = 0.0f;
              }
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 8; e += 2) {
                const float z0 = fmaf(alpha, gg[i + e], bg[e]), z1 = fmaf(alpha, gg[i + e + 1], bg[e + 1]);
                const float y0 = silu_times(z0, fmaf(alpha, uu[i + e], bu[e]));
                const float y1 = silu_times(z1, fmaf(alpha, uu[i + e + 1], bu[e + 1]));
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(y0, y1);
                w[e / 2] = *reinterpret_cast<const uint32_t*>(&b2);
              }
              *reinterpret_cast<uint4*>(atom + sw128(rl, 2 * hc + i / 8)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (hc + 1 < 4) tmem_wait_ld();
          }
        }
        acc_phase ^= 1u;
        // the h tile is an operand of the U' MMA (async proxy) and the source of the optional store
        fence_proxy_async_smem();
        __syncwarp();
        if (args.store_h && lane == 0) {
          tma_store_2d(&tmH, smem_addr(atom) + static_cast<uint32_t>(q * 32 * 128), n_blk * kHalf + h * 64,
                       m_blk * 128 + q * 32);
          bulk_commit_group();
        }
        // both CTAs' h tiles are the U' MMA's A operand: ready once all 16 warps have arrived (the
        // issuer waits for the slot that carries the tile's L1s' slice on its own)
        if (lane == 0) mbar_arrive_release_cluster(cluster_map(h_full_bar, 0));
        // pass 2: this row's four 16-column blocks of h, quantized for the next layer exactly as
        // kernel 1 would quantize them (rows past M get zero codes and scales, as kernel 1 writes)
        if (row < args.M_pad) {
#pragma unroll
          for (int hc = 0; hc < 4; ++hc) {
            const int k = n_blk * kHalf + h * 64 + 16 * hc;  // next-layer K column of the block
            const uint4 x0 = *reinterpret_cast<const uint4*>(atom + sw128(rl, 2 * hc));
            const uint4 x1 = *reinterpret_cast<const uint4*>(atom + sw128(rl, 2 * hc + 1));
            const uint32_t wx[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
            float v[16];
            float amax = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 l = __ldg(reinterpret_cast<const float4*>(args.inv_lambda2 + k) + j);
              const float2 p0 = mul2_rn(make_float2(__uint_as_float(wx[2 * j] << 16), __uint_as_float(wx[2 * j] & 0xFFFF0000u)),
                                        make_float2(l.x, l.y));
              const float2 p1 =
                  mul2_rn(make_float2(__uint_as_float(wx[2 * j + 1] << 16), __uint_as_float(wx[2 * j + 1] & 0xFFFF0000u)),
                          make_float2(l.z, l.w));
              v[4 * j] = p0.x;
              v[4 * j + 1] = p0.y;
              v[4 * j + 2] = p1.x;
              v[4 * j + 3] = p1.y;
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(v[e]));
            // kernel 1's scale rule: the reciprocal multiply, with the exact division only near an
            // E4M3 rounding boundary or below E4M3's normal range (the same code either way)
            float qs = __fmul_rn(amax, rd6);
            if (scale_needs_division(qs)) qs = __fdiv_rn(amax, d6);
            uint32_t sc = row < args.M ? cvt_e4m3(qs) : 0u;
            uint2 codes = make_uint2(0u, 0u);
            if (sc != 0) {
              const float rr = rs_tab[sc];
              const float2 r2 = make_float2(rr, rr);
              float qv[16];
#pragma unroll
              for (int e = 0; e < 16; e += 2) {
                const float2 p = mul2_rn(make_float2(v[e], v[e + 1]), r2);
                qv[e] = p.x;
                qv[e + 1] = p.y;
              }
              codes.x = cvt_e2m1x8(*reinterpret_cast<const float(*)[8]>(qv));
              codes.y = cvt_e2m1x8(*reinterpret_cast<const float(*)[8]>(qv + 8));
            }
            *reinterpret_cast<uint2*>(args.codes2 + static_cast<size_t>(row) * (args.K2 >> 1) + (k >> 1)) = codes;
            args.sf2[act_sf_offset(row, k >> 4, args.K2)] = static_cast<uint8_t>(sc);
          }
        }
        if (n_blk == n_end - 1) {
          ++useq;
          prev_m_pair = m_pair;
          prev_split = split;
        }
      }
    }
    if (ok && useq > 0 && h == 0) drain_u(prev_m_pair, prev_split);
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

// The most column splits a unit schedule uses (the partials buffer holds this many slices).
constexpr int kMaxUSplits = 8;

// U' = sum over splits of the partial sums (in split order), stored as kernel 1 stores U: u =
// fp32(U' * fp32(1 / alpha')) with alpha' = fp32(g_x' g_w'), as bf16 hi = bf16(u) and lo =
// bf16(u - hi); rows past M are zero. Also writes alpha'. A thread issues all its partial loads
// before the first sum, so their latencies overlap.
__global__ void finalize_u_kernel(const float* __restrict__ partials, int splits, int M, int M_pad, int r,
                                  const float* g_x2, const float* g_w2, __nv_bfloat16* __restrict__ U,
                                  float* alpha_out) {
  grid_dependency_wait();  // the partial sums of the kernel before it on the stream
  grid_launch_dependents();
  const float alpha = __fmul_rn(*g_x2, *g_w2);
  const float cinv = __frcp_rn(alpha);
  const size_t total = static_cast<size_t>(M_pad) * r;
  if (blockIdx.x == 0 && threadIdx.x == 0) *alpha_out = alpha;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(i / r);
    float pv[kMaxUSplits];
#pragma unroll
    for (int sp = 0; sp < kMaxUSplits; ++sp)
      pv[sp] = (m < M && sp < splits) ? partials[static_cast<size_t>(sp) * total + i] : 0.0f;
    float s = 0.0f;
#pragma unroll
    for (int sp = 0; sp < kMaxUSplits; ++sp)
      if (sp < splits) s += pv[sp];
    const float v = __fmul_rn(s, cinv);
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    U[i] = hi;
    U[total + i] = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(hi)));
  }
}

}  // namespace fused
}  // namespace svdq
