// Kernel 2: block-scaled NVFP4 GEMM on the 5th-generation tensor cores (tcgen05), with the
// low-rank up-projection and the bias / SwiGLU epilogue fused in.
//
// Method ("Bringing Nunchaku 4-bit diffusion inference to Diffusers", "SVDQuant deep dive"): the
// branch's up-projection (X L1) L2 is fused with the 4-bit GEMM; here it is one extra bf16 MMA
// (K = r) into the same TMEM accumulator, with U pre-divided by alpha = g_x g_w so that a single
// scale applies at the end. The fused QKV / SwiGLU epilogues follow the fused NVFP4 GEMMs of
// "FLUX 3 Image Klein on NVIDIA Blackwell", method 1.
//
// Structure: persistent clusters of two CTAs (one per SM) that share each 256 x n_tile output tile
// through the CTA-pair form of the tensor-core MMA (cta_group::2): the even CTA issues every MMA of
// the pair; rows 0..127 of A, of the accumulator and of the output belong to the even CTA, rows
// 128..255 to the odd one, and each CTA stages half of B's n_tile rows. Per CTA (14 warps):
//   warp 0       TMA producer: per 256-wide K step, its 128 A rows and n_tile/2 B rows (128B-
//                swizzled 2-D tiles) plus the scale-factor atoms (its own 128 A rows; all n_tile B
//                rows) as 1-D bulk copies, into a STAGES-deep ring on this CTA's own barriers.
//                Before a tile's K loop, ring slots carry U_hi, U_lo (its 128 rows) and its half
//                of L2^T in chunks of 32 columns of r.
//   warp 1       TMEM allocation for the pair; in the even CTA also the MMA issuer: per ring slot
//                it waits for the slot's barrier in the even CTA (8 arrivals: the scale writers of
//                both CTAs), issues 4 x tcgen05.mma kind::mxf4nvf4 (M=256, N=n_tile, K=64; at
//                n_tile 384 each as N=256 + N=128) or the low-rank kind::f16 MMAs, and multicasts
//                one commit to the slot's empty barrier in both CTAs.
//   warps 2..9   epilogue: two warps per 32-lane TMEM quadrant, each half of the tile's columns:
//                tcgen05.ld, y = alpha acc (+ bias), SwiGLU on interleaved gate/up columns, into a
//                swizzled staging buffer, TMA store. The accumulator goes back to the issuer (a
//                remote arrive) as soon as its last columns are in registers.
//   warps 10..13 scale-factor writers: per ring slot, wait for this CTA's data, copy the scale
//                atoms from shared memory into one of the TMEM scale buffers with tcgen05.st (each
//                warp its lane quadrant), then arrive on the issuer's barrier in the even CTA.
//                Measured on B200, every tcgen05.cp costs ~64 tensor-pipe cycles whatever its
//                shape, so copying 12 atoms per K step with tcgen05.cp starved the MMAs; stores
//                from four warps run beside the MMAs without slowing them.
// TMEM (512 columns): the accumulator (n_tile columns; two buffers when n_tile = 128) and 4 scale
// buffers of 16 + 16 * ceil(n_tile / 128) columns (2 beside the 384-column accumulator). Measured
// on B200: with only 2 scale buffers the commit -> writer -> remote arrive -> issuer round trip
// (~900 cycles across the pair) could not hide under a 256-wide K step; and one CTA per 128 x 192
// tile had to stream 48 KB per 384-cycle K step from L2 per SM, above what a B200 SM sustained in
// isolation (~75-90 B per cycle), against 38 KB per 512 cycles here.
// The 384-wide tile (4-stage ring) issues each K chunk as two MMAs, N = 256 and N = 128, on the
// same A: 48 KB per CTA per 768-cycle K step, 16 % fewer operand bytes per flop than at 256, for a
// kernel whose time follows the bytes it streams from L2.
// Every mbarrier wait is bounded (global timer); a wait that runs out records a status bit, sets
// a shared abort flag so that the other roles of the CTA stop too, and the kernel drains its own
// copies and MMAs before the cluster-wide barrier that precedes freeing TMEM.
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
  int m_tiles, m_pairs, n_tiles, k_iters, num_tiles;  // num_tiles = m_pairs * n_tiles pair tiles
  int ldy, out_f32, epi;                              // epi bit 0: bias, bit 1: SwiGLU
};

// Shared memory and TMEM layout of the pair GEMM. SCALES: the block-scaled NVFP4 format, whose
// ring slots also carry the K step's scale atoms and whose scale factors sit in TMEM buffers.
template <bool SCALES, int N_TILE, int STAGES>
struct PairGemmLayout {
  static constexpr int kBRows = N_TILE / 2;  // rows of B staged by each CTA of the pair
  static constexpr int kA = 128 * 128;       // 128 rows x 128 bytes of codes (one K step)
  static constexpr int kB = kBRows * 128;
  static constexpr int kSfAtomsB = (N_TILE + 127) / 128;
  static constexpr int kSfa = SCALES ? 4 * 512 : 0;
  static constexpr int kSfb = SCALES ? 4 * kSfAtomsB * 512 : 0;
  static constexpr int kStage = kA + kB + kSfa + kSfb;
  static constexpr int kOffB = kA;
  static constexpr int kOffSfa = kA + kB;
  static constexpr int kOffSfb = kA + kB + kSfa;
  // a low-rank slot holds U_hi (offset 0), U_lo (kOffULo), this CTA's half of L2^T (kOffB) and, for
  // a format whose L2^T is kept as a bf16 hi/lo pair, its lo half (kOffL2Lo)
  static constexpr int kOffL2Lo = kOffB + kBRows * 32 * 2;
  // TMEM scale-factor buffer (one K step): SFA 4 MMAs x 4 columns, then SFB 4 MMAs x 4 x atoms.
  // Four buffers beside an accumulator of up to 256 columns; two beside the 384-column one.
  static constexpr int kSfCols = SCALES ? 16 + 16 * kSfAtomsB : 0;
  static constexpr int kSfBufs = SCALES ? (N_TILE > 256 ? 2 : 4) : 0;
  static constexpr int kAccBufs = (2 * N_TILE + kSfBufs * kSfCols <= 512) ? 2 : 1;
  static constexpr int kColSf = kAccBufs * N_TILE;  // kSfBufs buffers of kSfCols columns from here
  // epilogue staging: 8 warps x 4 KB (two 32 x 32 bf16 boxes or one fp32 box in flight)
  static constexpr int kStageOutWarp = 4096;
  static constexpr int kOutOff = STAGES * kStage;
  static constexpr int kBarOff = kOutOff + 8 * kStageOutWarp;
  // full[STAGES], empty[STAGES], sf_land[STAGES], accf[kAccBufs], acce[kAccBufs], drain, sf_full[kSfBufs]
  static constexpr int kNumBars = 3 * STAGES + 2 * kAccBufs + 1 + kSfBufs;
  static constexpr int kSmem = kBarOff + kNumBars * 8 + 16 + 1024;
  static_assert(kStage % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(kOffL2Lo % 512 == 0, "64B-swizzled boxes start on 512-byte boundaries");
  static_assert(kOffL2Lo + kBRows * 32 * 2 <= kStage, "a low-rank slot fits a ring stage");
  static_assert(kColSf + kSfBufs * kSfCols <= 512, "TMEM budget");
  static_assert(kSfBufs <= STAGES, "a scale buffer's previous slot must still own its ring stage");
  static_assert(kSmem <= 232448, "shared memory budget");
  static_assert(N_TILE <= 256 || (SCALES && N_TILE == 384), "the 384-wide tile is an NVFP4 tile");
};
template <int N_TILE, int STAGES>
using GemmLayout = PairGemmLayout<true, N_TILE, STAGES>;

// Low-rank operands move in chunks of rc = min(r, 32) columns: U_hi, U_lo (128 x rc each) and this
// CTA's half of L2^T (n_tile/2 x rc), all bf16 with rc*2-byte rows (32B or 64B swizzle), one ring
// slot per chunk.
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
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t num_clusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}

// The block-scaled NVFP4 format of the pair GEMM (a policy of pair_gemm_kernel): E2M1 x E2M1 with
// one UE4M3 scale per 16 K-elements of A and B, the scales written into TMEM by the writer warps;
// the low-rank branch as U_hi L2 + U_lo L2 (two bf16 MMAs per 16 columns of r); the epilogue scale
// y = alpha acc (+ bias) with one alpha = g_x g_w for the whole tile.
struct Nvfp4Gemm {
  using Args = GemmArgs;
  static constexpr bool kScales = true;
  static constexpr bool kL2HiLo = false;
  // the MMAs of a 256-element K step: four of K = 64 (32 bytes of codes per row); the SFA of MMA j
  // at tsf + 4j, its SFB atoms (128 tile columns each) from tsf + 16 + 4 SF_ATOMS_B j on
  template <int N_TILE, int SF_ATOMS_B>
  __device__ static void kstep(uint32_t d, uint32_t la, uint32_t lb, uint32_t hi_ab, uint32_t tsf,
                               uint32_t accumulate) {
    if constexpr (N_TILE <= 256) {
      constexpr uint32_t id = idesc_nvfp4(256, N_TILE);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        mma_nvfp4_pair_warp(d, desc_join(la + 2u * j, hi_ab), desc_join(lb + 2u * j, hi_ab), id, tsf + 4 * j,
                            tsf + 16 + 4 * SF_ATOMS_B * j, j == 0 ? accumulate : 1u);
    } else {
      // 384 columns as N = 256 (accumulator columns 0..255; the first 128 rows of each CTA's B box,
      // SFB atoms 3j and 3j + 1) and N = 128 (columns 256..383; the box's last 64 rows, 16 KB on,
      // SFB atom 3j + 2), both on the same A
      constexpr uint32_t id_a = idesc_nvfp4(256, 256), id_b = idesc_nvfp4(256, N_TILE - 256);
      constexpr uint32_t kB2 = (128 * 128) >> 4;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint64_t a = desc_join(la + 2u * j, hi_ab);
        const uint32_t acc = j == 0 ? accumulate : 1u;
        mma_nvfp4_pair_warp(d, a, desc_join(lb + 2u * j, hi_ab), id_a, tsf + 4 * j, tsf + 16 + 4 * SF_ATOMS_B * j,
                            acc);
        mma_nvfp4_pair_warp(d + 256, a, desc_join(lb + kB2 + 2u * j, hi_ab), id_b, tsf + 4 * j,
                            tsf + 16 + 4 * SF_ATOMS_B * j + 8, acc);
      }
    }
  }
  // per tile row: y = alpha acc (+ bias) for 8 accumulator columns g0.. (GEMM order) of v[off..]
  struct Epi {
    float alpha;
    __device__ Epi(const Args& a, int srow) : alpha(*a.alpha) { (void)srow; }
    template <bool BIAS, class V>
    __device__ void apply8(const Args&, V& v, int off, int g0, const __nv_bfloat16* bias8) const {
      (void)g0;
      if constexpr (BIAS) {
        float b[8];
        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(bias8)), b);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[off + j] = fmaf(alpha, v[off + j], b[j]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[off + j] = alpha * v[off + j];
      }
    }
  };
};

constexpr int kGemmThreads = 448;

// Tile order: groups of kGroupPairs row pairs (256 rows each); inside a group the row pairs vary
// fastest, then the n_tile column blocks. The ~74 pairs in flight then share a few A slabs (a
// group's A rows, 8 x 256 x K/2 bytes) and sweep B, so A is fetched from DRAM about once even when
// the output stream evicts older lines from L2.
constexpr int kGroupPairs = 8;
__device__ __forceinline__ void tile_coords(int tile, int m_pairs, int n_tiles, int& m_pair, int& n_blk) {
  const int group_tiles = kGroupPairs * n_tiles;
  const int g = tile / group_tiles;
  const int first = g * kGroupPairs;
  const int gm = m_pairs - first < kGroupPairs ? m_pairs - first : kGroupPairs;
  const int local = tile - g * group_tiles;
  m_pair = first + local % gm;
  n_blk = local / gm;
}

// The pair GEMM body, one template for the formats: F supplies the MMA kind, whether scale factors
// travel with the ring, the low-rank operand layout and the epilogue's column scales.
template <class F, int N_TILE, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    pair_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmL2,
                     const __grid_constant__ CUtensorMap tmY, const typename F::Args args) {
  using L = PairGemmLayout<F::kScales, N_TILE, STAGES>;
  constexpr int kSfBufs = L::kSfBufs, kAccBufs = L::kAccBufs;
  extern __shared__ uint8_t smem_raw[];
  // the same offsets in both CTAs: the pair MMA addresses the odd CTA's operands by this CTA's
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  // full: in the even CTA, the A / B (or low-rank) bytes of both CTAs of a ring slot (the pair
  // loads complete there); sf_land: this CTA's scale-factor bytes of a slot
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto sf_land_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
  auto accf_bar = [&](int b) { return bar0 + 8u * (3 * STAGES + b); };
  auto acce_bar = [&](int b) { return bar0 + 8u * (3 * STAGES + kAccBufs + b); };
  const uint32_t drain_bar = bar0 + 8u * (3 * STAGES + 2 * kAccBufs);
  auto sf_full_bar = [&](int b) { return bar0 + 8u * (3 * STAGES + 2 * kAccBufs + 1 + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBarOff + L::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = args.r;
  const uint32_t rank = cluster_ctarank();  // 0: issues the pair's MMAs
  const int pair0 = static_cast<int>(cluster_id_x()), npairs = static_cast<int>(num_clusters_x());

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);   // the even CTA's producer arrives (with both CTAs' byte count)
      mbar_init(empty_bar(s), 1);
      mbar_init(sf_land_bar(s), 1);
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), 16);  // 8 epilogue warps in each CTA
    }
    mbar_init(drain_bar, 1);
    for (int b = 0; b < kSfBufs; ++b) mbar_init(sf_full_bar(b), 8);  // 4 writer warps in each CTA
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
  // The set-up above touches no global memory, so it overlaps the end of the previous kernel on the
  // stream (programmatic launch); everything below may read what that kernel wrote.
  grid_dependency_wait();
  grid_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  unsigned* status = &g_svdq_status;
  const uint64_t wait_ns = args.wait_ns;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // Per ring slot: this CTA's scale atoms (1-D bulk copies onto its own sf_land barrier, first,
      // so that the writers can store them while A and B are still in flight), then its 128 A rows
      // and n_tile/2 B rows as CTA-pair TMA loads that complete on the even CTA's full barrier; the
      // even CTA's producer expects the bytes of both CTAs there.
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      const int rc = r < kLrChunk ? r : kLrChunk;
      const uint32_t lr_bytes = static_cast<uint32_t>((2 * 128 + (F::kL2HiLo ? 2 : 1) * L::kBRows) * rc * 2);
      const int sf_row_stride = args.K >> 6;  // 64-wide K atoms per 128-row block
      const bool leader = rank == 0;
      bool ok = true;
      for (int tile = pair0; ok && tile < args.num_tiles; tile += npairs) {
        int m_pair, n_blk;
        tile_coords(tile, args.m_pairs, args.n_tiles, m_pair, n_blk);
        const int m_blk = 2 * m_pair + static_cast<int>(rank);
        const int b_row = n_blk * N_TILE + static_cast<int>(rank) * L::kBRows;
        for (int c0 = 0; c0 < r; c0 += kLrChunk) {
          if (!(ok = mbar_wait_bounded(empty_bar(stage), phase ^ 1u, wait_ns, status, kStatusProducer, abort_flag)))
            break;
          const uint32_t sa = sbase + stage * L::kStage;
          if constexpr (F::kScales) mbar_arrive(sf_land_bar(stage));  // no scales in a low-rank slot
          const uint32_t fb = cluster_map(full_bar(stage), 0);
          if (leader) mbar_arrive_expect_tx(full_bar(stage), 2 * lr_bytes);
          tma_load_2d_pair(sa, &tmU, c0, m_blk * 128, fb);
          tma_load_2d_pair(sa + kOffULo, &tmU, c0, args.M_pad + m_blk * 128, fb);
          tma_load_2d_pair(sa + L::kOffB, &tmL2, c0, b_row, fb);
          if constexpr (F::kL2HiLo) tma_load_2d_pair(sa + L::kOffL2Lo, &tmL2, c0, args.N + b_row, fb);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        // an odd CTA past the last 128-row block loads zero-filled codes (rows past the tensor) and
        // the last block's scales; none of its rows are stored
        const int m_sf = m_blk < args.m_tiles ? m_blk : args.m_tiles - 1;
        for (int kt = 0; kt < args.k_iters; ++kt) {
          if (!(ok = mbar_wait_bounded(empty_bar(stage), phase ^ 1u, wait_ns, status, kStatusProducer, abort_flag)))
            break;
          const uint32_t sa = sbase + stage * L::kStage;
          if constexpr (F::kScales) {
            const uint8_t* sfa_tile = args.sfa + (static_cast<size_t>(m_sf) * sf_row_stride << 9);
            const uint8_t* sfb_tile = args.sfb + (static_cast<size_t>(n_blk) * sf_row_stride * L::kSfAtomsB << 9);
            mbar_arrive_expect_tx(sf_land_bar(stage), L::kSfa + L::kSfb);
            bulk_load(sa + L::kOffSfa, sfa_tile + (static_cast<size_t>(kt) * 4 << 9), L::kSfa, sf_land_bar(stage));
            bulk_load(sa + L::kOffSfb, sfb_tile + (static_cast<size_t>(kt) * 4 * L::kSfAtomsB << 9), L::kSfb,
                      sf_land_bar(stage));
          } else {
            (void)m_sf;
            (void)sf_row_stride;
          }
          const uint32_t fb = cluster_map(full_bar(stage), 0);
          if (leader) mbar_arrive_expect_tx(full_bar(stage), 2 * (L::kA + L::kB));
          tma_load_2d_pair(sa, &tmA, kt * 128, m_blk * 128, fb);
          tma_load_2d_pair(sa + L::kOffB, &tmB, kt * 128, b_row, fb);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Drain: every copy this thread started has landed before the CTA may exit. A slot's release
      // (its MMAs have read it, so all its copies landed) shows it; after an abort the bounded
      // wait's limit, far longer than any copy takes, does.
      for (int s = 0; s < STAGES; ++s)
        if (armed & (1u << s))
          mbar_wait_bounded(empty_bar(s), (armed_parity >> s) & 1u, wait_ns, status, kStatusDrain, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (even CTA)
    // Per ring slot: wait for the slot's bytes of both CTAs (full) and, with scale factors, for its
    // scale buffer (the writers of both CTAs arrive there once the slot's scales are in TMEM); the
    // MMAs; one commit multicast to the slot's empty barrier in both CTAs (the writers also take it
    // as the release of the scale buffer that slot used). The waits sit before the slot's first
    // MMA: placed between queued MMAs, a barrier wait measurably stalled the tensor pipe on B200.
    // The whole warp runs this loop (warp-uniform operands); elect.sync inside the MMA and commit
    // helpers picks the issuing lane, and a wait succeeds only when it succeeds in every lane.
    if (rank == 0) {
      auto wait_slot = [&](int stage_, uint32_t phase_, int sfb_, uint32_t sf_phase_) -> bool {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(full_bar(stage_), phase_, wait_ns, status, kStatusMma,
                                                       abort_flag)))
          return false;
        if constexpr (!F::kScales) return true;
        return __all_sync(0xffffffffu, mbar_wait_bounded_cluster(sf_full_bar(sfb_), sf_phase_, wait_ns, status,
                                                                 kStatusMma, abort_flag)) != 0;
      };
      const int num_tiles = args.num_tiles, k_iters = args.k_iters;
      const int rc = r < kLrChunk ? r : kLrChunk;
      const int nj = rc >> 4;
      // the low-rank MMAs span the tile like the K steps: one of N = n_tile, or 256 + 128 columns
      constexpr int kLrN = N_TILE <= 256 ? N_TILE : 256;
      const uint32_t idesc_lr = idesc_bf16(256, kLrN);
      const uint32_t idesc_lr2 = idesc_bf16(256, N_TILE > 256 ? N_TILE - 256 : 16);
      // descriptor halves: low = start address / 16 | LBO (16 B) / 16 << 16; high = SBO / 16 |
      // version 1 | swizzle mode << 29
      const uint32_t lo0 = (sbase >> 4) | (1u << 16);
      const uint32_t hi_ab = (1024u >> 4) | (1u << 14) | (2u << 29);
      const uint32_t hi_lr = ((8u * rc * 2u) >> 4) | (1u << 14) | (lr_swizzle_mode(rc) << 29);
      const uint32_t tsf0 = tmem + L::kColSf;
      constexpr uint16_t kBoth = 3;
      int stage = 0, sfb = 0, acc = 0;
      uint32_t phase = 0, sf_phase = 0, acc_phase = 0;
      bool ok = true;
      auto next_slot = [&]() {
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        if constexpr (F::kScales) {
          if (++sfb == kSfBufs) { sfb = 0; sf_phase ^= 1u; }
        }
      };
      for (int tile = pair0; ok && tile < num_tiles; tile += npairs) {
        if (!(ok = __all_sync(0xffffffffu, mbar_wait_bounded_cluster(acce_bar(acc), acc_phase ^ 1u, wait_ns, status,
                                                                     kStatusMma, abort_flag)) != 0))
          break;
        const uint32_t d = tmem + static_cast<uint32_t>(acc * N_TILE);
        uint32_t accumulate = 0;
        for (int c0 = 0; c0 < r; c0 += kLrChunk) {
          if (!(ok = wait_slot(stage, phase, sfb, sf_phase))) break;
          tc_fence_after();
          const uint32_t lo = lo0 + stage * (L::kStage >> 4);
          for (int j = 0; j < nj; ++j) {
            const uint64_t u_hi = desc_join(lo + 2u * j, hi_lr);
            const uint64_t u_lo = desc_join(lo + (kOffULo >> 4) + 2u * j, hi_lr);
            const uint64_t l_hi = desc_join(lo + (L::kOffB >> 4) + 2u * j, hi_lr);
            mma_bf16_pair_warp(d, u_hi, l_hi, idesc_lr, accumulate);
            if constexpr (N_TILE > 256) {
              // columns 256..383: the last 64 rows of each CTA's L2^T box
              const uint64_t l_hi2 = desc_join(lo + ((L::kOffB + 128 * rc * 2) >> 4) + 2u * j, hi_lr);
              mma_bf16_pair_warp(d + 256, u_hi, l_hi2, idesc_lr2, accumulate);
              mma_bf16_pair_warp(d + 256, u_lo, l_hi2, idesc_lr2, 1u);
            }
            mma_bf16_pair_warp(d, u_lo, l_hi, idesc_lr, 1u);
            if constexpr (F::kL2HiLo)
              mma_bf16_pair_warp(d, u_hi, desc_join(lo + (L::kOffL2Lo >> 4) + 2u * j, hi_lr), idesc_lr, 1u);
            accumulate = 1;
          }
          tc_commit_pair_mc_warp(empty_bar(stage), kBoth);
          next_slot();
        }
        if (!ok) break;
        for (int kt = 0; kt < k_iters; ++kt) {
          if (!(ok = wait_slot(stage, phase, sfb, sf_phase))) break;
          tc_fence_after();
          const uint32_t la = lo0 + stage * (L::kStage >> 4);
          const uint32_t lb = la + (L::kOffB >> 4);
          F::template kstep<N_TILE, L::kSfAtomsB>(d, la, lb, hi_ab, tsf0 + sfb * L::kSfCols, accumulate);
          accumulate = 1;
          tc_commit_pair_mc_warp(empty_bar(stage), kBoth);
          next_slot();
        }
        if (!ok) break;
        tc_commit_pair_mc_warp(accf_bar(acc), kBoth);
        if (++acc == kAccBufs) { acc = 0; acc_phase ^= 1u; }
      }
      // Drain: all issued MMAs complete before TMEM may be freed.
      tc_commit_pair_mc_warp(drain_bar, 1);
      __all_sync(0xffffffffu, mbar_wait_bounded(drain_bar, 0, wait_ns, status, kStatusDrain, nullptr));
    }
  } else if (warp >= 10) {
    // ------------------------------------------------------------------ scale-factor writers (warps 10..13)
    // Each warp owns one TMEM lane quadrant and writes into it the replicated scale-factor layout
    // the block-scaled MMA reads: for a 128-row atom, lane l, column c holds the 4 E4M3 scales of
    // row l + 32 c -- exactly bytes [16 l, 16 l + 16) of the 512-byte atom in shared memory. Every
    // ring slot (low-rank chunks too, which carry no scales) is reported to the issuer's barrier.
    // The writers wait only for this CTA's scale bytes (sf_land), not for A and B, so their work
    // overlaps the rest of the slot's copies; the issuer waits for A and B itself. A format without
    // scale factors leaves these warps idle.
    if constexpr (F::kScales) {
      const int q = warp & 3;
      int stage = 0, sfb = 0, slots_done = 0;
      uint32_t phase = 0;
      const int lr_slots = (r + kLrChunk - 1) / kLrChunk;
      bool ok = true;
      for (int tile = pair0; ok && tile < args.num_tiles; tile += npairs) {
        for (int slot = 0; slot < lr_slots + args.k_iters; ++slot) {
          const bool got_data =
              mbar_wait_bounded(sf_land_bar(stage), phase, wait_ns, status, kStatusEpilogue, abort_flag);
          if (!__all_sync(0xffffffffu, got_data)) { ok = false; break; }
          const bool has_sf = slot >= lr_slots;
          // read the stage's scale atoms now; only the TMEM stores wait for the buffer
          uint4 fa[4], fb[4 * L::kSfAtomsB];
          if (has_sf) {
            const uint8_t* sfs = smem + stage * L::kStage + L::kOffSfa + lane * 16;
#pragma unroll
            for (int i = 0; i < 4; ++i) fa[i] = *reinterpret_cast<const uint4*>(sfs + 512 * i);
#pragma unroll
            for (int i = 0; i < 4 * L::kSfAtomsB; ++i)
              fb[i] = *reinterpret_cast<const uint4*>(smem + stage * L::kStage + L::kOffSfb + lane * 16 + 512 * i);
          }
          // Every slot, with scales or not, first waits for the release of the slot kSfBufs back
          // (the previous one on barrier sfb, whose MMAs read this scale buffer): then no CTA can
          // arrive for this slot while that slot's phase still waits for the other CTA's writers.
          // That slot is at most STAGES back, so its ring stage has not been released a second time.
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
          if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
          if (has_sf) {
            tc_fence_after();
            const uint32_t tsf = tmem + (static_cast<uint32_t>(q * 32) << 16) + L::kColSf + sfb * L::kSfCols;
            tmem_st_x16(tsf, fa);
#pragma unroll
            for (int h = 0; h < L::kSfAtomsB; ++h) {
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
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..9)
    // Warp (q, h): TMEM lane quadrant q = warp % 4, half h of the tile's 32-column output chunks.
    // A round loads up to 64 accumulator columns (tcgen05.ld), converts them (column scales, bias,
    // SwiGLU; bf16 results stay packed in registers) and, after the last round's loads, hands the
    // accumulator back before any store: the issuer's next tile then waits only for the loads.
    // Each 32 x 32 output block goes through a swizzled staging box (64B swizzle for bf16 rows,
    // 128B for fp32: conflict-free 16-byte writes) and a TMA tensor store that clips rows >= M.
    const int q = warp & 3, h = (warp - 2) >> 2;
    const bool has_bias = (args.epi & 1) != 0;
    const bool swiglu = (args.epi & 2) != 0;
    const bool f32 = args.out_f32 != 0;
    const int hN = args.N >> 1;
    uint8_t* stage_out = smem + L::kOutOff + (warp - 2) * L::kStageOutWarp;
    // 32-column output chunks of a tile, split between the two warps of a quadrant
    constexpr int kPlainPerWarp = N_TILE / 64;  // chunks per warp without SwiGLU
    constexpr int kGluChunks = N_TILE / 64;     // output chunks per tile with SwiGLU
    const int glu_beg = h * ((kGluChunks + 1) >> 1);
    const int glu_end = h ? kGluChunks : ((kGluChunks + 1) >> 1);
    int acc = 0;
    uint32_t acc_phase = 0;
    // a staging box is reused once the store issued from it has finished reading it
    auto store_box = [&](uint8_t* dst, int row0, int col0) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&tmY, smem_addr(dst), col0, row0);
        bulk_commit_group();
      }
    };
    auto pack_bf16 = [&](const float (&v)[32], uint32_t (&pk)[16]) {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
      }
    };
    // staging: two 2 KB bf16 boxes or one 4 KB fp32 box per warp; a box is rewritten once the
    // store issued from it has finished reading it
    auto write_box_bf16 = [&](const uint32_t (&pk)[16], int b) {
      uint8_t* dst = stage_out + b * 2048;
      // 64-byte rows, 4 chunks; chunk j of row `lane` lives at j ^ ((lane / 2) % 4)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(dst + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
    };
    auto boxes_free = [&]() {
      if (lane == 0) bulk_wait_group_read<0>();
      __syncwarp();
    };
    auto emit_f32 = [&](const float (&v)[32], int row0, int col0) {
      uint8_t* dst = stage_out;
      if (lane == 0) bulk_wait_group_read<0>();
      __syncwarp();
      // 128-byte rows, 8 chunks of 16 bytes; chunk j of row `lane` lives at j ^ (lane % 8)
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float4*>(dst + lane * 128 + ((j ^ (lane & 7)) << 4)) =
            make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      store_box(dst, row0, col0);
    };
    // y = scale(g) * acc (+ bias[n]) for 8 values of accumulator (GEMM) columns g0.. and output
    // (bias) columns n0..
    // (v is a register array; `off` is a compile-time constant after unrolling, so it stays one)
    auto affine8 = [&](const typename F::Epi& ep, auto& v, int off, int g0, int n0) {
      if (has_bias) ep.template apply8<true>(args, v, off, g0, args.bias + n0);
      else ep.template apply8<false>(args, v, off, g0, nullptr);
    };
    auto affine = [&](const typename F::Epi& ep, float (&v)[32], int g0, int n0) {
      if (has_bias) {
#pragma unroll
        for (int i = 0; i < 32; i += 8) ep.template apply8<true>(args, v, i, g0 + i, args.bias + n0 + i);
      } else {
#pragma unroll
        for (int i = 0; i < 32; i += 8) ep.template apply8<false>(args, v, i, g0 + i, nullptr);
      }
    };
    auto release_acc = [&]() {
      // all of this warp's accumulator columns are in registers: hand the buffer back to the issuer
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_map(acce_bar(acc), 0));
    };
    for (int tile = pair0; tile < args.num_tiles; tile += npairs) {
      int m_pair, n_blk;
      tile_coords(tile, args.m_pairs, args.n_tiles, m_pair, n_blk);
      const int m_blk = 2 * m_pair + static_cast<int>(rank);
      // warp-uniform outcome: tcgen05.ld below is a .sync.aligned warp instruction
      const bool got = mbar_wait_bounded(accf_bar(acc), acc_phase, wait_ns, status, kStatusEpilogue, abort_flag);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int row0 = m_blk * 128 + q * 32;
      // rows past M_pad (an odd CTA past the last block) are never stored; a row scale is read
      // from a valid row
      const typename F::Epi ep(args, row0 + lane < args.M_pad ? row0 + lane : args.M_pad - 1);
      const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * N_TILE);
      if (!swiglu && !f32) {
        // bf16 out, 64 columns per load round: chunks 0 and 1 are scaled, packed and written into
        // the two staging boxes, later chunks stay packed in registers; the accumulator is released
        // after the last round's loads and only then are the boxes stored (measured on B200:
        // staging and storing each chunk before the next load took ~700 cycles per chunk, all of it
        // on the issuer's path to the next tile). The 384-wide tile's six chunks per warp load their
        // last two rounds one chunk at a time, which keeps the packed chunks and the loaded ones
        // within the register budget.
        const int c_beg = h * kPlainPerWarp;
        uint32_t pk[kPlainPerWarp > 2 ? kPlainPerWarp - 2 : 1][16];
        boxes_free();
#pragma unroll
        for (int i = 0; i < kPlainPerWarp; i += (kPlainPerWarp > 4 && i >= 4) ? 1 : 2) {
          const bool pair = !(kPlainPerWarp > 4 && i >= 4) && i + 1 < kPlainPerWarp;
          float v[2][32];
          tmem_ld_32x32(tb + (c_beg + i) * 32, v[0]);
          if (pair) tmem_ld_32x32(tb + (c_beg + i + 1) * 32, v[1]);
          tmem_wait_ld();
          if (i + (pair ? 2 : 1) >= kPlainPerWarp) release_acc();
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int j = i + u;
            if (j < kPlainPerWarp && (u == 0 || pair)) {
              const int g0 = n_blk * N_TILE + (c_beg + j) * 32;
              affine(ep, v[u], g0, g0);
              if (j < 2) {
                uint32_t t[16];
                pack_bf16(v[u], t);
                write_box_bf16(t, j);
              } else {
                pack_bf16(v[u], pk[j - 2]);
              }
            }
          }
        }
#pragma unroll
        for (int j = 0; j < kPlainPerWarp; ++j) {
          if (j >= 2) {
            // box j % 2 is free once the store issued from it two chunks ago has read it
            if (lane == 0) bulk_wait_group_read<1>();
            __syncwarp();
            write_box_bf16(pk[j - 2], j & 1);
          }
          store_box(stage_out + (j & 1) * 2048, row0, n_blk * N_TILE + (c_beg + j) * 32);
        }
      } else if (!swiglu) {
        // fp32 out: chunk by chunk (the whole tile would not fit in registers)
        const int c_beg = h * kPlainPerWarp;
#pragma unroll 1
        for (int i = 0; i < kPlainPerWarp; ++i) {
          float v[32];
          tmem_ld_32x32(tb + (c_beg + i) * 32, v);
          tmem_wait_ld();
          if (i + 1 == kPlainPerWarp) release_acc();
          const int g0 = n_blk * N_TILE + (c_beg + i) * 32;
          affine(ep, v, g0, g0);
          emit_f32(v, row0, g0);
        }
      } else if constexpr (N_TILE <= 256) {
        // SwiGLU (tiles up to 256 wide; the host packs SwiGLU weights no wider): output chunk c
        // pairs gate columns c*32.. with up columns n_tile/2 + c*32.. (at most two chunks per warp,
        // one staging box each); gate GEMM column g, output (and gate bias) column j, up bias
        // column hN + j
        constexpr int kHalf = N_TILE / 2;
        const int n_mine = glu_end - glu_beg;
        if (!f32) {
          // bf16 out: 16-column halves of the chunks, the next half's gate/up loads in flight while
          // one is scaled and activated; the accumulator is released after the last load, then
          // the packed rows are staged and stored
          boxes_free();
          const int nh = 2 * n_mine;
          float g[2][16], u[2][16];
          auto load_half = [&](int hc, float (&gg)[16], float (&uu)[16]) {
            const int col = (glu_beg + (hc >> 1)) * 32 + 16 * (hc & 1);
            tmem_ld_32x16(tb + col, gg);
            tmem_ld_32x16(tb + kHalf + col, uu);
          };
          load_half(0, g[0], u[0]);
          tmem_wait_ld();
          constexpr int kMaxHalves = 2 * ((kGluChunks + 1) / 2);
#pragma unroll
          for (int hc = 0; hc < kMaxHalves; ++hc) {
            if (hc < nh) {
              if (hc + 1 < nh) load_half(hc + 1, g[(hc + 1) & 1], u[(hc + 1) & 1]);
              else release_acc();
              const int off = (glu_beg + (hc >> 1)) * 32 + 16 * (hc & 1);
              const int j0 = n_blk * kHalf + off;
              const int g0 = n_blk * N_TILE + off;
              float (&gg)[16] = g[hc & 1];
              float (&uu)[16] = u[hc & 1];
              // 16 outputs of row `lane` -> two 16-byte chunks of staging box hc / 2 (64B swizzle)
              uint8_t* box_row = stage_out + (hc >> 1) * 2048 + lane * 64;
#pragma unroll
              for (int i = 0; i < 16; i += 8) {
                affine8(ep, gg, i, g0 + i, j0 + i);
                affine8(ep, uu, i, g0 + kHalf + i, hN + j0 + i);
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                  const float z0 = gg[i + e], z1 = gg[i + e + 1];
                  const float y0 = silu_times(z0, uu[i + e]);
                  const float y1 = silu_times(z1, uu[i + e + 1]);
                  const __nv_bfloat162 b2 = __floats2bfloat162_rn(y0, y1);
                  w[e / 2] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                const int j = 2 * (hc & 1) + i / 8;
                *reinterpret_cast<uint4*>(box_row + ((j ^ ((lane >> 1) & 3)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
              }
              if (hc + 1 < nh) tmem_wait_ld();
            }
          }
#pragma unroll
          for (int c = 0; c < 2; ++c)
            if (c < n_mine) store_box(stage_out + c * 2048, row0, n_blk * kHalf + (glu_beg + c) * 32);
        } else {
#pragma unroll 1
          for (int c = 0; c < n_mine; ++c) {
            const int cc = glu_beg + c;
            float gt[32], up[32];
            tmem_ld_32x32(tb + cc * 32, gt);
            tmem_ld_32x32(tb + kHalf + cc * 32, up);
            tmem_wait_ld();
            if (c + 1 == n_mine) release_acc();
            const int j0 = n_blk * kHalf + cc * 32;
            const int g0 = n_blk * N_TILE + cc * 32;
            affine(ep, gt, g0, j0);
            affine(ep, up, g0 + kHalf, hN + j0);
            // the same arithmetic as the bf16 path, so that bf16 output = bf16(fp32 output)
#pragma unroll
            for (int i = 0; i < 32; ++i) gt[i] = silu_times(gt[i], up[i]);
            emit_f32(gt, row0, j0);
          }
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

}  // namespace svdq
