// C ABI of the sm_100a W4A4 + low-rank linear layer (declared in include/svdq.h): argument checks,
// buffer layouts, TMA descriptor construction and kernel launches. One translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>
#include <string>

#include "svdq.h"
#include "svdq_fp8r.cuh"
#include "svdq_fused.cuh"
#include "svdq_gemm.cuh"
#include "svdq_ptx.cuh"
#include "svdq_quant.cuh"

namespace {

thread_local std::string g_last_error;
std::atomic<unsigned long long> g_wait_ns{2000000000ull};

svdq_status fail(svdq_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
svdq_status fail(svdq_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

#define SVDQ_CUDA(call)                                                                         \
  do {                                                                                          \
    cudaError_t e_ = (call);                                                                    \
    if (e_ != cudaSuccess) return fail(SVDQ_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ per-device state
struct DeviceState {
  bool ready = false;
  int sm_count = 0;
  int max_pairs[4] = {0, 0, 0, 0};  // co-resident CTA pairs of the GEMM kernel for n_tile 256, 192, 128, 384
  int k1_clusters[4][4] = {};     // co-resident kernel-1 clusters, by r (0/16/32/64) and size - 1 (1..4)
  svdq_status status = SVDQ_OK;
  std::string error;
};
std::mutex g_dev_mu;
DeviceState g_dev[64];

constexpr int kStagesTile256 = 5;
constexpr int kStagesTile192 = 5;
constexpr int kStagesTile128 = 6;
constexpr int kStagesTile384 = 4;

using Encode = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                            const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                            CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
Encode g_encode = nullptr;

svdq_status device_ready(int* dev_out, int* sm_out) {
  int dev = 0;
  SVDQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(SVDQ_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    int major = 0, minor = 0, sms = 0;
    SVDQ_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    SVDQ_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    SVDQ_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    if (major != 10 || minor != 0)
      return fail(SVDQ_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a only", dev, major,
                  minor);
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      SVDQ_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
      if (fn == nullptr || q != cudaDriverEntryPointSuccess)
        return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled not available from the driver");
      g_encode = reinterpret_cast<Encode>(fn);
    }
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::pair_gemm_kernel<svdq::Nvfp4Gemm, 256, kStagesTile256>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   svdq::GemmLayout<256, kStagesTile256>::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::pair_gemm_kernel<svdq::Nvfp4Gemm, 192, kStagesTile192>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   svdq::GemmLayout<192, kStagesTile192>::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::pair_gemm_kernel<svdq::Nvfp4Gemm, 128, kStagesTile128>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   svdq::GemmLayout<128, kStagesTile128>::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::pair_gemm_kernel<svdq::Nvfp4Gemm, 384, kStagesTile384>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   svdq::GemmLayout<384, kStagesTile384>::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::quant_act_kernel<0, svdq::Nvfp4Act>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   svdq::Q1Layout<0>::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::quant_act_kernel<16, svdq::Nvfp4Act>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   svdq::Q1Layout<16>::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::quant_act_kernel<32, svdq::Nvfp4Act>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   svdq::Q1Layout<32>::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::quant_act_kernel<64, svdq::Nvfp4Act>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   svdq::Q1Layout<64>::kSmem));
    // How many CTA pairs of each GEMM instantiation can be resident at once: the persistent grid
    // never asks for more (pairs must sit on two SMs of one GPC, so this can be below sms / 2).
    auto max_pairs = [&](const void* fn, int smem, int* out) -> svdq_status {
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
      cfg.blockDim = dim3(svdq::kGemmThreads, 1, 1);
      cfg.dynamicSmemBytes = static_cast<size_t>(smem);
      int n = 0;
      SVDQ_CUDA(cudaOccupancyMaxActiveClusters(&n, fn, &cfg));
      if (n <= 0) return fail(SVDQ_ERR_CUDA, "GEMM kernel cannot be resident as CTA pairs");
      *out = n;
      return SVDQ_OK;
    };
    if (svdq_status s = max_pairs(reinterpret_cast<const void*>(svdq::pair_gemm_kernel<svdq::Nvfp4Gemm, 256, kStagesTile256>),
                                  svdq::GemmLayout<256, kStagesTile256>::kSmem, &st.max_pairs[0]);
        s != SVDQ_OK)
      return s;
    if (svdq_status s = max_pairs(reinterpret_cast<const void*>(svdq::pair_gemm_kernel<svdq::Nvfp4Gemm, 192, kStagesTile192>),
                                  svdq::GemmLayout<192, kStagesTile192>::kSmem, &st.max_pairs[1]);
        s != SVDQ_OK)
      return s;
    if (svdq_status s = max_pairs(reinterpret_cast<const void*>(svdq::pair_gemm_kernel<svdq::Nvfp4Gemm, 128, kStagesTile128>),
                                  svdq::GemmLayout<128, kStagesTile128>::kSmem, &st.max_pairs[2]);
        s != SVDQ_OK)
      return s;
    if (svdq_status s = max_pairs(reinterpret_cast<const void*>(svdq::pair_gemm_kernel<svdq::Nvfp4Gemm, 384, kStagesTile384>),
                                  svdq::GemmLayout<384, kStagesTile384>::kSmem, &st.max_pairs[3]);
        s != SVDQ_OK)
      return s;
    // how many kernel-1 clusters of 1, 2, 3 and 4 CTAs (one CTA per SM) can be resident at once
    // (a cluster's CTAs share a GPC, so fewer 4-clusters than sms / 4 may fit)
    auto k1_clusters = [&](const void* fn, int smem, int* out) -> svdq_status {
      for (int ci = 0; ci < 4; ++ci) {
        const int c = ci + 1;
        cudaLaunchConfig_t cfg{};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = c;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(c * (sms / c), 1, 1);
        cfg.blockDim = dim3(svdq::kQ1Threads, 1, 1);
        cfg.dynamicSmemBytes = static_cast<size_t>(smem);
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        SVDQ_CUDA(cudaOccupancyMaxActiveClusters(&n, fn, &cfg));
        out[ci] = n;
      }
      return SVDQ_OK;
    };
    if (svdq_status s = k1_clusters(reinterpret_cast<const void*>(svdq::quant_act_kernel<0, svdq::Nvfp4Act>), svdq::Q1Layout<0>::kSmem,
                                    st.k1_clusters[0]);
        s != SVDQ_OK)
      return s;
    if (svdq_status s = k1_clusters(reinterpret_cast<const void*>(svdq::quant_act_kernel<16, svdq::Nvfp4Act>),
                                    svdq::Q1Layout<16>::kSmem, st.k1_clusters[1]);
        s != SVDQ_OK)
      return s;
    if (svdq_status s = k1_clusters(reinterpret_cast<const void*>(svdq::quant_act_kernel<32, svdq::Nvfp4Act>),
                                    svdq::Q1Layout<32>::kSmem, st.k1_clusters[2]);
        s != SVDQ_OK)
      return s;
    if (svdq_status s = k1_clusters(reinterpret_cast<const void*>(svdq::quant_act_kernel<64, svdq::Nvfp4Act>),
                                    svdq::Q1Layout<64>::kSmem, st.k1_clusters[3]);
        s != SVDQ_OK)
      return s;
    st.sm_count = sms;
    st.ready = true;
  }
  if (dev_out) *dev_out = dev;
  if (sm_out) *sm_out = st.sm_count;
  return SVDQ_OK;
}

svdq_status make_tmap(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                      uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return SVDQ_OK;
}

// The low-rank operands travel in chunks of at most 32 columns of r (one ring slot each).
CUtensorMapSwizzle lr_swizzle(int r) { return r == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B; }

bool valid_r(int r) { return r == 0 || r == 16 || r == 32 || r == 64; }

// The 384-wide NVFP4 tile (two pair MMAs per K chunk): a weight without the SwiGLU interleave whose
// N is a multiple of 768, so that its blob has the same size as at 256 (N / 128 scale atoms per K
// atom either way) and svdq_weight_bytes need not know whether a weight is SwiGLU.
bool wide_tile_ok(int N, int swiglu) { return !swiglu && N % 768 == 0; }

// GEMM tile width along N: the widest that divides N, for the fewest operand bytes streamed per
// flop: 384 (where wide_tile_ok and `wide`: the NVFP4 GEMM), else 256, 192, 128. SVDQ_N_TILE
// overrides it with another valid width.
int choose_n_tile(int N, int swiglu, bool wide) {
  const char* env = getenv("SVDQ_N_TILE");
  if (env != nullptr) {
    const int t = atoi(env);
    if ((t == 256 || t == 192 || t == 128) && N % t == 0) return t;
    if (t == 384 && wide && wide_tile_ok(N, swiglu)) return t;
  }
  if (wide && wide_tile_ok(N, swiglu)) return 384;
  if (N % 256 == 0) return 256;
  if (N % 192 == 0) return 192;
  if (N % 128 == 0) return 128;
  return 0;
}
// A GEMM tile width a descriptor of an NVFP4 weight may hold.
bool valid_n_tile(int N, int n_tile, int swiglu) {
  if (n_tile == 384) return wide_tile_ok(N, swiglu);
  return (n_tile == 256 || n_tile == 192 || n_tile == 128) && N % n_tile == 0;
}

struct WeightLayout {
  size_t codes, scales, gw, inv_lambda, l1t, l2t, total;
};
WeightLayout weight_layout(int N, int K, int r, int n_tile) {
  WeightLayout l{};
  size_t off = 0;
  l.codes = off;
  off = align_up(off + static_cast<size_t>(N) * K / 2);
  l.scales = off;
  off = align_up(off + static_cast<size_t>(N / n_tile) * (K / 64) * ((n_tile + 127) / 128) * 512);
  l.gw = off;
  off = align_up(off + 4);
  l.inv_lambda = off;
  off = align_up(off + static_cast<size_t>(K) * 4);
  l.l1t = off;
  off = align_up(off + static_cast<size_t>(r) * K * 2);
  l.l2t = off;
  off = align_up(off + static_cast<size_t>(N) * r * 2);
  l.total = off;
  return l;
}

struct ActLayout {
  size_t codes, scales, u, alpha, total;
  int M_pad;
};
ActLayout act_layout(int M, int K, int r) {
  ActLayout l{};
  l.M_pad = (M + 127) / 128 * 128;
  size_t off = 0;
  l.codes = off;
  off = align_up(off + static_cast<size_t>(l.M_pad) * K / 2);
  l.scales = off;
  off = align_up(off + static_cast<size_t>(l.M_pad / 128) * (K / 64) * 512);
  l.u = off;
  off = align_up(off + static_cast<size_t>(l.M_pad) * r * 2 * 2);  // hi and lo halves
  l.alpha = off;
  off = align_up(off + 4);
  l.total = off;
  return l;
}

bool shape_ok(int N, int K, int r) {
  return N > 0 && K > 0 && K % 256 == 0 && valid_r(r) && K <= (1 << 20) && N <= (1 << 20) &&
         choose_n_tile(N, 0, false) > 0;
}

// The descriptors are plain structs that a caller may also fill by hand: before a launch reads
// through them, check that they describe a layout that svdq_pack_weight / svdq_act_bind can produce.
svdq_status check_weight(const svdq_weight* w) {
  const int t = w->n_tile;
  if (w->N <= 0 || !valid_n_tile(w->N, t, w->swiglu_interleaved) || w->N > (1 << 20) || w->K <= 0 ||
      w->K % 256 != 0 || w->K > (1 << 20) || !valid_r(w->r))
    return fail(SVDQ_ERR_INVALID_ARG, "weight descriptor N=%d K=%d r=%d n_tile=%d is not one svdq_pack_weight makes",
                w->N, w->K, w->r, t);
  if (w->codes == nullptr || w->scales == nullptr || w->g_w == nullptr || w->inv_lambda == nullptr ||
      (w->r > 0 && (w->L1s_t == nullptr || w->L2_t == nullptr)))
    return fail(SVDQ_ERR_INVALID_ARG, "weight descriptor has a null buffer");
  return SVDQ_OK;
}

svdq_status check_act(const svdq_act* a) {
  if (a->M < 1 || a->M >= (1 << 24) || a->K <= 0 || a->K % 256 != 0 || a->K > (1 << 20) || !valid_r(a->r) ||
      a->M_pad != (a->M + 127) / 128 * 128)
    return fail(SVDQ_ERR_INVALID_ARG, "act descriptor M=%d M_pad=%d K=%d r=%d is not one svdq_act_bind makes", a->M,
                a->M_pad, a->K, a->r);
  if (a->codes == nullptr || a->scales == nullptr || a->alpha == nullptr || (a->r > 0 && a->U == nullptr))
    return fail(SVDQ_ERR_INVALID_ARG, "act descriptor has a null buffer");
  return SVDQ_OK;
}

// Descriptor of a packed weight blob at `b`: the pointers of weight_layout(N, K, r, n_tile) and
// the TMA descriptors of its codes and L2^T, which hold absolute addresses and so are encoded for
// this copy of the blob. svdq_pack_weight and svdq_weight_bind both fill descriptors here.
svdq_status fill_weight_desc(uint8_t* b, int N, int K, int r, int swiglu, int n_tile, svdq_weight* out) {
  const WeightLayout l = weight_layout(N, K, r, n_tile);
  svdq_weight w{};
  w.N = N;
  w.K = K;
  w.r = r;
  w.swiglu_interleaved = swiglu ? 1 : 0;
  w.n_tile = n_tile;
  w.codes = b + l.codes;
  w.scales = b + l.scales;
  w.g_w = reinterpret_cast<float*>(b + l.gw);
  w.inv_lambda = reinterpret_cast<float*>(b + l.inv_lambda);
  w.L1s_t = b + l.l1t;
  w.L2_t = b + l.l2t;
  static_assert(sizeof(w.tmap) >= 2 * sizeof(CUtensorMap), "tmap storage");
  CUtensorMap tmB, tmL2;
  std::memset(&tmL2, 0, sizeof(tmL2));
  // each CTA of a GEMM pair stages half of a tile's n_tile rows
  if (svdq_status s = make_tmap(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.codes, K / 2, N, K / 2, 128, n_tile / 2,
                                CU_TENSOR_MAP_SWIZZLE_128B);
      s != SVDQ_OK)
    return s;
  if (r > 0) {
    if (svdq_status s = make_tmap(&tmL2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w.L2_t, r, N, static_cast<uint64_t>(r) * 2,
                                  r < 32 ? r : 32, n_tile / 2, lr_swizzle(r));
        s != SVDQ_OK)
      return s;
  }
  std::memcpy(&w.tmap[0][0], &tmB, sizeof(CUtensorMap));
  std::memcpy(&w.tmap[1][0], &tmL2, sizeof(CUtensorMap));
  *out = w;
  return SVDQ_OK;
}

int grid_for(size_t work_items, int per_block, int sm_count) {
  size_t blocks = (work_items + per_block - 1) / per_block;
  size_t cap = static_cast<size_t>(sm_count) * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return static_cast<int>(blocks);
}

svdq_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, "launch of %s failed: %s", what, cudaGetErrorString(e));
  return SVDQ_OK;
}

// Both kernels of a layer are launched with programmatic stream serialization: a kernel may be
// scheduled while the previous kernel on the stream is finishing, so its barrier and TMEM set-up
// overlap that kernel's tail; its first global access waits for that grid (griddepcontrol.wait).
void set_programmatic(cudaLaunchAttribute& a) {
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
}

// The pair GEMMs: clusters of 2 CTAs are compiled into the kernel, so the one launch attribute is
// the programmatic one.
template <typename... P, typename... A>
cudaError_t launch_pair_gemm(void (*kern)(P...), int ctas, int smem, cudaStream_t st, A&&... args) {
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  set_programmatic(attr[0]);
  cfg.gridDim = dim3(ctas, 1, 1);
  cfg.blockDim = dim3(svdq::kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

}  // namespace

extern "C" {

int svdq_abi_version(void) { return SVDQ_ABI_VERSION; }

const char* svdq_status_str(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_UNSUPPORTED: return "unsupported shape, alignment or device";
    case SVDQ_ERR_CUDA: return "CUDA error";
    case SVDQ_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

const char* svdq_last_error(void) { return g_last_error.c_str(); }

size_t svdq_weight_bytes(int N, int K, int r) {
  if (!shape_ok(N, K, r)) return 0;
  return weight_layout(N, K, r, choose_n_tile(N, 0, true)).total;
}

size_t svdq_weight_bytes_tiled(int N, int K, int r, int n_tile) {
  if (N <= 0 || K <= 0 || K % 256 != 0 || K > (1 << 20) || N > (1 << 20) || !valid_r(r) ||
      !valid_n_tile(N, n_tile, 0))
    return 0;
  return weight_layout(N, K, r, n_tile).total;
}

size_t svdq_act_bytes(int M, int K, int r) {
  if (M < 1 || M >= (1 << 24) || K <= 0 || K % 256 != 0 || !valid_r(r)) return 0;
  return act_layout(M, K, r).total;
}

svdq_status svdq_set_wait_limit_ns(unsigned long long ns) {
  if (ns < 1000000ull || ns > 60000000000ull) return fail(SVDQ_ERR_INVALID_ARG, "wait limit %llu ns out of range", ns);
  g_wait_ns.store(ns);
  return SVDQ_OK;
}

svdq_status svdq_act_bind(int M, int K, int r, void* dst, size_t dst_bytes, svdq_act* out) {
  if (out == nullptr || dst == nullptr) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  const size_t need = svdq_act_bytes(M, K, r);
  if (need == 0) return fail(SVDQ_ERR_UNSUPPORTED, "act shape M=%d K=%d r=%d unsupported", M, K, r);
  if (dst_bytes < need) return fail(SVDQ_ERR_INVALID_ARG, "act buffer %zu bytes < %zu", dst_bytes, need);
  if (reinterpret_cast<uintptr_t>(dst) % kAlign) return fail(SVDQ_ERR_UNSUPPORTED, "act buffer not 256-byte aligned");
  const ActLayout l = act_layout(M, K, r);
  uint8_t* b = static_cast<uint8_t*>(dst);
  out->M = M;
  out->K = K;
  out->r = r;
  out->M_pad = l.M_pad;
  out->codes = b + l.codes;
  out->scales = b + l.scales;
  out->U = b + l.u;
  out->alpha = reinterpret_cast<float*>(b + l.alpha);
  return SVDQ_OK;
}

svdq_status svdq_pack_weight(const float* R_nk, const uint16_t* L1s_kr, const uint16_t* L2_rn,
                             const float* inv_lambda, int N, int K, int r, int swiglu, void* dst, size_t dst_bytes,
                             svdq_weight* out, svdq_stream_t stream) {
  if (out == nullptr || R_nk == nullptr || inv_lambda == nullptr || dst == nullptr)
    return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (r > 0 && (L1s_kr == nullptr || L2_rn == nullptr)) return fail(SVDQ_ERR_INVALID_ARG, "null L1s / L2 with r > 0");
  if (!shape_ok(N, K, r)) return fail(SVDQ_ERR_UNSUPPORTED, "weight shape N=%d K=%d r=%d unsupported", N, K, r);
  if (swiglu && (N % 2 != 0)) return fail(SVDQ_ERR_UNSUPPORTED, "SwiGLU needs N even");
  if (!aligned16(R_nk) || !aligned16(inv_lambda) || (r > 0 && (!aligned16(L1s_kr) || !aligned16(L2_rn))))
    return fail(SVDQ_ERR_UNSUPPORTED, "inputs must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(dst) % kAlign) return fail(SVDQ_ERR_UNSUPPORTED, "dst not 256-byte aligned");
  const int n_tile = choose_n_tile(N, swiglu, true);
  const WeightLayout l = weight_layout(N, K, r, n_tile);
  if (dst_bytes < l.total) return fail(SVDQ_ERR_INVALID_ARG, "weight buffer %zu bytes < %zu", dst_bytes, l.total);
  int dev, sms;
  if (svdq_status s = device_ready(&dev, &sms); s != SVDQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* b = static_cast<uint8_t*>(dst);

  svdq_weight w{};
  if (svdq_status s = fill_weight_desc(b, N, K, r, swiglu, n_tile, &w); s != SVDQ_OK) return s;

  SVDQ_CUDA(cudaMemsetAsync(b + l.scales, 0, l.gw - l.scales + 4, st));  // pad rows of the scale layout, amax
  SVDQ_CUDA(cudaMemcpyAsync(w.inv_lambda, inv_lambda, static_cast<size_t>(K) * 4, cudaMemcpyDeviceToDevice, st));
  const size_t n4 = static_cast<size_t>(N) * K / 4;
  svdq::amax_f32_kernel<<<grid_for(n4, 256, sms), 256, 0, st>>>(R_nk, n4, reinterpret_cast<unsigned*>(w.g_w));
  if (svdq_status s = check_launch("amax_f32_kernel"); s != SVDQ_OK) return s;
  svdq::finalize_scale_kernel<<<1, 1, 0, st>>>(w.g_w);
  if (svdq_status s = check_launch("finalize_scale_kernel"); s != SVDQ_OK) return s;
  const size_t halves = static_cast<size_t>(N) * K / 8;
  svdq::pack_quant_kernel<<<grid_for(halves, 256, sms), 256, 0, st>>>(
      R_nk, N, K, n_tile, w.swiglu_interleaved, w.g_w, static_cast<uint8_t*>(w.codes), static_cast<uint8_t*>(w.scales));
  if (svdq_status s = check_launch("pack_quant_kernel"); s != SVDQ_OK) return s;
  if (r > 0) {
    svdq::transpose_l1_kernel<<<grid_for(static_cast<size_t>(K) * r, 256, sms), 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(L1s_kr), K, r, static_cast<__nv_bfloat16*>(w.L1s_t));
    if (svdq_status s = check_launch("transpose_l1_kernel"); s != SVDQ_OK) return s;
    svdq::pack_l2_kernel<<<grid_for(static_cast<size_t>(N) * r, 256, sms), 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(L2_rn), N, r, n_tile, w.swiglu_interleaved,
        static_cast<__nv_bfloat16*>(w.L2_t));
    if (svdq_status s = check_launch("pack_l2_kernel"); s != SVDQ_OK) return s;
  }
  *out = w;
  return SVDQ_OK;
}

svdq_status svdq_weight_bind(int N, int K, int r, int swiglu, int n_tile, void* blob, size_t blob_bytes,
                             svdq_weight* out) {
  if (out == nullptr || blob == nullptr) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (N <= 0 || K <= 0 || K % 256 != 0 || K > (1 << 20) || N > (1 << 20) || !valid_r(r) ||
      !valid_n_tile(N, n_tile, swiglu))
    return fail(SVDQ_ERR_UNSUPPORTED, "weight shape N=%d K=%d r=%d n_tile=%d swiglu=%d unsupported", N, K, r, n_tile,
                swiglu);
  if (reinterpret_cast<uintptr_t>(blob) % kAlign) return fail(SVDQ_ERR_UNSUPPORTED, "blob not 256-byte aligned");
  const WeightLayout l = weight_layout(N, K, r, n_tile);
  if (blob_bytes < l.total) return fail(SVDQ_ERR_INVALID_ARG, "weight blob %zu bytes < %zu", blob_bytes, l.total);
  int dev, sms;
  if (svdq_status s = device_ready(&dev, &sms); s != SVDQ_OK) return s;
  // the TMA descriptors hold absolute addresses: they are encoded for this copy of the blob
  return fill_weight_desc(static_cast<uint8_t*>(blob), N, K, r, swiglu, n_tile, out);
}

svdq_status svdq_calibrate_act(const uint16_t* X, int M, const svdq_weight* w, float* g_x_out, svdq_stream_t stream) {
  if (X == nullptr || w == nullptr || g_x_out == nullptr) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (svdq_status s = check_weight(w); s != SVDQ_OK) return s;
  if (M < 1 || M >= (1 << 24)) return fail(SVDQ_ERR_UNSUPPORTED, "M=%d unsupported", M);
  if (!aligned16(X)) return fail(SVDQ_ERR_UNSUPPORTED, "X must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(g_x_out) & 3u) return fail(SVDQ_ERR_UNSUPPORTED, "g_x_out must be 4-byte aligned");
  int dev, sms;
  if (svdq_status s = device_ready(&dev, &sms); s != SVDQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SVDQ_CUDA(cudaMemsetAsync(g_x_out, 0, 4, st));
  // 128 column chunks of 8 per block along x; rows split over y so that ~16 blocks land per SM
  const int per_row = w->K / 8;
  const int gx = (per_row + 127) / 128;
  int gy = sms * 16 / gx;
  if (gy > M) gy = M;
  if (gy > 65535) gy = 65535;
  if (gy < 1) gy = 1;
  svdq::act_amax_kernel<<<dim3(gx, gy), 128, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(X), w->inv_lambda,
                                                      M, w->K, reinterpret_cast<unsigned*>(g_x_out));
  if (svdq_status s = check_launch("act_amax_kernel"); s != SVDQ_OK) return s;
  svdq::finalize_scale_kernel<<<1, 1, 0, st>>>(g_x_out);
  return check_launch("finalize_scale_kernel");
}

svdq_status svdq_quantize_act(const uint16_t* X, const svdq_weight* w, const float* g_x, const svdq_act* act,
                              svdq_stream_t stream) {
  if (X == nullptr || w == nullptr || g_x == nullptr || act == nullptr) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (act->K != w->K || act->r != w->r)
    return fail(SVDQ_ERR_INVALID_ARG, "act (K=%d r=%d) does not match weight (K=%d r=%d)", act->K, act->r, w->K, w->r);
  if (svdq_status s = check_weight(w); s != SVDQ_OK) return s;
  if (svdq_status s = check_act(act); s != SVDQ_OK) return s;
  if (!aligned16(X)) return fail(SVDQ_ERR_UNSUPPORTED, "X must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(g_x) & 3u) return fail(SVDQ_ERR_UNSUPPORTED, "g_x must be 4-byte aligned");
  int dev, sms;
  if (svdq_status s = device_ready(&dev, &sms); s != SVDQ_OK) return s;
  const int K = act->K, r = w->r, M = act->M;
  CUtensorMap tmX, tmL1;
  std::memset(&tmL1, 0, sizeof(tmL1));
  if (svdq_status s = make_tmap(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, static_cast<uint64_t>(K) * 2, 64, 128,
                                CU_TENSOR_MAP_SWIZZLE_128B);
      s != SVDQ_OK)
    return s;
  if (r > 0) {
    if (svdq_status s = make_tmap(&tmL1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->L1s_t, K, r,
                                  static_cast<uint64_t>(K) * 2, 64, r, CU_TENSOR_MAP_SWIZZLE_128B);
        s != SVDQ_OK)
      return s;
  }
  // One CTA per SM; K is split across the largest cluster of 2, 3 or 4 CTAs whose clusters for all
  // row tiles are resident at once (cudaOccupancyMaxActiveClusters: clusters must fit inside GPCs),
  // so small M fills more SMs and nothing runs as a second wave. Measured on B200 at M = 4608 (36 row
  // tiles): only 32 clusters of 4 are resident, and at K = 12288 3-CTA clusters (108 CTAs) take
  // 47 us against 57 us for 2-CTA ones (72 CTAs). SVDQ_K1_CLUSTER overrides the size; every CTA
  // keeps whole 64-column K steps.
  const int m_tiles = act->M_pad / 128;
  int csize = 1;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    const int* mc = g_dev[dev].k1_clusters[r == 0 ? 0 : r == 16 ? 1 : r == 32 ? 2 : 3];
    for (int c = 2; c <= 4; ++c)
      if (m_tiles <= mc[c - 1] && K % (64 * c) == 0) csize = c;
  }
  if (const char* env = getenv("SVDQ_K1_CLUSTER"); env != nullptr) {
    const int c = atoi(env);
    if (c >= 1 && c <= 4 && K % (64 * c) == 0) csize = c;
  }
  svdq::QuantActArgs a;
  a.inv_lambda = w->inv_lambda;
  a.g_x = g_x;
  a.g_w = w->g_w;
  a.codes = static_cast<uint8_t*>(act->codes);
  a.sf = static_cast<uint8_t*>(act->scales);
  a.U = static_cast<__nv_bfloat16*>(act->U);
  a.alpha = act->alpha;
  a.wait_ns = g_wait_ns.load();
  a.M = M;
  a.K = K;
  a.M_pad = act->M_pad;
  a.k_per_cta = K / csize;

  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  set_programmatic(attr[1]);
  cfg.gridDim = dim3(m_tiles * csize, 1, 1);
  cfg.blockDim = dim3(svdq::kQ1Threads, 1, 1);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaSuccess;
  switch (r) {
    case 0:
      cfg.dynamicSmemBytes = svdq::Q1Layout<0>::kSmem;
      e = cudaLaunchKernelEx(&cfg, svdq::quant_act_kernel<0, svdq::Nvfp4Act>, tmX, tmL1, a);
      break;
    case 16:
      cfg.dynamicSmemBytes = svdq::Q1Layout<16>::kSmem;
      e = cudaLaunchKernelEx(&cfg, svdq::quant_act_kernel<16, svdq::Nvfp4Act>, tmX, tmL1, a);
      break;
    case 32:
      cfg.dynamicSmemBytes = svdq::Q1Layout<32>::kSmem;
      e = cudaLaunchKernelEx(&cfg, svdq::quant_act_kernel<32, svdq::Nvfp4Act>, tmX, tmL1, a);
      break;
    case 64:
      cfg.dynamicSmemBytes = svdq::Q1Layout<64>::kSmem;
      e = cudaLaunchKernelEx(&cfg, svdq::quant_act_kernel<64, svdq::Nvfp4Act>, tmX, tmL1, a);
      break;
    default: return fail(SVDQ_ERR_UNSUPPORTED, "r=%d unsupported", r);
  }
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, "launch of quant_act_kernel failed: %s", cudaGetErrorString(e));
  return check_launch("quant_act_kernel");
}

svdq_status svdq_gemm(const svdq_act* act, const svdq_weight* w, const uint16_t* bias, svdq_epilogue epi, void* Y,
                      svdq_out_dtype out_dtype, svdq_stream_t stream) {
  if (act == nullptr || w == nullptr || Y == nullptr) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (act->K != w->K || act->r != w->r) return fail(SVDQ_ERR_INVALID_ARG, "act does not match weight");
  if (svdq_status s = check_weight(w); s != SVDQ_OK) return s;
  if (svdq_status s = check_act(act); s != SVDQ_OK) return s;
  if (epi < SVDQ_EPI_NONE || epi > SVDQ_EPI_BIAS_SWIGLU) return fail(SVDQ_ERR_INVALID_ARG, "bad epilogue %d", epi);
  if (out_dtype != SVDQ_OUT_BF16 && out_dtype != SVDQ_OUT_F32) return fail(SVDQ_ERR_INVALID_ARG, "bad out dtype");
  const bool has_bias = (epi & 1) != 0, swiglu = (epi & 2) != 0;
  if (has_bias && bias == nullptr) return fail(SVDQ_ERR_INVALID_ARG, "epilogue needs a bias");
  if (swiglu && !w->swiglu_interleaved) return fail(SVDQ_ERR_INVALID_ARG, "SwiGLU needs a weight packed with swiglu=1");
  if (!swiglu && w->swiglu_interleaved) return fail(SVDQ_ERR_INVALID_ARG, "weight packed for SwiGLU");
  if (!aligned16(Y) || (bias != nullptr && !aligned16(bias))) return fail(SVDQ_ERR_UNSUPPORTED, "Y / bias alignment");
  const int n_tile = w->n_tile;
  int dev, sms;
  if (svdq_status s = device_ready(&dev, &sms); s != SVDQ_OK) return s;

  const int K = w->K, r = w->r;
  CUtensorMap tmA, tmU;
  std::memset(&tmU, 0, sizeof(tmU));
  if (svdq_status s = make_tmap(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, act->codes, K / 2, act->M_pad, K / 2, 128, 128,
                                CU_TENSOR_MAP_SWIZZLE_128B);
      s != SVDQ_OK)
    return s;
  if (r > 0) {
    if (svdq_status s = make_tmap(&tmU, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act->U, r, 2 * static_cast<uint64_t>(act->M_pad),
                                  static_cast<uint64_t>(r) * 2, r < 32 ? r : 32, 128, lr_swizzle(r));
        s != SVDQ_OK)
      return s;
  }
  CUtensorMap tmB, tmL2;  // properly aligned copies of the descriptors cached in the weight
  std::memcpy(&tmB, &w->tmap[0][0], sizeof(CUtensorMap));
  std::memcpy(&tmL2, &w->tmap[1][0], sizeof(CUtensorMap));

  svdq::GemmArgs g{};
  g.sfa = static_cast<const uint8_t*>(act->scales);
  g.sfb = static_cast<const uint8_t*>(w->scales);
  g.alpha = act->alpha;
  g.bias = reinterpret_cast<const __nv_bfloat16*>(bias);
  g.Y = Y;
  g.wait_ns = g_wait_ns.load();
  g.M = act->M;
  g.M_pad = act->M_pad;
  g.N = w->N;
  g.K = K;
  g.r = r;
  g.m_tiles = act->M_pad / 128;
  g.m_pairs = (g.m_tiles + 1) / 2;
  g.n_tiles = w->N / n_tile;
  g.k_iters = K / 256;
  g.num_tiles = g.m_pairs * g.n_tiles;
  g.ldy = swiglu ? w->N / 2 : w->N;
  g.out_f32 = out_dtype == SVDQ_OUT_F32 ? 1 : 0;
  g.epi = static_cast<int>(epi);
  CUtensorMap tmY;
  if (svdq_status s = make_tmap(&tmY, g.out_f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y,
                                static_cast<uint64_t>(g.ldy), static_cast<uint64_t>(act->M),
                                static_cast<uint64_t>(g.ldy) * (g.out_f32 ? 4 : 2), 32, 32,
                                g.out_f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
      s != SVDQ_OK)
    return s;
  int max_pairs = 0;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    max_pairs = g_dev[dev].max_pairs[n_tile == 256 ? 0 : n_tile == 192 ? 1 : n_tile == 128 ? 2 : 3];
  }
  const int pairs = g.num_tiles < max_pairs ? g.num_tiles : max_pairs;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (n_tile == 384)
    e = launch_pair_gemm(svdq::pair_gemm_kernel<svdq::Nvfp4Gemm, 384, kStagesTile384>, 2 * pairs,
                         svdq::GemmLayout<384, kStagesTile384>::kSmem, st, tmA, tmB, tmU, tmL2, tmY, g);
  else if (n_tile == 256)
    e = launch_pair_gemm(svdq::pair_gemm_kernel<svdq::Nvfp4Gemm, 256, kStagesTile256>, 2 * pairs,
                         svdq::GemmLayout<256, kStagesTile256>::kSmem, st, tmA, tmB, tmU, tmL2, tmY, g);
  else if (n_tile == 192)
    e = launch_pair_gemm(svdq::pair_gemm_kernel<svdq::Nvfp4Gemm, 192, kStagesTile192>, 2 * pairs,
                         svdq::GemmLayout<192, kStagesTile192>::kSmem, st, tmA, tmB, tmU, tmL2, tmY, g);
  else
    e = launch_pair_gemm(svdq::pair_gemm_kernel<svdq::Nvfp4Gemm, 128, kStagesTile128>, 2 * pairs,
                         svdq::GemmLayout<128, kStagesTile128>::kSmem, st, tmA, tmB, tmU, tmL2, tmY, g);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, "launch of pair_gemm_kernel failed: %s", cudaGetErrorString(e));
  return check_launch("pair_gemm_kernel (NVFP4)");
}

svdq_status svdq_export_weight(const svdq_weight* w, uint8_t* codes, uint8_t* scales, svdq_stream_t stream) {
  if (w == nullptr || codes == nullptr || scales == nullptr) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (svdq_status s = check_weight(w); s != SVDQ_OK) return s;
  int dev, sms;
  if (svdq_status s = device_ready(&dev, &sms); s != SVDQ_OK) return s;
  const size_t total = static_cast<size_t>(w->N) * (w->K / 16);
  svdq::export_weight_kernel<<<grid_for(total, 256, sms), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(w->codes), static_cast<const uint8_t*>(w->scales), w->N, w->K, w->n_tile,
      w->swiglu_interleaved, codes, scales);
  return check_launch("export_weight_kernel");
}

svdq_status svdq_export_act(const svdq_act* act, uint8_t* codes, uint8_t* scales, svdq_stream_t stream) {
  if (act == nullptr || codes == nullptr || scales == nullptr) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (svdq_status s = check_act(act); s != SVDQ_OK) return s;
  int dev, sms;
  if (svdq_status s = device_ready(&dev, &sms); s != SVDQ_OK) return s;
  const size_t total = static_cast<size_t>(act->M) * (act->K / 16);
  svdq::export_act_kernel<<<grid_for(total, 256, sms), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(act->codes), static_cast<const uint8_t*>(act->scales), act->M, act->K, codes,
      scales);
  return check_launch("export_act_kernel");
}

svdq_status svdq_device_status(int reset) {
  SVDQ_CUDA(cudaDeviceSynchronize());
  unsigned v = 0;
  SVDQ_CUDA(cudaMemcpyFromSymbol(&v, svdq::g_svdq_status, sizeof(v)));
  if (reset) {
    const unsigned z = 0;
    SVDQ_CUDA(cudaMemcpyToSymbol(svdq::g_svdq_status, &z, sizeof(z)));
  }
  if (v != 0) return fail(SVDQ_ERR_TIMEOUT, "device wait ran out (status bits 0x%x)", v);
  return SVDQ_OK;
}

svdq_status svdq_watchdog_selftest(unsigned long long limit_ns, svdq_stream_t stream) {
  if (limit_ns < 1000ull || limit_ns > 1000000000ull) return fail(SVDQ_ERR_INVALID_ARG, "limit out of range");
  int dev, sms;
  if (svdq_status s = device_ready(&dev, &sms); s != SVDQ_OK) return s;
  svdq::watchdog_selftest_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  return check_launch("watchdog_selftest_kernel");
}

}  // extern "C"

// ================================================================== row-wise FP8 (W8A8) variant
namespace {

constexpr int kFp8Stages256 = 6;
constexpr int kFp8Stages192 = 6;
constexpr int kFp8Stages128 = 8;

struct Fp8rState {
  bool ready = false;
  int max_pairs[3] = {0, 0, 0};  // co-resident CTA pairs of the FP8 GEMM for n_tile 256, 192, 128
};
Fp8rState g_fp8r[64];

svdq_status fp8r_max_pairs(const void* fn, int smem, int sms, int* out) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
  cfg.blockDim = dim3(svdq::kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  int n = 0;
  SVDQ_CUDA(cudaOccupancyMaxActiveClusters(&n, fn, &cfg));
  if (n <= 0) return fail(SVDQ_ERR_CUDA, "FP8 GEMM kernel cannot be resident as CTA pairs");
  *out = n;
  return SVDQ_OK;
}

// The FP8 kernels are set up on the first FP8 call on a device, apart from the NVFP4 set-up (which
// never depends on them).
svdq_status fp8r_ready(int* dev_out, int* sm_out) {
  int dev = 0, sms = 0;
  if (svdq_status s = device_ready(&dev, &sms); s != SVDQ_OK) return s;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  Fp8rState& st = g_fp8r[dev];
  if (!st.ready) {
    using L256 = svdq::PairGemmLayout<false, 256, kFp8Stages256>;
    using L192 = svdq::PairGemmLayout<false, 192, kFp8Stages192>;
    using L128 = svdq::PairGemmLayout<false, 128, kFp8Stages128>;
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::pair_gemm_kernel<svdq::fp8r::Fp8Gemm, 256, kFp8Stages256>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, L256::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::pair_gemm_kernel<svdq::fp8r::Fp8Gemm, 192, kFp8Stages192>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, L192::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::pair_gemm_kernel<svdq::fp8r::Fp8Gemm, 128, kFp8Stages128>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, L128::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::quant_act_kernel<0, svdq::fp8r::RowAct>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, svdq::Q1Layout<0>::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::quant_act_kernel<16, svdq::fp8r::RowAct>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, svdq::Q1Layout<16>::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::quant_act_kernel<32, svdq::fp8r::RowAct>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, svdq::Q1Layout<32>::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::quant_act_kernel<64, svdq::fp8r::RowAct>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, svdq::Q1Layout<64>::kSmem));
    if (svdq_status s = fp8r_max_pairs(reinterpret_cast<const void*>(svdq::pair_gemm_kernel<svdq::fp8r::Fp8Gemm, 256, kFp8Stages256>),
                                       L256::kSmem, sms, &st.max_pairs[0]);
        s != SVDQ_OK)
      return s;
    if (svdq_status s = fp8r_max_pairs(reinterpret_cast<const void*>(svdq::pair_gemm_kernel<svdq::fp8r::Fp8Gemm, 192, kFp8Stages192>),
                                       L192::kSmem, sms, &st.max_pairs[1]);
        s != SVDQ_OK)
      return s;
    if (svdq_status s = fp8r_max_pairs(reinterpret_cast<const void*>(svdq::pair_gemm_kernel<svdq::fp8r::Fp8Gemm, 128, kFp8Stages128>),
                                       L128::kSmem, sms, &st.max_pairs[2]);
        s != SVDQ_OK)
      return s;
    st.ready = true;
  }
  if (dev_out) *dev_out = dev;
  if (sm_out) *sm_out = sms;
  return SVDQ_OK;
}

struct Fp8rWeightLayout {
  size_t codes, scales, inv_lambda, l1t, l2t, total;
};
Fp8rWeightLayout fp8r_weight_layout(int N, int K, int r) {
  Fp8rWeightLayout l{};
  size_t off = 0;
  l.codes = off;
  off = align_up(off + static_cast<size_t>(N) * K);
  l.scales = off;
  off = align_up(off + static_cast<size_t>(N) * 4);
  l.inv_lambda = off;
  off = align_up(off + static_cast<size_t>(K) * 4);
  l.l1t = off;
  off = align_up(off + static_cast<size_t>(r) * K * 2);
  l.l2t = off;
  off = align_up(off + static_cast<size_t>(N) * r * 2 * 2);  // hi and lo halves
  l.total = off;
  return l;
}

struct Fp8rActLayout {
  size_t codes, s_x, rs_x, u, total;
  int M_pad;
};
Fp8rActLayout fp8r_act_layout(int M, int K, int r) {
  Fp8rActLayout l{};
  l.M_pad = (M + 127) / 128 * 128;
  size_t off = 0;
  l.codes = off;
  off = align_up(off + static_cast<size_t>(l.M_pad) * K);
  l.s_x = off;
  off = align_up(off + static_cast<size_t>(l.M_pad) * 4);
  l.rs_x = off;
  off = align_up(off + static_cast<size_t>(l.M_pad) * 4);
  l.u = off;
  off = align_up(off + static_cast<size_t>(l.M_pad) * r * 2 * 2);  // hi and lo halves
  l.total = off;
  return l;
}

svdq_status check_fp8r_weight(const svdq_fp8r_weight* w) {
  const int t = w->n_tile;
  if ((t != 256 && t != 192 && t != 128) || w->N <= 0 || w->N % t != 0 || w->N > (1 << 20) || w->K <= 0 ||
      w->K % 256 != 0 || w->K > (1 << 20) || !valid_r(w->r))
    return fail(SVDQ_ERR_INVALID_ARG,
                "FP8 weight descriptor N=%d K=%d r=%d n_tile=%d is not one svdq_fp8r_pack_weight makes", w->N, w->K,
                w->r, t);
  if (w->codes == nullptr || w->row_scale == nullptr || w->inv_lambda == nullptr ||
      (w->r > 0 && (w->L1s_t == nullptr || w->L2_t == nullptr)))
    return fail(SVDQ_ERR_INVALID_ARG, "FP8 weight descriptor has a null buffer");
  return SVDQ_OK;
}

svdq_status check_fp8r_act(const svdq_fp8r_act* a) {
  if (a->M < 1 || a->M >= (1 << 24) || a->K <= 0 || a->K % 256 != 0 || a->K > (1 << 20) || !valid_r(a->r) ||
      a->M_pad != (a->M + 127) / 128 * 128)
    return fail(SVDQ_ERR_INVALID_ARG,
                "FP8 act descriptor M=%d M_pad=%d K=%d r=%d is not one svdq_fp8r_act_bind makes", a->M, a->M_pad,
                a->K, a->r);
  if (a->codes == nullptr || a->row_scale == nullptr || a->row_rscale == nullptr || (a->r > 0 && a->U == nullptr))
    return fail(SVDQ_ERR_INVALID_ARG, "FP8 act descriptor has a null buffer");
  return SVDQ_OK;
}

}  // namespace

extern "C" {

size_t svdq_fp8r_weight_bytes(int N, int K, int r) {
  if (!shape_ok(N, K, r)) return 0;
  return fp8r_weight_layout(N, K, r).total;
}

size_t svdq_fp8r_act_bytes(int M, int K, int r) {
  if (M < 1 || M >= (1 << 24) || K <= 0 || K % 256 != 0 || K > (1 << 20) || !valid_r(r)) return 0;
  return fp8r_act_layout(M, K, r).total;
}

svdq_status svdq_fp8r_act_bind(int M, int K, int r, void* dst, size_t dst_bytes, svdq_fp8r_act* out) {
  if (out == nullptr || dst == nullptr) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  const size_t need = svdq_fp8r_act_bytes(M, K, r);
  if (need == 0) return fail(SVDQ_ERR_UNSUPPORTED, "FP8 act shape M=%d K=%d r=%d unsupported", M, K, r);
  if (dst_bytes < need) return fail(SVDQ_ERR_INVALID_ARG, "FP8 act buffer %zu bytes < %zu", dst_bytes, need);
  if (reinterpret_cast<uintptr_t>(dst) % kAlign) return fail(SVDQ_ERR_UNSUPPORTED, "act buffer not 256-byte aligned");
  const Fp8rActLayout l = fp8r_act_layout(M, K, r);
  uint8_t* b = static_cast<uint8_t*>(dst);
  out->M = M;
  out->K = K;
  out->r = r;
  out->M_pad = l.M_pad;
  out->codes = b + l.codes;
  out->row_scale = reinterpret_cast<float*>(b + l.s_x);
  out->row_rscale = reinterpret_cast<float*>(b + l.rs_x);
  out->U = b + l.u;
  return SVDQ_OK;
}

svdq_status svdq_fp8r_pack_weight(const float* R_nk, const uint16_t* L1s_kr, const uint16_t* L2_rn,
                                  const float* inv_lambda, int N, int K, int r, int swiglu, void* dst,
                                  size_t dst_bytes, svdq_fp8r_weight* out, svdq_stream_t stream) {
  if (out == nullptr || R_nk == nullptr || inv_lambda == nullptr || dst == nullptr)
    return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (r > 0 && (L1s_kr == nullptr || L2_rn == nullptr)) return fail(SVDQ_ERR_INVALID_ARG, "null L1s / L2 with r > 0");
  if (!shape_ok(N, K, r)) return fail(SVDQ_ERR_UNSUPPORTED, "weight shape N=%d K=%d r=%d unsupported", N, K, r);
  if (!aligned16(R_nk) || !aligned16(inv_lambda) || (r > 0 && (!aligned16(L1s_kr) || !aligned16(L2_rn))))
    return fail(SVDQ_ERR_UNSUPPORTED, "inputs must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(dst) % kAlign) return fail(SVDQ_ERR_UNSUPPORTED, "dst not 256-byte aligned");
  const int n_tile = choose_n_tile(N, swiglu, false);
  const Fp8rWeightLayout l = fp8r_weight_layout(N, K, r);
  if (dst_bytes < l.total) return fail(SVDQ_ERR_INVALID_ARG, "FP8 weight buffer %zu bytes < %zu", dst_bytes, l.total);
  int dev, sms;
  if (svdq_status s = fp8r_ready(&dev, &sms); s != SVDQ_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* b = static_cast<uint8_t*>(dst);

  svdq_fp8r_weight w{};
  w.N = N;
  w.K = K;
  w.r = r;
  w.swiglu_interleaved = swiglu ? 1 : 0;
  w.n_tile = n_tile;
  w.codes = b + l.codes;
  w.row_scale = reinterpret_cast<float*>(b + l.scales);
  w.inv_lambda = reinterpret_cast<float*>(b + l.inv_lambda);
  w.L1s_t = b + l.l1t;
  w.L2_t = b + l.l2t;

  SVDQ_CUDA(cudaMemcpyAsync(w.inv_lambda, inv_lambda, static_cast<size_t>(K) * 4, cudaMemcpyDeviceToDevice, st));
  svdq::fp8r::pack_weight_kernel<<<grid_for(static_cast<size_t>(N) * 32, 256, sms), 256, 0, st>>>(
      R_nk, N, K, n_tile, w.swiglu_interleaved, static_cast<uint8_t*>(w.codes), w.row_scale);
  if (svdq_status s = check_launch("fp8r::pack_weight_kernel"); s != SVDQ_OK) return s;
  if (r > 0) {
    svdq::transpose_l1_kernel<<<grid_for(static_cast<size_t>(K) * r, 256, sms), 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(L1s_kr), K, r, static_cast<__nv_bfloat16*>(w.L1s_t));
    if (svdq_status s = check_launch("transpose_l1_kernel"); s != SVDQ_OK) return s;
    svdq::fp8r::pack_l2_kernel<<<grid_for(static_cast<size_t>(N) * r, 256, sms), 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(L2_rn), w.row_scale, N, r, n_tile, w.swiglu_interleaved,
        static_cast<__nv_bfloat16*>(w.L2_t));
    if (svdq_status s = check_launch("fp8r::pack_l2_kernel"); s != SVDQ_OK) return s;
  }
  static_assert(sizeof(w.tmap) >= 2 * sizeof(CUtensorMap), "tmap storage");
  CUtensorMap tmB, tmL2;
  std::memset(&tmL2, 0, sizeof(tmL2));
  // each CTA of a GEMM pair stages half of a tile's n_tile rows; one K step is 128 bytes of a row
  if (svdq_status s = make_tmap(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.codes, K, N, K, 128, n_tile / 2,
                                CU_TENSOR_MAP_SWIZZLE_128B);
      s != SVDQ_OK)
    return s;
  if (r > 0) {
    // rows 0..N-1: hi halves, rows N..2N-1: lo halves
    if (svdq_status s = make_tmap(&tmL2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w.L2_t, r, 2 * static_cast<uint64_t>(N),
                                  static_cast<uint64_t>(r) * 2, r < 32 ? r : 32, n_tile / 2, lr_swizzle(r));
        s != SVDQ_OK)
      return s;
  }
  std::memcpy(&w.tmap[0][0], &tmB, sizeof(CUtensorMap));
  std::memcpy(&w.tmap[1][0], &tmL2, sizeof(CUtensorMap));
  *out = w;
  return SVDQ_OK;
}

svdq_status svdq_fp8r_quantize_act(const uint16_t* X, const svdq_fp8r_weight* w, const svdq_fp8r_act* act,
                                   svdq_stream_t stream) {
  if (X == nullptr || w == nullptr || act == nullptr) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (act->K != w->K || act->r != w->r)
    return fail(SVDQ_ERR_INVALID_ARG, "act (K=%d r=%d) does not match weight (K=%d r=%d)", act->K, act->r, w->K, w->r);
  if (svdq_status s = check_fp8r_weight(w); s != SVDQ_OK) return s;
  if (svdq_status s = check_fp8r_act(act); s != SVDQ_OK) return s;
  if (!aligned16(X)) return fail(SVDQ_ERR_UNSUPPORTED, "X must be 16-byte aligned");
  int dev, sms;
  if (svdq_status s = fp8r_ready(&dev, &sms); s != SVDQ_OK) return s;
  const int K = act->K, r = w->r, M = act->M;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // row scales first: the quantizing pass needs each row's amax before its first code
  {
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    set_programmatic(attr[0]);
    cfg.gridDim = dim3(grid_for(static_cast<size_t>(act->M_pad) * 32, 256, sms), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e =
        cudaLaunchKernelEx(&cfg, svdq::fp8r::act_row_scale_kernel, reinterpret_cast<const __nv_bfloat16*>(X),
                           static_cast<const float*>(w->inv_lambda), M, act->M_pad, K, act->row_scale, act->row_rscale);
    if (e != cudaSuccess)
      return fail(SVDQ_ERR_CUDA, "launch of fp8r::act_row_scale_kernel failed: %s", cudaGetErrorString(e));
  }
  if (svdq_status s = check_launch("fp8r::act_row_scale_kernel"); s != SVDQ_OK) return s;
  CUtensorMap tmX, tmL1;
  std::memset(&tmL1, 0, sizeof(tmL1));
  if (svdq_status s = make_tmap(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, static_cast<uint64_t>(K) * 2, 64, 128,
                                CU_TENSOR_MAP_SWIZZLE_128B);
      s != SVDQ_OK)
    return s;
  if (r > 0) {
    if (svdq_status s = make_tmap(&tmL1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->L1s_t, K, r,
                                  static_cast<uint64_t>(K) * 2, 64, r, CU_TENSOR_MAP_SWIZZLE_128B);
        s != SVDQ_OK)
      return s;
  }
  // K split over a cluster exactly as for the NVFP4 kernel 1 (the same kernel body and resources)
  const int m_tiles = act->M_pad / 128;
  int csize = 1;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    const int* mc = g_dev[dev].k1_clusters[r == 0 ? 0 : r == 16 ? 1 : r == 32 ? 2 : 3];
    for (int c = 2; c <= 4; ++c)
      if (m_tiles <= mc[c - 1] && K % (64 * c) == 0) csize = c;
  }
  svdq::fp8r::ActArgs a;
  a.inv_lambda = w->inv_lambda;
  a.rs_x = act->row_rscale;
  a.codes = static_cast<uint8_t*>(act->codes);
  a.U = static_cast<__nv_bfloat16*>(act->U);
  a.wait_ns = g_wait_ns.load();
  a.M = M;
  a.K = K;
  a.M_pad = act->M_pad;
  a.k_per_cta = K / csize;

  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  set_programmatic(attr[1]);
  cfg.gridDim = dim3(m_tiles * csize, 1, 1);
  cfg.blockDim = dim3(svdq::kQ1Threads, 1, 1);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaSuccess;
  switch (r) {
    case 0:
      cfg.dynamicSmemBytes = svdq::Q1Layout<0>::kSmem;
      e = cudaLaunchKernelEx(&cfg, svdq::quant_act_kernel<0, svdq::fp8r::RowAct>, tmX, tmL1, a);
      break;
    case 16:
      cfg.dynamicSmemBytes = svdq::Q1Layout<16>::kSmem;
      e = cudaLaunchKernelEx(&cfg, svdq::quant_act_kernel<16, svdq::fp8r::RowAct>, tmX, tmL1, a);
      break;
    case 32:
      cfg.dynamicSmemBytes = svdq::Q1Layout<32>::kSmem;
      e = cudaLaunchKernelEx(&cfg, svdq::quant_act_kernel<32, svdq::fp8r::RowAct>, tmX, tmL1, a);
      break;
    case 64:
      cfg.dynamicSmemBytes = svdq::Q1Layout<64>::kSmem;
      e = cudaLaunchKernelEx(&cfg, svdq::quant_act_kernel<64, svdq::fp8r::RowAct>, tmX, tmL1, a);
      break;
    default: return fail(SVDQ_ERR_UNSUPPORTED, "r=%d unsupported", r);
  }
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, "launch of the row-wise FP8 quant_act_kernel failed: %s", cudaGetErrorString(e));
  return check_launch("quant_act_kernel (row-wise FP8)");
}

svdq_status svdq_fp8r_gemm(const svdq_fp8r_act* act, const svdq_fp8r_weight* w, const uint16_t* bias,
                           svdq_epilogue epi, void* Y, svdq_out_dtype out_dtype, svdq_stream_t stream) {
  if (act == nullptr || w == nullptr || Y == nullptr) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (act->K != w->K || act->r != w->r) return fail(SVDQ_ERR_INVALID_ARG, "act does not match weight");
  if (svdq_status s = check_fp8r_weight(w); s != SVDQ_OK) return s;
  if (svdq_status s = check_fp8r_act(act); s != SVDQ_OK) return s;
  if (epi < SVDQ_EPI_NONE || epi > SVDQ_EPI_BIAS_SWIGLU) return fail(SVDQ_ERR_INVALID_ARG, "bad epilogue %d", epi);
  if (out_dtype != SVDQ_OUT_BF16 && out_dtype != SVDQ_OUT_F32) return fail(SVDQ_ERR_INVALID_ARG, "bad out dtype");
  const bool has_bias = (epi & 1) != 0, swiglu = (epi & 2) != 0;
  if (has_bias && bias == nullptr) return fail(SVDQ_ERR_INVALID_ARG, "epilogue needs a bias");
  if (swiglu && !w->swiglu_interleaved) return fail(SVDQ_ERR_INVALID_ARG, "SwiGLU needs a weight packed with swiglu=1");
  if (!swiglu && w->swiglu_interleaved) return fail(SVDQ_ERR_INVALID_ARG, "weight packed for SwiGLU");
  if (!aligned16(Y) || (bias != nullptr && !aligned16(bias))) return fail(SVDQ_ERR_UNSUPPORTED, "Y / bias alignment");
  const int n_tile = w->n_tile;
  int dev, sms;
  if (svdq_status s = fp8r_ready(&dev, &sms); s != SVDQ_OK) return s;

  const int K = w->K, r = w->r;
  CUtensorMap tmA, tmU;
  std::memset(&tmU, 0, sizeof(tmU));
  if (svdq_status s = make_tmap(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, act->codes, K, act->M_pad, K, 128, 128,
                                CU_TENSOR_MAP_SWIZZLE_128B);
      s != SVDQ_OK)
    return s;
  if (r > 0) {
    if (svdq_status s = make_tmap(&tmU, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act->U, r, 2 * static_cast<uint64_t>(act->M_pad),
                                  static_cast<uint64_t>(r) * 2, r < 32 ? r : 32, 128, lr_swizzle(r));
        s != SVDQ_OK)
      return s;
  }
  CUtensorMap tmB, tmL2;  // properly aligned copies of the descriptors cached in the weight
  std::memcpy(&tmB, &w->tmap[0][0], sizeof(CUtensorMap));
  std::memcpy(&tmL2, &w->tmap[1][0], sizeof(CUtensorMap));

  svdq::fp8r::GemmArgs g{};
  g.s_x = act->row_scale;
  g.s_w = w->row_scale;
  g.bias = reinterpret_cast<const __nv_bfloat16*>(bias);
  g.Y = Y;
  g.wait_ns = g_wait_ns.load();
  g.M = act->M;
  g.M_pad = act->M_pad;
  g.N = w->N;
  g.K = K;
  g.r = r;
  g.m_tiles = act->M_pad / 128;
  g.m_pairs = (g.m_tiles + 1) / 2;
  g.n_tiles = w->N / n_tile;
  g.k_iters = K / 128;
  g.num_tiles = g.m_pairs * g.n_tiles;
  g.ldy = swiglu ? w->N / 2 : w->N;
  g.out_f32 = out_dtype == SVDQ_OUT_F32 ? 1 : 0;
  g.epi = static_cast<int>(epi);
  CUtensorMap tmY;
  if (svdq_status s = make_tmap(&tmY, g.out_f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y,
                                static_cast<uint64_t>(g.ldy), static_cast<uint64_t>(act->M),
                                static_cast<uint64_t>(g.ldy) * (g.out_f32 ? 4 : 2), 32, 32,
                                g.out_f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
      s != SVDQ_OK)
    return s;
  int max_pairs = 0;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    max_pairs = g_fp8r[dev].max_pairs[n_tile == 256 ? 0 : n_tile == 192 ? 1 : 2];
  }
  const int pairs = g.num_tiles < max_pairs ? g.num_tiles : max_pairs;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (n_tile == 256)
    e = launch_pair_gemm(svdq::pair_gemm_kernel<svdq::fp8r::Fp8Gemm, 256, kFp8Stages256>, 2 * pairs,
                         svdq::PairGemmLayout<false, 256, kFp8Stages256>::kSmem, st, tmA, tmB, tmU, tmL2, tmY, g);
  else if (n_tile == 192)
    e = launch_pair_gemm(svdq::pair_gemm_kernel<svdq::fp8r::Fp8Gemm, 192, kFp8Stages192>, 2 * pairs,
                         svdq::PairGemmLayout<false, 192, kFp8Stages192>::kSmem, st, tmA, tmB, tmU, tmL2, tmY, g);
  else
    e = launch_pair_gemm(svdq::pair_gemm_kernel<svdq::fp8r::Fp8Gemm, 128, kFp8Stages128>, 2 * pairs,
                         svdq::PairGemmLayout<false, 128, kFp8Stages128>::kSmem, st, tmA, tmB, tmU, tmL2, tmY, g);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, "launch of pair_gemm_kernel failed: %s", cudaGetErrorString(e));
  return check_launch("pair_gemm_kernel (row-wise FP8)");
}

svdq_status svdq_fp8r_export_weight(const svdq_fp8r_weight* w, uint8_t* codes, float* scales, svdq_stream_t stream) {
  if (w == nullptr || codes == nullptr || scales == nullptr) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (svdq_status s = check_fp8r_weight(w); s != SVDQ_OK) return s;
  if (!aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u))
    return fail(SVDQ_ERR_UNSUPPORTED, "codes must be 16-byte and scales 4-byte aligned");
  int dev, sms;
  if (svdq_status s = fp8r_ready(&dev, &sms); s != SVDQ_OK) return s;
  const size_t total = static_cast<size_t>(w->N) * (w->K / 16);
  svdq::fp8r::export_weight_kernel<<<grid_for(total, 256, sms), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(w->codes), w->row_scale, w->N, w->K, w->n_tile, w->swiglu_interleaved, codes,
      scales);
  return check_launch("fp8r::export_weight_kernel");
}

svdq_status svdq_fp8r_export_act(const svdq_fp8r_act* act, uint8_t* codes, float* scales, svdq_stream_t stream) {
  if (act == nullptr || codes == nullptr || scales == nullptr) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (svdq_status s = check_fp8r_act(act); s != SVDQ_OK) return s;
  int dev, sms;
  if (svdq_status s = fp8r_ready(&dev, &sms); s != SVDQ_OK) return s;
  // the activation codes are already canonical row-major; rows >= M are padding
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SVDQ_CUDA(cudaMemcpyAsync(codes, act->codes, static_cast<size_t>(act->M) * act->K, cudaMemcpyDeviceToDevice, st));
  SVDQ_CUDA(cudaMemcpyAsync(scales, act->row_scale, static_cast<size_t>(act->M) * 4, cudaMemcpyDeviceToDevice, st));
  return SVDQ_OK;
}

}  // extern "C"

// ================================================================== MLP chain: kernel 1 fused into SwiGLU
namespace {

constexpr int kFusedStages = 5;
constexpr int kMaxSplits = svdq::fused::kMaxUSplits;

struct FusedState {
  bool ready = false;
  int max_pairs[3] = {0, 0, 0};  // r_next 16, 32, 64
};
FusedState g_fused[64];

svdq_status fused_ready(int* dev_out, int* sm_out) {
  int dev = 0, sms = 0;
  if (svdq_status s = device_ready(&dev, &sms); s != SVDQ_OK) return s;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  FusedState& st = g_fused[dev];
  if (!st.ready) {
    using L16 = svdq::fused::Layout<kFusedStages, 16>;
    using L32 = svdq::fused::Layout<kFusedStages, 32>;
    using L64 = svdq::fused::Layout<kFusedStages, 64>;
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::fused::gemm_swiglu_quant_kernel<kFusedStages, 16>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, L16::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::fused::gemm_swiglu_quant_kernel<kFusedStages, 32>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, L32::kSmem));
    SVDQ_CUDA(cudaFuncSetAttribute(svdq::fused::gemm_swiglu_quant_kernel<kFusedStages, 64>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, L64::kSmem));
    if (svdq_status s = fp8r_max_pairs(
            reinterpret_cast<const void*>(svdq::fused::gemm_swiglu_quant_kernel<kFusedStages, 16>), L16::kSmem, sms,
            &st.max_pairs[0]);
        s != SVDQ_OK)
      return s;
    if (svdq_status s = fp8r_max_pairs(
            reinterpret_cast<const void*>(svdq::fused::gemm_swiglu_quant_kernel<kFusedStages, 32>), L32::kSmem, sms,
            &st.max_pairs[1]);
        s != SVDQ_OK)
      return s;
    if (svdq_status s = fp8r_max_pairs(
            reinterpret_cast<const void*>(svdq::fused::gemm_swiglu_quant_kernel<kFusedStages, 64>), L64::kSmem, sms,
            &st.max_pairs[2]);
        s != SVDQ_OK)
      return s;
    st.ready = true;
  }
  if (dev_out) *dev_out = dev;
  if (sm_out) *sm_out = sms;
  return SVDQ_OK;
}

}  // namespace

extern "C" {

size_t svdq_mlp_scratch_bytes(int M, int r_next) {
  if (M < 1 || M >= (1 << 24) || !(r_next == 16 || r_next == 32 || r_next == 64)) return 0;
  const size_t m_pad = static_cast<size_t>((M + 127) / 128 * 128);
  return static_cast<size_t>(kMaxSplits) * m_pad * static_cast<size_t>(r_next) * 4;
}

svdq_status svdq_gemm_swiglu_quant(const svdq_act* act, const svdq_weight* w, const uint16_t* bias,
                                   const svdq_weight* w_next, const float* g_x_next, const svdq_act* act_next,
                                   void* scratch, size_t scratch_bytes, uint16_t* H, svdq_stream_t stream) {
  if (act == nullptr || w == nullptr || w_next == nullptr || g_x_next == nullptr || act_next == nullptr ||
      scratch == nullptr)
    return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (act->K != w->K || act->r != w->r) return fail(SVDQ_ERR_INVALID_ARG, "act does not match weight");
  if (svdq_status s = check_weight(w); s != SVDQ_OK) return s;
  if (svdq_status s = check_act(act); s != SVDQ_OK) return s;
  if (svdq_status s = check_weight(w_next); s != SVDQ_OK) return s;
  if (svdq_status s = check_act(act_next); s != SVDQ_OK) return s;
  if (!w->swiglu_interleaved || w->n_tile != 256)
    return fail(SVDQ_ERR_UNSUPPORTED, "the fused MLP path takes a SwiGLU weight packed with 256-wide tiles");
  if (w_next->swiglu_interleaved) return fail(SVDQ_ERR_INVALID_ARG, "the next layer's weight is packed for SwiGLU");
  if (w_next->K != w->N / 2) return fail(SVDQ_ERR_INVALID_ARG, "next layer K=%d != N/2=%d", w_next->K, w->N / 2);
  if (act_next->M != act->M || act_next->K != w_next->K || act_next->r != w_next->r)
    return fail(SVDQ_ERR_INVALID_ARG, "next act (M=%d K=%d r=%d) does not match", act_next->M, act_next->K,
                act_next->r);
  const int r2 = w_next->r;
  if (r2 != 16 && r2 != 32 && r2 != 64) return fail(SVDQ_ERR_UNSUPPORTED, "next layer rank %d not in 16/32/64", r2);
  const size_t need = svdq_mlp_scratch_bytes(act->M, r2);
  if (scratch_bytes < need) return fail(SVDQ_ERR_INVALID_ARG, "scratch %zu bytes < %zu", scratch_bytes, need);
  if (!aligned16(scratch) || (bias != nullptr && !aligned16(bias)) || (H != nullptr && !aligned16(H)) ||
      (reinterpret_cast<uintptr_t>(g_x_next) & 3u))
    return fail(SVDQ_ERR_UNSUPPORTED, "scratch / bias / H / g_x_next alignment");
  int dev, sms;
  if (svdq_status s = fused_ready(&dev, &sms); s != SVDQ_OK) return s;

  const int K = w->K, r = w->r, N = w->N, K2 = w_next->K;
  CUtensorMap tmA, tmU, tmH, tmL1n;
  std::memset(&tmU, 0, sizeof(tmU));
  std::memset(&tmH, 0, sizeof(tmH));
  if (svdq_status s = make_tmap(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, act->codes, K / 2, act->M_pad, K / 2, 128, 128,
                                CU_TENSOR_MAP_SWIZZLE_128B);
      s != SVDQ_OK)
    return s;
  if (r > 0) {
    if (svdq_status s = make_tmap(&tmU, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act->U, r, 2 * static_cast<uint64_t>(act->M_pad),
                                  static_cast<uint64_t>(r) * 2, r < 32 ? r : 32, 128, lr_swizzle(r));
        s != SVDQ_OK)
      return s;
  }
  // the next layer's L1s^T [r2][K2]: per tile, 64-column boxes of this CTA's r2/2 rows
  if (svdq_status s = make_tmap(&tmL1n, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w_next->L1s_t, K2, r2,
                                static_cast<uint64_t>(K2) * 2, 64, r2 / 2, CU_TENSOR_MAP_SWIZZLE_128B);
      s != SVDQ_OK)
    return s;
  if (H != nullptr) {
    // h [M][N/2] bf16, stored from the 128B-swizzled h tile in 64 x 32 boxes
    if (svdq_status s = make_tmap(&tmH, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, H, static_cast<uint64_t>(N / 2),
                                  static_cast<uint64_t>(act->M), static_cast<uint64_t>(N / 2) * 2, 64, 32,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
        s != SVDQ_OK)
      return s;
  }
  CUtensorMap tmB, tmL2;
  std::memcpy(&tmB, &w->tmap[0][0], sizeof(CUtensorMap));
  std::memcpy(&tmL2, &w->tmap[1][0], sizeof(CUtensorMap));

  svdq::fused::Args a{};
  a.sfa = static_cast<const uint8_t*>(act->scales);
  a.sfb = static_cast<const uint8_t*>(w->scales);
  a.alpha = act->alpha;
  a.bias = reinterpret_cast<const __nv_bfloat16*>(bias);
  a.wait_ns = g_wait_ns.load();
  a.M = act->M;
  a.M_pad = act->M_pad;
  a.N = N;
  a.K = K;
  a.r = r;
  a.m_tiles = act->M_pad / 128;
  a.m_pairs = (a.m_tiles + 1) / 2;
  a.n_tiles = N / 256;
  a.k_iters = K / 256;
  a.store_h = H != nullptr ? 1 : 0;
  a.inv_lambda2 = w_next->inv_lambda;
  a.g_x2 = g_x_next;
  a.codes2 = static_cast<uint8_t*>(act_next->codes);
  a.sf2 = static_cast<uint8_t*>(act_next->scales);
  a.partials = static_cast<float*>(scratch);
  a.K2 = K2;
  int max_pairs = 0;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    max_pairs = g_fused[dev].max_pairs[r2 == 16 ? 0 : r2 == 32 ? 1 : 2];
  }
  // column splits: enough units to about fill the resident pairs, each a sweep over n_tiles/splits tiles
  int splits = max_pairs / a.m_pairs;
  if (splits < 1) splits = 1;
  if (splits > kMaxSplits) splits = kMaxSplits;
  if (splits > a.n_tiles) splits = a.n_tiles;
  a.splits = splits;
  a.num_units = a.m_pairs * splits;
  const int pairs = a.num_units < max_pairs ? a.num_units : max_pairs;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (r2) {
    case 16:
      e = launch_pair_gemm(svdq::fused::gemm_swiglu_quant_kernel<kFusedStages, 16>, 2 * pairs,
                           svdq::fused::Layout<kFusedStages, 16>::kSmem, st, tmA, tmB, tmU, tmL2, tmH, tmL1n, a);
      break;
    case 32:
      e = launch_pair_gemm(svdq::fused::gemm_swiglu_quant_kernel<kFusedStages, 32>, 2 * pairs,
                           svdq::fused::Layout<kFusedStages, 32>::kSmem, st, tmA, tmB, tmU, tmL2, tmH, tmL1n, a);
      break;
    default:
      e = launch_pair_gemm(svdq::fused::gemm_swiglu_quant_kernel<kFusedStages, 64>, 2 * pairs,
                           svdq::fused::Layout<kFusedStages, 64>::kSmem, st, tmA, tmB, tmU, tmL2, tmH, tmL1n, a);
      break;
  }
  if (e != cudaSuccess)
    return fail(SVDQ_ERR_CUDA, "launch of fused::gemm_swiglu_quant_kernel failed: %s", cudaGetErrorString(e));
  if (svdq_status s = check_launch("fused::gemm_swiglu_quant_kernel"); s != SVDQ_OK) return s;
  {
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    set_programmatic(attr[0]);
    cfg.gridDim = dim3(grid_for(static_cast<size_t>(act_next->M_pad) * r2, 256, sms), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, svdq::fused::finalize_u_kernel, static_cast<const float*>(scratch), splits, act->M,
                           act_next->M_pad, r2, g_x_next, static_cast<const float*>(w_next->g_w),
                           static_cast<__nv_bfloat16*>(act_next->U), act_next->alpha);
  }
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, "launch of fused::finalize_u_kernel failed: %s", cudaGetErrorString(e));
  return check_launch("fused::finalize_u_kernel");
}

}  // extern "C"


// ================================================================== MLP chain without caller scratch
// svdq_gemm_swiglu_quant needs a scratch buffer for the column-split partial sums of U'. Some
// callers have none to lend and cannot allocate one; this entry point serves them from a buffer
// that lives in the library's own device image: a file-scope array of fixed size that every GPU
// which loads the library holds until the process exits. In host code the array's name is only a
// host-side stand-in, so its device address is looked up once per device (cudaGetSymbolAddress,
// with that device current) and handed to the kernels like any caller's scratch pointer.
namespace {

constexpr size_t kMlpBuiltinScratchBytes = SVDQ_MLP_BUILTIN_SCRATCH_BYTES;  // 8 MiB
static __device__ __align__(256) unsigned char g_mlp_builtin_scratch[kMlpBuiltinScratchBytes];

struct BuiltinScratchState {
  bool ready = false;
  void* ptr = nullptr;
};
BuiltinScratchState g_builtin_scratch[64];

// The device address of g_mlp_builtin_scratch on the current device (looked up on first use).
svdq_status builtin_scratch_ptr(void** out) {
  int dev = 0;
  SVDQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(SVDQ_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  BuiltinScratchState& st = g_builtin_scratch[dev];
  if (!st.ready) {
    void* p = nullptr;
    SVDQ_CUDA(cudaGetSymbolAddress(&p, g_mlp_builtin_scratch));
    if (p == nullptr || (reinterpret_cast<uintptr_t>(p) & 255u) != 0)
      return fail(SVDQ_ERR_CUDA, "built-in scratch has no usable device address");
    st.ptr = p;
    st.ready = true;
  }
  *out = st.ptr;
  return SVDQ_OK;
}

}  // namespace

extern "C" {

svdq_status svdq_gemm_swiglu_quant_noscratch(const svdq_act* act, const svdq_weight* w, const uint16_t* bias,
                                             const svdq_weight* w_next, const float* g_x_next,
                                             const svdq_act* act_next, uint16_t* H, svdq_stream_t stream) {
  if (act == nullptr || w == nullptr || w_next == nullptr || g_x_next == nullptr || act_next == nullptr)
    return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  const size_t need = svdq_mlp_scratch_bytes(act->M, w_next->r);
  if (need == 0)
    return fail(SVDQ_ERR_UNSUPPORTED, "M=%d with next-layer rank %d unsupported", act->M, w_next->r);
  if (need > kMlpBuiltinScratchBytes)
    return fail(SVDQ_ERR_UNSUPPORTED,
                "M=%d at next-layer rank %d needs %zu bytes of scratch, more than the %zu-byte built-in buffer; "
                "pass a buffer to svdq_gemm_swiglu_quant instead",
                act->M, w_next->r, need, kMlpBuiltinScratchBytes);
  void* scratch = nullptr;
  if (svdq_status s = builtin_scratch_ptr(&scratch); s != SVDQ_OK) return s;
  return svdq_gemm_swiglu_quant(act, w, bias, w_next, g_x_next, act_next, scratch, kMlpBuiltinScratchBytes, H,
                                stream);
}

}  // extern "C"
