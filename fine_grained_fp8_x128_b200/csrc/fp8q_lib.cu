// fp8q: the C ABI declared in include/fp8q.h.  Host-side argument checks,
// TMA descriptor construction and kernel launches; every kernel lives in the
// headers included below (one translation unit, so the device status word is a
// single module variable).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/fp8q.h"
#include "device_common.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "gemm_pertensor.cuh"
#include "mx.cuh"
#include "quant.cuh"

namespace {

constexpr int kMaxDevices = 64;

std::mutex g_mu;

struct DeviceInfo {
  bool ready = false;
  int sm_count = 0;
  bool gemm_attr[2][2][3] = {};   // [grouped][row mode][output mode]
  bool q2_attr = false;
  bool rq_attr = false;
  int rq_per_sm = 0;
  bool pair_attr[2][3] = {};       // [row mode][output mode]
  bool pt_attr[2] = {};            // per-tensor GEMM [output mode]
  int pt_clusters[2] = {};
  int pair_clusters[2][3] = {};    // co-resident CTA pairs per kernel instance
  int q1_per_sm = 0;               // resident blocks per SM of each quantizer
  int q1g_per_sm = 0;
  int q1s_per_sm = 0;
  int q1p_per_sm = 0;
  int q1e5_per_sm = 0;
  int q1gr_per_sm = 0;
  int q1sc_per_sm = 0;
  int q1scr_per_sm = 0;
  int q2e5_per_sm = 0;
  bool q2e5_attr = false;
  int pt_amax_per_sm = 0;
  int pt_cast_per_sm = 0;
  int q2_per_sm = 0;
  int qw_per_sm = 0;
  bool qd_attr = false;            // both-orientation quantizer
  int qd_per_sm = 0;
  bool mx_attr = false;            // UE8M0 block-scaled GEMM (study)
  int qmx_per_sm = 0;
  int qwmx_per_sm = 0;
};

// Resident blocks per SM of a kernel (cached per device); at least 1.
template <class Kern>
int blocks_per_sm(int* cache, Kern kern, int threads, size_t smem) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (*cache == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem) != cudaSuccess || n < 1) n = 1;
    *cache = n;
  }
  return *cache;
}

DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

fp8q_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8Q_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return FP8Q_ERR_CUDA;
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) return FP8Q_ERR_UNSUPPORTED;   // sm_100a code only
    d.ready = true;
  }
  *out = &d;
  return FP8Q_OK;
}

fp8q_status encoder(PFN_cuTensorMapEncodeTiled_v12000* out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return FP8Q_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  *out = g_encode;
  return FP8Q_OK;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

fp8q_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

int64_t grid_for(int64_t items, int sm_count, int per_sm) {
  int64_t g = static_cast<int64_t>(sm_count) * per_sm;
  if (items < g) g = items;
  return g < 1 ? 1 : g;
}

// K-major E4M3 operand [rows][ld] viewed as a 2D tensor {K, rows}; box
// {128 bytes, box_rows} with the 128-byte swizzle the UMMA descriptors expect.
fp8q_status make_tmap(CUtensorMap* map, const void* base, int64_t K, int64_t rows, int64_t ld, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  fp8q_status st = encoder(&enc);
  if (st != FP8Q_OK) return st;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld)};
  cuuint32_t box[2] = {128u, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8Q_OK : FP8Q_ERR_CUDA;
}

// FP32 matrix [outer][ld] viewed as a 2D tensor {inner, outer}; box
// {box_inner, box_outer}, no swizzle.  The pair GEMM loads its scale factors
// with these (ld must be a multiple of 4, the base 16-byte aligned).
fp8q_status make_tmap_f32(CUtensorMap* map, const float* base, int64_t inner, int64_t outer, int64_t ld,
                          uint32_t box_inner, uint32_t box_outer) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  fp8q_status st = encoder(&enc);
  if (st != FP8Q_OK) return st;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 4u};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8Q_OK : FP8Q_ERR_CUDA;
}

// Output matrix [rows][ld] of E4M3 codes (esz 1), BF16 (esz 2) or FP32 (esz 4)
// for the GEMMs' tile-end tensor stores: box {128 bytes, 32 rows}, 128-byte
// swizzle (the layout of the epilogues' staging buffers).
fp8q_status make_tmap_out(CUtensorMap* map, void* base, int64_t cols, int64_t rows, int64_t ld, int esz) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  fp8q_status st = encoder(&enc);
  if (st != FP8Q_OK) return st;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * esz)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esz), 32u};
  cuuint32_t estr[2] = {1u, 1u};
  const CUtensorMapDataType dt = esz == 4   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                            : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUresult r = enc(map, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8Q_OK : FP8Q_ERR_CUDA;
}

template <bool G, int MODE, int OUT>
fp8q_status launch_gemm(DeviceInfo* dev, const CUtensorMap& ta, const CUtensorMap& tb, const fp8q::GemmArgs& args,
                        int grid, cudaStream_t stream) {
  // the output's tensor map for the tile-end stores of full 32-row boxes
  CUtensorMap td;
  const int esz = OUT == fp8q::kOutF32 ? 4 : (OUT == fp8q::kOutE4m3 ? 1 : 2);
  fp8q_status st = make_tmap_out(&td, args.d, args.N, args.M, args.ldd, esz);
  if (st != FP8Q_OK) return st;
  const uint32_t smem = (G ? fp8q::GemmSmemLayout::bytes_grouped : fp8q::GemmSmemLayout::bytes_dense) + 1024;
  auto kern = fp8q::gemm_blockscaled_kernel<G, MODE, OUT>;
  bool& attr = dev->gemm_attr[G ? 1 : 0][MODE == FP8Q_SFB_ROW ? 1 : 0][OUT];
  if (!attr) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
        cudaSuccess)
      return FP8Q_ERR_CUDA;
    attr = true;
  }
  kern<<<grid, fp8q::kGemmThreads, smem, stream>>>(ta, tb, td, args);
  return launch_status();
}

template <int MODE, int OUT>
fp8q_status launch_gemm_pair(DeviceInfo* dev, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsa,
                             const CUtensorMap& tsb, const CUtensorMap& td, const fp8q::GemmArgs& args,
                             int64_t pair_tiles, cudaStream_t stream) {
  const uint32_t smem = fp8q::PairSmemLayout::bytes + 1024;
  auto kern = fp8q::gemm_pair_kernel<MODE, OUT>;
  const int mi = MODE == FP8Q_SFB_ROW ? 1 : 0, fi = OUT;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(fp8q::kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!dev->pair_attr[mi][fi]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
          cudaSuccess)
        return FP8Q_ERR_CUDA;
      cfg.gridDim = dim3(2 * (dev->sm_count / 2), 1, 1);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) n = dev->sm_count / 2;
      dev->pair_clusters[mi][fi] = n;
      dev->pair_attr[mi][fi] = true;
    }
  }
  const int64_t clusters = pair_tiles < dev->pair_clusters[mi][fi] ? pair_tiles : dev->pair_clusters[mi][fi];
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  if (cudaLaunchKernelEx(&cfg, kern, ta, tb, tsa, tsb, td, args) != cudaSuccess) return FP8Q_ERR_CUDA;
  return launch_status();
}

// The per-tensor baseline GEMM: the same cluster launch as the pair kernel.
template <int OUT>
fp8q_status launch_gemm_pertensor(DeviceInfo* dev, const CUtensorMap& ta, const CUtensorMap& tb,
                                  const fp8q::GemmArgs& args, const float* sa, const float* sb, int64_t pair_tiles,
                                  cudaStream_t stream) {
  const uint32_t smem = fp8q::PtSmemLayout::bytes + 1024;
  auto kern = fp8q::gemm_pertensor_pair_kernel<OUT>;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(fp8q::kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!dev->pt_attr[OUT]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
          cudaSuccess)
        return FP8Q_ERR_CUDA;
      cfg.gridDim = dim3(2 * (dev->sm_count / 2), 1, 1);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) n = dev->sm_count / 2;
      dev->pt_clusters[OUT] = n;
      dev->pt_attr[OUT] = true;
    }
  }
  const int64_t clusters = pair_tiles < dev->pt_clusters[OUT] ? pair_tiles : dev->pt_clusters[OUT];
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  if (cudaLaunchKernelEx(&cfg, kern, ta, tb, args, sa, sb) != cudaSuccess) return FP8Q_ERR_CUDA;
  return launch_status();
}

// Chunks of the dispatch layout's counting sort: about 256 entries each, at
// most 512 (a fixed rule, so the workspace size needs no device query).
int64_t layout_chunks(int64_t n) {
  int64_t c = (n + 255) / 256;
  return c < 1 ? 1 : (c > 512 ? 512 : c);
}

// L2 tile order of the pair kernel: tiles run through groups of group_m
// 256-row tile pairs, m fastest.  Keep whichever operand fits in about 40% of
// the 126 MB L2 resident and stream the other once: A resident -> one group
// over all of M; B resident -> groups of one tile pair (all of N sweeps past
// each 256 rows of A).  Otherwise groups of 16 tile pairs when their rows of A
// take at most 32 MiB, else 8 (2048 rows): each group streams all of B once,
// so fewer groups re-read B fewer times, as long as a wave's A rows and B
// columns still fit the L2.  On B200 (same box, alternating) 16 took Fprop
// (K = 7168, 29 MiB of A per group) from 936 to 921 us, left Wgrad (K = 8192)
// as it was, and made Dgrad (K = 18432, 72 MiB) 1 % slower; smaller groups
// sized to the L2 measured more DRAM bytes, not fewer.
int64_t pair_group_m(int64_t m_pairs, int64_t a_bytes, int64_t b_bytes, int64_t K) {
  const int64_t kResident = 48ll << 20;
  if (a_bytes <= kResident) return m_pairs < 1 ? 1 : m_pairs;
  if (b_bytes <= kResident) return 1;
  const int64_t g = 16 * 256 * K <= (32ll << 20) ? 16 : 8;
  return m_pairs < g ? m_pairs : g;
}

// Dense kernel choice set by fp8q_debug_force_dense_kernel (a test hook):
// FP8Q_DENSE_AUTO, FP8Q_DENSE_SINGLE or FP8Q_DENSE_PAIR.
std::atomic<int> g_dense_choice{FP8Q_DENSE_AUTO};

// Which dense kernel runs: the CTA-pair kernel (256 x 256 tiles) when A has
// more than one 128-row tile (the faster of the two on B200, both in short
// bursts and under the power cap), else the one-CTA kernel (128 x 256 tiles),
// which wastes no tensor-core rows on a short A.  The pair kernel TMA-loads
// the scale factors, so it also needs both scale arrays 16-byte aligned with
// leading dimensions that are multiples of 4 floats.  A forced choice applies
// where the kernel can run (the tests run both).
bool use_pair_kernel(int64_t M, const float* sfa, int64_t ld_sfa, const float* sfb, int64_t ld_sfb) {
  const bool fits = aligned(sfa, 16) && aligned(sfb, 16) && ld_sfa % 4 == 0 && ld_sfb % 4 == 0;
  const int choice = g_dense_choice.load(std::memory_order_relaxed);
  if (!fits || choice == FP8Q_DENSE_SINGLE) return false;
  if (choice == FP8Q_DENSE_PAIR) return true;
  return M > fp8q::BM;
}

// Dense GEMM launch for one scale mode: the pair or the one-CTA kernel, and
// the output mode (the FP8 output exists for 128x128-block B scales only).
template <int MODE>
fp8q_status dense_launch(DeviceInfo* dev, bool pair, int out, const CUtensorMap& ta, const CUtensorMap& tb,
                         const CUtensorMap& tsa, const CUtensorMap& tsb, const CUtensorMap& td,
                         const fp8q::GemmArgs& args, int64_t pair_tiles, int grid, cudaStream_t s) {
  if (out == fp8q::kOutF32)
    return pair ? launch_gemm_pair<MODE, fp8q::kOutF32>(dev, ta, tb, tsa, tsb, td, args, pair_tiles, s)
                : launch_gemm<false, MODE, fp8q::kOutF32>(dev, ta, tb, args, grid, s);
  if constexpr (MODE == FP8Q_SFB_BLOCK128) {
    if (out == fp8q::kOutE4m3)
      return pair ? launch_gemm_pair<MODE, fp8q::kOutE4m3>(dev, ta, tb, tsa, tsb, td, args, pair_tiles, s)
                  : launch_gemm<false, MODE, fp8q::kOutE4m3>(dev, ta, tb, args, grid, s);
  }
  return pair ? launch_gemm_pair<MODE, fp8q::kOutBf16>(dev, ta, tb, tsa, tsb, td, args, pair_tiles, s)
              : launch_gemm<false, MODE, fp8q::kOutBf16>(dev, ta, tb, args, grid, s);
}

// Body of both dense GEMM entry points.  out: fp8q::kOutBf16 / kOutF32 / kOutE4m3
// (d = E4M3 codes [M][ldd], sfd[(n/128) * ld_sfd + m] the scales of their 1x128 tiles).
fp8q_status gemm_dense(const void* a, int64_t lda, const float* sfa, int64_t ld_sfa, const void* b, int64_t ldb,
                       const float* sfb, int64_t ld_sfb, int sfb_mode, void* d, int64_t ldd, int out, float* sfd,
                       int64_t ld_sfd, int64_t M, int64_t N, int64_t K, void* stream, uint32_t idesc_fmt = 0) {
  const int64_t kIntMax = 0x7FFFFFFF;
  if (M < 1 || N < 128 || K < 128 || N % 128 != 0 || K % 128 != 0) return FP8Q_ERR_INVALID_ARG;
  if (M > kIntMax || N > kIntMax || K > kIntMax) return FP8Q_ERR_UNSUPPORTED;
  if (lda < K || ldb < K || ldd < N || ld_sfa < M) return FP8Q_ERR_INVALID_ARG;
  if (sfb_mode != FP8Q_SFB_BLOCK128 && sfb_mode != FP8Q_SFB_ROW) return FP8Q_ERR_INVALID_ARG;
  if (sfb_mode == FP8Q_SFB_BLOCK128 && ld_sfb < K / 128) return FP8Q_ERR_INVALID_ARG;
  if (sfb_mode == FP8Q_SFB_ROW && ld_sfb < N) return FP8Q_ERR_INVALID_ARG;
  if (a == nullptr || b == nullptr || sfa == nullptr || sfb == nullptr || d == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (out == fp8q::kOutE4m3) {
    if (sfb_mode != FP8Q_SFB_BLOCK128) return FP8Q_ERR_UNSUPPORTED;
    if (sfd == nullptr || ld_sfd < M) return FP8Q_ERR_INVALID_ARG;
    if (!aligned(sfd, 4)) return FP8Q_ERR_ALIGNMENT;
  }
  const int64_t esz = out == fp8q::kOutF32 ? 4 : (out == fp8q::kOutE4m3 ? 1 : 2);
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(d, 16) || !aligned(sfa, 4) || !aligned(sfb, 4) ||
      lda % 16 != 0 || ldb % 16 != 0 || (ldd * esz) % 16 != 0)
    return FP8Q_ERR_ALIGNMENT;
  if (sfb_mode == FP8Q_SFB_ROW && (!aligned(sfb, 16) || ld_sfb % 4 != 0)) return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  const bool pair = use_pair_kernel(M, sfa, ld_sfa, sfb, ld_sfb);
  CUtensorMap ta, tb, tsa, tsb, td;
  if ((st = make_tmap(&ta, a, K, M, lda, fp8q::BM)) != FP8Q_OK) return st;
  if ((st = make_tmap(&tb, b, K, N, ldb, pair ? fp8q::BN / 2 : fp8q::BN)) != FP8Q_OK) return st;
  if (pair) {
    // sa[K/128][ld_sfa]: 128 row scales per load
    if ((st = make_tmap_f32(&tsa, sfa, M, K / 128, ld_sfa, fp8q::BM, 1)) != FP8Q_OK) return st;
    // sb: [K/128][ld_sfb] per-column scales, 256 per load; or [N/128][ld_sfb]
    // block scales, 4 chunks x the tile's 2 column blocks per load
    st = sfb_mode == FP8Q_SFB_ROW ? make_tmap_f32(&tsb, sfb, N, K / 128, ld_sfb, fp8q::BN, 1)
                                  : make_tmap_f32(&tsb, sfb, K / 128, N / 128, ld_sfb, 4, 2);
    if (st != FP8Q_OK) return st;
    // the tile-end tensor stores (BF16 and FP32 outputs of the 128x128-block mode)
    if (out == fp8q::kOutE4m3 || sfb_mode == FP8Q_SFB_ROW) td = tb;
    else if ((st = make_tmap_out(&td, d, N, M, ldd, static_cast<int>(esz))) != FP8Q_OK) return st;
  } else {
    tsa = tb;   // not read by the one-CTA kernel
    tsb = tb;
    td = tb;
  }
  fp8q::GemmArgs args{};
  args.sfa = sfa;
  args.ld_sfa = ld_sfa;
  args.sfb = sfb;
  args.ld_sfb = ld_sfb;
  args.d = d;
  args.ldd = ldd;
  args.sfd = sfd;
  args.ld_sfd = ld_sfd;
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.num_n_tiles = static_cast<int>((N + fp8q::BN - 1) / fp8q::BN);
  args.num_k_chunks = static_cast<int>(K / fp8q::BK);
  args.num_m_tiles = static_cast<int>((M + fp8q::BM - 1) / fp8q::BM);
  args.group_offsets = nullptr;
  args.G = 1;
  args.idesc_fmt = idesc_fmt;
  const int64_t tiles = static_cast<int64_t>(args.num_m_tiles) * args.num_n_tiles;
  if (tiles > kIntMax) return FP8Q_ERR_UNSUPPORTED;
  const int grid = static_cast<int>(tiles < dev->sm_count ? tiles : dev->sm_count);
  const int64_t m_pairs = (M + 2 * fp8q::BM - 1) / (2 * fp8q::BM);
  const int64_t pair_tiles = m_pairs * args.num_n_tiles;
  args.group_m = static_cast<int>(pair_group_m(m_pairs, M * K, N * K, K));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return sfb_mode == FP8Q_SFB_BLOCK128
             ? dense_launch<FP8Q_SFB_BLOCK128>(dev, pair, out, ta, tb, tsa, tsb, td, args, pair_tiles, grid, s)
             : dense_launch<FP8Q_SFB_ROW>(dev, pair, out, ta, tb, tsa, tsb, td, args, pair_tiles, grid, s);
}

// Body of both grouped GEMM entry points (out: kOutBf16 or kOutE4m3).
fp8q_status gemm_grouped(const void* a, int64_t lda, const float* sfa, int64_t ld_sfa, const void* w,
                         const float* sfw, const int32_t* group_offsets, int64_t G, int64_t M_total, void* d,
                         int64_t ldd, int out, float* sfd, int64_t ld_sfd, int64_t N, int64_t K, void* stream) {
  const int64_t kIntMax = 0x7FFFFFFF;
  if (G < 1 || M_total < 0 || N < 128 || K < 128 || N % 128 != 0 || K % 128 != 0) return FP8Q_ERR_INVALID_ARG;
  if (G > fp8q::kMaxGroups || M_total > kIntMax || G * N > kIntMax || K > kIntMax) return FP8Q_ERR_UNSUPPORTED;
  if (lda < K || ldd < N || ld_sfa < M_total) return FP8Q_ERR_INVALID_ARG;
  if (out == fp8q::kOutE4m3 && ld_sfd < M_total) return FP8Q_ERR_INVALID_ARG;
  if (M_total == 0) return FP8Q_OK;
  if (a == nullptr || w == nullptr || sfa == nullptr || sfw == nullptr || group_offsets == nullptr || d == nullptr ||
      (out == fp8q::kOutE4m3 && sfd == nullptr))
    return FP8Q_ERR_INVALID_ARG;
  const int64_t esz = out == fp8q::kOutE4m3 ? 1 : 2;
  if (!aligned(a, 16) || !aligned(w, 16) || !aligned(d, 16) || !aligned(sfa, 4) || !aligned(sfw, 4) ||
      !aligned(group_offsets, 4) || lda % 16 != 0 || (ldd * esz) % 16 != 0 ||
      (out == fp8q::kOutE4m3 && !aligned(sfd, 4)))
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  CUtensorMap ta, tb;
  if ((st = make_tmap(&ta, a, K, M_total, lda, fp8q::BM)) != FP8Q_OK) return st;
  if ((st = make_tmap(&tb, w, K, G * N, K, fp8q::BN)) != FP8Q_OK) return st;
  fp8q::GemmArgs args{};
  args.sfa = sfa;
  args.ld_sfa = ld_sfa;
  args.sfb = sfw;
  args.ld_sfb = K / 128;
  args.d = d;
  args.ldd = ldd;
  args.sfd = sfd;
  args.ld_sfd = ld_sfd;
  args.M = static_cast<int>(M_total);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.num_n_tiles = static_cast<int>((N + fp8q::BN - 1) / fp8q::BN);
  args.num_k_chunks = static_cast<int>(K / fp8q::BK);
  args.num_m_tiles = 0;
  args.group_offsets = group_offsets;
  args.G = static_cast<int>(G);
  // upper bound on the device-side tile count: every expert wastes at most one partial m-tile
  const int64_t bound = ((M_total + fp8q::BM - 1) / fp8q::BM + G) * args.num_n_tiles;
  if (bound > kIntMax) return FP8Q_ERR_UNSUPPORTED;
  const int grid = static_cast<int>(bound < dev->sm_count ? bound : dev->sm_count);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return out == fp8q::kOutE4m3 ? launch_gemm<true, FP8Q_SFB_BLOCK128, fp8q::kOutE4m3>(dev, ta, tb, args, grid, s)
                               : launch_gemm<true, FP8Q_SFB_BLOCK128, fp8q::kOutBf16>(dev, ta, tb, args, grid, s);
}

}  // namespace

// Body of the 1x128 quantizer entries, for either FP8 format.
template <int kFmt>
fp8q_status quant_1x128_impl(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, int64_t ldq, float* sf,
                             int64_t ld_sf, void* stream) {
  if (M < 0 || K < 0 || K % 128 != 0 || ldx < K || ldq < K || ld_sf < M) return FP8Q_ERR_INVALID_ARG;
  if (M == 0 || K == 0) return FP8Q_OK;
  if (x == nullptr || q == nullptr || sf == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(sf, 4) || ldx % 8 != 0 || ldq % 16 != 0)
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  const int64_t KB = K / 128;
  const int64_t items = ((M + fp8q::kQ1Rows - 1) / fp8q::kQ1Rows) * KB;
  const int per_sm = blocks_per_sm(kFmt == fp8q::kFmtE4M3 ? &dev->q1_per_sm : &dev->q1e5_per_sm, fp8q::quant_act_1x128_kernel<false, kFmt>, fp8q::kQ1Threads, 0);
  const int64_t grid = grid_for(items, dev->sm_count, per_sm);
  fp8q::quant_act_1x128_kernel<false, kFmt><<<static_cast<unsigned>(grid), fp8q::kQ1Threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), M, KB, ldx, static_cast<uint8_t*>(q), ldq, sf, ld_sf, nullptr, M);
  return launch_status();
}

// Body of the 128x1 quantizer entries, for either FP8 format.
template <int kFmt>
fp8q_status quant_128x1_impl(const void* x, int64_t T, int64_t C, int64_t ldx, void* qt, int64_t ldqt, float* sf,
                             int64_t ld_sf, void* stream) {
  if (T < 0 || C < 0 || T % 128 != 0 || C % 8 != 0 || ldx < C || ldqt < T || ld_sf < C) return FP8Q_ERR_INVALID_ARG;
  if (T == 0 || C == 0) return FP8Q_OK;
  if (x == nullptr || qt == nullptr || sf == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(qt, 16) || !aligned(sf, 4) || ldx % 8 != 0 || ldqt % 16 != 0)
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    bool& attr = kFmt == fp8q::kFmtE4M3 ? dev->q2_attr : dev->q2e5_attr;
    if (!attr) {
      if (cudaFuncSetAttribute(fp8q::quant_act_128x1_kernel<kFmt>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               fp8q::kQTSmem) != cudaSuccess)
        return FP8Q_ERR_CUDA;
      attr = true;
    }
  }
  const int64_t items = (T / 128) * ((C + fp8q::kQTCols - 1) / fp8q::kQTCols);
  const int per_sm = blocks_per_sm(kFmt == fp8q::kFmtE4M3 ? &dev->q2_per_sm : &dev->q2e5_per_sm,
                                   fp8q::quant_act_128x1_kernel<kFmt>, fp8q::kQTThreads, fp8q::kQTSmem);
  const int64_t grid = grid_for(items, dev->sm_count, per_sm);
  fp8q::quant_act_128x1_kernel<kFmt><<<static_cast<unsigned>(grid), fp8q::kQTThreads, fp8q::kQTSmem,
                                 static_cast<cudaStream_t>(stream)>>>(static_cast<const __nv_bfloat16*>(x), T, C, ldx,
                                                                      static_cast<uint8_t*>(qt), ldqt, sf, ld_sf);
  return launch_status();
}

// Body of both scatter quantizer entries.
template <bool kRowScales>
fp8q_status quant_scatter_impl(const void* x, int64_t M_src, int64_t K, int64_t ldx, const int32_t* pos, int k,
                               int64_t M_out, void* q, int64_t ldq, float* sf, int64_t ld_sf, void* stream) {
  if (M_src < 0 || M_out < 0 || K < 0 || K % 128 != 0 || ldx < K || ldq < K || ld_sf < (kRowScales ? K / 128 : M_out) || k < 1 ||
      k > fp8q::kScatterMaxK)
    return FP8Q_ERR_INVALID_ARG;
  if (M_src == 0 || M_out == 0 || K == 0) return FP8Q_OK;
  if (x == nullptr || pos == nullptr || q == nullptr || sf == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(sf, 4) || !aligned(pos, 4) || ldx % 8 != 0 || ldq % 16 != 0)
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  const int64_t KB = K / 128;
  const int64_t items = ((M_src + fp8q::kQ1Rows - 1) / fp8q::kQ1Rows) * KB;
  auto kern = fp8q::quant_act_1x128_scatter_kernel<kRowScales>;
  const int per_sm = blocks_per_sm(kRowScales ? &dev->q1scr_per_sm : &dev->q1sc_per_sm, kern, fp8q::kQ1Threads, 0);
  const int64_t grid = grid_for(items, dev->sm_count, per_sm);
  kern<<<static_cast<unsigned>(grid), fp8q::kQ1Threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), M_src, KB, ldx, pos, k, M_out, static_cast<uint8_t*>(q), ldq, sf, ld_sf);
  return launch_status();
}

extern "C" {

int fp8q_version(void) { return 100; }

const char* fp8q_status_string(fp8q_status s) {
  switch (s) {
    case FP8Q_OK: return "ok";
    case FP8Q_ERR_INVALID_ARG: return "invalid argument";
    case FP8Q_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case FP8Q_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case FP8Q_ERR_CUDA: return "CUDA error";
    case FP8Q_ERR_TIMEOUT: return "device-side bounded wait gave up";
    case FP8Q_ERR_SCRATCH_LIMIT: return "request needs more scratch than the fixed no-allocation array holds";
    case FP8Q_ERR_BOUNDS: return "device-side bounds check failed (checked build)";
    default: return "unknown status";
  }
}

int fp8q_build_checks(void) {
#ifdef FP8Q_CHECKS
  return 1;
#else
  return 0;
#endif
}

fp8q_status fp8q_device_status(void* stream, int* out_code) {
  if (out_code == nullptr) return FP8Q_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int word = 0;
  const unsigned int zero = 0;
  if (cudaMemcpyFromSymbolAsync(&word, fp8q::g_status, sizeof(word), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(fp8q::g_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return FP8Q_ERR_CUDA;
  *out_code = static_cast<int>(word);
  if (word == 0) return FP8Q_OK;
  // bits 0-7 hold the FP8Q_ERR_* code of the first report
  const unsigned int code = word & 0xFFu;
  return code == FP8Q_ERR_INVALID_ARG || code == FP8Q_ERR_TIMEOUT || code == FP8Q_ERR_BOUNDS
             ? static_cast<fp8q_status>(code)
             : FP8Q_ERR_CUDA;
}

fp8q_status fp8q_quant_act_1x128(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, int64_t ldq,
                                 float* sf, int64_t ld_sf, void* stream) {
  return quant_1x128_impl<fp8q::kFmtE4M3>(x, M, K, ldx, q, ldq, sf, ld_sf, stream);
}

fp8q_status fp8q_quant_act_1x128_e5m2(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, int64_t ldq,
                                      float* sf, int64_t ld_sf, void* stream) {
  return quant_1x128_impl<fp8q::kFmtE5M2>(x, M, K, ldx, q, ldq, sf, ld_sf, stream);
}

fp8q_status fp8q_quant_act_1x128_gather(const void* x, int64_t M_src, int64_t K, int64_t ldx, const int32_t* rows,
                                        int64_t M, void* q, int64_t ldq, float* sf, int64_t ld_sf, void* stream) {
  if (M_src < 0 || M < 0 || K < 0 || K % 128 != 0 || ldx < K || ldq < K || ld_sf < M) return FP8Q_ERR_INVALID_ARG;
  if (M == 0 || K == 0) return FP8Q_OK;
  if (x == nullptr || rows == nullptr || q == nullptr || sf == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(sf, 4) || !aligned(rows, 4) || ldx % 8 != 0 || ldq % 16 != 0)
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  const int64_t KB = K / 128;
  const int64_t items = ((M + fp8q::kQ1Rows - 1) / fp8q::kQ1Rows) * KB;
  const int per_sm = blocks_per_sm(&dev->q1g_per_sm, fp8q::quant_act_1x128_kernel<true>, fp8q::kQ1Threads, 0);
  const int64_t grid = grid_for(items, dev->sm_count, per_sm);
  fp8q::quant_act_1x128_kernel<true><<<static_cast<unsigned>(grid), fp8q::kQ1Threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), M, KB, ldx, static_cast<uint8_t*>(q), ldq, sf, ld_sf, rows, M_src);
  return launch_status();
}

fp8q_status fp8q_quant_act_1x128_scatter(const void* x, int64_t M_src, int64_t K, int64_t ldx, const int32_t* pos,
                                         int k, int64_t M_out, void* q, int64_t ldq, float* sf, int64_t ld_sf,
                                         void* stream) {
  return quant_scatter_impl<false>(x, M_src, K, ldx, pos, k, M_out, q, ldq, sf, ld_sf, stream);
}

fp8q_status fp8q_quant_act_1x128_scatter_rowscales(const void* x, int64_t M_src, int64_t K, int64_t ldx,
                                                   const int32_t* pos, int k, int64_t M_out, void* q, int64_t ldq,
                                                   float* sf, int64_t ld_sf, void* stream) {
  return quant_scatter_impl<true>(x, M_src, K, ldx, pos, k, M_out, q, ldq, sf, ld_sf, stream);
}

fp8q_status fp8q_quant_act_1x128_gather_rowscales(const void* x, int64_t M_src, int64_t K, int64_t ldx,
                                                  const int32_t* rows, int64_t M, void* q, int64_t ldq, float* sf,
                                                  int64_t ld_sf, void* stream) {
  if (M_src < 0 || M < 0 || K < 0 || K % 128 != 0 || ldx < K || ldq < K || ld_sf < K / 128)
    return FP8Q_ERR_INVALID_ARG;
  if (M == 0 || K == 0) return FP8Q_OK;
  if (x == nullptr || rows == nullptr || q == nullptr || sf == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(sf, 4) || !aligned(rows, 4) || ldx % 8 != 0 || ldq % 16 != 0)
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  const int64_t KB = K / 128;
  const int64_t items = ((M + fp8q::kQ1Rows - 1) / fp8q::kQ1Rows) * KB;
  auto kern = fp8q::quant_act_1x128_kernel<true, fp8q::kFmtE4M3, true>;
  const int per_sm = blocks_per_sm(&dev->q1gr_per_sm, kern, fp8q::kQ1Threads, 0);
  const int64_t grid = grid_for(items, dev->sm_count, per_sm);
  kern<<<static_cast<unsigned>(grid), fp8q::kQ1Threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), M, KB, ldx, static_cast<uint8_t*>(q), ldq, sf, ld_sf, rows, M_src);
  return launch_status();
}

int64_t fp8q_moe_dispatch_layout_workspace(int64_t n_entries, int num_experts) {
  if (n_entries <= 0 || num_experts <= 0) return 0;
  const int64_t chunks = layout_chunks(n_entries);
  return 2 * chunks * num_experts;
}

fp8q_status fp8q_moe_dispatch_layout(const int32_t* expert_ids, int64_t n_entries, int k, int num_experts,
                                     int32_t* rows, int32_t* pos, int32_t* offsets, int32_t* workspace,
                                     int64_t workspace_len, void* stream) {
  if (n_entries < 0 || k < 1 || num_experts < 1 || num_experts > fp8q::kLayoutMaxExperts || n_entries % k != 0)
    return FP8Q_ERR_INVALID_ARG;
  if (n_entries > 0x7FFFFFFF) return FP8Q_ERR_UNSUPPORTED;
  if (offsets == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (n_entries > 0 && (expert_ids == nullptr || rows == nullptr || pos == nullptr || workspace == nullptr))
    return FP8Q_ERR_INVALID_ARG;
  if (workspace_len < fp8q_moe_dispatch_layout_workspace(n_entries, num_experts)) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(offsets, 4) || (n_entries > 0 && (!aligned(expert_ids, 4) || !aligned(rows, 4) ||
                                                 !aligned(pos, 4) || !aligned(workspace, 4))))
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n_entries == 0) {
    if (cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (num_experts + 1), s) != cudaSuccess) return FP8Q_ERR_CUDA;
    return FP8Q_OK;
  }
  const int64_t chunks = layout_chunks(n_entries);
  const int64_t chunk = (n_entries + chunks - 1) / chunks;
  int32_t* hist = workspace;
  int32_t* starts = workspace + chunks * num_experts;
  fp8q::moe_layout_hist_kernel<<<static_cast<unsigned>(chunks), 256, 0, s>>>(expert_ids, n_entries, num_experts, chunk,
                                                                            hist);
  if ((st = launch_status()) != FP8Q_OK) return st;
  fp8q::moe_layout_scan_kernel<<<1, fp8q::kLayoutMaxExperts, 0, s>>>(hist, static_cast<int>(chunks), num_experts,
                                                                    offsets, starts);
  if ((st = launch_status()) != FP8Q_OK) return st;
  fp8q::moe_layout_scatter_kernel<<<static_cast<unsigned>(chunks), 32, 0, s>>>(expert_ids, n_entries, k, num_experts,
                                                                               chunk, starts, rows, pos);
  return launch_status();
}

fp8q_status fp8q_gather_rows_fp8(const void* q_in, int64_t ldq_in, const float* sf_in, int64_t ld_sf_in, int64_t M_in,
                                 const int32_t* rows, int64_t M_out, int64_t K, void* q_out, int64_t ldq_out,
                                 float* sf_out, int64_t ld_sf_out, void* stream) {
  if (M_in < 0 || M_out < 0 || K < 0 || K % 128 != 0 || ldq_in < K || ldq_out < K || ld_sf_in < K / 128 ||
      ld_sf_out < M_out)
    return FP8Q_ERR_INVALID_ARG;
  if (M_out == 0 || K == 0) return FP8Q_OK;
  if (q_in == nullptr || sf_in == nullptr || rows == nullptr || q_out == nullptr || sf_out == nullptr)
    return FP8Q_ERR_INVALID_ARG;
  if (!aligned(q_in, 16) || !aligned(q_out, 16) || ldq_in % 16 != 0 || ldq_out % 16 != 0 || !aligned(sf_in, 4) ||
      !aligned(sf_out, 4) || !aligned(rows, 4))
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  const int64_t grid = grid_for((M_out + 7) / 8, dev->sm_count, 8);
  fp8q::gather_rows_fp8_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(q_in), ldq_in, sf_in, ld_sf_in, M_in, rows, M_out, K, static_cast<uint8_t*>(q_out),
      ldq_out, sf_out, ld_sf_out);
  return launch_status();
}

fp8q_status fp8q_moe_regroup_order(const int32_t* all_offsets, int world, int rank, int num_experts, int64_t M_recv,
                                   int32_t* rows, int32_t* expert_offsets, void* stream) {
  if (world < 1 || rank < 0 || rank >= world || num_experts < 1 || num_experts > fp8q::kLayoutMaxExperts ||
      num_experts % world != 0 || M_recv < 0)
    return FP8Q_ERR_INVALID_ARG;
  if (M_recv > 0x7FFFFFFF) return FP8Q_ERR_UNSUPPORTED;
  if (all_offsets == nullptr || expert_offsets == nullptr || (M_recv > 0 && rows == nullptr))
    return FP8Q_ERR_INVALID_ARG;
  if (!aligned(all_offsets, 4) || !aligned(expert_offsets, 4) || !aligned(rows, 4)) return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  const int64_t grid = grid_for((M_recv + fp8q::kRegroupOrderThreads - 1) / fp8q::kRegroupOrderThreads,
                                dev->sm_count, 1);
  fp8q::moe_regroup_order_kernel<<<static_cast<unsigned>(grid), fp8q::kRegroupOrderThreads, 0,
                                   static_cast<cudaStream_t>(stream)>>>(all_offsets, world, rank, num_experts, M_recv,
                                                                        rows, expert_offsets);
  return launch_status();
}

fp8q_status fp8q_quant_act_1x128_scaled(const void* x, int64_t M, int64_t K, int64_t ldx, const float* sf,
                                        int64_t ld_sf, void* q, int64_t ldq, float* amax, int64_t ld_amax,
                                        unsigned long long* clipped, void* stream) {
  if (M < 0 || K < 0 || K % 128 != 0 || ldx < K || ldq < K || ld_sf < M) return FP8Q_ERR_INVALID_ARG;
  if (amax != nullptr && ld_amax < M) return FP8Q_ERR_INVALID_ARG;
  if (M == 0 || K == 0) return FP8Q_OK;
  if (x == nullptr || sf == nullptr || q == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(sf, 4) || ldx % 8 != 0 || ldq % 16 != 0 ||
      (amax != nullptr && !aligned(amax, 4)) || (clipped != nullptr && !aligned(clipped, 8)))
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  const int64_t KB = K / 128;
  const int64_t items = ((M + fp8q::kQ1Rows - 1) / fp8q::kQ1Rows) * KB;
  const int per_sm = blocks_per_sm(&dev->q1s_per_sm, fp8q::quant_act_1x128_scaled_kernel, fp8q::kQ1Threads, 0);
  const int64_t grid = grid_for(items, dev->sm_count, per_sm);
  fp8q::quant_act_1x128_scaled_kernel<<<static_cast<unsigned>(grid), fp8q::kQ1Threads, 0,
                                        static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), M, KB, ldx, sf, ld_sf, static_cast<uint8_t*>(q), ldq, amax, ld_amax,
      clipped);
  return launch_status();
}

fp8q_status fp8q_quant_act_1x128_percentile(const void* x, int64_t M, int64_t K, int64_t ldx, int rank, void* q,
                                            int64_t ldq, float* sf, int64_t ld_sf, unsigned long long* clipped,
                                            void* stream) {
  if (M < 0 || K < 0 || K % 128 != 0 || ldx < K || ldq < K || ld_sf < M || rank < 1 || rank > 128)
    return FP8Q_ERR_INVALID_ARG;
  if (M == 0 || K == 0) return FP8Q_OK;
  if (x == nullptr || q == nullptr || sf == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(sf, 4) || ldx % 8 != 0 || ldq % 16 != 0 ||
      (clipped != nullptr && !aligned(clipped, 8)))
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  const int64_t KB = K / 128;
  const int64_t items = ((M + fp8q::kQ1Rows - 1) / fp8q::kQ1Rows) * KB;
  const int per_sm = blocks_per_sm(&dev->q1p_per_sm, fp8q::quant_act_1x128_percentile_kernel, fp8q::kQ1Threads, 0);
  const int64_t grid = grid_for(items, dev->sm_count, per_sm);
  fp8q::quant_act_1x128_percentile_kernel<<<static_cast<unsigned>(grid), fp8q::kQ1Threads, 0,
                                            static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), M, KB, ldx, rank, static_cast<uint8_t*>(q), ldq, sf, ld_sf, clipped);
  return launch_status();
}

fp8q_status fp8q_quant_pertensor(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, int64_t ldq,
                                 float* amax_scale, void* stream) {
  if (M < 0 || K < 0 || K % 8 != 0 || ldx < K || ldq < K) return FP8Q_ERR_INVALID_ARG;
  if (amax_scale == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (M > 0 && K > 0 && (x == nullptr || q == nullptr)) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(amax_scale, 4) || (M > 0 && K > 0 && (!aligned(x, 16) || !aligned(q, 8) || ldx % 8 != 0 ||
                                                      ldq % 8 != 0)))
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // amax starts at zero (an empty tensor keeps it, and s = 1e-12)
  if (cudaMemsetAsync(amax_scale, 0, sizeof(float), s) != cudaSuccess) return FP8Q_ERR_CUDA;
  const int64_t words = M * (K / 8);
  if (words > 0) {
    const int per_sm = blocks_per_sm(&dev->pt_amax_per_sm, fp8q::quant_pertensor_amax_kernel, fp8q::kPtQThreads, 0);
    const int64_t grid = grid_for((words + fp8q::kPtQThreads - 1) / fp8q::kPtQThreads, dev->sm_count, per_sm);
    fp8q::quant_pertensor_amax_kernel<<<static_cast<unsigned>(grid), fp8q::kPtQThreads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), M, K, ldx, reinterpret_cast<unsigned int*>(amax_scale));
    if ((st = launch_status()) != FP8Q_OK) return st;
  }
  const int per_sm = blocks_per_sm(&dev->pt_cast_per_sm, fp8q::quant_pertensor_cast_kernel, fp8q::kPtQThreads, 0);
  const int64_t grid = grid_for((words + fp8q::kPtQThreads - 1) / fp8q::kPtQThreads, dev->sm_count, per_sm);
  fp8q::quant_pertensor_cast_kernel<<<static_cast<unsigned>(grid), fp8q::kPtQThreads, 0, s>>>(
      static_cast<const __nv_bfloat16*>(x), M, K, ldx, static_cast<uint8_t*>(q), ldq, amax_scale, amax_scale + 1);
  return launch_status();
}

fp8q_status fp8q_gemm_pertensor(const void* a, int64_t lda, const float* scale_a, const void* b, int64_t ldb,
                                const float* scale_b, void* d, int64_t ldd, int d_dtype, int64_t M, int64_t N,
                                int64_t K, void* stream) {
  const int64_t kIntMax = 0x7FFFFFFF;
  if (M < 1 || N < 128 || K < 128 || N % 128 != 0 || K % 128 != 0) return FP8Q_ERR_INVALID_ARG;
  if (M > kIntMax || N > kIntMax || K > kIntMax) return FP8Q_ERR_UNSUPPORTED;
  if (lda < K || ldb < K || ldd < N) return FP8Q_ERR_INVALID_ARG;
  if (d_dtype != FP8Q_OUT_BF16 && d_dtype != FP8Q_OUT_F32) return FP8Q_ERR_INVALID_ARG;
  if (a == nullptr || b == nullptr || scale_a == nullptr || scale_b == nullptr || d == nullptr)
    return FP8Q_ERR_INVALID_ARG;
  const int64_t esz = d_dtype == FP8Q_OUT_F32 ? 4 : 2;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(d, 16) || !aligned(scale_a, 4) || !aligned(scale_b, 4) ||
      lda % 16 != 0 || ldb % 16 != 0 || (ldd * esz) % 16 != 0)
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  CUtensorMap ta, tb;
  if ((st = make_tmap(&ta, a, K, M, lda, fp8q::BM)) != FP8Q_OK) return st;
  if ((st = make_tmap(&tb, b, K, N, ldb, fp8q::BN / 2)) != FP8Q_OK) return st;
  fp8q::GemmArgs args{};
  args.d = d;
  args.ldd = ldd;
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.num_n_tiles = static_cast<int>((N + fp8q::BN - 1) / fp8q::BN);
  args.num_k_chunks = static_cast<int>(K / fp8q::BK);
  args.num_m_tiles = static_cast<int>((M + fp8q::BM - 1) / fp8q::BM);
  args.G = 1;
  const int64_t m_pairs = (M + 2 * fp8q::BM - 1) / (2 * fp8q::BM);
  const int64_t pair_tiles = m_pairs * args.num_n_tiles;
  if (pair_tiles > kIntMax) return FP8Q_ERR_UNSUPPORTED;
  args.group_m = static_cast<int>(pair_group_m(m_pairs, M * K, N * K, K));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d_dtype == FP8Q_OUT_F32
             ? launch_gemm_pertensor<fp8q::kOutF32>(dev, ta, tb, args, scale_a, scale_b, pair_tiles, s)
             : launch_gemm_pertensor<fp8q::kOutBf16>(dev, ta, tb, args, scale_a, scale_b, pair_tiles, s);
}

fp8q_status fp8q_scale_history_update(int policy, float alpha, const float* amax, float* hist, float* sf, int64_t n,
                                      void* stream) {
  if (policy < FP8Q_POLICY_PREVIOUS || policy > FP8Q_POLICY_DECAYED_MAX || n < 0) return FP8Q_ERR_INVALID_ARG;
  if (!(alpha >= 0.0f && alpha <= 1.0f)) return FP8Q_ERR_INVALID_ARG;
  if (n == 0) return FP8Q_OK;
  if (amax == nullptr || hist == nullptr || sf == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(amax, 4) || !aligned(hist, 4) || !aligned(sf, 4)) return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  const int64_t grid = grid_for((n + 255) / 256, dev->sm_count, 8);
  fp8q::scale_history_update_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      policy, alpha, amax, hist, sf, n);
  return launch_status();
}

fp8q_status fp8q_requant_1x128_to_128x1(const void* q, int64_t T, int64_t C, int64_t ldq, const float* sf_in,
                                        int64_t ld_sf_in, void* qt, int64_t ldqt, float* sf, int64_t ld_sf,
                                        void* stream) {
  if (T < 0 || C < 0 || T % 128 != 0 || C % 128 != 0 || ldq < C || ld_sf_in < T || ldqt < T || ld_sf < C)
    return FP8Q_ERR_INVALID_ARG;
  if (T == 0 || C == 0) return FP8Q_OK;
  if (q == nullptr || sf_in == nullptr || qt == nullptr || sf == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(sf_in, 16) || !aligned(qt, 16) || !aligned(sf, 4) || ldq % 16 != 0 ||
      ld_sf_in % 4 != 0 || ldqt % 16 != 0)
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!dev->rq_attr) {
      if (cudaFuncSetAttribute(fp8q::requant_1x128_to_128x1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               fp8q::kRQSmem) != cudaSuccess)
        return FP8Q_ERR_CUDA;
      dev->rq_attr = true;
    }
  }
  const int64_t items = (T / 128) * (C / 128);
  const int per_sm =
      blocks_per_sm(&dev->rq_per_sm, fp8q::requant_1x128_to_128x1_kernel, fp8q::kQTThreads, fp8q::kRQSmem);
  const int64_t grid = grid_for(items, dev->sm_count, per_sm);
  fp8q::requant_1x128_to_128x1_kernel<<<static_cast<unsigned>(grid), fp8q::kQTThreads, fp8q::kRQSmem,
                                        static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(q), T, C, ldq, sf_in, ld_sf_in, static_cast<uint8_t*>(qt), ldqt, sf, ld_sf);
  return launch_status();
}

fp8q_status fp8q_quant_act_dual(const void* x, int64_t T, int64_t C, int64_t ldx, void* q, int64_t ldq, float* sf,
                                int64_t ld_sf, void* qt, int64_t ldqt, float* sft, int64_t ld_sft, void* stream) {
  if (T < 0 || C < 0 || T % 128 != 0 || C % 128 != 0 || ldx < C || ldq < C || ld_sf < T || ldqt < T ||
      ld_sft < C)
    return FP8Q_ERR_INVALID_ARG;
  if (T == 0 || C == 0) return FP8Q_OK;
  if (x == nullptr || q == nullptr || sf == nullptr || qt == nullptr || sft == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(qt, 16) || !aligned(sf, 4) || !aligned(sft, 4) ||
      ldx % 8 != 0 || ldq % 16 != 0 || ldqt % 16 != 0)
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  auto kern = fp8q::quant_act_dual_kernel<fp8q::kFmtE4M3>;
  const int smem = fp8q::kQTSmem;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!dev->qd_attr) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return FP8Q_ERR_CUDA;
      dev->qd_attr = true;
    }
  }
  const int64_t items = (T / 128) * (C / 128);
  const int per_sm = blocks_per_sm(&dev->qd_per_sm, kern, fp8q::kQTThreads, smem);
  const int64_t grid = grid_for(items, dev->sm_count, per_sm);
  kern<<<static_cast<unsigned>(grid), fp8q::kQTThreads, smem, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), T, C, ldx, static_cast<uint8_t*>(q), ldq, sf, ld_sf,
      static_cast<uint8_t*>(qt), ldqt, sft, ld_sft);
  return launch_status();
}

fp8q_status fp8q_quant_act_128x1(const void* x, int64_t T, int64_t C, int64_t ldx, void* qt, int64_t ldqt,
                                 float* sf, int64_t ld_sf, void* stream) {
  return quant_128x1_impl<fp8q::kFmtE4M3>(x, T, C, ldx, qt, ldqt, sf, ld_sf, stream);
}

fp8q_status fp8q_quant_act_128x1_e5m2(const void* x, int64_t T, int64_t C, int64_t ldx, void* qt, int64_t ldqt,
                                      float* sf, int64_t ld_sf, void* stream) {
  return quant_128x1_impl<fp8q::kFmtE5M2>(x, T, C, ldx, qt, ldqt, sf, ld_sf, stream);
}

fp8q_status fp8q_quant_w_128x128(const void* w, int64_t N, int64_t K, int64_t ldw, void* q, int64_t ldq, float* sf,
                                 int64_t ld_sf, void* qt, int64_t ldqt, float* sft, int64_t ld_sft, void* stream) {
  if (N < 0 || K < 0 || N % 128 != 0 || K % 128 != 0 || ldw < K || ldq < K || ld_sf < K / 128)
    return FP8Q_ERR_INVALID_ARG;
  if (qt != nullptr && ldqt < N) return FP8Q_ERR_INVALID_ARG;
  if (sft != nullptr && ld_sft < N / 128) return FP8Q_ERR_INVALID_ARG;
  if (N == 0 || K == 0) return FP8Q_OK;
  if (w == nullptr || q == nullptr || sf == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(q, 16) || !aligned(sf, 4) || ldw % 8 != 0 || ldq % 16 != 0)
    return FP8Q_ERR_ALIGNMENT;
  if (qt != nullptr && (!aligned(qt, 16) || ldqt % 16 != 0)) return FP8Q_ERR_ALIGNMENT;
  if (sft != nullptr && !aligned(sft, 4)) return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  const int64_t NB = N / 128, KB = K / 128;
  const int per_sm = blocks_per_sm(&dev->qw_per_sm, fp8q::quant_w_128x128_kernel, fp8q::kQWThreads, 0);
  const int64_t grid = grid_for(NB * KB, dev->sm_count, per_sm);
  fp8q::quant_w_128x128_kernel<<<static_cast<unsigned>(grid), fp8q::kQWThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(w), NB, KB, ldw, static_cast<uint8_t*>(q), ldq, sf, ld_sf,
      static_cast<uint8_t*>(qt), ldqt, sft, ld_sft);
  return launch_status();
}

fp8q_status fp8q_gemm_blockscaled(const void* a, int64_t lda, const float* sfa, int64_t ld_sfa, const void* b,
                                  int64_t ldb, const float* sfb, int64_t ld_sfb, int sfb_mode, void* d, int64_t ldd,
                                  int d_dtype, int64_t M, int64_t N, int64_t K, void* stream) {
  if (d_dtype != FP8Q_OUT_BF16 && d_dtype != FP8Q_OUT_F32) return FP8Q_ERR_INVALID_ARG;
  return gemm_dense(a, lda, sfa, ld_sfa, b, ldb, sfb, ld_sfb, sfb_mode, d, ldd,
                    d_dtype == FP8Q_OUT_F32 ? fp8q::kOutF32 : fp8q::kOutBf16, nullptr, 0, M, N, K, stream);
}

fp8q_status fp8q_gemm_blockscaled_fmt(const void* a, int a_fmt, int64_t lda, const float* sfa, int64_t ld_sfa,
                                      const void* b, int b_fmt, int64_t ldb, const float* sfb, int64_t ld_sfb,
                                      int sfb_mode, void* d, int64_t ldd, int d_dtype, int64_t M, int64_t N, int64_t K,
                                      void* stream) {
  if (d_dtype != FP8Q_OUT_BF16 && d_dtype != FP8Q_OUT_F32) return FP8Q_ERR_INVALID_ARG;
  if ((a_fmt != FP8Q_FMT_E4M3 && a_fmt != FP8Q_FMT_E5M2) || (b_fmt != FP8Q_FMT_E4M3 && b_fmt != FP8Q_FMT_E5M2))
    return FP8Q_ERR_INVALID_ARG;
  return gemm_dense(a, lda, sfa, ld_sfa, b, ldb, sfb, ld_sfb, sfb_mode, d, ldd,
                    d_dtype == FP8Q_OUT_F32 ? fp8q::kOutF32 : fp8q::kOutBf16, nullptr, 0, M, N, K, stream,
                    fp8q::umma_idesc_formats(static_cast<uint32_t>(a_fmt), static_cast<uint32_t>(b_fmt)));
}

fp8q_status fp8q_gemm_blockscaled_q1x128(const void* a, int64_t lda, const float* sfa, int64_t ld_sfa, const void* b,
                                         int64_t ldb, const float* sfb, int64_t ld_sfb, void* dq, int64_t lddq,
                                         float* sfd, int64_t ld_sfd, int64_t M, int64_t N, int64_t K, void* stream) {
  return gemm_dense(a, lda, sfa, ld_sfa, b, ldb, sfb, ld_sfb, FP8Q_SFB_BLOCK128, dq, lddq, fp8q::kOutE4m3, sfd,
                    ld_sfd, M, N, K, stream);
}

fp8q_status fp8q_grouped_gemm_blockscaled(const void* a, int64_t lda, const float* sfa, int64_t ld_sfa, const void* w,
                                          const float* sfw, const int32_t* group_offsets, int64_t G, int64_t M_total,
                                          void* d, int64_t ldd, int64_t N, int64_t K, void* stream) {
  return gemm_grouped(a, lda, sfa, ld_sfa, w, sfw, group_offsets, G, M_total, d, ldd, fp8q::kOutBf16, nullptr, 0, N, K,
                      stream);
}

fp8q_status fp8q_grouped_gemm_blockscaled_q1x128(const void* a, int64_t lda, const float* sfa, int64_t ld_sfa,
                                                 const void* w, const float* sfw, const int32_t* group_offsets,
                                                 int64_t G, int64_t M_total, void* dq, int64_t lddq, float* sfd,
                                                 int64_t ld_sfd, int64_t N, int64_t K, void* stream) {
  return gemm_grouped(a, lda, sfa, ld_sfa, w, sfw, group_offsets, G, M_total, dq, lddq, fp8q::kOutE4m3, sfd, ld_sfd, N,
                      K, stream);
}

fp8q_status fp8q_debug_cast_e4m3_bits(uint32_t start, int64_t count, void* out, void* stream) {
  if (count < 0 || count > (int64_t(1) << 32)) return FP8Q_ERR_INVALID_ARG;
  if (count == 0) return FP8Q_OK;
  if (out == nullptr) return FP8Q_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  const int64_t pairs = (count + 1) / 2;
  const int64_t grid = grid_for((pairs + 255) / 256, dev->sm_count, 16);
  fp8q::cast_e4m3_bits_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      start, count, static_cast<uint8_t*>(out));
  return launch_status();
}

fp8q_status fp8q_kernel_clock_counters(unsigned long long* out, int reset) {
  if (out == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return FP8Q_ERR_CUDA;
  if (cudaMemcpyFromSymbol(out, fp8q::g_kernel_clock, sizeof(unsigned long long) * 12) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  if (reset) {
    const unsigned long long zero[12] = {};
    if (cudaMemcpyToSymbol(fp8q::g_kernel_clock, zero, sizeof(zero)) != cudaSuccess) return FP8Q_ERR_CUDA;
  }
  return FP8Q_OK;
}

fp8q_status fp8q_debug_force_dense_kernel(int choice) {
  if (choice != FP8Q_DENSE_AUTO && choice != FP8Q_DENSE_SINGLE && choice != FP8Q_DENSE_PAIR)
    return FP8Q_ERR_INVALID_ARG;
  g_dense_choice.store(choice, std::memory_order_relaxed);
  return FP8Q_OK;
}

fp8q_status fp8q_debug_wait_timeout(int64_t budget_cycles, void* stream) {
  if (budget_cycles < 1 || budget_cycles > (int64_t(1) << 34)) return FP8Q_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  fp8q::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<long long>(budget_cycles));
  return launch_status();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// fp8q_moe_dispatch_layout_noalloc: the dispatch layout with its scratch in a
// fixed array of this library's device module instead of a caller workspace.
// For callers that cannot allocate device memory at the time they call (see
// the declaration in fp8q.h).  The array is FP8Q_LAYOUT_NOALLOC_SCRATCH_INTS
// int32 (1 MiB) and every device that loads the library holds it until the
// process exits.
// ---------------------------------------------------------------------------
static __device__ __align__(256) int32_t g_layout_scratch[FP8Q_LAYOUT_NOALLOC_SCRATCH_INTS];

namespace {

int32_t* g_layout_scratch_ptr[kMaxDevices] = {};

// Device address of g_layout_scratch on the current device.  In host code the
// array's name stands for a host-side shadow, not device memory, so the
// address is looked up once per device (with that device current) and kept.
fp8q_status layout_scratch_address(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8Q_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_layout_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess || p == nullptr) return FP8Q_ERR_CUDA;
    g_layout_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_layout_scratch_ptr[dev];
  return FP8Q_OK;
}

}  // namespace

extern "C" fp8q_status fp8q_moe_dispatch_layout_noalloc(const int32_t* expert_ids, int64_t n_entries, int k,
                                                        int num_experts, int32_t* rows, int32_t* pos,
                                                        int32_t* offsets, void* stream) {
  if (n_entries < 0 || k < 1 || num_experts < 1 || num_experts > fp8q::kLayoutMaxExperts || n_entries % k != 0)
    return FP8Q_ERR_INVALID_ARG;
  if (n_entries > 0x7FFFFFFF) return FP8Q_ERR_UNSUPPORTED;
  // the scratch this request needs must fit the fixed array
  if (fp8q_moe_dispatch_layout_workspace(n_entries, num_experts) > FP8Q_LAYOUT_NOALLOC_SCRATCH_INTS)
    return FP8Q_ERR_SCRATCH_LIMIT;
  if (offsets == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (n_entries > 0 && (expert_ids == nullptr || rows == nullptr || pos == nullptr)) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(offsets, 4) ||
      (n_entries > 0 && (!aligned(expert_ids, 4) || !aligned(rows, 4) || !aligned(pos, 4))))
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  int32_t* scratch = nullptr;
  if ((st = layout_scratch_address(&scratch)) != FP8Q_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n_entries == 0) {
    // offsets are all zero; no kernel runs and the scratch is not touched
    if (cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (num_experts + 1), s) != cudaSuccess) return FP8Q_ERR_CUDA;
    return FP8Q_OK;
  }
  // Every scratch word the kernels read is written earlier in the same call
  // (per-chunk histograms, then per-chunk starts), so nothing needs clearing.
  const int64_t chunks = layout_chunks(n_entries);
  const int64_t chunk = (n_entries + chunks - 1) / chunks;
  int32_t* hist = scratch;
  int32_t* starts = scratch + chunks * num_experts;
  fp8q::moe_layout_hist_kernel<<<static_cast<unsigned>(chunks), 256, 0, s>>>(expert_ids, n_entries, num_experts, chunk,
                                                                            hist);
  if ((st = launch_status()) != FP8Q_OK) return st;
  fp8q::moe_layout_scan_kernel<<<1, fp8q::kLayoutMaxExperts, 0, s>>>(hist, static_cast<int>(chunks), num_experts,
                                                                    offsets, starts);
  if ((st = launch_status()) != FP8Q_OK) return st;
  fp8q::moe_layout_scatter_kernel<<<static_cast<unsigned>(chunks), 32, 0, s>>>(expert_ids, n_entries, k, num_experts,
                                                                               chunk, starts, rows, pos);
  return launch_status();
}

// ---------------------------------------------------------------------------
// Power-of-two (UE8M0) scales on the hardware block-scaled MMA: the
// throughput study beside the method (mx.cuh).
// ---------------------------------------------------------------------------
extern "C" fp8q_status fp8q_quant_act_1x128_ue8m0(const void* x, int64_t M, int64_t K, int64_t ldx, void* q,
                                                  int64_t ldq, uint32_t* sf_mx, void* stream) {
  if (M < 0 || K < 0 || K % 128 != 0 || ldx < K || ldq < K) return FP8Q_ERR_INVALID_ARG;
  if (M == 0 || K == 0) return FP8Q_OK;
  if (x == nullptr || q == nullptr || sf_mx == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (M > 0x7FFFFFFF) return FP8Q_ERR_UNSUPPORTED;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(sf_mx, 16) || ldx % 8 != 0 || ldq % 16 != 0)
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  const int64_t KB = K / 128;
  const int64_t items = ((M + 127) / 128) * (128 / fp8q::kQ1Rows) * KB;
  const int per_sm = blocks_per_sm(&dev->qmx_per_sm, fp8q::quant_act_1x128_ue8m0_kernel, fp8q::kQ1Threads, 0);
  const int64_t grid = grid_for(items, dev->sm_count, per_sm);
  fp8q::quant_act_1x128_ue8m0_kernel<<<static_cast<unsigned>(grid), fp8q::kQ1Threads, 0,
                                       static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), M, KB, ldx, static_cast<uint8_t*>(q), ldq, sf_mx);
  return launch_status();
}

extern "C" fp8q_status fp8q_quant_w_128x128_ue8m0(const void* w, int64_t N, int64_t K, int64_t ldw, void* q,
                                                  int64_t ldq, uint32_t* sf_mx, void* stream) {
  if (N < 0 || K < 0 || N % 128 != 0 || K % 128 != 0 || ldw < K || ldq < K) return FP8Q_ERR_INVALID_ARG;
  if (N == 0 || K == 0) return FP8Q_OK;
  if (w == nullptr || q == nullptr || sf_mx == nullptr) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(q, 16) || !aligned(sf_mx, 16) || ldw % 8 != 0 || ldq % 16 != 0)
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  const int64_t NB = N / 128, KB = K / 128;
  const int per_sm = blocks_per_sm(&dev->qwmx_per_sm, fp8q::quant_w_128x128_ue8m0_kernel, fp8q::kQWThreads, 0);
  const int64_t grid = grid_for(NB * KB, dev->sm_count, per_sm);
  fp8q::quant_w_128x128_ue8m0_kernel<<<static_cast<unsigned>(grid), fp8q::kQWThreads, 0,
                                       static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(w), NB, KB, ldw, static_cast<uint8_t*>(q), ldq, sf_mx);
  return launch_status();
}

extern "C" fp8q_status fp8q_gemm_mxf8_ue8m0(const void* a, int64_t lda, const uint32_t* sfa_mx, const void* b,
                                            int64_t ldb, const uint32_t* sfb_mx, void* d, int64_t ldd, int64_t M,
                                            int64_t N, int64_t K, void* stream) {
  const int64_t kIntMax = 0x7FFFFFFF;
  if (M < 1 || N < 256 || K < 128 || K % 128 != 0) return FP8Q_ERR_INVALID_ARG;
  if (N % 256 != 0) return FP8Q_ERR_UNSUPPORTED;   // whole 256-column tiles only (the study's shapes)
  if (M > kIntMax || N > kIntMax || K > kIntMax) return FP8Q_ERR_UNSUPPORTED;
  if (lda < K || ldb < K || ldd < N) return FP8Q_ERR_INVALID_ARG;
  if (a == nullptr || b == nullptr || sfa_mx == nullptr || sfb_mx == nullptr || d == nullptr)
    return FP8Q_ERR_INVALID_ARG;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(d, 16) || !aligned(sfa_mx, 16) || !aligned(sfb_mx, 16) ||
      lda % 16 != 0 || ldb % 16 != 0 || (ldd * 2) % 16 != 0)
    return FP8Q_ERR_ALIGNMENT;
  DeviceInfo* dev = nullptr;
  fp8q_status st = device_info(&dev);
  if (st != FP8Q_OK) return st;
  CUtensorMap ta, tb;
  if ((st = make_tmap(&ta, a, K, M, lda, fp8q::BM)) != FP8Q_OK) return st;
  if ((st = make_tmap(&tb, b, K, N, ldb, fp8q::BN)) != FP8Q_OK) return st;
  fp8q::MxArgs args{};
  args.sfa = sfa_mx;
  args.sfb = sfb_mx;
  args.d = d;
  args.ldd = ldd;
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.num_m_tiles = static_cast<int>((M + fp8q::BM - 1) / fp8q::BM);
  args.num_n_tiles = static_cast<int>(N / fp8q::BN);
  args.num_k_chunks = static_cast<int>(K / fp8q::BK);
  const int64_t tiles = static_cast<int64_t>(args.num_m_tiles) * args.num_n_tiles;
  if (tiles > kIntMax) return FP8Q_ERR_UNSUPPORTED;
  const uint32_t smem = fp8q::MxSmemLayout::bytes + 1024;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!dev->mx_attr) {
      if (cudaFuncSetAttribute(fp8q::gemm_mx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem)) != cudaSuccess)
        return FP8Q_ERR_CUDA;
      dev->mx_attr = true;
    }
  }
  const int grid = static_cast<int>(tiles < dev->sm_count ? tiles : dev->sm_count);
  fp8q::gemm_mx_kernel<<<grid, fp8q::kGemmThreads, smem, static_cast<cudaStream_t>(stream)>>>(ta, tb, args);
  return launch_status();
}
