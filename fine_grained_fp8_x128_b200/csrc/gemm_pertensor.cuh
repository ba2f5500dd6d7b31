// Per-tensor FP8 baseline: one scale for each whole operand, the scheme that
// fine-grained scaling is measured against ("FP8 Mixed Precision: DeepSeek-V3
// Training Architecture", section 1, the per-tensor baseline of its error
// comparison; "Introduction to LLM Quantization", "Fine-grained
// Quantization", which contrasts it with per-group scaling).
//
//   amax  = max |x| over the tensor          (quant_pertensor_amax_kernel)
//   s     = max(fl32(amax / 448), fl32(1e-12))
//   q     = e4m3(fl32(x / s))                 (quant_pertensor_cast_kernel)
//   D     = (s_a * s_b) * sum_k q_a[m,k] q_b[n,k]   (gemm_pertensor_pair_kernel)
//
// The GEMM keeps the whole K reduction in the tensor cores' TMEM accumulator:
// with one scale per operand nothing has to be applied per K chunk, so there
// is no promotion step on the CUDA cores.  It is the fine-grained GEMM's
// CTA-pair kernel (256 x 256 tiles, cta_group::2, the same TMA loads and MMA
// descriptors) with the per-chunk promote replaced by one scaled read of the
// finished tile.  The barriers therefore split into the usual four:
//   full[s]   (leader)     TMA bytes of stage s landed            (expect_tx)
//   empty[s]  (both CTAs)  the MMAs reading stage s completed     (commit)
//   tfull[b]  (both CTAs)  TMEM buffer b holds a finished tile    (commit)
//   tempty[b] (leader)     both CTAs' epilogues read buffer b     (16 arrivals)
// Two TMEM buffers of 256 columns let the MMAs of tile i+1 run while the
// epilogue drains tile i.  Every wait is bounded, as in the other GEMMs.
#pragma once

#include "gemm_pair.cuh"

namespace fp8q {

constexpr int kPtStages = 6;
constexpr uint32_t kPtOutStageBytes = 4096;     // per epilogue warp: 32 rows x 128 bytes
struct PtSmemLayout {
  static constexpr uint32_t stages = 0;
  static constexpr uint32_t out_stage = stages + kPtStages * kPairStageBytes;
  static constexpr uint32_t bars = out_stage + kEpiWarps * kPtOutStageBytes;
  // full[S], empty[S], tfull[2], tempty[2]
  static constexpr uint32_t nbars = 2 * kPtStages + 4;
  static constexpr uint32_t misc = bars + nbars * 8;
  static constexpr uint32_t bytes = misc + 16;
};
static_assert(PtSmemLayout::bytes + 1024 <= 232448, "shared memory budget");

// ---------------------------------------------------------------------------
// Quantizer, pass 1: amax over all of x [M][ldx] (K columns).  A grid-stride
// loop over 16-byte words; per-lane 16x2 magnitude maxima, a warp and a block
// reduction, one atomicMax per block on the float's bits (non-negative floats
// order like their bit patterns).  *amax must be zero before the launch.
// ---------------------------------------------------------------------------
constexpr int kPtQThreads = 256;

__global__ void __launch_bounds__(kPtQThreads)
quant_pertensor_amax_kernel(const __nv_bfloat16* __restrict__ x, int64_t M, int64_t K, int64_t ldx,
                            unsigned int* __restrict__ amax_bits) {
  __shared__ uint32_t red[kPtQThreads / 32];
  const int64_t wpr = K / 8;                         // 16-byte words per row
  const int64_t words = M * wpr;
  uint32_t m2 = 0;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(kPtQThreads) + threadIdx.x; i < words;
       i += static_cast<int64_t>(gridDim.x) * kPtQThreads) {
    const int64_t r = i / wpr;
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(x + r * ldx) + (i - r * wpr));
    m2 = amax2(m2, v.x); m2 = amax2(m2, v.y); m2 = amax2(m2, v.z); m2 = amax2(m2, v.w);
  }
  uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < kPtQThreads / 32 ? red[threadIdx.x] : 0u;
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (threadIdx.x == 0 && m != 0) atomicMax(amax_bits, __float_as_uint(__uint_as_float(m << 16)));
  }
}

// Pass 2: s = tile_scale(amax) and the E4M3 codes.  The reciprocal form of the
// cast is exact here for the same reason as in the tile quantizers: every
// element is at most amax, and s = tile_scale(amax).  Block 0 stores s.
__global__ void __launch_bounds__(kPtQThreads)
quant_pertensor_cast_kernel(const __nv_bfloat16* __restrict__ x, int64_t M, int64_t K, int64_t ldx,
                            uint8_t* __restrict__ q, int64_t ldq, const float* __restrict__ amax,
                            float* __restrict__ scale) {
  const float s = tile_scale(*amax);
  const float nr = -__frcp_rn(s);
  if (blockIdx.x == 0 && threadIdx.x == 0) *scale = s;
  const int64_t wpr = K / 8;
  const int64_t words = M * wpr;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(kPtQThreads) + threadIdx.x; i < words;
       i += static_cast<int64_t>(gridDim.x) * kPtQThreads) {
    const int64_t r = i / wpr;
    const int64_t c = i - r * wpr;
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(x + r * ldx) + c);
    uint2 o;
    o.x = quant_words(v.x, v.y, nr, s);
    o.y = quant_words(v.z, v.w, nr, s);
    *reinterpret_cast<uint2*>(q + r * ldq + 8 * c) = o;
  }
}

// ---------------------------------------------------------------------------
// The GEMM.  A [M][K] and B [N][K] E4M3, K-major; scales: device floats
// s_a = *scales_a, s_b = *scales_b; D [M][ldd] BF16 or FP32.
// ---------------------------------------------------------------------------
template <int kOut>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_pertensor_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                           const GemmArgs p, const float* __restrict__ scale_a, const float* __restrict__ scale_b) {
  const KernelClock kclock = kernel_clock_begin();
  extern __shared__ uint8_t pt_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pt_smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PtSmemLayout::bars);
  uint64_t* full = bars;
  uint64_t* empty = bars + kPtStages;
  uint64_t* tfull = bars + 2 * kPtStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PtSmemLayout::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + PtSmemLayout::misc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nk = p.num_k_chunks;
  const uint32_t rank = cluster_ctarank();          // 0 = leader
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  const int num_m_pairs = (p.M + 2 * BM - 1) / (2 * BM);
  const int total_tiles = num_m_pairs * p.num_n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPtStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], 2 * kEpiWarps); }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
  }
  if (warp == 9) { tmem_alloc_pair(tmem_slot, 512); tmem_relinquish_pair(); }
  tc_fence_before();
  cluster_sync_all();          // both CTAs' barriers exist before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto tile_rows = [&](int t, int& a_row0, int& n0) {
    const int per_group = p.group_m * p.num_n_tiles;
    const int grp = t / per_group;
    const int first_m = grp * p.group_m;
    const int gm = min(p.group_m, num_m_pairs - first_m);
    const int within = t - grp * per_group;
    a_row0 = (first_m + within % gm) * 2 * BM + static_cast<int>(rank) * BM;
    n0 = (within / gm) * BN;
  };

  if (warp >= kEpiWarps) {
    setmaxnreg_dec40();
    if (warp == 8) {
      // ---------------- TMA producer (both CTAs, one lane) ----------------
      if (lane == 0) {
        const uint32_t leader_full0 = mapa_shared(smem_u32(&full[0]), 0);
        int it = 0;
        bool ok = true;
        for (int t = cluster; ok && t < total_tiles; t += nclusters) {
          int a_row0, n0;
          tile_rows(t, a_row0, n0);
          const int b_row0 = n0 + static_cast<int>(rank) * (BN / 2);
          for (int kc = 0; kc < nk; ++kc, ++it) {
            const int s = it % kPtStages;
            const uint32_t ph = (it / kPtStages) & 1;
            if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, WAIT_PRODUCER_EMPTY)) { ok = false; break; }
            uint8_t* st = smem + PtSmemLayout::stages + s * kPairStageBytes;
            const uint32_t leader_full = leader_full0 + static_cast<uint32_t>(s) * 8u;
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * kPairStageBytes);
            tma_load_2d_pair(st, &tmap_a, leader_full, kc * BK, a_row0);
            tma_load_2d_pair(st + kPairABytes, &tmap_b, leader_full, kc * BK, b_row0);
          }
        }
        if (!ok && rank == 0) {
          for (int j = max(0, it - kPtStages); j < it; ++j)
            mbar_wait(&full[j % kPtStages], (j / kPtStages) & 1, nullptr, WAIT_DRAIN, 1ll << 22);
        }
      }
      __syncwarp();
    } else if (warp == 9 && rank == 0) {
      // ---------------- MMA issuer (leader CTA, one lane) ----------------
      if (lane == 0) {
        const uint32_t idesc = umma_idesc_e4m3_f32(2 * BM, BN);
        bool ok = true;
        int it = 0, ti = 0;
        for (int t = cluster; ok && t < total_tiles; t += nclusters, ++ti) {
          const int b = ti & 1;
          if (!mbar_wait(&tempty[b], ((ti >> 1) & 1) ^ 1, abort_flag, WAIT_MMA_TMEM_EMPTY)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * BN);
          for (int kc = 0; kc < nk; ++kc, ++it) {
            const int s = it % kPtStages;
            if (!mbar_wait(&full[s], (it / kPtStages) & 1, abort_flag, WAIT_MMA_FULL)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + PtSmemLayout::stages + s * kPairStageBytes);
            const uint32_t b_addr = a_addr + kPairABytes;
#pragma unroll
            for (int k = 0; k < BK / 32; ++k)
              umma_f8f6f4_pair(d_tmem, umma_desc_k_sw128(a_addr + 32 * k), umma_desc_k_sw128(b_addr + 32 * k), idesc,
                               (kc > 0 || k > 0) ? 1u : 0u);
            umma_commit_pair(&empty[s], 0x3);
          }
          if (ok) umma_commit_pair(&tfull[b], 0x3);
        }
        if (!ok && it > 0) {
          const int j = it - 1;
          mbar_wait(&empty[j % kPtStages], (j / kPtStages) & 1, nullptr, WAIT_DRAIN, 1ll << 26);
        }
      }
      __syncwarp();
    }
  } else {
    // ---------------- epilogue (warps 0-7, both CTAs) ----------------
    setmaxnreg_inc232();
    const int quad = warp & 3;
    const int half = warp >> 2;
    const uint32_t t_lane = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t leader_tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const float scale = __fmul_rn(*scale_a, *scale_b);
    float2 acc[64];
    int ti = 0;
    for (int t = cluster; t < total_tiles; t += nclusters, ++ti) {
      int a_row0, n0;
      tile_rows(t, a_row0, n0);
      const int ncol0 = n0 + half * 128;
      const int b = ti & 1;
      if (!warp_wait(&tfull[b], (ti >> 1) & 1, abort_flag, WAIT_EPI_TMEM_FULL)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + t_lane + static_cast<uint32_t>(b * BN + half * 128);
      uint32_t v[64];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        tmem_ld_32x32b_x64_sync(taddr + 64 * h, v);
        const float2 sc = f2(scale);
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[32 * h + j] = fmul2(f2u(v[2 * j], v[2 * j + 1]), sc);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_tempty0 + static_cast<uint32_t>(b) * 8u);   // buffer b is free
      if (ncol0 < p.N) {
        const int row0 = a_row0 + quad * 32;
        store_rows128_staged<kOut>(acc, lane, row0, min(32, p.M - row0), ncol0, p,
                                   reinterpret_cast<uint4*>(smem + PtSmemLayout::out_stage + warp * kPtOutStageBytes));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();          // the peer's shared memory and TMEM are no longer in use
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
  kernel_clock_end(CLOCK_PERTENSOR, kclock);
}

}  // namespace fp8q
