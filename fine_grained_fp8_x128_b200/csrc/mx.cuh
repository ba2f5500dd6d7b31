// Power-of-two (UE8M0) scales on the hardware block-scaled MMA -- a throughput
// study beside the method, not the method itself.
//
// The pages define the tile scale as s = amax/448, a full FP32 value ("FP8
// Mixed Precision: DeepSeek-V3 Training Architecture", section 1, eq. s_W),
// which is why the block-scaled GEMM of gemm.cuh / gemm_pair.cuh promotes each
// 128-wide K chunk on the CUDA cores.  sm_100a's tcgen05.mma kind::mxf8f6f4
// applies per-row scales itself, inside the tensor core, but only powers of
// two (UE8M0 bytes: b stands for 2^(b - 127)), one per 32 elements of K.
// Here the method's tiles are kept (1x128 activations, 128x128 weight blocks)
// and each scale is rounded UP to the next power of two,
//   s2 = 2^ceil(log2 t),  t = max(fl32(amax / 448), fl32(1e-12)),
// so no element saturates; q = e4m3(fl32(x / s2)).  The GEMM then accumulates
// all of K in TMEM with no promotion on the CUDA cores -- the four 32-wide
// K-blocks of a 128-wide chunk carry the same scale.
//
// Scale factors live in TMEM during the MMA.  They reach it from shared
// memory with tcgen05.cp.32x128b.warpx4, which copies 32 rows of 16 bytes into
// TMEM lanes 0-31 and repeats them in the other three lane quarters.  The
// source layout (an "atom" of 128 rows x 4 K-blocks) puts the four UE8M0
// bytes of row r = r0 + 32 * r1 (K-block j in byte j) in 32-bit word
// 4 * r0 + r1 of a 512-byte block.  The quantizers below write their scales
// directly in that layout, one atom per (128-row block, 128-wide K chunk):
//   sf_mx[(kb * row_blocks + r / 128) * 128 + 4 * (r % 32) + (r % 128) / 32].
#pragma once

#include "gemm.cuh"
#include "quant.cuh"

namespace fp8q {

// Word of row r, K chunk kb in the scale-atom array (row_blocks atoms per chunk).
__host__ __device__ __forceinline__ int64_t mx_atom_word(int64_t r, int64_t kb, int64_t row_blocks) {
  return (kb * row_blocks + (r >> 7)) * 128 + 4 * (r & 31) + ((r >> 5) & 3);
}

// Smallest power of two >= t, for a positive normal t below 2^127.
__device__ __forceinline__ float pow2_ceil(float t) {
  uint32_t b = __float_as_uint(t);
  if (b & 0x7FFFFFu) b = (b & 0xFF800000u) + 0x800000u;
  return __uint_as_float(b);
}

// The UE8M0 byte of a power of two (its biased exponent), in all four bytes:
// the four 32-wide K-blocks of a 128-wide chunk share the scale.
__device__ __forceinline__ uint32_t ue8m0_word(float s2) {
  return ((__float_as_uint(s2) >> 23) & 0xFFu) * 0x01010101u;
}
constexpr uint32_t kUe8m0One = 0x7F7F7F7Fu;   // 2^0 in every byte (padding rows)

// ---------------------------------------------------------------------------
// 1x128 tiles with power-of-two scales: the tiling of quant_act_1x128_kernel
// (4 lanes per tile, a 256-thread block over 64 rows of one K chunk), the
// scale rounded up to a power of two, the scale written as a UE8M0 word of the
// atom layout.  Rows from M up to the next multiple of 128 get the word of 1.0
// so the GEMM never reads an unwritten scale.  The division by a power of two
// is exact, so the cast of x * (1/s2) equals the cast of fl32(x / s2).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kQ1Threads)
quant_act_1x128_ue8m0_kernel(const __nv_bfloat16* __restrict__ x, int64_t M, int64_t KB, int64_t ldx,
                             uint8_t* __restrict__ q, int64_t ldq, uint32_t* __restrict__ sf_mx) {
  const int tid = threadIdx.x;
  const int sub = tid & 3;
  const int tile = tid >> 2;
  const int64_t row_blocks = (M + 127) / 128;
  const int64_t items = (row_blocks * 128 / kQ1Rows) * KB;   // padding rows included
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
    Q1Slice cur;
    q1_load<false>(cur, x, M, KB, ldx, nullptr, 0, it, tile, sub);
    const int64_t rb = it / KB;
    const int64_t kb = it - rb * KB;
    const int64_t row = rb * kQ1Rows + tile;
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m2 = amax2(m2, cur.v[i].x); m2 = amax2(m2, cur.v[i].y);
      m2 = amax2(m2, cur.v[i].z); m2 = amax2(m2, cur.v[i].w);
    }
    float m = amax2_value(m2);
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    const float s = pow2_ceil(tile_scale(m));
    const float nr = -__frcp_rn(s);   // exact: s is a power of two
    if (row < M) {
      uint8_t* dst = q + row * ldq + kb * 128 + sub * 8;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint2 o;
        o.x = quant_words(cur.v[i].x, cur.v[i].y, nr, s);
        o.y = quant_words(cur.v[i].z, cur.v[i].w, nr, s);
        *reinterpret_cast<uint2*>(dst + 32 * i) = o;
      }
    }
    if (sub == 0) sf_mx[mx_atom_word(row, kb, row_blocks)] = row < M ? ue8m0_word(s) : kUe8m0One;
  }
}

// ---------------------------------------------------------------------------
// 128x128 weight blocks with power-of-two scales: the tiling of
// quant_w_128x128_kernel (one 256-thread block per weight block, an 8x8
// sub-block per thread), without the transposed copy.  Every row of the block
// carries the block's scale, so the block's atom is 128 equal words.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kQWThreads, 3)
quant_w_128x128_ue8m0_kernel(const __nv_bfloat16* __restrict__ w, int64_t NB, int64_t KB, int64_t ldw,
                             uint8_t* __restrict__ q, int64_t ldq, uint32_t* __restrict__ sf_mx) {
  __shared__ float warp_max[kQWThreads / 32];
  const int tid = threadIdx.x;
  const int a = tid >> 4;
  const int b = tid & 15;
  const int64_t items = NB * KB;
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
    const int64_t nb = it / KB;
    const int64_t kb = it - nb * KB;
    const int64_t n0 = nb * 128, k0 = kb * 128;
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      v[i] = __ldg(reinterpret_cast<const uint4*>(w + (n0 + 8 * a + i) * ldw + k0 + 8 * b));
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      m2 = amax2(m2, v[i].x); m2 = amax2(m2, v[i].y);
      m2 = amax2(m2, v[i].z); m2 = amax2(m2, v[i].w);
    }
    float m = amax2_value(m2);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((tid & 31) == 0) warp_max[tid >> 5] = m;
    __syncthreads();
    m = warp_max[0];
#pragma unroll
    for (int i = 1; i < kQWThreads / 32; ++i) m = fmaxf(m, warp_max[i]);
    const float s = pow2_ceil(tile_scale(m));
    const float nr = -__frcp_rn(s);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      *reinterpret_cast<uint2*>(q + (n0 + 8 * a + i) * ldq + k0 + 8 * b) =
          make_uint2(quant_words(v[i].x, v[i].y, nr, s), quant_words(v[i].z, v[i].w, nr, s));
    if (tid < 128) sf_mx[(kb * NB + nb) * 128 + tid] = ue8m0_word(s);
    __syncthreads();   // warp_max is reused by the next block
  }
}

// ---------------------------------------------------------------------------
// GEMM on tcgen05.mma kind::mxf8f6f4 with UE8M0 block scales:
//   D[m,n] = sum_k (qa[m,k] * 2^ea[m,k/32]) * (qb[n,k] * 2^eb[n,k/32])
// accumulated in FP32 in TMEM over all of K, BF16 out.  One persistent CTA
// per SM, 128 x 256 output tiles (cta_group::1):
//   warps 0-7: epilogue.  After a tile's last MMA, warp w reads TMEM lanes
//              32*(w%4) (its rows) and columns 128*(w/4) (its half) -- all
//              128 columns at once -- hands TMEM back, then converts to BF16
//              and stores through a 2 KB staging buffer.
//   warp 8   : producer (lane 0): TMA loads of A (128 x 128 B) and B
//              (256 x 128 B), and bulk copies of the chunk's scale atoms
//              (512 B for A's 128 rows, 1 KB for B's 256 rows) into stage s.
//   warp 9   : MMA issuer (lane 0) and TMEM owner: per chunk, three
//              tcgen05.cp of the scale atoms into the stage's TMEM columns,
//              then four MMAs of K = 32, K-block j taking byte j of the
//              scale words (scale-factor ids in the instruction descriptor),
//              one commit that frees the stage.
// TMEM: the accumulator in columns 0-255; stage s's scales in columns
// 256 + 16 s (A: 4 columns) and 264 + 16 s (B: 8 columns).  One accumulator:
// the first MMA of the next tile waits until the epilogue has read this one
// (a few hundred cycles against the tile's K/128 x 512).
// Every wait is bounded and reports through the status word, as in gemm.cuh.
// ---------------------------------------------------------------------------
constexpr int kMxStages = 4;
constexpr uint32_t kMxSfaBytes = 512;
constexpr uint32_t kMxSfbBytes = 1024;
constexpr uint32_t kMxAccCols = 256;
constexpr uint32_t kMxSfCols = 16;   // per stage: A at +0 (4 columns), B at +8 (8 columns)

struct MxSmemLayout {
  static constexpr uint32_t stages = 0;                                          // A | B per stage
  static constexpr uint32_t sf = stages + kMxStages * kStageBytes;              // SFA | SFB per stage
  static constexpr uint32_t out_stage = sf + kMxStages * (kMxSfaBytes + kMxSfbBytes);
  static constexpr uint32_t bars = out_stage + kEpiWarps * 2048;
  // full[S], empty[S], acc_full, acc_empty
  static constexpr uint32_t nbars = 2 * kMxStages + 2;
  static constexpr uint32_t misc = bars + nbars * 8;
  static constexpr uint32_t bytes = misc + 16;
};

struct MxArgs {
  const uint32_t* sfa;   // [K/128][ceil(M/128)][128] scale-atom words
  const uint32_t* sfb;   // [K/128][N/128][128]
  void* d;               // BF16 [M][ldd]
  int64_t ldd;
  int M, N, K;
  int num_m_tiles, num_n_tiles, num_k_chunks;
};

// Shared-memory descriptor of a scale atom for tcgen05.cp: no swizzle, 8-row
// core matrices of 16-byte rows, consecutive (stride 128 B); one core matrix
// along the 16-byte row, so the leading offset is unused.
__device__ __forceinline__ uint64_t mx_sf_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  return d;
}

__device__ __forceinline__ void tmem_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Instruction descriptor of kind::mxf8f6f4: E4M3 x E4M3 (formats 0), K-major
// operands, N >> 3 at bits 17-22, UE8M0 scales (bit 23), M >> 4 at bits
// 24-28, scale-factor ids of B (bits 4-5) and A (bits 29-30).
__host__ __device__ constexpr uint32_t mx_idesc(uint32_t M, uint32_t N, uint32_t sf_id) {
  return (sf_id << 4) | ((N >> 3) << 17) | (1u << 23) | ((M >> 4) << 24) | (sf_id << 29);
}

__device__ __forceinline__ void umma_mxf8f6f4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t tmem_sfa, uint32_t tmem_sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
          tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(tmem_sfa), "r"(tmem_sfb), "r"(accumulate)
      : "memory");
}

__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_mx_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
               const MxArgs p) {
  const KernelClock kclock = kernel_clock_begin();
  extern __shared__ uint8_t mx_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(mx_smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + MxSmemLayout::bars);
  uint64_t* full = bars;
  uint64_t* empty = bars + kMxStages;
  uint64_t* acc_full = bars + 2 * kMxStages;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + MxSmemLayout::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + MxSmemLayout::misc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nk = p.num_k_chunks;
  const int total_tiles = p.num_m_tiles * p.num_n_tiles;
  const int64_t m_blocks = p.num_m_tiles;   // 128-row scale atoms per K chunk of A
  const int64_t n_blocks = p.N / 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMxStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8 && lane == 0) { prefetch_tmap(&tmap_a); prefetch_tmap(&tmap_b); }
  if (warp == 9) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // tile t -> (first row, first column): 16-tile groups along M for L2 reuse
  auto tile_origin = [&](int t, int& m0, int& n0) {
    const int per_group = kGroupM * p.num_n_tiles;
    const int grp = t / per_group;
    const int first_m = grp * kGroupM;
    const int gm = min(kGroupM, p.num_m_tiles - first_m);
    const int within = t - grp * per_group;
    m0 = (first_m + within % gm) * BM;
    n0 = (within / gm) * BN;
  };

  if (warp == 8) {
    // ---------------- producer (one lane) ----------------
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
        int m0, n0;
        tile_origin(t, m0, n0);
        for (int kc = 0; kc < nk; ++kc, ++it) {
          const int s = it % kMxStages;
          if (!mbar_wait(&empty[s], ((it / kMxStages) & 1) ^ 1, abort_flag, WAIT_PRODUCER_EMPTY)) { ok = false; break; }
          uint8_t* st = smem + MxSmemLayout::stages + s * kStageBytes;
          uint8_t* sf = smem + MxSmemLayout::sf + s * (kMxSfaBytes + kMxSfbBytes);
          mbar_arrive_expect_tx(&full[s], kStageBytes + kMxSfaBytes + kMxSfbBytes);
          tma_load_2d_nohint(st, &tmap_a, &full[s], kc * BK, m0);
          tma_load_2d_nohint(st + kABytes, &tmap_b, &full[s], kc * BK, n0);
          bulk_load(sf, p.sfa + (static_cast<int64_t>(kc) * m_blocks + m0 / 128) * 128, kMxSfaBytes, &full[s]);
          bulk_load(sf + kMxSfaBytes, p.sfb + (static_cast<int64_t>(kc) * n_blocks + n0 / 128) * 128, kMxSfbBytes,
                    &full[s]);
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA exits (short waits)
        for (int j = max(0, it - kMxStages); j < it; ++j)
          mbar_wait(&full[j % kMxStages], (j / kMxStages) & 1, nullptr, WAIT_DRAIN, 1ll << 22);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------- MMA issuer (one lane) ----------------
    if (lane == 0) {
      int it = 0, tile_i = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x, ++tile_i) {
        // the epilogue has read the previous tile's accumulator
        if (!mbar_wait(acc_empty, (tile_i & 1) ^ 1, abort_flag, WAIT_MMA_TMEM_EMPTY)) { ok = false; break; }
        tc_fence_after();
        for (int kc = 0; kc < nk; ++kc, ++it) {
          const int s = it % kMxStages;
          if (!mbar_wait(&full[s], (it / kMxStages) & 1, abort_flag, WAIT_MMA_FULL)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + MxSmemLayout::stages + s * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
          const uint32_t sf_addr = smem_u32(smem + MxSmemLayout::sf + s * (kMxSfaBytes + kMxSfbBytes));
          const uint32_t t_sfa = tmem_base + kMxAccCols + kMxSfCols * static_cast<uint32_t>(s);
          const uint32_t t_sfb = t_sfa + 8;
          tmem_cp_32x128b_warpx4(t_sfa, mx_sf_desc(sf_addr));
          tmem_cp_32x128b_warpx4(t_sfb, mx_sf_desc(sf_addr + kMxSfaBytes));
          tmem_cp_32x128b_warpx4(t_sfb + 4, mx_sf_desc(sf_addr + kMxSfaBytes + 512));
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            umma_mxf8f6f4(tmem_base, umma_desc_k_sw128(a_addr + 32 * k), umma_desc_k_sw128(b_addr + 32 * k),
                          mx_idesc(BM, BN, static_cast<uint32_t>(k)), t_sfa, t_sfb, (kc > 0 || k > 0) ? 1u : 0u);
          umma_commit(&empty[s]);   // the stage (operands and scale atoms) may be refilled
        }
        if (!ok) break;
        umma_commit(acc_full);      // the tile's accumulator is complete
      }
      if (!ok && it > 0) {
        const int j = it - 1;
        mbar_wait(&empty[j % kMxStages], (j / kMxStages) & 1, nullptr, WAIT_DRAIN, 1ll << 26);
      }
    }
    __syncwarp();
  } else if (warp < kEpiWarps) {
    // ---------------- epilogue (warps 0-7) ----------------
    const int quad = warp & 3;
    const int half = warp >> 2;
    const uint32_t t_lane = static_cast<uint32_t>(quad * 32) << 16;
    uint4* stage = reinterpret_cast<uint4*>(smem + MxSmemLayout::out_stage + warp * 2048);
    GemmArgs g{};
    g.d = p.d;
    g.ldd = p.ldd;
    int tile_i = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++tile_i) {
      int m0, n0;
      tile_origin(t, m0, n0);
      if (!warp_wait(acc_full, tile_i & 1, abort_flag, WAIT_EPI_TMEM_FULL)) break;
      tc_fence_after();
      uint32_t v0[64], v1[64];
      const uint32_t taddr = tmem_base + t_lane + static_cast<uint32_t>(half * 128);
      tmem_ld_32x32b_x64_sync(taddr, v0);
      tmem_ld_32x32b_x64_sync(taddr + 64, v1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);   // the accumulator may be overwritten
      float2 acc[64];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        acc[j] = f2u(v0[2 * j], v0[2 * j + 1]);
        acc[32 + j] = f2u(v1[2 * j], v1[2 * j + 1]);
      }
      const int row0 = m0 + quad * 32;
      const int rows_valid = min(32, p.M - row0);
      const int ncol0 = n0 + half * 128;
      if (rows_valid > 0 && ncol0 < p.N)
        store_rows128_staged4<kOutBf16>(acc, lane, row0, rows_valid, ncol0, g, stage);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
  kernel_clock_end(CLOCK_MX, kclock);
}

}  // namespace fp8q
