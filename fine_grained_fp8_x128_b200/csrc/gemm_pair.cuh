// Dense block-scaled FP8 GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same arithmetic as gemm.cuh -- D[m,n] = sum_kb sa[m,kb] * sb(n,kb) * P_kb[m,n]
// with a TMEM accumulator per 128-wide K chunk and FP32 promotion on the CUDA
// cores ("FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section 3;
// "Introduction to LLM Quantization", "Fine-grained Quantization" Steps 1-4) --
// but a cluster of two CTAs on two SMs computes one 256 x 256 output tile:
//   * each CTA loads its own 128 rows of A and its own 128-row half of B
//     (32 KB per K chunk instead of the 48 KB a lone 128 x 256 CTA needs) with
//     cta_group::2 TMA loads whose completion is counted on the leader CTA's
//     barrier -- no multicast loads;
//   * the leader CTA issues tcgen05.mma.cta_group::2 (M = 256, N = 256), which
//     reads both CTAs' shared memory and writes each CTA's 128 x 256 FP32 chunk
//     result into that CTA's TMEM;
//   * each CTA promotes and stores its own 128 rows, exactly as the single-CTA
//     kernel does, and hands TMEM buffers back to the leader's MMA warp with a
//     remote arrive on the leader's go[] barrier.
// Warp roles, TMEM double buffering, the go/done barrier pair per stage (one
// wait and one commit per chunk in the MMA warp) and the bounded waits are
// those of gemm.cuh.  Here go[s] lives on the leader and counts the leader's
// expect_tx, both CTAs' TMA bytes and 16 epilogue warps; done[s] is signalled
// in both CTAs by one multicast commit.
// The scale factors travel with the operands: each CTA TMA-loads chunk c's
// row scales of its 128 rows and the B scales of the tile (the two 128x128
// block scales, or the 256 per-column scales in FP8Q_SFB_ROW) into slot
// c % kPairScaleSlots of a ring, counted on go[], so the epilogue reads them
// from shared memory after done(c) with no load latency and no barrier of
// their own.  The slot is refilled (chunk c + kPairScaleSlots) after done(c +
// kPairScaleSlots - S), which needs every epilogue warp's release of chunk
// c + kPairScaleSlots - S - 2 >= c + 1, issued after the warp's last read of
// slot c; a proxy fence before each release orders those reads before the
// refill.
// At the end of a tile each epilogue warp writes its 32 rows x 128 columns
// through two 4 KB shared buffers with TMA tensor stores (store_rows128_tma), so
// the global writes complete in the background while the warp returns to the
// next tile's chunks.  The FP8 output keeps the staged 16-byte stores of
// stage_store_pass (with its scales), and the FP8Q_SFB_ROW mode's 16x256b
// fragments are stored directly.
#pragma once

#include "gemm.cuh"

namespace fp8q {

#ifndef FP8Q_PAIR_STAGES
#define FP8Q_PAIR_STAGES 4
#endif
constexpr int kPairStages = FP8Q_PAIR_STAGES;
constexpr uint32_t kPairABytes = 128 * BK;                    // 16 KB
constexpr uint32_t kPairBBytes = 128 * BK;                    // 16 KB (half of the 256-row B tile)
constexpr uint32_t kPairStageBytes = kPairABytes + kPairBBytes;
constexpr int kPairScaleSlots = 8;                            // scale ring (>= S + 3)
static_assert(kPairScaleSlots >= kPairStages + 3, "a scale slot may be refilled while still being read");
// One slot: B scales at 0 (256 per-column floats, or a 4 x 2 box of block
// scales: chunks (c & ~3)..+3 of the tile's two 128-column blocks), the 128
// row scales of this CTA at 1024.
constexpr uint32_t kPairSlotBytes = 2048;
constexpr uint32_t kPairSlotSa = 1024;
constexpr uint32_t kPairSaBytes = 128 * 4;
template <int kSfbMode>
__host__ __device__ constexpr uint32_t pair_sb_bytes() { return kSfbMode == FP8Q_SFB_ROW ? BN * 4 : 4 * 2 * 4; }

constexpr uint32_t kPairOutStageBytes = 8192;                 // per epilogue warp: two buffers of 32 rows x 128 bytes
struct PairSmemLayout {
  static constexpr uint32_t stages = 0;
  static constexpr uint32_t scales = stages + kPairStages * kPairStageBytes;
  static constexpr uint32_t out_stage = scales + kPairScaleSlots * kPairSlotBytes;
  static constexpr uint32_t bars = out_stage + kEpiWarps * kPairOutStageBytes;
  // go[S], done[S]
  static constexpr uint32_t nbars = 2 * kPairStages;
  static constexpr uint32_t misc = bars + nbars * 8;
  static constexpr uint32_t bytes = misc + 16;
};

// Per-column scales (FP8Q_SFB_ROW) on 16x256b fragments (tmem_ld_16x256b_x8x2_sync):
// the thread holds 4 rows x 16 columns; acc[32g + 4k + 2i + j] += v[...] *
// (sa[2g + i] * sb[8k + 2c + j]) with c = lane % 4.  Each column-scale pair is
// one 8-byte shared load (shared by 8 lanes) used for all 4 rows, where a
// 32x32b row fragment would need all 128 column scales in every thread.
// The scales are read from shared memory by the caller before the TMEM load
// (load_rows16_scales), so their latency hides behind it.
struct Rows16Scales {
  float sa[4];     // rows l4, l4 + 8, l4 + 16, l4 + 24
  float2 sb[8];    // column pairs 8k + 2c, +1
};
__device__ __forceinline__ void load_rows16_scales(Rows16Scales& sc, const float* sa_rows, const float* sb_cols,
                                                   bool with_sa) {
  if (with_sa) {
#pragma unroll
    for (int q = 0; q < 4; ++q) sc.sa[q] = sa_rows[8 * ((q & 1) + 2 * (q >> 1))];
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) sc.sb[k] = *reinterpret_cast<const float2*>(sb_cols + 8 * k);
}
__device__ __forceinline__ void promote_rows16(float2* acc, const uint32_t (&v)[64], const Rows16Scales& sc) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float2 sb = sc.sb[k];
#pragma unroll
    for (int q = 0; q < 4; ++q) {   // q = 2g + i
      const int x = 32 * (q >> 1) + 4 * k + 2 * (q & 1);
      const float2 c = fmul2(make_float2(sb.x, sb.y), f2(sc.sa[q]));
      acc[x / 2] = ffma2(f2u(v[x], v[x + 1]), c, acc[x / 2]);
    }
  }
}

// ---------------------------------------------------------------------------
// Tile-end stores through TMA.  A warp's 32 rows x 128 columns leave in passes
// of 32 rows x 128 bytes: the warp writes each pass into one of its two 4 KB
// shared buffers in the TMA's 128-byte-swizzled layout (16-byte chunk j of row
// r at chunk j ^ (r % 8)) and one lane issues a tensor store of the box.  The
// passes go out back to back; the warp waits for the TMA to have read the
// buffers only when it next refills them (the FP32 output's third pass, or the
// next tile's stores), so the global writes complete in the background while
// the warp returns to the next tile's chunks.  Rows past M are clipped by the
// tensor map.
// ---------------------------------------------------------------------------
// 32x32b fragments (thread = row `lane`, acc[j] = columns 2j, 2j+1 of the
// warp's 128): BF16 in 2 passes of 64 columns, FP32 in 4 passes of 32.
template <int kOut>
__device__ __forceinline__ void store_rows128_tma(const float2* acc, int lane, int row0, int ncol0,
                                                  const CUtensorMap* tmap_d, uint8_t* buf) {
  auto issue = [&](uint8_t* b, int x) {
    fence_proxy_async_shared();
    __syncwarp();
    if (lane == 0) tma_store_2d(tmap_d, b, x, row0);
  };
  if (lane == 0) bulk_wait_group_read0();   // the previous tile's stores have read both buffers
  __syncwarp();
  if (kOut == kOutF32) {
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      if (h == 2) {
        if (lane == 0) { bulk_commit_group(); bulk_wait_group_read0(); }
        __syncwarp();
      }
      uint4* stage = reinterpret_cast<uint4*>(buf + 4096 * (h & 1));
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float2 a = acc[16 * h + 2 * j], b = acc[16 * h + 2 * j + 1];
        stage[lane * 8 + (j ^ (lane & 7))] =
            make_uint4(__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(b.x), __float_as_uint(b.y));
      }
      issue(buf + 4096 * (h & 1), ncol0 + 32 * h);
    }
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint4* stage = reinterpret_cast<uint4*>(buf + 4096 * h);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 v = __float22bfloat162_rn(acc[32 * h + 4 * j + e]);
          w[e] = *reinterpret_cast<const uint32_t*>(&v);
        }
        stage[lane * 8 + (j ^ (lane & 7))] = make_uint4(w[0], w[1], w[2], w[3]);
      }
      issue(buf + 4096 * h, ncol0 + 64 * h);
    }
  }
  if (lane == 0) bulk_commit_group();
  __syncwarp();
}

template <int kSfbMode, int kOut>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                 const __grid_constant__ CUtensorMap tmap_sa, const __grid_constant__ CUtensorMap tmap_sb,
                 const __grid_constant__ CUtensorMap tmap_d, const GemmArgs p) {
  const KernelClock kclock = kernel_clock_begin();
  extern __shared__ uint8_t pair_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pair_smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PairSmemLayout::bars);
  uint64_t* go = bars;
  uint64_t* done = bars + kPairStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PairSmemLayout::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + PairSmemLayout::misc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nk = p.num_k_chunks;
  const uint32_t rank = cluster_ctarank();          // 0 = leader
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  const int num_m_pairs = (p.M + 2 * BM - 1) / (2 * BM);
  const int total_tiles = num_m_pairs * p.num_n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) { mbar_init(&go[s], 1 + 2 * kEpiWarps); mbar_init(&done[s], 1); }
    // both TMEM buffers start free: the epilogues' share of go[] for chunks 0 and 1
    for (int w = 0; w < 2 * kEpiWarps; ++w) { mbar_arrive(&go[0]); mbar_arrive(&go[1 % kPairStages]); }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_sa);
    prefetch_tmap(&tmap_sb);
  }
  if (warp == 9) { tmem_alloc_pair(tmem_slot, 512); tmem_relinquish_pair(); }
  tc_fence_before();
  cluster_sync_all();          // both CTAs' barriers exist before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // pair tile t -> first row of this CTA's half and first column
  auto tile_rows = [&](int t, int& a_row0, int& n0) {
    const int per_group = p.group_m * p.num_n_tiles;
    const int grp = t / per_group;
    const int first_m = grp * p.group_m;
    const int gm = min(p.group_m, num_m_pairs - first_m);
    const int within = t - grp * per_group;
    const int mt = first_m + within % gm;
    const int nt = within / gm;
    a_row0 = mt * 2 * BM + static_cast<int>(rank) * BM;
    n0 = nt * BN;
  };

  if (warp >= kEpiWarps) {
    setmaxnreg_dec40();
    if (warp == 8) {
      // ---------------- TMA producer (both CTAs, one lane) ----------------
      if (lane == 0) {
        const uint32_t leader_go0 = mapa_shared(smem_u32(&go[0]), 0);
        int it = 0;
        bool ok = true;
        for (int t = cluster; ok && t < total_tiles; t += nclusters) {
          int a_row0, n0;
          tile_rows(t, a_row0, n0);
          const int b_row0 = n0 + static_cast<int>(rank) * (BN / 2);
          for (int kc = 0; kc < nk; ++kc, ++it) {
            const int s = it % kPairStages;
            const uint32_t ph = (it / kPairStages) & 1;
            if (!mbar_wait(&done[s], ph ^ 1, abort_flag, WAIT_PRODUCER_EMPTY)) { ok = false; break; }
            uint8_t* st = smem + PairSmemLayout::stages + s * kPairStageBytes;
            const uint32_t leader_go = leader_go0 + static_cast<uint32_t>(s) * 8u;
            uint8_t* slot = smem + PairSmemLayout::scales + (it % kPairScaleSlots) * kPairSlotBytes;
            if (rank == 0)   // both CTAs' operand and scale bytes
              mbar_arrive_expect_tx(&go[s], 2 * (kPairStageBytes + kPairSaBytes + pair_sb_bytes<kSfbMode>()));
            tma_load_2d_pair(st, &tmap_a, leader_go, kc * BK, a_row0);
            tma_load_2d_pair(st + kPairABytes, &tmap_b, leader_go, kc * BK, b_row0);
            // sa[kc][a_row0 .. +127] (rows past M read as zero)
            tma_load_2d_pair(slot + kPairSlotSa, &tmap_sa, leader_go, a_row0, kc);
            if (kSfbMode == FP8Q_SFB_ROW)   // sb[kc][n0 .. n0+255] (columns past N read as zero)
              tma_load_2d_pair(slot, &tmap_sb, leader_go, n0, kc);
            else                            // sb[n0/128 .. +1][(kc & ~3) .. +3]: a 16-byte aligned group
              tma_load_2d_pair(slot, &tmap_sb, leader_go, kc & ~3, n0 / 128);
          }
        }
        if (!ok && rank == 0) {
          // short waits: go[] also counts epilogue arrivals that may never come
          for (int j = max(0, it - kPairStages); j < it; ++j)
            mbar_wait(&go[j % kPairStages], (j / kPairStages) & 1, nullptr, WAIT_DRAIN, 1ll << 22);
        }
      }
      __syncwarp();
    } else if (warp == 9 && rank == 0) {
      // ---------------- MMA issuer (leader CTA, one lane) ----------------
      if (lane == 0) {
        const uint32_t idesc = umma_idesc_e4m3_f32(2 * BM, BN) | p.idesc_fmt;
        const int total_chunks =
            ((total_tiles - cluster + nclusters - 1) / nclusters) * nk;
        bool ok = true;
        int it = 0;
        for (; ok && it < total_chunks; ++it) {
          const int s = it % kPairStages;
          const int b = it & 1;
          if (!mbar_wait(&go[s], (it / kPairStages) & 1, abort_flag, WAIT_MMA_FULL)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + PairSmemLayout::stages + s * kPairStageBytes);
          const uint32_t b_addr = a_addr + kPairABytes;
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * BN);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            umma_f8f6f4_pair(d_tmem, umma_desc_k_sw128(a_addr + 32 * k), umma_desc_k_sw128(b_addr + 32 * k), idesc,
                             k > 0 ? 1u : 0u);
          umma_commit_pair(&done[s], 0x3);
        }
        if (!ok && it > 0) {
          const int j = it - 1;
          mbar_wait(&done[j % kPairStages], (j / kPairStages) & 1, nullptr, WAIT_DRAIN, 1ll << 26);
        }
      }
      __syncwarp();
    }
  } else {
    // ---------------- promotion + epilogue (warps 0-7, both CTAs) ----------------
    setmaxnreg_inc232();
    const int quad = warp & 3;
    const int half = warp >> 2;
    const int r_in_tile = quad * 32 + lane;
    const uint32_t t_lane = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t leader_go0 = mapa_shared(smem_u32(&go[0]), 0);
    float2 acc[64];
    int it = 0;
    bool ok = true;
    for (int t = cluster; ok && t < total_tiles; t += nclusters) {
      int a_row0, n0;
      tile_rows(t, a_row0, n0);
      const int ncol0 = n0 + half * 128;
      const bool vcol = ncol0 < p.N;
#pragma unroll
      for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
      for (int kc = 0; kc < nk; ++kc, ++it) {
        const int b = it & 1;
        const int s = it % kPairStages;
        if (!warp_wait(&done[s], (it / kPairStages) & 1, abort_flag, WAIT_EPI_TMEM_FULL)) { ok = false; break; }
        // this chunk's scales landed with its operands (go[] counted their bytes)
        const float* slot = reinterpret_cast<const float*>(smem + PairSmemLayout::scales +
                                                           (it % kPairScaleSlots) * kPairSlotBytes);
        tc_fence_after();
        const uint32_t taddr = tmem_base + t_lane + static_cast<uint32_t>(b * BN + half * 128);
        uint32_t v[64];
        // FP8Q_SFB_ROW, 16x256b fragments: rows 32*quad + {l4, l4+8, l4+16, l4+24}
        // with l4 = lane/4; columns 8k + 2*(lane%4) + {0,1} of each 64-column half
        const float* sa_rows = slot + kPairSlotSa / 4 + quad * 32 + (lane >> 2);
        // the scales are read before the TMEM loads so that their shared-memory
        // latency overlaps the loads instead of following them
        Rows16Scales sc;
        float scale = 0.0f;
        if (kSfbMode == FP8Q_SFB_ROW) {
          load_rows16_scales(sc, sa_rows, slot + half * 128 + 2 * (lane & 3), true);
          tmem_ld_16x256b_x8x2_sync(taddr, v);
          promote_rows16(acc, v, sc);
          load_rows16_scales(sc, sa_rows, slot + half * 128 + 64 + 2 * (lane & 3), false);
          tmem_ld_16x256b_x8x2_sync(taddr + 64, v);
        } else {
          scale = slot[kPairSlotSa / 4 + r_in_tile] * slot[half * 4 + (kc & 3)];
          tmem_ld_32x32b_x64_sync(taddr, v);
          promote64(acc, v, scale);
          tmem_ld_32x32b_x64_sync(taddr + 64, v);
        }
        // scale slots read so far (ordinary loads) are refilled by TMA (async
        // proxy) only after releases like this one: order across proxies
        fence_proxy_async_shared();
        tc_fence_before();
        __syncwarp();
        if (lane == 0)   // buffer b is free for chunk it + 2
          mbar_arrive_cluster(leader_go0 + static_cast<uint32_t>((it + 2) % kPairStages) * 8u);
        if (kSfbMode == FP8Q_SFB_ROW) {
          promote_rows16(acc + 32, v, sc);
        } else {
          promote64(acc + 32, v, scale);
        }
      }
      if (!ok) break;
      const int row0 = a_row0 + quad * 32;
      uint8_t* out_buf = smem + PairSmemLayout::out_stage + warp * kPairOutStageBytes;
      if (kSfbMode == FP8Q_SFB_ROW) {
        // 16x256b fragments: acc[64h + 32g + 4k + 2i + j] is row 32*quad + 16g +
        // 8i + lane/4, column 64h + 8k + 2*(lane%4) + j of this half; 4 lanes
        // write one 32-byte sector of a row per group k.  (Tensor stores of
        // these fragments measured slower on B200, twice: their staging raised
        // the register pressure of the chunk loop.)
        if (vcol) {
#pragma unroll
          for (int g = 0; g < 2; ++g) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int r = a_row0 + quad * 32 + 16 * g + 8 * i + (lane >> 2);
              if (r >= p.M) continue;
              const int64_t base = static_cast<int64_t>(r) * p.ldd + ncol0 + 2 * (lane & 3);
#pragma unroll
              for (int k = 0; k < 16; ++k) {   // k < 8: first 64 columns, k >= 8: second
                if (!chk(ncol0 + 8 * k + 2 * (lane & 3) + 1, p.N, CHK_GEMM_D)) continue;
                const int x = 64 * (k >> 3) + 32 * g + 4 * (k & 7) + 2 * i;
                const float x0 = acc[x / 2].x, x1 = acc[x / 2].y;
                if (kOut == kOutF32) {
                  *reinterpret_cast<float2*>(static_cast<float*>(p.d) + base + 8 * k) = make_float2(x0, x1);
                } else {
                  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
                  *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(p.d) + base + 8 * k) = h;
                }
              }
            }
          }
        }
      } else if (vcol && row0 < p.M && chk(ncol0 + 127, p.N, CHK_GEMM_D)) {
        if (kOut == kOutE4m3)
          store_rows128_staged<kOut>(acc, lane, row0, min(32, p.M - row0), ncol0, p,
                                     reinterpret_cast<uint4*>(out_buf));
        else
          store_rows128_tma<kOut>(acc, lane, row0, ncol0, &tmap_d, out_buf);
      }
    }
    if (lane == 0) bulk_wait_group0();   // this warp's tensor stores are complete before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();          // the peer's shared memory and TMEM are no longer in use
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
  kernel_clock_end(CLOCK_PAIR, kclock);
}

}  // namespace fp8q
