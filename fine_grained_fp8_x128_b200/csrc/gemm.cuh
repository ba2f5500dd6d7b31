// Block-scaled FP8 GEMM for sm_100a: TMA -> shared memory ring -> tcgen05.mma
// (kind::f8f6f4, E4M3 x E4M3 -> FP32 in tensor memory) -> per-128-K-chunk
// promotion into FP32 registers on the CUDA cores -> BF16/FP32 store.
//
//   D[m,n] = sum_kb sa[m,kb] * sb(n,kb) * P_kb[m,n],
//   P_kb   = sum over the 128 K of chunk kb of A[m,k] * B[n,k]   (tensor cores)
//
// "FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section 3
// "Decoupled Accumulation in Tensor Core GEMMs": FP8 products on the tensor
// cores, FP32 accumulation, scales s_A * s_B applied in FP32; "Introduction to
// LLM Quantization", "Fine-grained Quantization" Step 4 (rescale on the CUDA
// cores) and "3. Increasing accumulation Quantization" (promotion at an
// interval N_C, here 128 = one scale chunk).
//
// Scale factors are FP32 amax/448 values, not powers of two, so the hardware
// block-scaled MMA (UE8M0 scales) cannot apply them; every chunk gets its own
// TMEM accumulator and the scale multiply happens in the TMEM -> register path.
//
// CTA organisation (one persistent CTA per SM, 384 threads):
//   warps 0-7  : promotion + epilogue.  Warp w reads TMEM lanes 32*(w%4).. (its
//                rows) and columns 128*(w/4).. (its half of the 256-wide tile);
//                each thread keeps 128 FP32 accumulators of one output row.
//   warp 8     : TMA producer (lane 0 runs the loop).
//   warp 9     : MMA issuer (lane 0); owns the TMEM allocation.
//   warps 10-11: idle (they complete the third warpgroup for setmaxnreg).
// Pipelines:
//   smem ring  : kStages x (A 128x128 + B 256x128 E4M3).
//   tile-end   : two 4 KB staging buffers per epilogue warp for the tensor stores.
//   TMEM       : 2 chunk accumulators of 128 lanes x 256 FP32 columns (all 512
//                columns): the MMAs of chunk c+1 overlap the promotion of c.
//   row scales : (FP8Q_SFB_ROW only) a ring of per-chunk B scale vectors.
// Two mbarriers per ring stage carry all of it, so the MMA warp does one wait
// and one commit per chunk (each extra wait or commit between two chunks' MMAs
// leaves the tensor pipe idle for tens of cycles):
//   go[s]   (count 1 + 8): chunk c's operands have landed in stage s = c % S
//           (producer's expect_tx + TMA bytes) AND its TMEM buffer c % 2 is
//           free (one arrive per epilogue warp when chunk c-2 was read out).
//   done[s] (count 1): chunk c's MMAs have completed (one tcgen05.commit):
//           stage s may be refilled and TMEM buffer c % 2 may be read.
// Every wait is bounded (see mbar_wait) and reports through the status word.
#pragma once

#include "device_common.cuh"
#include "quant.cuh"

namespace fp8q {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int kStages = 3;
#ifndef FP8Q_SB_RING
#define FP8Q_SB_RING 8
#endif
constexpr int kSbRing = FP8Q_SB_RING;
constexpr int kGemmThreads = 384;
constexpr int kEpiWarps = 8;
constexpr uint32_t kABytes = BM * BK;               // 16 KB
constexpr uint32_t kBBytes = BN * BK;               // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes; // 48 KB
constexpr uint32_t kSbBytes = BN * 4;               // 1 KB
// Tile-end staging per epilogue warp: two 4 KB buffers (32 rows x 128 bytes
// each), so a tile's tensor stores leave without waiting for one another.
constexpr uint32_t kOutStageBytes = 8192;
constexpr int kMaxGroups = 1024;
constexpr int kGroupM = 16;                          // L2 swizzle: m-tiles per group

struct GemmSmemLayout {
  // offsets from the 1024-aligned base
  static constexpr uint32_t stages = 0;
  static constexpr uint32_t sb_ring = stages + kStages * kStageBytes;
  static constexpr uint32_t out_stage = sb_ring + kSbRing * kSbBytes;   // 8 epilogue warps x 8 KB, 1024-aligned
  static constexpr uint32_t bars = out_stage + 8 * kOutStageBytes;
  // barriers: go[S], done[S], sbfull[R], sbempty[R]
  static constexpr uint32_t nbars = 2 * kStages + 2 * kSbRing;
  static constexpr uint32_t misc = bars + nbars * 8;           // tmem base, abort flag
  static constexpr uint32_t prefix = misc + 16;                // grouped: tile prefix [G+1]
  static constexpr uint32_t offs = prefix + (kMaxGroups + 1) * 4;  // grouped: clamped offsets [G+1]
  static constexpr uint32_t bytes_dense = prefix;
  static constexpr uint32_t bytes_grouped = offs + (kMaxGroups + 1) * 4;
};

struct GemmArgs {
  const float* sfa;
  int64_t ld_sfa;
  const float* sfb;      // dense: per sfb_mode; grouped: sfw [G][N/128][K/128]
  int64_t ld_sfb;
  void* d;               // BF16 / FP32 output, or E4M3 codes (kOut == kOutE4m3)
  int64_t ldd;
  float* sfd;            // kOut == kOutE4m3: scales of the output's 1x128 tiles, sfd[(n/128) * ld_sfd + m]
  int64_t ld_sfd;
  int M;                 // dense: rows of A; grouped: M_total
  int N;
  int K;
  int num_n_tiles;
  int num_k_chunks;
  int num_m_tiles;       // dense only
  const int32_t* group_offsets;  // grouped only
  int G;
  int group_m;           // pair kernel: 256-row tiles per L2 group (tiles run m-fastest within a group)
  uint32_t idesc_fmt;    // operand formats OR-ed into the MMA instruction descriptor (0: both E4M3)
};

// Which output tile a linear tile id denotes.
struct TileCoord {
  int a_row0;     // first row of A (TMA y coordinate)
  int row_end;    // one past the last valid output row
  int n0;         // first output column
  int b_row0;     // first row of B in its tensor map (grouped: g*N + n0)
  int group;      // expert (grouped) or 0
};

template <bool kGrouped>
__device__ __forceinline__ TileCoord tile_coord(int t, const GemmArgs& p, const int* prefix,
                                                const int* offs) {
  TileCoord c;
  if (!kGrouped) {
    const int per_group = kGroupM * p.num_n_tiles;
    const int grp = t / per_group;
    const int first_m = grp * kGroupM;
    const int gm = min(kGroupM, p.num_m_tiles - first_m);
    const int within = t - grp * per_group;
    const int mt = first_m + within % gm;
    const int nt = within / gm;
    c.a_row0 = mt * BM;
    c.row_end = min(p.M, c.a_row0 + BM);
    c.n0 = nt * BN;
    c.b_row0 = c.n0;
    c.group = 0;
  } else {
    // largest g with prefix[g] <= t (empty experts share a prefix and are skipped)
    int lo = 0, hi = p.G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const int local = t - prefix[g];
    const int rows = offs[g + 1] - offs[g];
    const int mtiles = (rows + BM - 1) / BM;
    const int mt = local % mtiles;
    const int nt = local / mtiles;
    c.a_row0 = offs[g] + mt * BM;
    c.row_end = min(offs[g + 1], c.a_row0 + BM);
    c.n0 = nt * BN;
    c.b_row0 = g * p.N + c.n0;
    c.group = g;
  }
  return c;
}

// Output modes of the GEMM kernels.
constexpr int kOutBf16 = 0;   // round-to-nearest-even BF16
constexpr int kOutF32 = 1;    // FP32
constexpr int kOutE4m3 = 2;   // the next layer's operand: BF16-rounded rows quantized in 1x128 tiles

// One pass of a warp's staged store: lane l brings 8 16-byte chunks of row l
// (128 consecutive bytes of its output row); they go through the warp's 4 KB
// shared buffer -- chunk j of row r at chunk slot j ^ (r & 7), so each group
// of 8 lanes covers all 32 banks on the way in and on the way out -- and leave
// as 16-byte global stores in which the warp covers 4 whole 128-byte row
// segments at a time (instead of 32 scattered 16-byte pieces).  Rows at or
// past rows_valid are not written.  Every lane of the warp takes part.
__device__ __forceinline__ void stage_store_pass(uint4* stage, const uint4 (&chunk)[8], int lane, uint8_t* gbase,
                                                 int64_t ld_bytes, int rows_valid) {
#pragma unroll
  for (int j = 0; j < 8; ++j) stage[lane * 8 + (j ^ (lane & 7))] = chunk[j];
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 4 * i + (lane >> 3);
    const int c = lane & 7;
    const uint4 val = stage[r * 8 + (c ^ (r & 7))];
    if (r < rows_valid) *reinterpret_cast<uint4*>(gbase + r * ld_bytes + 16 * c) = val;
  }
  __syncwarp();
}

// stage_store_pass with 64-byte row segments and a 2 KB buffer: lane l brings
// 4 16-byte chunks of row l (chunk j of row r at slot j ^ ((r / 2) % 4), so 8
// consecutive rows cover all 32 banks both ways); each 16-byte global store of
// the warp covers 8 whole 64-byte row segments.
__device__ __forceinline__ void stage_store_pass4(uint4* stage, const uint4 (&chunk)[4], int lane, uint8_t* gbase,
                                                  int64_t ld_bytes, int rows_valid) {
#pragma unroll
  for (int j = 0; j < 4; ++j) stage[lane * 4 + (j ^ ((lane >> 1) & 3))] = chunk[j];
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = 8 * i + (lane >> 2);
    const int c = lane & 3;
    const uint4 val = stage[r * 4 + (c ^ ((r >> 1) & 3))];
    if (r < rows_valid) *reinterpret_cast<uint4*>(gbase + r * ld_bytes + 16 * c) = val;
  }
  __syncwarp();
}


// The tile-end store of a warp whose 32 rows are all valid, through tensor
// stores of 128-byte boxes from two 4 KB buffers (the output's tensor map:
// SWIZZLE_128B, box 128 bytes x 32 rows; chunk j of row r at j ^ (r % 8)).  BF16: 64 columns per box, both boxes issued back to back;
// E4M3: all 128 codes of a row in one box; FP32: 32 columns per box, the two
// buffers used twice.  The warp waits only before it refills a buffer that a
// store may still be reading -- at the start of the next tile's stores -- so a
// tile's global writes overlap the next tile's chunks.
template <int kOut>
__device__ __forceinline__ void store_rows128_tma128(const float2* acc, int lane, int row0, int ncol0,
                                                     const GemmArgs& p, const CUtensorMap* tmap_d, uint8_t* buf) {
  auto put = [&](uint8_t* b, const uint4 (&chunk)[8]) {
    uint4* stage = reinterpret_cast<uint4*>(b);
#pragma unroll
    for (int j = 0; j < 8; ++j) stage[lane * 8 + (j ^ (lane & 7))] = chunk[j];
  };
  auto issue = [&](uint8_t* b, int x) {
    fence_proxy_async_shared();   // the buffer's generic-proxy writes, before the async-proxy read
    __syncwarp();
    if (lane == 0) tma_store_2d(tmap_d, b, x, row0);
  };
  if (lane == 0) bulk_wait_group_read0();   // the previous tile's stores have read both buffers
  __syncwarp();
  uint4 chunk[8];
  if (kOut == kOutF32) {
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      if (h == 2) {                  // the buffers come round again
        if (lane == 0) { bulk_commit_group(); bulk_wait_group_read0(); }
        __syncwarp();
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float2 a = acc[16 * h + 2 * j], b = acc[16 * h + 2 * j + 1];
        chunk[j] = make_uint4(__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(b.x), __float_as_uint(b.y));
      }
      put(buf + 4096 * (h & 1), chunk);
      issue(buf + 4096 * (h & 1), ncol0 + 32 * h);
    }
  } else {
    uint32_t w[64];   // BF16 pairs
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      const __nv_bfloat162 h = __float22bfloat162_rn(acc[j]);
      w[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    if (kOut == kOutBf16) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          chunk[j] = make_uint4(w[32 * h + 4 * j], w[32 * h + 4 * j + 1], w[32 * h + 4 * j + 2], w[32 * h + 4 * j + 3]);
        put(buf + 4096 * h, chunk);
        issue(buf + 4096 * h, ncol0 + 64 * h);
      }
    } else {
      uint32_t m2 = 0;
#pragma unroll
      for (int j = 0; j < 64; ++j) m2 = amax2_sx(m2, w[j]);
      const float s = tile_scale(amax2_value(amax2_sx_bits(m2)));
      const float nr = -__frcp_rn(s);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t c[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) c[e] = quant_words(w[8 * j + 2 * e], w[8 * j + 2 * e + 1], nr, s);
        chunk[j] = make_uint4(c[0], c[1], c[2], c[3]);
      }
      put(buf, chunk);
      issue(buf, ncol0);
      if (chk(row0 + lane, p.ld_sfd, CHK_GEMM_SFD)) p.sfd[static_cast<int64_t>(ncol0 / 128) * p.ld_sfd + row0 + lane] = s;
    }
  }
  if (lane == 0) bulk_commit_group();
  __syncwarp();
}

// store_rows128_staged through a 2 KB buffer: 8 passes of 16 FP32 columns, 4
// of 32 BF16 columns or 2 of 64 E4M3 codes.
template <int kOut>
__device__ __forceinline__ void store_rows128_staged4(const float2* acc, int lane, int row0, int rows_valid, int ncol0,
                                                      const GemmArgs& p, uint4* stage) {
  uint4 chunk[4];
  if (kOut == kOutF32) {
    uint8_t* base = reinterpret_cast<uint8_t*>(static_cast<float*>(p.d) + static_cast<int64_t>(row0) * p.ldd + ncol0);
#pragma unroll
    for (int h = 0; h < 8; ++h) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 a = acc[8 * h + 2 * j], b = acc[8 * h + 2 * j + 1];
        chunk[j] = make_uint4(__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(b.x), __float_as_uint(b.y));
      }
      stage_store_pass4(stage, chunk, lane, base + 64 * h, p.ldd * 4, rows_valid);
    }
  } else {
    uint32_t w[64];   // BF16 pairs
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      const __nv_bfloat162 h = __float22bfloat162_rn(acc[j]);
      w[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    if (kOut == kOutBf16) {
      uint8_t* base =
          reinterpret_cast<uint8_t*>(static_cast<__nv_bfloat16*>(p.d) + static_cast<int64_t>(row0) * p.ldd + ncol0);
#pragma unroll
      for (int h = 0; h < 4; ++h) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          chunk[j] = make_uint4(w[16 * h + 4 * j], w[16 * h + 4 * j + 1], w[16 * h + 4 * j + 2], w[16 * h + 4 * j + 3]);
        stage_store_pass4(stage, chunk, lane, base + 64 * h, p.ldd * 2, rows_valid);
      }
    } else {
      uint32_t m2 = 0;
#pragma unroll
      for (int j = 0; j < 64; ++j) m2 = amax2_sx(m2, w[j]);
      const float s = tile_scale(amax2_value(amax2_sx_bits(m2)));
      const float nr = -__frcp_rn(s);
      uint8_t* base = static_cast<uint8_t*>(p.d) + static_cast<int64_t>(row0) * p.ldd + ncol0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t c[4];
#pragma unroll
          for (int j = 0; j < 4; ++j)
            c[j] = quant_words(w[32 * h + 8 * i + 2 * j], w[32 * h + 8 * i + 2 * j + 1], nr, s);
          chunk[i] = make_uint4(c[0], c[1], c[2], c[3]);
        }
        stage_store_pass4(stage, chunk, lane, base + 64 * h, p.ldd, rows_valid);
      }
      if (lane < rows_valid && chk(row0 + lane, p.ld_sfd, CHK_GEMM_SFD))
        p.sfd[static_cast<int64_t>(ncol0 / 128) * p.ld_sfd + row0 + lane] = s;
    }
  }
}

// The warp's 32 rows x 128 columns (row row0 + lane in acc, columns ncol0 ..
// ncol0 + 127) through stage_store_pass: 4 passes of 32 FP32 columns, 2 of 64
// BF16 columns, or 1 of 128 E4M3 codes plus the row's tile scale.  In
// kOutE4m3 mode a thread's 128 values are one 1x128 tile: they are rounded to
// BF16 and quantized exactly as quant_act_1x128_kernel quantizes a BF16 row
// ("Fine-Grained FP8 Quantization in DeepSeek", section 2: per-tile amax,
// s = amax/448, E4M3 cast), so the result equals quantizing the BF16 output
// -- without writing or re-reading it.
template <int kOut>
__device__ __forceinline__ void store_rows128_staged(const float2* acc, int lane, int row0, int rows_valid, int ncol0,
                                                     const GemmArgs& p, uint4* stage) {
  if (rows_valid <= 0) return;
  uint4 chunk[8];
  if (kOut == kOutF32) {
    uint8_t* base = reinterpret_cast<uint8_t*>(static_cast<float*>(p.d) + static_cast<int64_t>(row0) * p.ldd + ncol0);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float2 a = acc[16 * h + 2 * j], b = acc[16 * h + 2 * j + 1];
        chunk[j] = make_uint4(__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(b.x), __float_as_uint(b.y));
      }
      stage_store_pass(stage, chunk, lane, base + 128 * h, p.ldd * 4, rows_valid);
    }
  } else {
    uint32_t w[64];   // BF16 pairs
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      const __nv_bfloat162 h = __float22bfloat162_rn(acc[j]);
      w[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    if (kOut == kOutBf16) {
      uint8_t* base =
          reinterpret_cast<uint8_t*>(static_cast<__nv_bfloat16*>(p.d) + static_cast<int64_t>(row0) * p.ldd + ncol0);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          chunk[j] = make_uint4(w[32 * h + 4 * j], w[32 * h + 4 * j + 1], w[32 * h + 4 * j + 2], w[32 * h + 4 * j + 3]);
        stage_store_pass(stage, chunk, lane, base + 128 * h, p.ldd * 2, rows_valid);
      }
    } else {
      uint32_t m2 = 0;
#pragma unroll
      for (int j = 0; j < 64; ++j) m2 = amax2_sx(m2, w[j]);
      const float s = tile_scale(amax2_value(amax2_sx_bits(m2)));
      const float nr = -__frcp_rn(s);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint32_t c[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) c[j] = quant_words(w[8 * i + 2 * j], w[8 * i + 2 * j + 1], nr, s);
        chunk[i] = make_uint4(c[0], c[1], c[2], c[3]);
      }
      stage_store_pass(stage, chunk, lane, static_cast<uint8_t*>(p.d) + static_cast<int64_t>(row0) * p.ldd + ncol0,
                       p.ldd, rows_valid);
      if (lane < rows_valid && chk(row0 + lane, p.ld_sfd, CHK_GEMM_SFD))
        p.sfd[static_cast<int64_t>(ncol0 / 128) * p.ld_sfd + row0 + lane] = s;
    }
  }
}

__device__ __forceinline__ void setmaxnreg_inc232() { asm volatile("setmaxnreg.inc.sync.aligned.u32 232;"); }
__device__ __forceinline__ void setmaxnreg_dec40() { asm volatile("setmaxnreg.dec.sync.aligned.u32 40;"); }

}  // namespace fp8q

namespace fp8q {

// acc[j] += v[j] * scale for 64 columns (packed FP32 pairs).
__device__ __forceinline__ void promote64(float2* acc, const uint32_t (&v)[64], float scale) {
  const float2 s = f2(scale);
#pragma unroll
  for (int j = 0; j < 32; ++j) acc[j] = ffma2(f2u(v[2 * j], v[2 * j + 1]), s, acc[j]);
}

// Per-column scales (FP8Q_SFB_ROW): acc[j] += v[j] * (sa * sb[j]).
__device__ __forceinline__ void promote64_rows(float2* acc, const uint32_t (&v)[64], float sa, const float* sb) {
  const float4* s4 = reinterpret_cast<const float4*>(sb);
  const float2 a = f2(sa);
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const float4 s = s4[q];
    const float2 c01 = fmul2(make_float2(s.x, s.y), a);
    const float2 c23 = fmul2(make_float2(s.z, s.w), a);
    acc[2 * q] = ffma2(f2u(v[4 * q + 0], v[4 * q + 1]), c01, acc[2 * q]);
    acc[2 * q + 1] = ffma2(f2u(v[4 * q + 2], v[4 * q + 3]), c23, acc[2 * q + 1]);
  }
}

// Grouped GEMMs, run by one warp before the main loop: clamp the device-side
// offsets into [0, M_total], force them nondecreasing (warp max-scan), write
// them to offs[0..G] and the exclusive prefix of each expert's tile count
// (ceil(rows / 128) * tiles_per_block) to prefix[0..G].  Offsets that had to
// be changed are reported through the status word (FP8Q_ERR_INVALID_ARG).
__device__ __forceinline__ void build_group_prefix(const GemmArgs& p, int* offs, int* prefix, int tiles_per_block,
                                                   int lane) {
  bool bad = false;
  int carry = 0;
  for (int g0 = 0; g0 <= p.G; g0 += 32) {
    const int g = g0 + lane;
    int o = 0;
    if (g <= p.G) {
      const int raw = p.group_offsets[g];
      o = min(max(raw, 0), p.M);
      bad |= (o != raw);
    }
    int m = o;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, m, d);
      if (lane >= d) m = max(m, v);
    }
    m = max(m, carry);
    if (g <= p.G) { bad |= (m != o); offs[g] = m; }
    carry = __shfl_sync(0xFFFFFFFFu, m, 31);
  }
  __syncwarp();
  if (lane == 0) bad |= (offs[0] != 0) || (offs[p.G] != p.M);
  int tcarry = 0;
  for (int g0 = 0; g0 < p.G; g0 += 32) {
    const int g = g0 + lane;
    const int tg = (g < p.G) ? ((offs[g + 1] - offs[g] + BM - 1) / BM) * tiles_per_block : 0;
    int s = tg;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, s, d);
      if (lane >= d) s += v;
    }
    if (g < p.G) prefix[g] = tcarry + s - tg;
    tcarry += __shfl_sync(0xFFFFFFFFu, s, 31);
  }
  if (lane == 0) prefix[p.G] = tcarry;
  bad = __any_sync(0xFFFFFFFFu, bad);
  if (bad && lane == 0 && blockIdx.x == 0) report_status(FP8Q_ERR_INVALID_ARG, BAD_GROUP_OFFSETS);
}

template <bool kGrouped, int kSfbMode, int kOut>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_blockscaled_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                        const __grid_constant__ CUtensorMap tmap_d, const GemmArgs p) {
  const KernelClock kclock = kernel_clock_begin();
  extern __shared__ uint8_t gemm_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + GemmSmemLayout::bars);
  uint64_t* go = bars;
  uint64_t* done = bars + kStages;
  uint64_t* sbfull = bars + 2 * kStages;
  uint64_t* sbempty = sbfull + kSbRing;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + GemmSmemLayout::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + GemmSmemLayout::misc + 4);
  int* prefix = reinterpret_cast<int*>(smem + GemmSmemLayout::prefix);
  int* offs = reinterpret_cast<int*>(smem + GemmSmemLayout::offs);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nk = p.num_k_chunks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&go[s], 1 + kEpiWarps); mbar_init(&done[s], 1); }
    for (int r = 0; r < kSbRing; ++r) { mbar_init(&sbfull[r], 1); mbar_init(&sbempty[r], kEpiWarps); }
    // both TMEM buffers start free: the epilogue's share of go[] for chunks 0 and 1
    for (int w = 0; w < kEpiWarps; ++w) { mbar_arrive(&go[0]); mbar_arrive(&go[1 % kStages]); }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8 && lane == 0) { prefetch_tmap(&tmap_a); prefetch_tmap(&tmap_b); }
  if (warp == 9) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  if (kGrouped && warp == 0) build_group_prefix(p, offs, prefix, p.num_n_tiles, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = kGrouped ? prefix[p.G] : p.num_m_tiles * p.num_n_tiles;

  if (warp >= kEpiWarps) {
    setmaxnreg_dec40();
    if (warp == 8) {
      // ---------------- TMA producer (one lane) ----------------
      if (lane == 0) {
        int it = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
          const TileCoord c = tile_coord<kGrouped>(t, p, prefix, offs);
          for (int kc = 0; kc < nk; ++kc, ++it) {
            const int s = it % kStages;
            const uint32_t ph = (it / kStages) & 1;
            if (!mbar_wait(&done[s], ph ^ 1, abort_flag, WAIT_PRODUCER_EMPTY)) { ok = false; break; }
            if (kSfbMode == FP8Q_SFB_ROW) {
              const int r = it % kSbRing;
              if (!mbar_wait(&sbempty[r], ((it / kSbRing) & 1) ^ 1, abort_flag, WAIT_PRODUCER_EMPTY)) { ok = false; break; }
              const uint32_t nbytes = static_cast<uint32_t>(min(BN, p.N - c.n0)) * 4u;
              mbar_arrive_expect_tx(&sbfull[r], nbytes);
              bulk_load(smem + GemmSmemLayout::sb_ring + r * kSbBytes,
                        p.sfb + static_cast<int64_t>(kc) * p.ld_sfb + c.n0, nbytes, &sbfull[r]);
            }
            uint8_t* st = smem + GemmSmemLayout::stages + s * kStageBytes;
            mbar_arrive_expect_tx(&go[s], kStageBytes);
            tma_load_2d_nohint(st, &tmap_a, &go[s], kc * BK, c.a_row0);
            tma_load_2d_nohint(st + kABytes, &tmap_b, &go[s], kc * BK, c.b_row0);
          }
        }
        if (!ok) {
          // error path: let the copies already in flight land before the CTA exits.
          // go[] also waits for epilogue arrivals that may never come, so each
          // wait is short; the copies themselves land within microseconds.
          for (int j = max(0, it - kStages); j < it; ++j)
            mbar_wait(&go[j % kStages], (j / kStages) & 1, nullptr, WAIT_DRAIN, 1ll << 22);
        }
      }
      __syncwarp();
    } else if (warp == 9) {
      // ---------------- MMA issuer (one lane) ----------------
      if (lane == 0) {
        const uint32_t idesc = umma_idesc_e4m3_f32(BM, BN) | p.idesc_fmt;
        const int total_chunks = ((total_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                                  static_cast<int>(gridDim.x)) * nk;
        bool ok = true;
        int it = 0;
        for (; ok && it < total_chunks; ++it) {
          const int s = it % kStages;
          const int b = it & 1;
          if (!mbar_wait(&go[s], (it / kStages) & 1, abort_flag, WAIT_MMA_FULL)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + GemmSmemLayout::stages + s * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * BN);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            umma_f8f6f4(d_tmem, umma_desc_k_sw128(a_addr + 32 * k), umma_desc_k_sw128(b_addr + 32 * k), idesc,
                        k > 0 ? 1u : 0u);
          umma_commit(&done[s]);
        }
        if (!ok && it > 0) {
          // error path: the last issued MMAs must finish reading shared memory
          const int j = it - 1;
          mbar_wait(&done[j % kStages], (j / kStages) & 1, nullptr, WAIT_DRAIN, 1ll << 26);
        }
      }
      __syncwarp();
    }
  } else {
    // ---------------- promotion + epilogue (warps 0-7) ----------------
    setmaxnreg_inc232();
    const int quad = warp & 3;
    const int half = warp >> 2;
    const int r_in_tile = quad * 32 + lane;
    const uint32_t t_lane = static_cast<uint32_t>(quad * 32) << 16;
    const int nb_per_group = p.N / 128;
    float2 acc[64];
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
      const TileCoord c = tile_coord<kGrouped>(t, p, prefix, offs);
      const int row = c.a_row0 + r_in_tile;
      const bool vrow = row < c.row_end;
      const int ncol0 = c.n0 + half * 128;
      const bool vcol = ncol0 < p.N;
#pragma unroll
      for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
      // Scale factors of chunk kc are loaded kScalePrefetch chunks ahead (a
      // register shift ring) so their L2 latency stays off the promotion path.
      const float* sa_ptr = p.sfa + row;
      const float* sb_ptr = kGrouped ? p.sfb + (static_cast<int64_t>(c.group) * nb_per_group + ncol0 / 128) * nk
                                     : p.sfb + static_cast<int64_t>(ncol0 / 128) * p.ld_sfb;
      auto load_sa = [&](int k) -> float {
        return (vrow && k < nk) ? __ldg(sa_ptr + static_cast<int64_t>(k) * p.ld_sfa) : 0.0f;
      };
      auto load_sb = [&](int k) -> float {
        return (kSfbMode == FP8Q_SFB_BLOCK128 && vcol && k < nk) ? __ldg(sb_ptr + k) : 0.0f;
      };
      float sa_q0 = load_sa(0), sa_q1 = load_sa(1), sa_q2 = load_sa(2), sa_q3 = load_sa(3);
      float sb_q0 = load_sb(0), sb_q1 = load_sb(1), sb_q2 = load_sb(2), sb_q3 = load_sb(3);
      for (int kc = 0; kc < nk; ++kc, ++it) {
        const int b = it & 1;
        const int s = it % kStages;
        const float sa = sa_q0;
        const float sbk = sb_q0;
        sa_q0 = sa_q1; sa_q1 = sa_q2; sa_q2 = sa_q3; sa_q3 = load_sa(kc + 4);
        sb_q0 = sb_q1; sb_q1 = sb_q2; sb_q2 = sb_q3; sb_q3 = load_sb(kc + 4);
        if (!warp_wait(&done[s], (it / kStages) & 1, abort_flag, WAIT_EPI_TMEM_FULL)) { ok = false; break; }
        const float* sbv = nullptr;
        int r = 0;
        if (kSfbMode == FP8Q_SFB_ROW) {
          r = it % kSbRing;
          if (!warp_wait(&sbfull[r], (it / kSbRing) & 1, abort_flag, WAIT_EPI_TMEM_FULL)) { ok = false; break; }
          sbv = reinterpret_cast<const float*>(smem + GemmSmemLayout::sb_ring + r * kSbBytes) + half * 128;
        }
        tc_fence_after();
        const float scale = sa * sbk;
        const uint32_t taddr = tmem_base + t_lane + static_cast<uint32_t>(b * BN + half * 128);
        // two 64-column TMEM reads (each waited for inside its own asm statement);
        // the buffer goes back to the MMA warp as soon as the second read has
        // landed, before its FMAs
        uint32_t v[64];
        tmem_ld_32x32b_x64_sync(taddr, v);
        if (kSfbMode == FP8Q_SFB_ROW) promote64_rows(acc, v, sa, sbv); else promote64(acc, v, scale);
        tmem_ld_32x32b_x64_sync(taddr + 64, v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&go[(it + 2) % kStages]);   // buffer b is free for chunk it + 2
        if (kSfbMode == FP8Q_SFB_ROW) promote64_rows(acc + 32, v, sa, sbv + 64); else promote64(acc + 32, v, scale);
        if (kSfbMode == FP8Q_SFB_ROW) {
          // the ring slot was read with ordinary loads and is refilled by a bulk
          // copy (async proxy): order the reads before the release across proxies
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sbempty[r]);
        }
      }
      if (!ok) break;
      if (vcol) {   // warp-uniform
        const int row0 = c.a_row0 + quad * 32;
        const int rows_valid = min(32, c.row_end - row0);
        uint8_t* out_buf = smem + GemmSmemLayout::out_stage + warp * kOutStageBytes;
        // a box of 32 full rows leaves as tensor stores; a part-filled box (the
        // last rows of an expert or of M) keeps the per-row staged stores, so
        // nothing is written past the expert's rows
        const bool inside = rows_valid <= 0 || (chk(row0, p.M, CHK_GROUP) && chk(row0 + rows_valid - 1, p.M, CHK_GROUP) &&
                                                chk(ncol0 + 127, p.N, CHK_GEMM_D));
        if (!inside) {
        } else if (rows_valid == 32) {
          store_rows128_tma128<kOut>(acc, lane, row0, ncol0, p, &tmap_d, out_buf);
        } else if (rows_valid > 0) {
          if (lane == 0) bulk_wait_group_read0();   // earlier tensor stores have read the buffer
          __syncwarp();
          store_rows128_staged4<kOut>(acc, lane, row0, rows_valid, ncol0, p, reinterpret_cast<uint4*>(out_buf));
        }
      }
    }
    if (lane == 0) bulk_wait_group0();   // this warp's tensor stores are complete before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
  kernel_clock_end(CLOCK_ONE_CTA, kclock);
}

}  // namespace fp8q
