// Online quantizers: 1x128 activation tiles, 128x1 transposed tiles, 128x128
// weight blocks.  All three are HBM-bound streaming kernels: 16-byte coalesced
// loads, a register/shuffle amax per tile, the scale s = amax/448 and the
// saturating E4M3 cast fused into one store pass.
//
// Passages: "Fine-Grained FP8 Quantization in DeepSeek", sections 2-3;
// "FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section 1 (eq. s_W,
// eq. W_FP8); "Introduction to LLM Quantization", "5) Online Quantization".
#pragma once

#include "device_common.cuh"

namespace fp8q {

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Lane-wise maximum magnitude of BF16 pairs.  For finite BF16 values |a| <= |b|
// exactly when their 15 low bits compare that way as unsigned integers, so one
// 16x2 integer max per word keeps both lanes' running maxima (m starts at 0).
__device__ __forceinline__ uint32_t amax2(uint32_t m, uint32_t w) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(m), "r"(w & 0x7FFF7FFFu));
  return r;
}
__device__ __forceinline__ float amax2_value(uint32_t m) { return fmaxf(bf16lo(m), bf16hi(m)); }

// The same running maximum in one instruction: max.xorsign.abs keeps the
// larger magnitude of each lane (its sign bit is the XOR of the inputs' signs,
// cleared by amax2_sx_bits at the end); .NaN keeps a NaN, as the integer form
// does (NaN patterns compare above every finite value and infinity).
__device__ __forceinline__ uint32_t amax2_sx(uint32_t m, uint32_t w) {
  uint32_t r;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(m), "r"(w));
  return r;
}
__device__ __forceinline__ uint32_t amax2_sx_bits(uint32_t m) { return m & 0x7FFF7FFFu; }

// Four BF16 values (two words) -> four E4M3 codes, one byte each in element
// order: q = e4m3(fl32(x / s)), with nr = -fl32(1/s) (see e4m3x2_neg_quot,
// which returns the codes with inverted signs; one XOR flips all four back).
constexpr uint32_t kFlipSigns = 0x80808080u;
template <int kFmt = kFmtE4M3>
__device__ __forceinline__ uint32_t quant_words(uint32_t w0, uint32_t w1, float nr, float s) {
  const uint32_t c0 = fp8x2_neg_quot<kFmt>(bf16lo(w0), bf16hi(w0), nr, nr, s, s);
  const uint32_t c1 = fp8x2_neg_quot<kFmt>(bf16lo(w1), bf16hi(w1), nr, nr, s, s);
  return (c0 | (c1 << 16)) ^ kFlipSigns;
}

// ---------------------------------------------------------------------------
// 1x128 tiles.  4 consecutive lanes own one tile (32 elements each, four
// 16-byte loads).  Lane `sub` reads bytes 16*sub + 64*i (i = 0..3) of the
// tile's 256, so each load instruction covers whole 32-byte sectors; its codes
// leave as four 8-byte stores at the matching offsets.  A 256-thread block
// covers 64 tiles: rows r0..r0+63 of one 128-column chunk kb, so the 64 scales
// it writes, sf[kb*ld_sf + r0 ..], are contiguous.  The loads of the block's
// next grid-stride item are issued before the current item is cast.
// With a row map (rows != nullptr) output row m is the quantization of source
// row rows[m] -- the gather of MoE dispatch fused into the quantizer; an index
// outside [0, M_src) gives the all-zero tile and records FP8Q_ERR_INVALID_ARG.
// kRowScales writes the scales row-major, sf[m * ld_sf + kb], the layout in
// which each row's scales travel with its codes through the dispatch exchange.
// ---------------------------------------------------------------------------
constexpr int kQ1Threads = 256;
constexpr int kQ1Rows = 64;

struct Q1Slice {
  uint4 v[4];
};

template <bool kGather>
__device__ __forceinline__ void q1_load(Q1Slice& d, const __nv_bfloat16* __restrict__ x, int64_t M, int64_t KB,
                                        int64_t ldx, const int32_t* __restrict__ rows, int64_t M_src, int64_t it,
                                        int tile, int sub) {
  const int64_t rb = it / KB;
  const int64_t kb = it - rb * KB;
  const int64_t row = rb * kQ1Rows + tile;
  int64_t src_row = row;
  if (kGather && row < M) {
    src_row = __ldg(rows + row);
    if (src_row < 0 || src_row >= M_src) {
      if (sub == 0 && kb == 0) report_status(FP8Q_ERR_INVALID_ARG, BAD_ROW_INDEX);
      src_row = -1;
    }
  }
  if (row < M && src_row >= 0) {
    const uint4* src = reinterpret_cast<const uint4*>(x + src_row * ldx + kb * 128 + sub * 8);
    if (kGather) {
      // a source row is read once per output row that maps to it: default
      // caching keeps the rows in the L2 between their reads
#pragma unroll
      for (int i = 0; i < 4; ++i) d.v[i] = __ldg(src + 4 * i);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) d.v[i] = __ldcs(src + 4 * i);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) d.v[i] = make_uint4(0, 0, 0, 0);
  }
}

template <bool kGather, int kFmt = kFmtE4M3, bool kRowScales = false>
__global__ void __launch_bounds__(kQ1Threads)
quant_act_1x128_kernel(const __nv_bfloat16* __restrict__ x, int64_t M, int64_t KB, int64_t ldx,
                       uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ sf, int64_t ld_sf,
                       const int32_t* __restrict__ rows, int64_t M_src) {
  const int tid = threadIdx.x;
  const int sub = tid & 3;           // 32-element slice within the tile
  const int tile = tid >> 2;         // 0..63: row within the block's 64 rows
  const int64_t row_blocks = (M + kQ1Rows - 1) / kQ1Rows;
  const int64_t items = row_blocks * KB;
  int64_t it = blockIdx.x;
  if (it >= items) return;
  Q1Slice cur, nxt;
  q1_load<kGather>(cur, x, M, KB, ldx, rows, M_src, it, tile, sub);
  for (; it < items; it += gridDim.x) {
    const int64_t it_next = it + gridDim.x;
    if (it_next < items) q1_load<kGather>(nxt, x, M, KB, ldx, rows, M_src, it_next, tile, sub);
    const int64_t rb = it / KB;
    const int64_t kb = it - rb * KB;
    const int64_t row = rb * kQ1Rows + tile;
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m2 = amax2_sx(m2, cur.v[i].x); m2 = amax2_sx(m2, cur.v[i].y);
      m2 = amax2_sx(m2, cur.v[i].z); m2 = amax2_sx(m2, cur.v[i].w);
    }
    float m = amax2_value(amax2_sx_bits(m2));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    const float s = tile_scale_fmt<kFmt>(m);
    const float nr = -__frcp_rn(s);
    if (row < M && chk(kb * 128 + sub * 8 + 32 * 3 + 7, ldq, CHK_Q1)) {
      uint8_t* dst = q + row * ldq + kb * 128 + sub * 8;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint2 o;
        o.x = quant_words<kFmt>(cur.v[i].x, cur.v[i].y, nr, s);
        o.y = quant_words<kFmt>(cur.v[i].z, cur.v[i].w, nr, s);
        if (kGather)
          __stcs(reinterpret_cast<uint2*>(dst + 32 * i), o);   // evict-first: leave the L2 to the source rows
        else
          *reinterpret_cast<uint2*>(dst + 32 * i) = o;
      }
      if (sub == 0) {
        if (kRowScales) {
          if (chk(kb, ld_sf, CHK_Q1_SF))
            sf[row * ld_sf + kb] = s;    // row-major [M][ld_sf >= K/128]: a row's scales travel with it
        } else if (chk(row, ld_sf, CHK_Q1_SF)) {
          sf[kb * ld_sf + row] = s;
        }
      }
    }
    cur = nxt;
  }
}

// ---------------------------------------------------------------------------
// Quantize once, scatter k times: the MoE dispatch from the token side.  Each
// source row's 1x128 tiles are quantized once (tiling and loads as above) and
// written to the k output rows pos[row * k + j] it is routed to, so that the
// same token is not re-read and re-quantized per routed copy.  A negative
// position (a dropped entry) is skipped; one at or above M_out records
// FP8Q_ERR_INVALID_ARG and is skipped.  Output rows no entry maps to are not
// written.  kRowScales writes the scales row-major (the exchange's send layout).
// ---------------------------------------------------------------------------
constexpr int kScatterMaxK = 64;

template <bool kRowScales = false>
__global__ void __launch_bounds__(kQ1Threads)
quant_act_1x128_scatter_kernel(const __nv_bfloat16* __restrict__ x, int64_t M, int64_t KB, int64_t ldx,
                               const int32_t* __restrict__ pos, int k, int64_t M_out, uint8_t* __restrict__ q,
                               int64_t ldq, float* __restrict__ sf, int64_t ld_sf) {
  const int tid = threadIdx.x;
  const int sub = tid & 3;
  const int tile = tid >> 2;
  const int64_t items = ((M + kQ1Rows - 1) / kQ1Rows) * KB;
  int64_t it = blockIdx.x;
  if (it >= items) return;
  Q1Slice cur, nxt;
  q1_load<false>(cur, x, M, KB, ldx, nullptr, 0, it, tile, sub);
  for (; it < items; it += gridDim.x) {
    const int64_t it_next = it + gridDim.x;
    if (it_next < items) q1_load<false>(nxt, x, M, KB, ldx, nullptr, 0, it_next, tile, sub);
    const int64_t rb = it / KB;
    const int64_t kb = it - rb * KB;
    const int64_t row = rb * kQ1Rows + tile;
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m2 = amax2_sx(m2, cur.v[i].x); m2 = amax2_sx(m2, cur.v[i].y);
      m2 = amax2_sx(m2, cur.v[i].z); m2 = amax2_sx(m2, cur.v[i].w);
    }
    float m = amax2_value(amax2_sx_bits(m2));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    const float s = tile_scale(m);
    const float nr = -__frcp_rn(s);
    if (row < M) {
      uint2 o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        o[i].x = quant_words(cur.v[i].x, cur.v[i].y, nr, s);
        o[i].y = quant_words(cur.v[i].z, cur.v[i].w, nr, s);
      }
      for (int j = 0; j < k; ++j) {
        const int64_t dst = __ldg(pos + row * k + j);
        if (dst < 0) continue;
        if (dst >= M_out) {
          if (sub == 0 && kb == 0) report_status(FP8Q_ERR_INVALID_ARG, BAD_ROW_INDEX);
          continue;
        }
        if (!chk(kb * 128 + sub * 8 + 32 * 3 + 7, ldq, CHK_SCATTER)) continue;
        uint8_t* d = q + dst * ldq + kb * 128 + sub * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) __stcs(reinterpret_cast<uint2*>(d + 32 * i), o[i]);
        if (sub == 0) {
          if (kRowScales) {
            if (chk(kb, ld_sf, CHK_SCATTER)) sf[dst * ld_sf + kb] = s;
          } else if (chk(dst, ld_sf, CHK_SCATTER)) {
            sf[kb * ld_sf + dst] = s;
          }
        }
      }
    }
    cur = nxt;
  }
}

// ---------------------------------------------------------------------------
// Scale policies ("Online Quantization During Training", section 4 and its
// worked example; "Introduction to LLM Quantization", "5) Online Quantization",
// delayed quantization): 1x128 tiles cast with GIVEN scales (a policy's, e.g.
// from a tile-maximum history) instead of their own maxima.  Same tiling as
// quant_act_1x128_kernel.  Each tile's maximum is recorded for the history
// update, and the elements the saturating cast clamps (|fl32(x / s)| > 464:
// above that, round-to-nearest-even would leave 448) are counted.  A given
// scale need not bound the tile, so the cast divides (IEEE) instead of using
// the reciprocal form, whose exactness was checked only for s = max|tile|/448.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kQ1Threads)
quant_act_1x128_scaled_kernel(const __nv_bfloat16* __restrict__ x, int64_t M, int64_t KB, int64_t ldx,
                              const float* __restrict__ sf_in, int64_t ld_sf_in, uint8_t* __restrict__ q, int64_t ldq,
                              float* __restrict__ amax_out, int64_t ld_amax, unsigned long long* __restrict__ clipped) {
  const int tid = threadIdx.x;
  const int sub = tid & 3;
  const int tile = tid >> 2;
  const int64_t items = ((M + kQ1Rows - 1) / kQ1Rows) * KB;
  unsigned int nclip = 0;
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
    const int64_t rb = it / KB;
    const int64_t kb = it - rb * KB;
    const int64_t row = rb * kQ1Rows + tile;
    Q1Slice cur;
    q1_load<false>(cur, x, M, KB, ldx, nullptr, 0, it, tile, sub);
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m2 = amax2(m2, cur.v[i].x); m2 = amax2(m2, cur.v[i].y);
      m2 = amax2(m2, cur.v[i].z); m2 = amax2(m2, cur.v[i].w);
    }
    float m = amax2_value(m2);
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    if (row < M) {
      const float s = sf_in[kb * ld_sf_in + row];
      uint8_t* dst = q + row * ldq + kb * 128 + sub * 8;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t w[4] = {cur.v[i].x, cur.v[i].y, cur.v[i].z, cur.v[i].w};
        uint32_t c[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float v0 = __fdiv_rn(bf16lo(w[2 * j]), s), v1 = __fdiv_rn(bf16hi(w[2 * j]), s);
          const float v2 = __fdiv_rn(bf16lo(w[2 * j + 1]), s), v3 = __fdiv_rn(bf16hi(w[2 * j + 1]), s);
          nclip += (fabsf(v0) > 464.0f) + (fabsf(v1) > 464.0f) + (fabsf(v2) > 464.0f) + (fabsf(v3) > 464.0f);
          c[j] = cvt_e4m3x2(v0, v1) | (cvt_e4m3x2(v2, v3) << 16);
        }
        *reinterpret_cast<uint2*>(dst + 32 * i) = make_uint2(c[0], c[1]);
      }
      if (sub == 0 && amax_out != nullptr) amax_out[kb * ld_amax + row] = m;
    }
  }
  if (clipped != nullptr) {
    const unsigned int warp_clip = __reduce_add_sync(0xFFFFFFFFu, nclip);
    if ((tid & 31) == 0 && warp_clip != 0) atomicAdd(clipped, static_cast<unsigned long long>(warp_clip));
  }
}

// ---------------------------------------------------------------------------
// Percentile clipping ("Online Quantization During Training", section 4): the
// tile's scale comes from its rank-th largest magnitude v (nearest-rank
// percentile; rank 1 is the online rule), s = max(fl32(v/448), fl32(1e-12)),
// and the values above v saturate.  Same tiling as quant_act_1x128_kernel.
//
// Selection: BF16 magnitudes order like their 15-bit patterns, so the four
// lanes of a tile walk the distinct magnitudes downwards from the maximum g:
// each round counts #(|x| >= g) and finds the largest magnitude below g, two
// 16x2 packed operations per word (bit 15 of (mag | 0x8000) - g is set exactly
// when mag >= g, with no borrow between the halves).  The walk stops at the
// first g whose count reaches rank, which is the rank-th largest magnitude.
// Every round raises the count by at least one, so it ends within rank rounds;
// the warp loops until all of its tiles are done, which keeps the shuffles
// warp-uniform.
//
// Cast: |x| <= v is cast without division (exact for every BF16 x, v with
// |x| <= v and s = tile_scale(v)) and never saturates.  A lane holding values
// above v recasts them from the IEEE quotient fl32(x / s) (which the 1e-12
// floor of s can keep small, and which can overflow to infinity: it is clamped
// to +-448 first) and counts those with |fl32(x / s)| > 464 as clipped.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t slice_rank_walk(const Q1Slice& d, uint32_t g, uint32_t* next) {
  const uint32_t gg = g * 0x00010001u;
  uint32_t cnt2 = 0, nm = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t w[4] = {d.v[i].x, d.v[i].y, d.v[i].z, d.v[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t ge = ((w[j] | 0x80008000u) - gg) & 0x80008000u;   // bit 15/31: mag >= g
      const uint32_t one = ge >> 15;
      cnt2 += one;
      const uint32_t below = w[j] & ~(ge - one) & 0x7FFF7FFFu;          // magnitudes < g, else 0
      asm("max.u16x2 %0, %0, %1;" : "+r"(nm) : "r"(below));
    }
  }
  *next = max(nm & 0xFFFFu, nm >> 16);
  return (cnt2 & 0xFFFFu) + (cnt2 >> 16);
}

__global__ void __launch_bounds__(kQ1Threads)
quant_act_1x128_percentile_kernel(const __nv_bfloat16* __restrict__ x, int64_t M, int64_t KB, int64_t ldx, int rank,
                                  uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ sf, int64_t ld_sf,
                                  unsigned long long* __restrict__ clipped) {
  const int tid = threadIdx.x;
  const int sub = tid & 3;
  const int tile = tid >> 2;
  const int64_t items = ((M + kQ1Rows - 1) / kQ1Rows) * KB;
  int64_t it = blockIdx.x;
  unsigned int nclip = 0;
  if (it < items) {
    Q1Slice cur, nxt;
    q1_load<false>(cur, x, M, KB, ldx, nullptr, 0, it, tile, sub);
    for (; it < items; it += gridDim.x) {
      const int64_t it_next = it + gridDim.x;
      if (it_next < items) q1_load<false>(nxt, x, M, KB, ldx, nullptr, 0, it_next, tile, sub);
      const int64_t rb = it / KB;
      const int64_t kb = it - rb * KB;
      const int64_t row = rb * kQ1Rows + tile;
      uint32_t m2 = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        m2 = amax2(m2, cur.v[i].x); m2 = amax2(m2, cur.v[i].y);
        m2 = amax2(m2, cur.v[i].z); m2 = amax2(m2, cur.v[i].w);
      }
      const uint32_t lane_max = max(m2 & 0xFFFFu, m2 >> 16);
      uint32_t g = max(lane_max, __shfl_xor_sync(0xFFFFFFFFu, lane_max, 1));
      g = max(g, __shfl_xor_sync(0xFFFFFFFFu, g, 2));
      bool done = rank <= 1;
      for (int round = 0; round < 128; ++round) {
        if (__all_sync(0xFFFFFFFFu, done)) break;
        uint32_t next;
        uint32_t cnt = slice_rank_walk(cur, g, &next);
        cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, 1);
        cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, 2);
        next = max(next, __shfl_xor_sync(0xFFFFFFFFu, next, 1));
        next = max(next, __shfl_xor_sync(0xFFFFFFFFu, next, 2));
        if (!done) {
          if (cnt >= static_cast<uint32_t>(rank)) done = true;
          else g = next;
        }
      }
      const float s = tile_scale(__uint_as_float(g << 16));
      const float nr = -__frcp_rn(s);
      if (row < M) {
        uint2 o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          o[i].x = quant_words(cur.v[i].x, cur.v[i].y, nr, s);
          o[i].y = quant_words(cur.v[i].z, cur.v[i].w, nr, s);
        }
        if (lane_max > g) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t w[4] = {cur.v[i].x, cur.v[i].y, cur.v[i].z, cur.v[i].w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const uint32_t bits = (w[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
              if ((bits & 0x7FFFu) > g) {
                const float qv = __fdiv_rn(__uint_as_float(bits << 16), s);
                nclip += fabsf(qv) > 464.0f;
                const uint32_t code = cvt_e4m3x2(fminf(fmaxf(qv, -448.0f), 448.0f), 0.0f) & 0xFFu;
                uint32_t& word = (e < 4) ? o[i].x : o[i].y;
                const int sh = 8 * (e & 3);
                word = (word & ~(0xFFu << sh)) | (code << sh);
              }
            }
          }
        }
        uint8_t* dst = q + row * ldq + kb * 128 + sub * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) *reinterpret_cast<uint2*>(dst + 32 * i) = o[i];
        if (sub == 0) sf[kb * ld_sf + row] = s;
      }
      cur = nxt;
    }
  }
  if (clipped != nullptr) {
    const unsigned int warp_clip = __reduce_add_sync(0xFFFFFFFFu, nclip);
    if ((tid & 31) == 0 && warp_clip != 0) atomicAdd(clipped, static_cast<unsigned long long>(warp_clip));
  }
}

// One history step per tile: h <- policy(h, amax), sf <- max(fl32(h / 448),
// fl32(1e-12)).  Policies: 0 previous step (h = a), 1 exponential history
// (h = fl32(fl32(alpha*h) + fl32(fl32(1 - alpha)*a))), 2 decaying maximum
// (h = max(a, fl32(alpha*h))); every operation rounded on its own.
__global__ void scale_history_update_kernel(int policy, float alpha, const float* __restrict__ a,
                                            float* __restrict__ h, float* __restrict__ sf, int64_t n) {
  const float beta = __fsub_rn(1.0f, alpha);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float ai = a[i];
    float nh;
    if (policy == 0) {
      nh = ai;
    } else if (policy == 1) {
      nh = __fadd_rn(__fmul_rn(alpha, h[i]), __fmul_rn(beta, ai));
    } else {
      nh = fmaxf(ai, __fmul_rn(alpha, h[i]));
    }
    h[i] = nh;
    sf[i] = tile_scale(nh);
  }
}

// ---------------------------------------------------------------------------
// 128x1 tiles along the token dimension, written transposed.  A 256-thread
// block stages 128-token x 128-channel BF16 tiles (32 KB) in shared memory
// with cp.async, double-buffered so the next tile's copy overlaps this one's
// cast.  Thread t owns the channel pair p = t % 64 for the 32-token
// quarter r = t / 64: a bank-conflict-free 32-bit shared load per token gives
// both channels, the four quarters' maxima combine through shared memory, and
// the codes go back through the staged tile as [channel][128 tokens] rows so
// that the block writes whole 128-byte rows of qt.
// ---------------------------------------------------------------------------
constexpr int kQTThreads = 256;
constexpr int kQTCols = 128;
constexpr int kQTTileBytes = 128 * kQTCols * 2;                 // 32 KB staged BF16 tile
constexpr int kQTSmem = 2 * kQTTileBytes + 4 * kQTCols * 4;     // double buffer + per-quarter maxima

// Stage item `it` (128 tokens x up to 128 channels) into `tile` with cp.async.
__device__ __forceinline__ void qt_stage(uint32_t* tile, const __nv_bfloat16* __restrict__ x, int64_t C, int64_t ldx,
                                         int64_t col_blocks, int64_t it, int tid) {
  const int64_t tb = it / col_blocks;
  const int64_t c0 = (it - tb * col_blocks) * kQTCols;
  const int64_t ncols = (C - c0) < kQTCols ? (C - c0) : kQTCols;   // multiple of 8
  const int chunks_per_row = static_cast<int>(ncols / 8);
  for (int i = tid; i < 128 * (kQTCols / 8); i += kQTThreads) {
    const int rr = i / (kQTCols / 8);
    const int cc = i % (kQTCols / 8);
    if (cc < chunks_per_row) cp_async16(&tile[rr * (kQTCols / 2) + cc * 4], x + (tb * 128 + rr) * ldx + c0 + cc * 8);
  }
  cp_async_commit();
}

// Write the 128x1 codes of a 128-token x ncols tile transposed (qt rows c0 +
// c, columns tb*128 ..), through 16 KB of shared memory that every thread has
// finished reading.  Thread (p = tid % 64, r = tid / 64) holds channel 2p's
// tokens 32r .. +15 and +16 .. +31 in codes[0], codes[1], and channel 2p+1's
// in codes[2], codes[3].  Channel row c keeps its 16-byte chunk j at slot
// j ^ ((c / 2) % 8), so the 8 lanes of a wavefront hit 8 different bank
// groups both when the rows are written and when they are read back; each
// warp store instruction then writes 4 whole 128-byte rows of qt.
__device__ __forceinline__ void qt_store_transposed(uint8_t* smem16k, const uint4 (&codes)[4], bool active,
                                                    int64_t tb, int64_t c0, int64_t ncols,
                                                    uint8_t* __restrict__ qt, int64_t ldqt, int64_t qt_rows, int tid) {
  const int p = tid & 63;
  const int r = tid >> 6;
  __syncthreads();
  uint4* crows = reinterpret_cast<uint4*>(smem16k);
  if (active) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = 2 * r + h;
      crows[(2 * p) * 8 + (j ^ (p & 7))] = codes[h];
      crows[(2 * p + 1) * 8 + (j ^ (p & 7))] = codes[2 + h];
    }
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  for (int row = 4 * warp + (lane >> 3); row < ncols; row += 4 * (kQTThreads / 32)) {
    const int j = lane & 7;
    if (chk(c0 + row, qt_rows, CHK_QT) && chk(tb * 128 + 16 * j + 15, ldqt, CHK_QT))
      *reinterpret_cast<uint4*>(qt + (c0 + row) * ldqt + tb * 128 + 16 * j) = crows[row * 8 + (j ^ ((row >> 1) & 7))];
  }
}

// Cast one staged BF16 tile -- 128 tokens x ncols (<= 128) channels, row t
// at tile_bytes + 256 t -- as 128x1 tiles: each channel's maximum over the
// 128 tokens (the four token quarters combine through qmax), its scale into
// sf[tb * ld_sf + c0 + c], and its 128 codes transposed into row c0 + c of
// qt.  The staged tile is overwritten by the transposed codes.  Every thread
// of the block calls it (it synchronizes the block).
template <int kFmt = kFmtE4M3>
__device__ __forceinline__ void qt_cast_staged(uint8_t* tile_bytes, float* qmax, int64_t tb, int64_t c0,
                                               int64_t ncols, uint8_t* __restrict__ qt, int64_t ldqt,
                                               float* __restrict__ sf, int64_t ld_sf, int64_t C, int tid) {
  const int p = tid & 63;          // channel pair
  const int r = tid >> 6;          // token quarter
  constexpr int kWords = kQTCols / 2;   // 64 words per staged row
  const uint32_t* tile = reinterpret_cast<const uint32_t*>(tile_bytes);
  const bool active = 2 * p < ncols;
  uint4 codes[4];                  // channel 2p: tokens 32r .. +15, +16 .. +31; then channel 2p+1
  float ma = 0.0f, mb = 0.0f;
  if (active) {
    uint32_t m2 = 0;   // channel 2p in the low half, 2p+1 in the high half
#pragma unroll 8
    for (int t = 32 * r; t < 32 * r + 32; ++t) m2 = amax2_sx(m2, tile[t * kWords + p]);
    m2 = amax2_sx_bits(m2);
    ma = bf16lo(m2);
    mb = bf16hi(m2);
  }
  qmax[r * kQTCols + 2 * p] = ma;
  qmax[r * kQTCols + 2 * p + 1] = mb;
  __syncthreads();
  if (active) {
    ma = fmaxf(fmaxf(qmax[2 * p], qmax[kQTCols + 2 * p]), fmaxf(qmax[2 * kQTCols + 2 * p], qmax[3 * kQTCols + 2 * p]));
    mb = fmaxf(fmaxf(qmax[2 * p + 1], qmax[kQTCols + 2 * p + 1]),
               fmaxf(qmax[2 * kQTCols + 2 * p + 1], qmax[3 * kQTCols + 2 * p + 1]));
    const float sa = tile_scale_fmt<kFmt>(ma), sb = tile_scale_fmt<kFmt>(mb);
    const float nra = -__frcp_rn(sa), nrb = -__frcp_rn(sb);
    const int64_t ca = c0 + 2 * p;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t oa[4], ob[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t a4 = 0, b4 = 0;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = 32 * r + 16 * h + 4 * j + 2 * e;
          const uint32_t w0 = tile[t * kWords + p];
          const uint32_t w1 = tile[(t + 1) * kWords + p];
          a4 |= fp8x2_neg_quot<kFmt>(bf16lo(w0), bf16lo(w1), nra, nra, sa, sa) << (16 * e);
          b4 |= fp8x2_neg_quot<kFmt>(bf16hi(w0), bf16hi(w1), nrb, nrb, sb, sb) << (16 * e);
        }
        oa[j] = a4 ^ kFlipSigns;
        ob[j] = b4 ^ kFlipSigns;
      }
      codes[h] = make_uint4(oa[0], oa[1], oa[2], oa[3]);
      codes[2 + h] = make_uint4(ob[0], ob[1], ob[2], ob[3]);
    }
    if (r == 0 && chk(ca + 1, ld_sf, CHK_QT_SF)) {
      sf[tb * ld_sf + ca] = sa;
      sf[tb * ld_sf + ca + 1] = sb;
    }
  }
  qt_store_transposed(tile_bytes, codes, active, tb, c0, ncols, qt, ldqt, C, tid);
}

template <int kFmt = kFmtE4M3>
__global__ void __launch_bounds__(kQTThreads)
quant_act_128x1_kernel(const __nv_bfloat16* __restrict__ x, int64_t T, int64_t C, int64_t ldx,
                       uint8_t* __restrict__ qt, int64_t ldqt, float* __restrict__ sf, int64_t ld_sf) {
  extern __shared__ __align__(128) uint8_t q2_smem[];
  float* qmax = reinterpret_cast<float*>(q2_smem + 2 * kQTTileBytes);   // [4 quarters][128 channels]
  const int tid = threadIdx.x;
  const int64_t col_blocks = (C + kQTCols - 1) / kQTCols;
  const int64_t items = (T / 128) * col_blocks;
  int64_t it = blockIdx.x;
  if (it >= items) return;
  int buf = 0;
  qt_stage(reinterpret_cast<uint32_t*>(q2_smem), x, C, ldx, col_blocks, it, tid);
  for (; it < items; it += gridDim.x, buf ^= 1) {
    // prefetch the next item into the other buffer while this one is cast
    const int64_t next = it + gridDim.x;
    if (next < items) {
      qt_stage(reinterpret_cast<uint32_t*>(q2_smem + (buf ^ 1) * kQTTileBytes), x, C, ldx, col_blocks, next, tid);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int64_t tb = it / col_blocks;
    const int64_t c0 = (it - tb * col_blocks) * kQTCols;
    const int64_t ncols = (C - c0) < kQTCols ? (C - c0) : kQTCols;
    qt_cast_staged<kFmt>(q2_smem + buf * kQTTileBytes, qmax, tb, c0, ncols, qt, ldqt, sf, ld_sf, C, tid);
    __syncthreads();   // this buffer is refilled two items later; the maxima are reused next item
  }
}

// ---------------------------------------------------------------------------
// Both tile orientations from one read: the 1x128 quantization (the operand of
// the forward GEMM or of Dgrad) and the 128x1 transposed quantization (the
// operand of Wgrad) of the same BF16 tensor ("Fine-Grained FP8 Quantization in
// DeepSeek", section 2 and section 4 "transpose layout"; "Introduction to LLM
// Quantization", "3) Backward propagation": the gradient is needed in both).
// Each 128-token x 128-channel tile is staged once in shared memory: its 128
// rows are 128 1x128 tiles, its 128 columns 128 128x1 tiles.  Codes and scales
// are those of quant_act_1x128_kernel and quant_act_128x1_kernel exactly.
//
// The staged tile is swizzled -- 16-byte chunk j of token row t at chunk
// j ^ (t % 16) -- so that both passes read it without bank conflicts: the
// 1x128 pass gives 4 lanes to a row (chunks sub + 4i, as in the 1x128
// kernel), the 128x1 pass gives a warp 32 consecutive channel-pair words of one
// row.  Requires C % 128 == 0 (whole tiles).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void dual_stage(uint32_t* tile, const __nv_bfloat16* __restrict__ x, int64_t ldx,
                                           int64_t col_blocks, int64_t it, int tid) {
  const int64_t tb = it / col_blocks;
  const int64_t c0 = (it - tb * col_blocks) * 128;
  for (int i = tid; i < 128 * 16; i += kQTThreads) {
    const int rr = i >> 4, cc = i & 15;
    cp_async16(&tile[rr * 64 + ((cc ^ (rr & 15)) << 2)], x + (tb * 128 + rr) * ldx + c0 + cc * 8);
  }
  cp_async_commit();
}

// The next tile is staged while this one is cast (two 32 KB buffers, 3 blocks
// per SM; one buffer and 6 blocks per SM measured 5 % slower on B200).
template <int kFmt = kFmtE4M3>
__global__ void __launch_bounds__(kQTThreads)
quant_act_dual_kernel(const __nv_bfloat16* __restrict__ x, int64_t T, int64_t C, int64_t ldx,
                      uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ sf, int64_t ld_sf,
                      uint8_t* __restrict__ qt, int64_t ldqt, float* __restrict__ sft, int64_t ld_sft) {
  extern __shared__ __align__(128) uint8_t qd_smem[];
  float* qmax = reinterpret_cast<float*>(qd_smem + 2 * kQTTileBytes);   // [4 quarters][128 channels]
  const int tid = threadIdx.x;
  const int64_t col_blocks = C / 128;
  const int64_t items = (T / 128) * col_blocks;
  int64_t it = blockIdx.x;
  if (it >= items) return;
  int buf = 0;
  dual_stage(reinterpret_cast<uint32_t*>(qd_smem), x, ldx, col_blocks, it, tid);
  for (; it < items; it += gridDim.x, buf ^= 1) {
    const int64_t next = it + gridDim.x;
    if (next < items) {
      dual_stage(reinterpret_cast<uint32_t*>(qd_smem + (buf ^ 1) * kQTTileBytes), x, ldx, col_blocks, next, tid);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int64_t tb = it / col_blocks;
    const int64_t cb = it - tb * col_blocks;
    uint8_t* tile_bytes = qd_smem + buf * kQTTileBytes;
    const uint4* tile16 = reinterpret_cast<const uint4*>(tile_bytes);
    const uint32_t* tile = reinterpret_cast<const uint32_t*>(tile_bytes);

    // ---- 1x128 tiles: the 128 token rows, 4 lanes a row, 64 rows a pass
    {
      const int sub = tid & 3;
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        const int r = 64 * pass + (tid >> 2);
        uint4 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = tile16[r * 16 + ((sub + 4 * i) ^ (r & 15))];
        uint32_t m2 = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          m2 = amax2_sx(m2, v[i].x); m2 = amax2_sx(m2, v[i].y);
          m2 = amax2_sx(m2, v[i].z); m2 = amax2_sx(m2, v[i].w);
        }
        float m = amax2_value(amax2_sx_bits(m2));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
        const float s = tile_scale_fmt<kFmt>(m);
        const float nr = -__frcp_rn(s);
        const int64_t row = tb * 128 + r;
        uint8_t* dst = q + row * ldq + cb * 128 + sub * 8;
        if (chk(row, T, CHK_Q1) && chk(cb * 128 + sub * 8 + 32 * 3 + 7, ldq, CHK_Q1)) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint2 o;
            o.x = quant_words<kFmt>(v[i].x, v[i].y, nr, s);
            o.y = quant_words<kFmt>(v[i].z, v[i].w, nr, s);
            *reinterpret_cast<uint2*>(dst + 32 * i) = o;
          }
        }
        if (sub == 0 && chk(row, ld_sf, CHK_Q1_SF)) sf[cb * ld_sf + row] = s;
      }
    }

    // ---- 128x1 tiles: the 128 channel columns (as qt_cast_staged, on the swizzled tile)
    {
      const int p = tid & 63;          // channel pair
      const int r = tid >> 6;          // token quarter
      uint4 codes[4];
      // word p of token row 32r + k sits at k * 64 + woff[k % 16] from row 32r
      // (32r is a multiple of 16, so the swizzle depends on k alone): the 16
      // offsets are formed once and every load below is a base plus a constant
      const uint32_t* trow = tile + 32 * r * 64;
      int woff[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) woff[c] = (((p >> 2) ^ c) << 2) + (p & 3);
      uint32_t m2 = 0;
#pragma unroll
      for (int k = 0; k < 32; ++k) m2 = amax2_sx(m2, trow[k * 64 + woff[k & 15]]);
      m2 = amax2_sx_bits(m2);
      float ma = bf16lo(m2), mb = bf16hi(m2);
      qmax[r * 128 + 2 * p] = ma;
      qmax[r * 128 + 2 * p + 1] = mb;
      __syncthreads();
      ma = fmaxf(fmaxf(qmax[2 * p], qmax[128 + 2 * p]), fmaxf(qmax[256 + 2 * p], qmax[384 + 2 * p]));
      mb = fmaxf(fmaxf(qmax[2 * p + 1], qmax[128 + 2 * p + 1]), fmaxf(qmax[256 + 2 * p + 1], qmax[384 + 2 * p + 1]));
      const float sa = tile_scale_fmt<kFmt>(ma), sb = tile_scale_fmt<kFmt>(mb);
      const float nra = -__frcp_rn(sa), nrb = -__frcp_rn(sb);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t oa[4], ob[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t a4 = 0, b4 = 0;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int k = 16 * h + 4 * j + 2 * e;   // token 32r + k
            const uint32_t w0 = trow[k * 64 + woff[k & 15]];
            const uint32_t w1 = trow[(k + 1) * 64 + woff[(k + 1) & 15]];
            a4 |= fp8x2_neg_quot<kFmt>(bf16lo(w0), bf16lo(w1), nra, nra, sa, sa) << (16 * e);
            b4 |= fp8x2_neg_quot<kFmt>(bf16hi(w0), bf16hi(w1), nrb, nrb, sb, sb) << (16 * e);
          }
          oa[j] = a4 ^ kFlipSigns;
          ob[j] = b4 ^ kFlipSigns;
        }
        codes[h] = make_uint4(oa[0], oa[1], oa[2], oa[3]);
        codes[2 + h] = make_uint4(ob[0], ob[1], ob[2], ob[3]);
      }
      if (r == 0 && chk(cb * 128 + 2 * p + 1, ld_sft, CHK_QT_SF)) {
        sft[tb * ld_sft + cb * 128 + 2 * p] = sa;
        sft[tb * ld_sft + cb * 128 + 2 * p + 1] = sb;
      }
      // the transposed codes leave through the tile's first 16 KB once every
      // thread has finished reading it (both passes)
      qt_store_transposed(tile_bytes, codes, true, tb, cb * 128, 128, qt, ldqt, C, tid);
    }
    __syncthreads();   // this buffer is refilled two items later; the maxima are reused next item
  }
}

// ---------------------------------------------------------------------------
// FP8 activation caching ("FP8 Mixed Precision: DeepSeek-V3 Training
// Architecture", section 4: activations are cached in FP8 for the backward
// pass, halving their memory).  The forward pass keeps only the 1x128-tile
// codes and scales it already made for Fprop; Wgrad needs the activation in
// 128x1 tiles along tokens, transposed.  This kernel rebuilds that operand
// from the cache: each element is dequantized to BF16, xh = RN_bf16(e4m3(q) *
// s) (the exact product rounded once), and the BF16 tile is quantized 128x1
// exactly as quant_act_128x1_kernel quantizes a BF16 activation.
//
// A 256-thread block handles 128 tokens x 128 channels (one 1x128 tile column
// kb, so one scale per token): the codes (16 KB) and the 128 token scales are
// staged with cp.async, double-buffered.  Thread (p, r) dequantizes channels
// 2p, 2p+1 of tokens 32r .. +31 into registers as BF16 pairs, the four token
// quarters combine their channel maxima through shared memory, and the codes
// leave transposed through the stage's code buffer (qt_store_transposed).
// ---------------------------------------------------------------------------
constexpr int kRQCodeBytes = 128 * 128;
constexpr int kRQStageBytes = kRQCodeBytes + 128 * 4;
constexpr int kRQSmem = 2 * kRQStageBytes + 4 * kQTCols * 4;

__device__ __forceinline__ void rq_stage(uint8_t* st, const uint8_t* __restrict__ q, int64_t ldq,
                                         const float* __restrict__ sf, int64_t ld_sf, int64_t col_blocks, int64_t it,
                                         int tid) {
  const int64_t tb = it / col_blocks;
  const int64_t kb = it - tb * col_blocks;
  for (int i = tid; i < 128 * 8; i += kQTThreads) {
    const int rr = i >> 3, cc = i & 7;
    cp_async16(st + rr * 128 + cc * 16, q + (tb * 128 + rr) * ldq + kb * 128 + cc * 16);
  }
  if (tid < 32) cp_async16(st + kRQCodeBytes + 16 * tid, sf + kb * ld_sf + tb * 128 + 4 * tid);
  cp_async_commit();
}

// The BF16 bits of the exact product c * s, rounded once to nearest-even,
// from p = fl32(c * s) and its exact error e = c * s - p: p rounds like the
// exact product unless p is itself a BF16 midpoint and e != 0, in which case
// the sign of e says on which side of the midpoint the product lies.
__device__ __forceinline__ uint32_t bf16_at_midpoint(float p, float e, uint32_t rne) {
  const uint32_t u = __float_as_uint(p);
  if ((u & 0xFFFFu) != 0x8000u || e == 0.0f) return rne;
  return (u >> 16) + (((e > 0.0f) == (p > 0.0f)) ? 1u : 0u);
}

// Two E4M3 codes (low byte first) -> the BF16 pair RN_bf16(code * s), low
// first.  Decoding: an E4M3 code's 7 magnitude bits shifted left by 20, read
// as FP32, are exactly 2^-120 times its value -- the 4 exponent bits land in
// the float's exponent field and the subnormal codes on FP32 subnormals with
// the same ratio -- so one exact multiply by 2^120 decodes two codes at once.
// The common case rounds both products with one packed conversion; the rare
// product that float32 rounding put on a BF16 midpoint is fixed by its error.
__device__ __forceinline__ uint32_t dequant_bf16x2(uint32_t c2, float s) {
  const uint32_t b0 = ((c2 & 0x7Fu) << 20) | ((c2 & 0x80u) << 24);
  const uint32_t b1 = ((c2 & 0x7F00u) << 12) | ((c2 & 0x8000u) << 16);
  const float2 v = fmul2(f2u(b0, b1), f2(0x1p120f));
  const float2 sv = f2(s);
  const float2 p = fmul2(v, sv);
  const __nv_bfloat162 h = __floats2bfloat162_rn(p.x, p.y);
  uint32_t r = *reinterpret_cast<const uint32_t*>(&h);
  const uint32_t u0 = __float_as_uint(p.x), u1 = __float_as_uint(p.y);
  if (((u0 & 0xFFFFu) == 0x8000u) | ((u1 & 0xFFFFu) == 0x8000u)) {
    const float2 e = ffma2(v, sv, make_float2(-p.x, -p.y));
    r = bf16_at_midpoint(p.x, e.x, r & 0xFFFFu) | (bf16_at_midpoint(p.y, e.y, r >> 16) << 16);
  }
  return r;
}

__global__ void __launch_bounds__(kQTThreads)
requant_1x128_to_128x1_kernel(const uint8_t* __restrict__ q, int64_t T, int64_t C, int64_t ldq,
                              const float* __restrict__ sf_in, int64_t ld_sf_in, uint8_t* __restrict__ qt,
                              int64_t ldqt, float* __restrict__ sf, int64_t ld_sf) {
  extern __shared__ __align__(128) uint8_t rq_smem[];
  float* qmax = reinterpret_cast<float*>(rq_smem + 2 * kRQStageBytes);   // [4 quarters][128 channels]
  const int tid = threadIdx.x;
  const int p = tid & 63;          // channel pair
  const int r = tid >> 6;          // token quarter
  const int64_t col_blocks = C / 128;
  const int64_t items = (T / 128) * col_blocks;
  int64_t it = blockIdx.x;
  if (it >= items) return;
  int buf = 0;
  rq_stage(rq_smem, q, ldq, sf_in, ld_sf_in, col_blocks, it, tid);
  for (; it < items; it += gridDim.x, buf ^= 1) {
    const int64_t next = it + gridDim.x;
    if (next < items) {
      rq_stage(rq_smem + (buf ^ 1) * kRQStageBytes, q, ldq, sf_in, ld_sf_in, col_blocks, next, tid);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    uint8_t* st = rq_smem + buf * kRQStageBytes;
    const float* tok_scale = reinterpret_cast<const float*>(st + kRQCodeBytes);
    // channels 2p, 2p+1 of tokens 32r .. 32r+31, dequantized to BF16 pairs
    uint32_t w[32];
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int t = 32 * r + i;
      const uint32_t c2 = *reinterpret_cast<const uint16_t*>(st + t * 128 + 2 * p);
      w[i] = dequant_bf16x2(c2, tok_scale[t]);
      m2 = amax2(m2, w[i]);
    }
    qmax[r * kQTCols + 2 * p] = bf16lo(m2);
    qmax[r * kQTCols + 2 * p + 1] = bf16hi(m2);
    __syncthreads();
    const float ma = fmaxf(fmaxf(qmax[2 * p], qmax[kQTCols + 2 * p]),
                           fmaxf(qmax[2 * kQTCols + 2 * p], qmax[3 * kQTCols + 2 * p]));
    const float mb = fmaxf(fmaxf(qmax[2 * p + 1], qmax[kQTCols + 2 * p + 1]),
                           fmaxf(qmax[2 * kQTCols + 2 * p + 1], qmax[3 * kQTCols + 2 * p + 1]));
    const float sa = tile_scale(ma), sb = tile_scale(mb);
    const float nra = -__frcp_rn(sa), nrb = -__frcp_rn(sb);
    uint4 codes[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t oa[4], ob[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t a4 = 0, b4 = 0;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int i = 16 * h + 4 * j + 2 * e;
          a4 |= e4m3x2_neg_quot(bf16lo(w[i]), bf16lo(w[i + 1]), nra, nra, sa, sa) << (16 * e);
          b4 |= e4m3x2_neg_quot(bf16hi(w[i]), bf16hi(w[i + 1]), nrb, nrb, sb, sb) << (16 * e);
        }
        oa[j] = a4 ^ kFlipSigns;
        ob[j] = b4 ^ kFlipSigns;
      }
      codes[h] = make_uint4(oa[0], oa[1], oa[2], oa[3]);
      codes[2 + h] = make_uint4(ob[0], ob[1], ob[2], ob[3]);
    }
    const int64_t tb = it / col_blocks;
    const int64_t c0 = (it - tb * col_blocks) * kQTCols;
    if (r == 0) {
      sf[tb * ld_sf + c0 + 2 * p] = sa;
      sf[tb * ld_sf + c0 + 2 * p + 1] = sb;
    }
    qt_store_transposed(st, codes, true, tb, c0, kQTCols, qt, ldqt, C, tid);
    __syncthreads();   // this stage buffer is refilled next item; the maxima are reused
  }
}

// ---------------------------------------------------------------------------
// 128x128 weight blocks, with the optional transposed copy for Dgrad.  One
// 256-thread block per weight block; thread t owns the 8x8 sub-block at rows
// 8*(t/16).., columns 8*(t%16)..: eight 16-byte row loads (16 lanes cover one
// 256-byte row), block amax via shuffles and shared memory, eight 8-byte Q
// stores, and, for Q^T, an in-register 8x8 byte transpose (byte permutes)
// whose rows go through a 16 KB shared buffer so that the block writes whole
// 128-byte rows of Q^T.
// ---------------------------------------------------------------------------
constexpr int kQWThreads = 256;

// 4x4 byte transpose: in a[i] = row i (byte j = column j); out c[j] = column j.
__device__ __forceinline__ void transpose4x4(const uint32_t a0, const uint32_t a1, const uint32_t a2,
                                             const uint32_t a3, uint32_t (&c)[4]) {
  const uint32_t t0 = __byte_perm(a0, a1, 0x5140);   // a0.b0 a1.b0 a0.b1 a1.b1
  const uint32_t t1 = __byte_perm(a0, a1, 0x7362);   // a0.b2 a1.b2 a0.b3 a1.b3
  const uint32_t t2 = __byte_perm(a2, a3, 0x5140);
  const uint32_t t3 = __byte_perm(a2, a3, 0x7362);
  c[0] = __byte_perm(t0, t2, 0x5410);
  c[1] = __byte_perm(t0, t2, 0x7632);
  c[2] = __byte_perm(t1, t3, 0x5410);
  c[3] = __byte_perm(t1, t3, 0x7632);
}

__global__ void __launch_bounds__(kQWThreads, 3)
quant_w_128x128_kernel(const __nv_bfloat16* __restrict__ w, int64_t NB, int64_t KB, int64_t ldw,
                       uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ sf, int64_t ld_sf,
                       uint8_t* __restrict__ qt, int64_t ldqt, float* __restrict__ sft, int64_t ld_sft) {
  __shared__ float warp_max[kQWThreads / 32];
  __shared__ __align__(16) uint2 tstage[128 * 16];   // the block's codes transposed: [k][16 x 8 n]
  const int tid = threadIdx.x;
  const int a = tid >> 4;        // rows 8a .. 8a+7
  const int b = tid & 15;        // cols 8b .. 8b+7
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
      m2 = amax2_sx(m2, v[i].x); m2 = amax2_sx(m2, v[i].y);
      m2 = amax2_sx(m2, v[i].z); m2 = amax2_sx(m2, v[i].w);
    }
    float m = amax2_value(amax2_sx_bits(m2));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((tid & 31) == 0) warp_max[tid >> 5] = m;
    __syncthreads();
    m = warp_max[0];
#pragma unroll
    for (int i = 1; i < kQWThreads / 32; ++i) m = fmaxf(m, warp_max[i]);
    const float s = tile_scale(m);
    const float nr = -__frcp_rn(s);
    uint32_t lo[8], hi[8];   // row i: bytes of columns 0-3 (lo) and 4-7 (hi)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      lo[i] = quant_words(v[i].x, v[i].y, nr, s);
      hi[i] = quant_words(v[i].z, v[i].w, nr, s);
      if (chk(n0 + 8 * a + i, NB * 128, CHK_QW) && chk(k0 + 8 * b + 7, ldq, CHK_QW))
        *reinterpret_cast<uint2*>(q + (n0 + 8 * a + i) * ldq + k0 + 8 * b) = make_uint2(lo[i], hi[i]);
    }
    if (qt != nullptr) {
      uint32_t c00[4], c01[4], c10[4], c11[4];   // c<rowhalf><colhalf>
      transpose4x4(lo[0], lo[1], lo[2], lo[3], c00);
      transpose4x4(hi[0], hi[1], hi[2], hi[3], c01);
      transpose4x4(lo[4], lo[5], lo[6], lo[7], c10);
      transpose4x4(hi[4], hi[5], hi[6], hi[7], c11);
      // Q^T rows k0 + 8b + j, columns n0 + 8a .. +7, through shared memory:
      // 8-byte chunk a of row kk at slot a ^ (kk / 8 % 16), so the 16 lanes of
      // a wavefront (16 rows, one chunk each) hit 16 different slots; read back
      // a warp instruction writes 2 whole 128-byte rows of qt.
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        tstage[(8 * b + j) * 16 + (a ^ b)] = make_uint2(c00[j], c10[j]);
        tstage[(8 * b + 4 + j) * 16 + (a ^ b)] = make_uint2(c01[j], c11[j]);
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int kk = 16 * i + (tid >> 4);   // 16 rows per pass over the block's 256 threads
        const int c = tid & 15;
        if (chk(k0 + kk, KB * 128, CHK_QW) && chk(n0 + 8 * c + 7, ldqt, CHK_QW))
          *reinterpret_cast<uint2*>(qt + (k0 + kk) * ldqt + n0 + 8 * c) = tstage[kk * 16 + (c ^ ((kk >> 3) & 15))];
      }
    }
    if (tid == 0) {
      if (chk(kb, ld_sf, CHK_QW)) sf[nb * ld_sf + kb] = s;
      if (sft != nullptr && chk(nb, ld_sft, CHK_QW)) sft[kb * ld_sft + nb] = s;
    }
    __syncthreads();   // warp_max is reused by the next block
  }
}

// ---------------------------------------------------------------------------
// Diagnostics: the E4M3 cast over consecutive FP32 bit patterns.
// ---------------------------------------------------------------------------
__global__ void cast_e4m3_bits_kernel(uint32_t start, int64_t count, uint8_t* __restrict__ out) {
  const int64_t pairs = (count + 1) / 2;
  for (int64_t p = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; p < pairs;
       p += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t b0 = start + static_cast<uint32_t>(2 * p);
    const uint32_t code = cvt_e4m3x2(__uint_as_float(b0), __uint_as_float(b0 + 1u));
    out[2 * p] = static_cast<uint8_t>(code & 0xFF);
    if (2 * p + 1 < count) out[2 * p + 1] = static_cast<uint8_t>(code >> 8);
  }
}

// One block waits on a barrier that nothing completes; the bounded wait gives
// up after `budget` clocks and records FP8Q_ERR_TIMEOUT.
__global__ void wait_timeout_kernel(long long budget) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, WAIT_DEBUG, budget);
  __syncthreads();
}

}  // namespace fp8q

namespace fp8q {

// ---------------------------------------------------------------------------
// MoE dispatch ("FP8 Mixed Precision: DeepSeek-V3 Training Architecture",
// section 4: tokens sent to their experts' GPUs are quantized to FP8 on the
// fly, halving the all-to-all's bytes).
//
// Layout: the (token, slot) entries i = t * k + j with expert ids[i] are put
// in expert-major order, ties in entry order (a stable counting sort): rows[m]
// is the token of output row m, pos[i] the output row of entry i, and
// offsets[e] .. offsets[e+1] the rows of expert e.  Experts are assigned to
// ranks in contiguous ranges, so the order is also destination-rank-major.
// Three launches, deterministic: per-chunk expert histograms, one block that
// scans them, and one warp per chunk that places its entries in order (equal
// experts within 32 entries are ranked with __match_any_sync).  An id outside
// [0, E) records FP8Q_ERR_INVALID_ARG and its entry is dropped (pos = -1).
// ---------------------------------------------------------------------------
constexpr int kLayoutMaxExperts = 1024;

__global__ void __launch_bounds__(256)
moe_layout_hist_kernel(const int32_t* __restrict__ ids, int64_t n, int E, int64_t chunk, int32_t* __restrict__ hist) {
  __shared__ int32_t cnt[kLayoutMaxExperts];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int64_t lo = blockIdx.x * chunk;
  const int64_t hi = lo + chunk < n ? lo + chunk : n;
  for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x) {
    const int32_t e = ids[i];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
    else report_status(FP8Q_ERR_INVALID_ARG, BAD_EXPERT_ID);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[static_cast<int64_t>(blockIdx.x) * E + e] = cnt[e];
}

// One block of kLayoutMaxExperts threads: offsets[e] = sum of the counts of
// experts < e; starts[b][e] = offsets[e] + the counts of expert e in chunks < b.
__global__ void __launch_bounds__(kLayoutMaxExperts)
moe_layout_scan_kernel(const int32_t* __restrict__ hist, int nchunks, int E, int32_t* __restrict__ offsets,
                       int32_t* __restrict__ starts) {
  __shared__ int32_t tot[kLayoutMaxExperts];
  const int e = threadIdx.x;
  int32_t t = 0;
  if (e < E)
    for (int b = 0; b < nchunks; ++b) t += hist[static_cast<int64_t>(b) * E + e];
  tot[e] = e < E ? t : 0;
  __syncthreads();
  // inclusive scan over the experts (Hillis-Steele in shared memory)
  for (int d = 1; d < kLayoutMaxExperts; d <<= 1) {
    const int32_t v = e >= d ? tot[e - d] : 0;
    __syncthreads();
    tot[e] += v;
    __syncthreads();
  }
  if (e < E) {
    int32_t base = tot[e] - t;                // exclusive
    offsets[e] = base;
    for (int b = 0; b < nchunks; ++b) {
      starts[static_cast<int64_t>(b) * E + e] = base;
      base += hist[static_cast<int64_t>(b) * E + e];
    }
    if (e == E - 1) offsets[E] = base;
  }
}

__global__ void __launch_bounds__(32)
moe_layout_scatter_kernel(const int32_t* __restrict__ ids, int64_t n, int k, int E, int64_t chunk,
                          const int32_t* __restrict__ starts, int32_t* __restrict__ rows, int32_t* __restrict__ pos) {
  __shared__ int32_t next[kLayoutMaxExperts];
  const int lane = threadIdx.x;
  for (int e = lane; e < E; e += 32) next[e] = starts[static_cast<int64_t>(blockIdx.x) * E + e];
  __syncwarp();
  const int64_t lo = blockIdx.x * chunk;
  const int64_t hi = lo + chunk < n ? lo + chunk : n;
  for (int64_t seg = lo; seg < hi; seg += 32) {
    const int64_t i = seg + lane;
    int32_t e = i < hi ? ids[i] : -1;
    if (e >= E) e = -1;
    const unsigned same = __match_any_sync(0xFFFFFFFFu, e);
    const int before = __popc(same & ((1u << lane) - 1u));
    int32_t p = -1;
    if (e >= 0) p = next[e] + before;
    __syncwarp();
    if (e >= 0 && before == 0) next[e] += __popc(same);
    __syncwarp();
    if (i < hi) {
      pos[i] = p;
      if (p >= 0 && chk(p, n, CHK_LAYOUT)) rows[p] = static_cast<int32_t>(i / k);
    }
  }
}

// ---------------------------------------------------------------------------
// Regroup order of an expert-parallel dispatch, from the all-gathered layout
// offsets table off[s][0..E] of every source rank s.  This rank owns experts
// rank*el .. rank*el + el - 1.  Received rows are source-major, each source's
// rows expert-major; the output is expert-major, each expert's rows
// source-major.  Piece p = e * world + s holds cnt[p] = off[s][g+1] - off[s][g]
// rows (g = rank*el + e), which arrive at recv_start[p] = (rows of sources < s)
// + off[s][g] - off[s][rank*el] and leave at out_start[p] = the exclusive sum
// of cnt over pieces < p.  Every block rebuilds the piece table (at most 1024
// pieces) in shared memory; each thread then places its output rows by a binary
// search over out_start.  Block 0 writes the experts' output offsets.
// ---------------------------------------------------------------------------
constexpr int kRegroupOrderThreads = 1024;

__global__ void __launch_bounds__(kRegroupOrderThreads)
moe_regroup_order_kernel(const int32_t* __restrict__ off, int world, int rank, int E, int64_t M_recv,
                         int32_t* __restrict__ rows, int32_t* __restrict__ expert_offsets) {
  __shared__ int32_t cnt[kLayoutMaxExperts];
  __shared__ int32_t out_start[kLayoutMaxExperts];
  __shared__ int32_t recv_start[kLayoutMaxExperts];
  __shared__ int32_t src_tot[kLayoutMaxExperts];
  __shared__ int bad;
  const int el = E / world;
  const int P = el * world;                 // = E <= kLayoutMaxExperts
  const int t = threadIdx.x;
  if (t == 0) bad = 0;
  __syncthreads();
  const int64_t ld = E + 1;
  // rows each source sends to this rank, then their exclusive prefix over sources
  int32_t mine = 0;
  if (t < world) {
    const int32_t lo = off[t * ld + rank * el], hi = off[t * ld + rank * el + el];
    mine = hi - lo;
    if (lo < 0 || mine < 0) { bad = 1; mine = 0; }
  }
  src_tot[t] = mine;
  __syncthreads();
  for (int d = 1; d < kRegroupOrderThreads; d <<= 1) {   // inclusive scan over sources
    const int32_t v = t >= d ? src_tot[t - d] : 0;
    __syncthreads();
    src_tot[t] += v;
    __syncthreads();
  }
  // the piece table: thread t owns piece p = t (expert p / world, source p % world)
  int32_t c = 0;
  if (t < P) {
    const int e = t / world, s = t % world;
    const int64_t g = static_cast<int64_t>(s) * ld + rank * el + e;
    c = off[g + 1] - off[g];
    const int32_t within = off[g] - off[static_cast<int64_t>(s) * ld + rank * el];
    if (c < 0 || within < 0) { bad = 1; c = 0; }
    recv_start[t] = (s > 0 ? src_tot[s - 1] : 0) + within;
  }
  cnt[t] = c;
  out_start[t] = c;
  __syncthreads();
  for (int d = 1; d < kRegroupOrderThreads; d <<= 1) {   // inclusive scan over pieces
    const int32_t v = t >= d ? out_start[t - d] : 0;
    __syncthreads();
    out_start[t] += v;
    __syncthreads();
  }
  const int32_t incl = out_start[t];
  __syncthreads();
  out_start[t] = incl - cnt[t];                           // exclusive
  __syncthreads();
  const int64_t total = P > 0 ? static_cast<int64_t>(out_start[P - 1]) + cnt[P - 1] : 0;
  if (blockIdx.x == 0) {
    if (t < el) expert_offsets[t] = out_start[t * world];
    if (t == 0) expert_offsets[el] = static_cast<int32_t>(total);
    if (t == 0 && (bad || total != M_recv)) report_status(FP8Q_ERR_INVALID_ARG, BAD_COUNT_TABLE);
  }
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t m = static_cast<int64_t>(blockIdx.x) * blockDim.x + t; m < M_recv; m += stride) {
    if (m >= total) { rows[m] = -1; continue; }
    // the last piece whose output range starts at or before m (empty pieces
    // share their start with the next non-empty one, which comes after them)
    int lo = 0, hi = P;                                   // out_start[lo] <= m < out_start[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (out_start[mid] <= m) lo = mid; else hi = mid;
    }
    const int32_t src = recv_start[lo] + static_cast<int32_t>(m - out_start[lo]);
    rows[m] = chk(src, M_recv, CHK_LAYOUT) ? src : -1;
  }
}

// ---------------------------------------------------------------------------
// Regroup of received FP8 rows: q_out row m = q_in row rows[m] (K bytes, 16-byte
// copies), and its K/128 scales from the row-major receive layout into the
// GEMM's K-chunk-major layout, sf_out[kb * ld_out + m].  One warp per row; each
// lane issues up to 8 of the row's 16-byte loads before their stores, so that
// enough bytes are in flight to keep the HBM busy (one load at a time per lane
// ran at ~4.1 TB/s).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
gather_rows_fp8_kernel(const uint8_t* __restrict__ q_in, int64_t ldq_in, const float* __restrict__ sf_in,
                       int64_t ld_sf_in, int64_t M_in, const int32_t* __restrict__ rows, int64_t M_out, int64_t K,
                       uint8_t* __restrict__ q_out, int64_t ldq_out, float* __restrict__ sf_out, int64_t ld_sf_out) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t KB = K / 128;
  for (int64_t m = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5); m < M_out; m += warps) {
    int64_t src = rows[m];
    if (src < 0 || src >= M_in) {
      if (lane == 0) report_status(FP8Q_ERR_INVALID_ARG, BAD_ROW_INDEX);
      src = -1;
    }
    const uint4* in = reinterpret_cast<const uint4*>(q_in + (src < 0 ? 0 : src) * ldq_in);
    uint4* out = reinterpret_cast<uint4*>(q_out + m * ldq_out);
    const int64_t n16 = K / 16;
    for (int64_t c0 = 0; c0 < n16; c0 += 32 * 8) {
      uint4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t c = c0 + 32 * j + lane;
        v[j] = (src < 0 || c >= n16) ? make_uint4(0, 0, 0, 0) : __ldcs(in + c);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t c = c0 + 32 * j + lane;
        if (c < n16) out[c] = v[j];
      }
    }
    for (int64_t kb = lane; kb < KB; kb += 32)
      sf_out[kb * ld_sf_out + m] = src < 0 ? 1e-12f : sf_in[src * ld_sf_in + kb];
  }
}

}  // namespace fp8q
