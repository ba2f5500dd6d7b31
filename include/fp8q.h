/*
 * fp8q -- fine-grained FP8 training matmuls for NVIDIA B200 (sm_100a).
 *
 * C ABI.  Every entry point takes plain pointers and sizes; no C++ or torch
 * types cross this boundary.  Page citations name the page title and section:
 *   "Fine-Grained FP8 Quantization in DeepSeek"                  (shivam2003.com)
 *   "FP8 Mixed Precision: DeepSeek-V3 Training Architecture"      (aifetchly)
 *   "Introduction to LLM Quantization"                            (medium)
 *   "Online Quantization During Training"                         (shivam2003.com)
 *
 * Conventions shared by every call:
 *  - Pointers named x, w, q, qt, sf, a, b, d, group_offsets are DEVICE memory
 *    owned by the caller.  The library never frees or retains them.
 *  - Sizes and leading dimensions (ld*) are element counts (int64_t).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Kernels are enqueued asynchronously on it; the call returns after host
 *    validation and launch.
 *  - Return value: FP8Q_OK or an error code.  Invalid arguments are reported
 *    synchronously and nothing is launched.  Nothing throws across the ABI.
 *  - Outputs are written entirely (no accumulation into an existing output).
 *    Inputs and outputs must not overlap.
 *  - Inputs are finite BF16 values; behaviour for Inf/NaN inputs is unspecified.
 *  - The library allocates no per-call memory.  Its only state is one
 *    device-side status word per device.  One call needs scratch space, and
 *    the caller passes it: fp8q_moe_dispatch_layout takes a workspace sized
 *    by fp8q_moe_dispatch_layout_workspace.
 *  - E4M3 is the OCP "E4M3FN" encoding (bias 7, max 448, no infinities).
 *    The cast is round-to-nearest-even with saturation to +-448.
 *  - Tile scale: s = max(fl32(amax / 448), fl32(1e-12)), IEEE FP32 division;
 *    q = e4m3(fl32(x / s)), IEEE FP32 division.  s is stored (dequantised
 *    value = decode(q) * s).
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int fp8q_status;

enum {
  FP8Q_OK = 0,
  FP8Q_ERR_INVALID_ARG = 1,  /* a size, leading dimension or mode is invalid    */
  FP8Q_ERR_ALIGNMENT = 2,    /* a pointer or leading dimension is misaligned    */
  FP8Q_ERR_UNSUPPORTED = 3,  /* valid request this build does not implement     */
  FP8Q_ERR_CUDA = 4,         /* a CUDA runtime/driver call or launch failed     */
  FP8Q_ERR_TIMEOUT = 5,      /* a kernel gave up a bounded wait (device status) */
  FP8Q_ERR_SCRATCH_LIMIT = 6, /* request exceeds a fixed no-allocation scratch    */
  FP8Q_ERR_BOUNDS = 7        /* checked build: a computed index left its buffer   */
};

/* Scale layouts for operand B of fp8q_gemm_blockscaled. */
enum {
  FP8Q_SFB_BLOCK128 = 0, /* 128x128 weight blocks: sfb[(n/128) * ld_sfb + kb], ld_sfb >= K/128 */
  FP8Q_SFB_ROW = 1       /* one scale per row and K chunk: sfb[kb * ld_sfb + n], ld_sfb >= N */
};

/* Scale-history policies of fp8q_scale_history_update. */
enum {
  FP8Q_POLICY_PREVIOUS = 0,    /* delayed: the previous step's tile maximum  */
  FP8Q_POLICY_EMA = 1,         /* exponential history of tile maxima         */
  FP8Q_POLICY_DECAYED_MAX = 2  /* running maximum that decays by alpha       */
};

/* Output element types of the GEMMs. */
enum {
  FP8Q_OUT_BF16 = 0, /* round-to-nearest-even BF16 */
  FP8Q_OUT_F32 = 1   /* FP32 */
};

/* FP8 operand formats (the method uses E4M3 everywhere; E5M2 is the gradient
 * variant of conventional FP8 recipes). */
enum {
  FP8Q_FMT_E4M3 = 0, /* 1-4-3, max 448 */
  FP8Q_FMT_E5M2 = 1  /* 1-5-2, max 57344 */
};

/* Library version (major*10000 + minor*100 + patch). */
int fp8q_version(void);

/* Static, NUL-terminated description of a status code. */
const char* fp8q_status_string(fp8q_status s);

/*
 * Synchronise `stream`, then read and clear this device's sticky device-side
 * status word.  *out_code receives the raw word: 0 when no kernel reported a
 * problem; otherwise bits 0-7 hold the FP8Q_ERR_* code of the first report and
 * bits 8-31 say where it happened (which wait gave up, or which input check
 * failed).  Returns FP8Q_OK for a clean word, else the code in bits 0-7:
 * FP8Q_ERR_TIMEOUT (a bounded wait gave up), FP8Q_ERR_INVALID_ARG (a
 * device-side input check failed: group offsets, a row index, an expert id
 * or a dispatch count table out of range) or, in a checked build only,
 * FP8Q_ERR_BOUNDS.  FP8Q_ERR_CUDA if reading the word failed.
 */
fp8q_status fp8q_device_status(void* stream, int* out_code);

/*
 * 1 if this library was built with device-side bounds checks (-DFP8Q_CHECKS,
 * `python fine_grained_fp8_x128_b200/build.py --checks`, libfp8q_checks.so),
 * else 0.  In a checked build the kernels compare each computed global index
 * of their stores (and of the dispatch's row maps) with the extent their
 * arguments give; an index outside it records FP8Q_ERR_BOUNDS and the site
 * in the device status word instead of being written, so a bad index shows
 * up as a status, not as a fault.  Results are otherwise bit-identical to
 * the unchecked build.
 */
int fp8q_build_checks(void);

/*
 * Online 1x128 activation quantization.
 * "Fine-Grained FP8 Quantization in DeepSeek", section 2 "Activations use 1x128
 * tiles"; "FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section 1
 * "Fine-Grained Tile and Block-Wise Scaling" (eq. s = max|tile|/448, eq. W_FP8);
 * "Introduction to LLM Quantization", "5) Online Quantization".
 *
 *   x  : BF16 [M][ldx], row-major (token m, channel k).
 *   q  : E4M3 bytes [M][ldq]; q[m*ldq + k].
 *   sf : FP32 scales, logical [M][K/128], stored K-chunk-major:
 *        sf[(k/128) * ld_sf + m] (the layout the GEMM reads for operand A).
 * Requirements: M >= 0, K % 128 == 0, ldx >= K, ldq >= K, ld_sf >= M;
 * x and q 16-byte aligned, ldx % 8 == 0, ldq % 16 == 0; sf 4-byte aligned
 * (else FP8Q_ERR_ALIGNMENT).  M == 0 or K == 0 launches nothing.
 */
fp8q_status fp8q_quant_act_1x128(const void* x, int64_t M, int64_t K, int64_t ldx,
                                 void* q, int64_t ldq, float* sf, int64_t ld_sf,
                                 void* stream);

/*
 * fp8q_quant_act_1x128 over a row gather: output row m quantizes input row
 * rows[m] of x.  This is the MoE dispatch's permutation (tokens copied to the
 * rows of their experts, one copy per routed expert) fused into the online
 * quantization, so the permuted BF16 activations never exist in HBM ("FP8
 * Mixed Precision: DeepSeek-V3 Training Architecture", section 2 "The MoE
 * Inter-Node All-to-All Communication Wall": dispatch activations travel in
 * FP8; "Fine-Grained FP8 Quantization in DeepSeek", section 2).
 *
 *   x    : BF16 [M_src][ldx] (source tokens).
 *   rows : device int32 [M]; each in [0, M_src).  An index outside that
 *          range makes the output row's tiles quantize zeros (q = 0,
 *          sf = 1e-12) and records FP8Q_ERR_INVALID_ARG in the device status
 *          word (read with fp8q_device_status).
 *   q, sf: as fp8q_quant_act_1x128 with M output rows.
 * Requirements: as fp8q_quant_act_1x128 plus M_src >= 0, rows 4-byte aligned.
 */
fp8q_status fp8q_quant_act_1x128_gather(const void* x, int64_t M_src, int64_t K, int64_t ldx,
                                        const int32_t* rows, int64_t M,
                                        void* q, int64_t ldq, float* sf, int64_t ld_sf,
                                        void* stream);

/*
 * MoE dispatch in FP8 ("FP8 Mixed Precision: DeepSeek-V3 Training
 * Architecture", section 4: tokens sent to their experts' GPUs are quantized
 * to FP8 on the fly, which halves the all-to-all traffic).  The exchange
 * itself is a collective (torch.distributed all_to_all_single over NCCL);
 * these calls are its device steps.
 *
 * fp8q_moe_dispatch_layout: a stable counting sort of the (token, slot)
 * entries i = t * k + j by expert id: output row m of the expert-major order
 * holds token rows[m]; entry i lands on row pos[i]; expert e owns rows
 * offsets[e] .. offsets[e+1] - 1.  Ties keep entry order.  With experts
 * assigned to ranks in contiguous ranges the order is also rank-major.
 *   expert_ids : device int32 [n_entries] (token-major, k per token).
 *   rows, pos  : device int32 [n_entries]; offsets: device int32 [num_experts + 1].
 *   workspace  : device int32, at least fp8q_moe_dispatch_layout_workspace(n_entries, num_experts).
 * Requirements: 1 <= num_experts <= 1024, k >= 1, n_entries % k == 0.  An id
 * outside [0, num_experts) drops its entry (pos = -1, no row) and records
 * FP8Q_ERR_INVALID_ARG in the device status word.  Three launches.
 */
int64_t fp8q_moe_dispatch_layout_workspace(int64_t n_entries, int num_experts);
fp8q_status fp8q_moe_dispatch_layout(const int32_t* expert_ids, int64_t n_entries, int k, int num_experts,
                                     int32_t* rows, int32_t* pos, int32_t* offsets,
                                     int32_t* workspace, int64_t workspace_len, void* stream);

/*
 * fp8q_moe_dispatch_layout for callers that cannot allocate device memory when
 * they call.  Some callers have no allocator to use: a plugin that a host
 * framework calls to enqueue work, where the framework owns all device memory
 * and hands the plugin no workspace; a runtime that reserved its whole memory
 * budget at start-up; a latency-critical path where cudaMalloc's implicit
 * device synchronisation is not allowed.  This entry point takes no workspace
 * and allocates nothing (no cudaMalloc, cudaFree or allocating library call):
 * its scratch is a fixed array of FP8Q_LAYOUT_NOALLOC_SCRATCH_INTS int32
 * (1 MiB) in the library's device module, which every GPU that loads the
 * library holds until the process exits.  The pages have no counterpart to
 * this call; it is an interface for such callers only.
 *   Arguments, results and device-side reports: as fp8q_moe_dispatch_layout
 *   (rows, pos, offsets are caller-owned device buffers).
 *   Limit: fp8q_moe_dispatch_layout_workspace(n_entries, num_experts) must not
 *   exceed FP8Q_LAYOUT_NOALLOC_SCRATCH_INTS (for 256 experts any n_entries; for
 *   1024 experts up to 32768 entries); a larger request returns
 *   FP8Q_ERR_SCRATCH_LIMIT and launches nothing.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and keeps it; make that
 *   first call before any stream capture.
 *   Every call shares the one array and it keeps the last call's contents.
 *   The call needs no cleared scratch: each word it reads it wrote earlier in
 *   the same call.  Calls whose kernels overlap on the GPU (other streams, or
 *   other host threads on the same device) race on the array: order them on
 *   one stream or with events.
 */
enum { FP8Q_LAYOUT_NOALLOC_SCRATCH_INTS = 262144 };
fp8q_status fp8q_moe_dispatch_layout_noalloc(const int32_t* expert_ids, int64_t n_entries, int k, int num_experts,
                                             int32_t* rows, int32_t* pos, int32_t* offsets, void* stream);

/*
 * The dispatch quantizer from the token side: each source row of x is
 * quantized once (1x128 tiles, exactly as fp8q_quant_act_1x128) and its codes
 * and scales are written to the k output rows pos[row * k + j] (j < k), the
 * positions fp8q_moe_dispatch_layout returns.  Equal to
 * fp8q_quant_act_1x128_gather over the inverse map, without quantizing a
 * token once per routed copy.
 *   x   : BF16 [M_src][ldx].   pos: device int32 [M_src][k]; a negative entry
 *         is skipped (a dropped entry), one >= M_out is skipped and records
 *         FP8Q_ERR_INVALID_ARG.  Output rows that no entry names are left as they are.
 *   q, sf: as fp8q_quant_act_1x128 with M_out output rows.
 * Requirements: as fp8q_quant_act_1x128_gather, plus 1 <= k <= 64, pos 4-byte aligned.
 */
fp8q_status fp8q_quant_act_1x128_scatter(const void* x, int64_t M_src, int64_t K, int64_t ldx,
                                         const int32_t* pos, int k, int64_t M_out,
                                         void* q, int64_t ldq, float* sf, int64_t ld_sf, void* stream);
/* The same with the scales written row-major, sf[m * ld_sf + kb] (ld_sf >=
 * K/128): the exchange's send layout. */
fp8q_status fp8q_quant_act_1x128_scatter_rowscales(const void* x, int64_t M_src, int64_t K, int64_t ldx,
                                                   const int32_t* pos, int k, int64_t M_out,
                                                   void* q, int64_t ldq, float* sf, int64_t ld_sf, void* stream);

/*
 * fp8q_quant_act_1x128_gather with the scales written row-major,
 * sf[m * ld_sf + kb] (ld_sf >= K/128): the send layout of the dispatch
 * exchange, in which a row's scales travel with its codes.
 */
fp8q_status fp8q_quant_act_1x128_gather_rowscales(const void* x, int64_t M_src, int64_t K, int64_t ldx,
                                                  const int32_t* rows, int64_t M, void* q, int64_t ldq,
                                                  float* sf, int64_t ld_sf, void* stream);

/*
 * Regroup of received FP8 rows into the grouped GEMM's layout: q_out row m =
 * q_in row rows[m], and its scales from the row-major receive layout
 * (sf_in[r * ld_sf_in + kb]) into sf_out[kb * ld_sf_out + m].  A row index
 * outside [0, M_in) writes a zero row with scale 1e-12 and records
 * FP8Q_ERR_INVALID_ARG.
 * Requirements: K % 128 == 0, ldq_in >= K, ldq_out >= K (both % 16 == 0,
 * q_in and q_out 16-byte aligned), ld_sf_in >= K/128, ld_sf_out >= M_out.
 */
fp8q_status fp8q_gather_rows_fp8(const void* q_in, int64_t ldq_in, const float* sf_in, int64_t ld_sf_in, int64_t M_in,
                                 const int32_t* rows, int64_t M_out, int64_t K, void* q_out, int64_t ldq_out,
                                 float* sf_out, int64_t ld_sf_out, void* stream);

/*
 * The regroup order of the dispatch exchange, built on the device from the
 * exchanged layout offsets, so that the host needs nothing from the exchange
 * but the split sizes.  Received rows arrive source-rank-major, each source's
 * rows expert-major (the send order of fp8q_moe_dispatch_layout); the grouped
 * GEMM wants them expert-major, each expert's rows source-major.  This call
 * writes rows[m] = the received row that becomes output row m, for use with
 * fp8q_gather_rows_fp8, and the local experts' output offsets.
 *   all_offsets    : device int32 [world][num_experts + 1]: every rank's
 *                    fp8q_moe_dispatch_layout offsets, rank-major (an all_gather).
 *   world, rank    : the group size and this rank; this rank's experts are
 *                    rank * el .. rank * el + el - 1, el = num_experts / world.
 *   M_recv         : the rows this rank receives (the sum of its split sizes).
 *   rows           : device int32 [M_recv] (caller-owned).
 *   expert_offsets : device int32 [el + 1] (caller-owned): local expert e owns
 *                    output rows expert_offsets[e] .. expert_offsets[e+1] - 1.
 * Requirements: 1 <= num_experts <= 1024, num_experts % world == 0,
 * 0 <= rank < world, M_recv < 2^31.  A table whose offsets decrease, or whose
 * received total differs from M_recv, records FP8Q_ERR_INVALID_ARG in the
 * device status word; output rows past the table's total get -1.  One launch,
 * no workspace.  The pages describe the exchange, not this bookkeeping
 * ("FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section 4).
 */
fp8q_status fp8q_moe_regroup_order(const int32_t* all_offsets, int world, int rank, int num_experts, int64_t M_recv,
                                   int32_t* rows, int32_t* expert_offsets, void* stream);

/*
 * 1x128 quantization with GIVEN tile scales -- a scale policy's (fixed
 * calibration, delayed, or a tile-maximum history) instead of the tiles' own
 * maxima.  "Online Quantization During Training", section 4 "Max scaling is
 * robust but noisy" and its worked example; "Introduction to LLM
 * Quantization", "5) Online Quantization", delayed quantization.
 *
 *   x      : BF16 [M][ldx].
 *   sf     : FP32 scales to apply, sf[(k/128) * ld_sf + m] (the layout
 *            fp8q_quant_act_1x128 writes), ld_sf >= M.
 *   q      : E4M3 [M][ldq], q = e4m3(fl32(x / s)) (IEEE division, RNE,
 *            saturating at +-448).
 *   amax   : optional FP32 [K/128][ld_amax]: each tile's current maximum
 *            |x| (the input of fp8q_scale_history_update); NULL to skip.
 *   clipped: optional device counter (8-byte aligned): += the number of
 *            elements the cast saturated, |fl32(x / s)| > 464; NULL to skip.
 * Requirements: as fp8q_quant_act_1x128, plus ld_amax >= M when amax is given.
 */
fp8q_status fp8q_quant_act_1x128_scaled(const void* x, int64_t M, int64_t K, int64_t ldx,
                                        const float* sf, int64_t ld_sf, void* q, int64_t ldq,
                                        float* amax, int64_t ld_amax, unsigned long long* clipped,
                                        void* stream);

/*
 * 1x128 quantization with percentile clipping: each tile's scale comes from
 * its rank-th largest magnitude v instead of its maximum, so the rank-1
 * values above v saturate ("Online Quantization During Training", section 4
 * "Max scaling is robust but noisy", percentile clipping).  The p-th
 * percentile of a tile by the nearest-rank rule is rank = 128 - ceil(128 p) + 1;
 * rank 1 gives exactly fp8q_quant_act_1x128.
 *
 *   x      : BF16 [M][ldx], finite values.
 *   rank   : 1..128; anything else is FP8Q_ERR_INVALID_ARG.
 *   q, sf  : as fp8q_quant_act_1x128, with s = max(fl32(v / 448), fl32(1e-12));
 *            q = e4m3(fl32(x / s)) (RNE, saturating at +-448).
 *   clipped: optional device counter (8-byte aligned): += the number of
 *            elements with |fl32(x / s)| > 464; NULL to skip.
 * Run time grows with rank (one pass over the tile's registers per distinct
 * magnitude above v); the policy is meant for ranks of a few.
 * Requirements: as fp8q_quant_act_1x128.
 */
fp8q_status fp8q_quant_act_1x128_percentile(const void* x, int64_t M, int64_t K, int64_t ldx, int rank,
                                            void* q, int64_t ldq, float* sf, int64_t ld_sf,
                                            unsigned long long* clipped, void* stream);

/*
 * One step of a per-tile scale history (same passages as above): for each of
 * the n tiles, hist <- policy(hist, amax) and sf <- max(fl32(hist / 448),
 * fl32(1e-12)), the scale the next step's fp8q_quant_act_1x128_scaled uses.
 *   FP8Q_POLICY_PREVIOUS    : hist = amax
 *   FP8Q_POLICY_EMA         : hist = fl32(fl32(alpha*hist) + fl32(fl32(1-alpha)*amax))
 *   FP8Q_POLICY_DECAYED_MAX : hist = max(amax, fl32(alpha*hist))
 * Each product and sum is rounded to FP32 on its own.
 *   amax, hist, sf : device FP32 [n] (hist updated in place).
 * Requirements: 0 <= alpha <= 1, n >= 0; pointers 4-byte aligned.
 */
fp8q_status fp8q_scale_history_update(int policy, float alpha, const float* amax, float* hist,
                                      float* sf, int64_t n, void* stream);

/*
 * Online 128x1 quantization along the token dimension, written transposed:
 * the layout both Wgrad operands need (dL/dW = x^T (dL/dz), "Introduction to
 * LLM Quantization", "3) Backward propagation"; "Fine-Grained FP8 Quantization
 * in DeepSeek", section 4: transpose layout).  Same tile rule as above with
 * tiles of 128 consecutive tokens of one channel.
 *
 *   x  : BF16 [T][ldx] (token t, channel c).
 *   qt : E4M3 [C][ldqt]; qt[c*ldqt + t].
 *   sf : FP32 [T/128][ld_sf]; sf[(t/128) * ld_sf + c]  (operand-A layout for
 *        a GEMM whose rows are channels and whose K is tokens).
 * Requirements: T % 128 == 0, C >= 0, C % 8 == 0, ldx >= C, ldqt >= T,
 * ld_sf >= C; x, qt 16-byte aligned, ldx % 8 == 0, ldqt % 16 == 0.
 */
fp8q_status fp8q_quant_act_128x1(const void* x, int64_t T, int64_t C, int64_t ldx,
                                 void* qt, int64_t ldqt, float* sf, int64_t ld_sf,
                                 void* stream);

/*
 * E5M2 gradient variant of fp8q_quant_act_1x128 and fp8q_quant_act_128x1
 * ("FP8 Mixed Precision: DeepSeek-V3 Training Architecture", "2. Universal
 * E4M3": conventional recipes keep gradients in E5M2, which DeepSeek replaces
 * with E4M3; "Introduction to LLM Quantization", "E4M3 vs E5M2").  The same
 * tile rule with the E5M2 maximum: s = max(fl32(amax / 57344), fl32(1e-12)),
 * q = e5m2(fl32(x / s)), round-to-nearest-even, saturating at +-57344.
 * Arguments, layouts and requirements as the E4M3 calls.
 */
fp8q_status fp8q_quant_act_1x128_e5m2(const void* x, int64_t M, int64_t K, int64_t ldx,
                                      void* q, int64_t ldq, float* sf, int64_t ld_sf, void* stream);
fp8q_status fp8q_quant_act_128x1_e5m2(const void* x, int64_t T, int64_t C, int64_t ldx,
                                      void* qt, int64_t ldqt, float* sf, int64_t ld_sf, void* stream);

/*
 * FP8 activation caching: rebuild Wgrad's 128x1 transposed operand from the
 * 1x128 FP8 copy the forward pass made ("FP8 Mixed Precision: DeepSeek-V3
 * Training Architecture", section 4: activations cached in FP8 for the
 * backward pass), so the BF16 activation need not be kept.
 *   xh[t][c] = RN_bf16(e4m3(q[t][c]) * s[t][c/128])   (exact product, rounded once)
 *   then exactly fp8q_quant_act_128x1 of xh.
 *
 *   q     : E4M3 [T][ldq], as fp8q_quant_act_1x128 wrote it (no NaN codes).
 *   sf_in : its scales, sf_in[(c/128) * ld_sf_in + t], ld_sf_in >= T.
 *   qt, sf: as fp8q_quant_act_128x1 (qt [C][ldqt], sf[(t/128) * ld_sf + c]).
 * Requirements: T % 128 == 0, C % 128 == 0, ldq >= C, ldqt >= T, ld_sf >= C;
 * q, qt 16-byte aligned, ldq % 16 == 0, ldqt % 16 == 0; sf_in 16-byte aligned
 * with ld_sf_in % 4 == 0; sf 4-byte aligned.
 */
fp8q_status fp8q_requant_1x128_to_128x1(const void* q, int64_t T, int64_t C, int64_t ldq,
                                        const float* sf_in, int64_t ld_sf_in,
                                        void* qt, int64_t ldqt, float* sf, int64_t ld_sf, void* stream);

/*
 * Both tile orientations of one BF16 tensor from a single read: the 1x128
 * quantization of fp8q_quant_act_1x128 (operand A of the forward GEMM and of
 * Dgrad) and the 128x1 transposed quantization of fp8q_quant_act_128x1
 * (operand A or B of Wgrad), bit for bit the same codes and scales as those two
 * calls.  The backward pass needs the gradient in both layouts ("Introduction
 * to LLM Quantization", "3) Backward propagation"; "Fine-Grained FP8
 * Quantization in DeepSeek", section 2 and section 4 "transpose layout"), and
 * so does the activation: each 128-token x 128-channel tile is read from HBM
 * once instead of twice.
 *   x   : BF16 [T][ldx] (token t, channel c).
 *   q   : E4M3 [T][ldq];  sf  : FP32 sf[(c/128) * ld_sf + t]   (as fp8q_quant_act_1x128).
 *   qt  : E4M3 [C][ldqt]; sft : FP32 sft[(t/128) * ld_sft + c] (as fp8q_quant_act_128x1).
 * Requirements: T % 128 == 0, C % 128 == 0, ldx >= C, ldq >= C, ldqt >= T,
 * ld_sf >= T, ld_sft >= C; x, q, qt 16-byte aligned, ldx % 8 == 0,
 * ldq % 16 == 0, ldqt % 16 == 0; sf, sft 4-byte aligned.
 */
fp8q_status fp8q_quant_act_dual(const void* x, int64_t T, int64_t C, int64_t ldx, void* q, int64_t ldq, float* sf,
                                int64_t ld_sf, void* qt, int64_t ldqt, float* sft, int64_t ld_sft, void* stream);

/*
 * 128x128 weight block quantization ("Fine-Grained FP8 Quantization in
 * DeepSeek", section 3 "Weights use 128x128 blocks"; "FP8 Mixed Precision",
 * eq. s_W = max|W_block| / 448).  Run once per optimizer step; the result is
 * reused by forward and backward ("Online Quantization During Training",
 * section 3 "Weights occupy a middle ground").
 *
 *   w   : BF16 [N][ldw] (output feature n, input feature k).
 *   q   : E4M3 [N][ldq].            sf : FP32 [N/128][ld_sf], sf[nb*ld_sf + kb].
 *   qt  : optional E4M3 W^T [K][ldqt] (NULL to skip) -- operand B of Dgrad.
 *   sft : optional FP32 [K/128][ld_sft] transposed scale grid (NULL to skip).
 * The block scale is invariant under transposition, so qt/sft are exactly the
 * quantization of W^T.
 * Requirements: N % 128 == 0, K % 128 == 0, ldw >= K, ldq >= K,
 * ld_sf >= K/128, (qt: ldqt >= N, ldqt % 16 == 0), (sft: ld_sft >= N/128);
 * w, q, qt 16-byte aligned, ldw % 8 == 0, ldq % 16 == 0.
 */
fp8q_status fp8q_quant_w_128x128(const void* w, int64_t N, int64_t K, int64_t ldw,
                                 void* q, int64_t ldq, float* sf, int64_t ld_sf,
                                 void* qt, int64_t ldqt, float* sft, int64_t ld_sft,
                                 void* stream);

/*
 * Block-scaled FP8 GEMM with FP32 promotion at every 128-wide K chunk:
 *   D[m,n] = sum_kb  sa[m,kb] * sb(n,kb) * ( sum_{k in chunk kb} A[m,k] * B[n,k] )
 * "FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section 3
 * "Decoupled Accumulation in Tensor Core GEMMs" (eq. C_ij, per K chunk);
 * "Introduction to LLM Quantization", "Fine-grained Quantization" Steps 1-4 and
 * "3. Increasing accumulation Quantization".  The chunk products run on the
 * tensor cores; the scale multiply and FP32 accumulation run on the CUDA cores.
 *
 *   a   : E4M3 [M][lda], K-major.   sfa : FP32 sfa[kb * ld_sfa + m], ld_sfa >= M.
 *   b   : E4M3 [N][ldb], K-major.   sfb : per sfb_mode (FP8Q_SFB_BLOCK128 for a
 *         128x128-block weight -- Fprop, Dgrad with b = W^T; FP8Q_SFB_ROW for
 *         per-row 128x1 tiles -- Wgrad).
 *   d   : [M][ldd] of d_dtype (FP8Q_OUT_BF16 or FP8Q_OUT_F32).
 * Requirements: M >= 1, N % 128 == 0, N >= 128, K % 128 == 0, K >= 128,
 * lda >= K, ldb >= K, ldd >= N; a, b 16-byte aligned, lda % 16 == 0,
 * ldb % 16 == 0; d 16-byte aligned and ldd * sizeof(elem) % 16 == 0.
 * The result is deterministic for fixed inputs.
 */
fp8q_status fp8q_gemm_blockscaled(const void* a, int64_t lda, const float* sfa, int64_t ld_sfa,
                                  const void* b, int64_t ldb, const float* sfb, int64_t ld_sfb,
                                  int sfb_mode, void* d, int64_t ldd, int d_dtype,
                                  int64_t M, int64_t N, int64_t K, void* stream);

/*
 * fp8q_gemm_blockscaled with the operands' FP8 formats given (FP8Q_FMT_E4M3
 * or FP8Q_FMT_E5M2 each): the E5M2 gradient variant runs Dgrad as
 * dY (E5M2) x W^T (E4M3) and Wgrad as dY^T (E5M2) x X^T (E4M3).  The tensor
 * cores take both formats in one instruction kind; nothing else changes.
 * Other arguments and requirements as fp8q_gemm_blockscaled; a format outside
 * the two is FP8Q_ERR_INVALID_ARG.
 */
fp8q_status fp8q_gemm_blockscaled_fmt(const void* a, int a_fmt, int64_t lda, const float* sfa, int64_t ld_sfa,
                                      const void* b, int b_fmt, int64_t ldb, const float* sfb, int64_t ld_sfb,
                                      int sfb_mode, void* d, int64_t ldd, int d_dtype,
                                      int64_t M, int64_t N, int64_t K, void* stream);

/*
 * fp8q_gemm_blockscaled (FP8Q_SFB_BLOCK128) whose output is the next layer's
 * FP8 input: the epilogue rounds each FP32 result to BF16, then quantizes
 * every 1x128 tile of the row exactly as fp8q_quant_act_1x128 does on that
 * BF16 row.  The result equals fp8q_gemm_blockscaled (BF16 out) followed by
 * fp8q_quant_act_1x128, bit for bit, without the BF16 round trip through HBM
 * ("Fine-Grained FP8 Quantization in DeepSeek", section 2: activations are
 * quantized online per 1x128 tile; "FP8 Mixed Precision: DeepSeek-V3 Training
 * Architecture", section 1: activations cached in FP8 for the next layer).
 *
 *   dq  : E4M3 [M][lddq].   sfd : FP32 sfd[(n/128) * ld_sfd + m], ld_sfd >= M.
 * Requirements: as fp8q_gemm_blockscaled with FP8Q_SFB_BLOCK128, plus
 * dq 16-byte aligned, lddq % 16 == 0, sfd 4-byte aligned.
 */
fp8q_status fp8q_gemm_blockscaled_q1x128(const void* a, int64_t lda, const float* sfa, int64_t ld_sfa,
                                         const void* b, int64_t ldb, const float* sfb, int64_t ld_sfb,
                                         void* dq, int64_t lddq, float* sfd, int64_t ld_sfd,
                                         int64_t M, int64_t N, int64_t K, void* stream);

/*
 * Grouped (MoE expert) block-scaled FP8 GEMM.  For each expert g, rows
 * [off[g], off[g+1]) of the expert-packed activations are multiplied by that
 * expert's 128x128-block weight, with the semantics of fp8q_gemm_blockscaled
 * (FP8Q_SFB_BLOCK128, BF16 out).  The per-expert sizes are read on the device
 * only: the host needs M_total (tokens * top_k) and nothing else, so no host
 * synchronisation is needed.  MoE context: "FP8 Mixed Precision: DeepSeek-V3
 * Training Architecture", sections 2 "The MoE Inter-Node All-to-All
 * Communication Wall" and 4 "Low-Precision Systems Co-Design".
 *
 *   a   : E4M3 [M_total][lda]; sfa[kb * ld_sfa + m], ld_sfa >= M_total.
 *   w   : E4M3 [G][N][K] (expert-major, rows K-major, packed).
 *   sfw : FP32 [G][N/128][K/128] packed.
 *   group_offsets : device int32 [G+1], nondecreasing, off[0] = 0,
 *         off[G] = M_total.  Offsets outside [0, M_total] are clamped and the
 *         device status word records FP8Q_ERR_INVALID_ARG.
 *   d   : BF16 [M_total][ldd].
 * Requirements: 1 <= G <= 1024 (larger G: FP8Q_ERR_UNSUPPORTED), M_total >= 0,
 * N % 128 == 0, K % 128 == 0, lda >= K,
 * ldd >= N; alignment as for fp8q_gemm_blockscaled.
 */
fp8q_status fp8q_grouped_gemm_blockscaled(const void* a, int64_t lda, const float* sfa, int64_t ld_sfa,
                                          const void* w, const float* sfw,
                                          const int32_t* group_offsets, int64_t G, int64_t M_total,
                                          void* d, int64_t ldd, int64_t N, int64_t K,
                                          void* stream);

/*
 * fp8q_grouped_gemm_blockscaled with the FP8 output of
 * fp8q_gemm_blockscaled_q1x128: each expert's rows come out as E4M3 1x128
 * tiles plus their scales, ready to be operand A of the next expert GEMM.
 *
 *   dq  : E4M3 [M_total][lddq].   sfd : FP32 sfd[(n/128) * ld_sfd + m],
 *         ld_sfd >= M_total.
 * Requirements: as fp8q_grouped_gemm_blockscaled plus dq 16-byte aligned,
 * lddq % 16 == 0, sfd 4-byte aligned.
 */
fp8q_status fp8q_grouped_gemm_blockscaled_q1x128(const void* a, int64_t lda, const float* sfa, int64_t ld_sfa,
                                                 const void* w, const float* sfw,
                                                 const int32_t* group_offsets, int64_t G, int64_t M_total,
                                                 void* dq, int64_t lddq, float* sfd, int64_t ld_sfd,
                                                 int64_t N, int64_t K, void* stream);

/*
 * Per-tensor FP8 baseline ("FP8 Mixed Precision: DeepSeek-V3 Training
 * Architecture", section 1: the per-tensor scaling that fine-grained tiles
 * improve on; "Introduction to LLM Quantization", "Fine-grained
 * Quantization").  Not part of the fine-grained path: it exists to measure
 * what the fine-grained scales cost in error and in GEMM throughput.
 *
 * fp8q_quant_pertensor: one scale for all of x [M][ldx] (K columns):
 *   amax = max |x|, s = max(fl32(amax / 448), fl32(1e-12)), q = e4m3(fl32(x / s)).
 *   amax_scale : device FP32 [2], written {amax, s} (4-byte aligned).
 *   q          : E4M3 [M][ldq].
 * Requirements: K % 8 == 0, ldx >= K, ldq >= K; x 16-byte aligned, ldx % 8 == 0;
 * q 8-byte aligned, ldq % 8 == 0.  Runs a memset and two kernels on `stream`.
 */
fp8q_status fp8q_quant_pertensor(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, int64_t ldq,
                                 float* amax_scale, void* stream);

/*
 * fp8q_gemm_pertensor: D[m,n] = (s_a * s_b) * sum_k A[m,k] * B[n,k], the whole
 * K reduction accumulated in the tensor cores' FP32 accumulator (no per-chunk
 * promotion: there is one scale per operand).
 *   scale_a, scale_b : device FP32 scalars (e.g. amax_scale + 1 of the call above).
 * Other arguments and requirements as fp8q_gemm_blockscaled (d_dtype
 * FP8Q_OUT_BF16 or FP8Q_OUT_F32).
 */
fp8q_status fp8q_gemm_pertensor(const void* a, int64_t lda, const float* scale_a, const void* b, int64_t ldb,
                                const float* scale_b, void* d, int64_t ldd, int d_dtype,
                                int64_t M, int64_t N, int64_t K, void* stream);

/* ---- power-of-two (UE8M0) scales on the block-scaled MMA: a study ------------
 * Not the pages' method.  The pages fix s = amax/448 ("FP8 Mixed Precision:
 * DeepSeek-V3 Training Architecture", section 1, eq. s_W), a full FP32 scale,
 * which is why fp8q_gemm_blockscaled promotes every 128-wide K chunk on the
 * CUDA cores.  The tensor core's block-scaled MMA (tcgen05.mma
 * kind::mxf8f6f4) applies scales itself but only powers of two (UE8M0: byte b
 * stands for 2^(b - 127)), one per 32 elements of K.  These calls keep the
 * method's tiles and round each scale UP to a power of two,
 *   s2 = 2^ceil(log2 t),  t = max(fl32(amax / 448), fl32(1e-12)),
 *   q  = e4m3(fl32(x / s2))   (no element saturates),
 * so that the GEMM can accumulate all of K in the tensor core: they measure
 * what the method's non-power-of-two scales cost.
 *
 * Scale layout ("scale atoms", the tensor core's scale-factor layout): one
 * 512-byte atom of 128 uint32 words per (128-row block rb, K chunk kb); row
 * r = 128 rb + r0 + 32 r1 (r0 < 32, r1 < 4) has word 4 r0 + r1, whose four
 * bytes are the UE8M0 scales of its four 32-wide K-blocks (all equal here):
 *   sf_mx[(kb * row_blocks + r / 128) * 128 + 4 * (r % 32) + (r % 128) / 32].
 * Arrays are 16-byte aligned, row_blocks = ceil(rows / 128).
 */

/*
 * 1x128 tiles with power-of-two scales.  x: BF16 [M][ldx]; q: E4M3 [M][ldq];
 * sf_mx: uint32 [K/128][ceil(M/128)][128] scale atoms (rows M .. up to the
 * next multiple of 128 get the word of 1.0).  Requirements as
 * fp8q_quant_act_1x128, plus sf_mx 16-byte aligned.
 */
fp8q_status fp8q_quant_act_1x128_ue8m0(const void* x, int64_t M, int64_t K, int64_t ldx, void* q, int64_t ldq,
                                       uint32_t* sf_mx, void* stream);

/*
 * 128x128 weight blocks with power-of-two scales.  w: BF16 [N][ldw];
 * q: E4M3 [N][ldq]; sf_mx: uint32 [K/128][N/128][128] scale atoms (every row
 * of a block carries the block's scale).  N % 128 == 0, K % 128 == 0.
 */
fp8q_status fp8q_quant_w_128x128_ue8m0(const void* w, int64_t N, int64_t K, int64_t ldw, void* q, int64_t ldq,
                                       uint32_t* sf_mx, void* stream);

/*
 * D = A . B^T on the block-scaled MMA with the scale atoms above, FP32
 * accumulation of all of K in tensor memory, BF16 out (RNE):
 *   D[m,n] = sum_k (qa[m,k] * sa2[m, k/128]) * (qb[n,k] * sb2[n, k/128]).
 *   a: E4M3 [M][lda] K-major, sfa_mx [K/128][ceil(M/128)][128];
 *   b: E4M3 [N][ldb] K-major, sfb_mx [K/128][N/128][128];  d: BF16 [M][ldd].
 * Requirements: M >= 1, K % 128 == 0, N % 256 == 0 (else FP8Q_ERR_UNSUPPORTED),
 * lda >= K, ldb >= K, ldd >= N; a, b, d, sfa_mx, sfb_mx 16-byte aligned,
 * lda % 16 == 0, ldb % 16 == 0, ldd % 8 == 0.
 */
fp8q_status fp8q_gemm_mxf8_ue8m0(const void* a, int64_t lda, const uint32_t* sfa_mx, const void* b, int64_t ldb,
                                 const uint32_t* sfb_mx, void* d, int64_t ldd, int64_t M, int64_t N, int64_t K,
                                 void* stream);

/*
 * Clock record of the GEMM kernels.  Every CTA of a GEMM kernel adds, on exit,
 * the SM-clock cycles and the nanoseconds (global timer) it ran; their ratio is
 * the effective SM clock inside those kernels -- under sustained FP8 load the
 * B200 lowers its clock to its power limit, which a sampled nvidia-smi reading
 * does not resolve.  out receives 4 kinds x {cycles, ns, CTAs} as 12
 * unsigned 64-bit counts: kind 0 the CTA-pair block-scaled GEMM, 1 the one-CTA
 * and grouped GEMM, 2 the per-tensor GEMM, 3 the UE8M0 study's GEMM.
 * Synchronises the device; reset != 0 clears the counters after the read.
 */
fp8q_status fp8q_kernel_clock_counters(unsigned long long* out, int reset);

/* ---- diagnostics (used by the test suite; not on the hot path) ---------- */

/*
 * Cast the `count` FP32 values whose bit patterns are start, start+1, ...
 * (wrapping modulo 2^32) with the same E4M3 conversion the quantizers use,
 * writing one byte each to out[0..count).  Lets a test compare the device cast
 * with an independent encoder over every FP32 input.  count <= 2^32.
 */
fp8q_status fp8q_debug_cast_e4m3_bits(uint32_t start, int64_t count, void* out, void* stream);

/*
 * Force which dense GEMM kernel fp8q_gemm_blockscaled and its variants use,
 * where it can run: FP8Q_DENSE_AUTO (the default: the CTA-pair kernel when
 * M > 128), FP8Q_DENSE_SINGLE (the one-CTA kernel) or FP8Q_DENSE_PAIR.  Both
 * kernels compute the same result; the tests run each.  Process-wide, takes
 * effect for later calls.  FP8Q_ERR_INVALID_ARG for another value.
 */
enum {
  FP8Q_DENSE_AUTO = 0,
  FP8Q_DENSE_SINGLE = 1,
  FP8Q_DENSE_PAIR = 2
};
fp8q_status fp8q_debug_force_dense_kernel(int choice);

/*
 * Launch one block that waits on a barrier no thread ever completes, with a
 * wait budget of `budget_cycles` SM clocks (1 <= budget <= 2^34).  The wait
 * gives up, records FP8Q_ERR_TIMEOUT in the device status word and the kernel
 * returns; fp8q_device_status() then reports it.  Exercises the same bounded
 * wait every pipeline wait in the library uses, without hanging the device.
 */
fp8q_status fp8q_debug_wait_timeout(int64_t budget_cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H */
