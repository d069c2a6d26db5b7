/*
 * sage.h -- C ABI of libsage.so, the B200 (sm_100a) SageAttention-family
 * quantized attention forward.
 *
 * The operation (citations are to the pages this library follows):
 *   - SageAttention2 Technical Report, abstract: smooth the inputs, quantize
 *     Q and K to low-bit integers at a fine (warp-level) granularity and
 *     (P~, V) to FP8, then run attention on the quantized operands.
 *   - SageAttention2++ summary, Sec. 2.1: Q and K (and P~) carry per-block
 *     scale factors, V a per-channel scale; Sec. 2: the kernel is
 *     FlashAttention-based (tiled, online softmax); Sec. 3: the PV matmul may
 *     accumulate in FP16 with P and V ranges narrowed to Pr = 224, Vr = 4.5
 *     (Sec. 3.1), two MMA results summed in FP16 before FP32 (Sec. 3.2).
 *   - SageAttention3 abstract: microscaling FP4 attention on Blackwell.
 * INT4 QK of the pages is INT8 here: sm_100a tcgen05 has no INT4 MMA.
 *
 * Conventions for every entry point:
 *   - Tensors are contiguous row-major [B, H, N, d] in fp16 or bf16 device
 *     memory; self-attention (query and key length N); softmax scale 1/sqrt(d).
 *   - The caller owns all device memory (inputs, output, workspace) and the
 *     stream.  The library never allocates, frees or synchronizes, except
 *     sage_check, which synchronizes the given stream.
 *   - All work is enqueued asynchronously on `stream` (0 = legacy default).
 *   - Supported: d in {64, 128}, N >= 1, 1 <= B*H <= 65535, B*H*Npad*d < 2^31
 *     where Npad = ceil(N / 128) * 128.  Other values return SAGE_ERR_UNSUPPORTED
 *     or SAGE_ERR_INVALID_ARG before any launch; a launch failure returns
 *     SAGE_ERR_CUDA.  sage_last_error() gives a message for the last non-OK
 *     status of the calling thread.
 *   - The kernels never trap.  Every wait inside them is bounded; a wait that
 *     runs out records an error word in the workspace and the kernel returns.
 *     sage_check() reports it as SAGE_ERR_TIMEOUT.
 */
#ifndef SAGE_H_
#define SAGE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SAGE_API __attribute__((visibility("default")))
#else
#define SAGE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sage_stream_t; /* same handle as cudaStream_t */

typedef enum {
  SAGE_OK = 0,
  SAGE_ERR_INVALID_ARG = 1,
  SAGE_ERR_UNSUPPORTED = 2,
  SAGE_ERR_CUDA = 3,
  SAGE_ERR_TIMEOUT = 4
} sage_status;

/* INT8 QK + FP8 PV with FP32 accumulation (SageAttention2, Sec. 2.1);
 * the same with the FP16 PV accumulator (SageAttention2++, Sec. 3);
 * microscaled FP4 (SageAttention3). */
typedef enum { SAGE_MODE_INT8_FP8 = 0, SAGE_MODE_INT8_FP8_F16ACC = 1, SAGE_MODE_NVFP4 = 2 } sage_mode;

typedef enum { SAGE_F16 = 0, SAGE_BF16 = 1 } sage_dtype;

/* Byte offsets into the workspace of each quantized buffer (INT8/FP8 modes).
 * Npad = ceil(N/128)*128, BH = B*H.  Every offset is 1024-byte aligned.
 *   q_codes  int8  [BH, Npad, d]   Q codes, one granule = 32 tokens; pad rows 0
 *   k_codes  int8  [BH, Npad, d]   smoothed K codes, one granule = 64 tokens
 *   vt_codes uint8 [BH, d, Npad]   e4m3 V codes, transposed (token-contiguous)
 *   q_scale  f32   [BH, Npad/32]   per-granule scale (absmax / 127), 0 for empty
 *   k_scale  f32   [BH, Npad/64]
 *   v_scale  f32   [BH, d]         per-channel scale absmax / Vr
 *   k_mean   f32   [BH, d]         per-channel mean of K over the N tokens
 *   q_mean   f32   [BH, d]         same for Q (written only when smooth_q)
 *   q_bias   f32   [BH, Npad]      sum_c q_mean[c] * (k - k_mean)[n, c] (smooth_q)
 *   error    int32 (one word)      0, or the code of a wait that ran out
 *   scratch  f32                   partial sums of the statistics pass
 * In the NVFP4 mode (SageAttention3 abstract):
 *   q_codes, k_codes  [BH, Npad, d/2]  two e2m1 codes per byte, low nibble =
 *                     even channel; block of 16 channels per scale
 *   vt_codes          [BH, d, Npad/2]  V^T, low nibble = even token; block of
 *                     16 tokens per scale
 *   q_scale, k_scale  ue4m3 block scales in 512-byte atoms, one atom per
 *                     (128-row tile, 64 channels): atom index
 *                     (bh * Npad/128 + row/128) * d/64 + channel/64, byte
 *                     16*(r%32) + 4*(r/32) + b within it, r = row % 128,
 *                     b = (channel % 64) / 16.  This is the layout the
 *                     tensor cores read block scales in.
 *   v_scale           the same atoms for V^T: index (bh * Npad/128 +
 *                     token/128) * 2 + (token%128)/64, r = channel (rows
 *                     d..127 of an atom are 0 when d = 64), b = (token%64)/16
 *   global_scale      fp32 [BH, 4]: Q, K, V global scales (max |x| / 2688), 0 */
typedef struct {
  size_t q_codes, k_codes, vt_codes, q_scale, k_scale, v_scale;
  size_t k_mean, q_mean, q_bias, global_scale, error, scratch;
  size_t total;
} sage_ws_layout;

/* Fill `out` with the workspace layout for a problem; returns its size in
 * out->total.  Pure host computation. */
SAGE_API sage_status sage_workspace_layout(int B, int H, int N, int d, int mode, sage_ws_layout* out);

/* Workspace bytes needed (0 if the arguments are unsupported). */
SAGE_API size_t sage_workspace_size(int B, int H, int N, int d, int mode);

/* Smoothing + quantization (SageAttention2 abstract; SageAttention2++ Sec.
 * 2.1, 3.1): K minus its per-channel mean over tokens; if smooth_q, Q minus
 * its mean and the bias mean_q . (k - mean_k) per key; INT8 Q (32-token
 * granules) and K (64-token granules) with scale absmax/127 and codes
 * round-to-nearest-even of x * (127/absmax); V to e4m3 per channel with
 * scale absmax/Vr (Vr = 448, or 4.5 in SAGE_MODE_INT8_FP8_F16ACC), stored
 * transposed.  q, k, v: device [B,H,N,d] of `dtype`.  ws: device workspace of
 * at least sage_workspace_size() bytes, 1024-byte aligned. */
SAGE_API sage_status sage_quantize_qkv(const void* q, const void* k, const void* v, int dtype, int B, int H, int N, int d,
                              int smooth_q, int mode, void* ws, size_t ws_bytes, sage_stream_t stream);

/* sage_quantize_qkv for callers that cannot allocate device memory.  (The
 * pages have no counterpart; this is a deployment variant.)  Code running
 * inside a CUDA-graph capture that must not grow the memory pool, a plugin
 * whose host framework owns every allocation, or a real-time loop that may
 * not call the allocator can pass its inputs and one output buffer but no
 * scratch area.  This entry point keeps the statistics scratch (per-chunk
 * partial sums) in a 16 MiB device array inside the library instead; every
 * GPU that loads this part of the library holds that array until the
 * process exits.  It calls no allocator.
 *   out: device buffer of at least sage_ws_layout.scratch bytes (everything
 *        the layout places before `scratch`), 1024-byte aligned; it receives
 *        the same codes, scales, means and bias as the workspace of
 *        sage_quantize_qkv, at the same offsets.
 *   Limit: 3*B*H*(Npad/64)*d + B*H*d words (INT8/FP8 modes) or
 *   7*B*H*(Npad/64)*d words (NVFP4) <= 4 Mi (16 MiB);
 *   larger problems return SAGE_ERR_UNSUPPORTED with the sizes in
 *   sage_last_error().
 *   The first call on a device looks up the array's device address once,
 *   with that device current; make that first call before any stream
 *   capture.  All calls share the array: calls that overlap on the GPU (on
 *   different streams, or on several host threads at once) race on it and
 *   must be serialized by the caller.  Nothing in the array needs to start at
 *   zero; each call overwrites what it reads. */
SAGE_API sage_status sage_quantize_qkv_static(const void* q, const void* k, const void* v, int dtype, int B, int H,
                                              int N, int d, int smooth_q, int mode, void* out, size_t out_bytes,
                                              sage_stream_t stream);

/* Fused attention on a workspace filled by sage_quantize_qkv with the same
 * (B,H,N,d,smooth_q,mode): per 128-query tile, for each 128-key tile, INT8
 * QK^T on the tensor cores, dequantize (scale_q * scale_k, plus the Q bias),
 * online softmax in base 2, P~ = e4m3(p * Pr) with Pr = 448 (224 in the F16ACC
 * mode), FP8 P~ V, and O = acc * scale_v / (Pr * l) (SageAttention2++ Sec. 2,
 * 2.1, 3).  SAGE_MODE_NVFP4 (SageAttention3 abstract): block-scaled e2m1 QK^T
 * and P~ V (tcgen05 kind::mxf4nvf4), P~ quantized per 16 keys with ue4m3
 * scales and global scale 1/(6*448); d must be 128 (SAGE_ERR_UNSUPPORTED
 * otherwise).  causal masks key j > query i.  out: device [B,H,N,d] of
 * `dtype`.  ws_bytes: at least sage_ws_layout.scratch (the quantized region;
 * the statistics scratch after it is not read), so the output buffer of
 * sage_quantize_qkv_static serves as well. */
SAGE_API sage_status sage_attn_quantized(const void* ws, size_t ws_bytes, void* out, int dtype, int B, int H, int N, int d,
                                int causal, int smooth_q, int mode, sage_stream_t stream);

/* sage_quantize_qkv followed by sage_attn_quantized: the drop-in attention
 * call ("plug-and-play", SageAttention2 abstract). */
SAGE_API sage_status sage_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int H, int N, int d,
                          int causal, int mode, int dtype, int smooth_q, void* ws, size_t ws_bytes,
                          sage_stream_t stream);

/* sage_attn_fwd with Q quantized inside the attention kernel: each CTA
 * loads its 128-row tiles of the caller's 16-bit Q and quantizes them itself
 * (the per-block Q quantization of the SageAttention2++ summary, Sec. 2.1,
 * fused into the FlashAttention-style kernel of Sec. 2) with the steps of
 * sage_quantize_qkv, so Q makes one trip from HBM instead of three (read,
 * codes written, codes read).  K and V are quantized beforehand (with
 * smooth_q, Q's means and the bias too).  The output is bit-identical to
 * sage_attn_fwd's; the workspace (sage_workspace_size bytes) afterwards holds
 * the K/V codes, scales, means and bias but not Q's codes or scales.
 * INT8/FP8 modes (SAGE_MODE_NVFP4 returns SAGE_ERR_UNSUPPORTED); other
 * arguments as for sage_attn_fwd; out must be 16-byte aligned.  Speed: the
 * saved Q traffic is largely offset by each CTA quantizing its Q tiles before
 * its first MMA: on a B200 the call runs within 0.3 % of sage_attn_fwd at
 * B4 H32 N32768 d128 and 2-3 % slower at B1 H32 N8192 d128 causal. */
SAGE_API sage_status sage_attn_fwd_fused(const void* q, const void* k, const void* v, void* out, int B, int H, int N,
                                         int d, int causal, int mode, int dtype, int smooth_q, void* ws,
                                         size_t ws_bytes, sage_stream_t stream);

/* sage_attn_fwd with the P~ and V quantization ranges chosen by the caller:
 * P~ = e4m3(p * Pr), V codes e4m3(v * Vr / absmax), O rescaled by 1 / Pr.
 * The SageAttention2++ summary (Sec. 3.1) narrows both so that an FP16
 * accumulator cannot overflow and picks Pr = 224, Vr = 4.5 among the pairs
 * that qualify; sage_attn_fwd uses those (448, 448 with the FP32
 * accumulator).  Pr and Vr must lie in (0, 448]; in
 * SAGE_MODE_INT8_FP8_F16ACC the worst 64-key FP16 partial, 64 * Pr * Vr,
 * must not exceed 65504 -- otherwise SAGE_ERR_INVALID_ARG.  SAGE_MODE_NVFP4
 * returns SAGE_ERR_UNSUPPORTED (its P~ scale is fixed).  Other arguments as
 * for sage_attn_fwd. */
SAGE_API sage_status sage_attn_fwd_ranges(const void* q, const void* k, const void* v, void* out, int B, int H,
                                          int N, int d, int causal, int mode, int dtype, int smooth_q, float Pr,
                                          float Vr, void* ws, size_t ws_bytes, sage_stream_t stream);

/* Grouped key/value heads and separate query and key lengths (decoding or
 * chunked prefill against a longer key cache, cross-attention, and models whose
 * query heads share key/value heads).  The pages' method per query head
 * (SageAttention2 abstract; SageAttention2++ summary Sec. 2, 2.1, 3) with:
 *   q, out [B, Hq, Nq, d]; k, v [B, Hkv, Nk, d]; Hq a multiple of Hkv; query
 *   head h reads key/value head h / (Hq / Hkv);
 *   K smoothed per key/value head over its Nk tokens, V scaled per channel of
 *   its key/value head, Q quantized per query head (smoothed with smooth_q,
 *   the bias mean_q(h) . k~ over the keys of h's key/value head);
 *   causal: query row i sees keys j <= i + Nk - Nq (the last query row sees
 *   all keys; needs Nq <= Nk, else SAGE_ERR_UNSUPPORTED).
 * INT8/FP8 modes only (SAGE_MODE_NVFP4 needs Hq == Hkv and Nq == Nk).  With
 * Hq == Hkv and Nq == Nk these are the per-head entry points above, with the
 * same workspace layout.  Workspace layout (sage_workspace_layout_gqa):
 * q_codes [B*Hq, Npq, d], q_scale [B*Hq, Npq/32], q_mean [B*Hq, d], q_bias
 * [B*Hq, Npk]; k_codes [B*Hkv, Npk, d], vt_codes [B*Hkv, d, Npk], k_scale
 * [B*Hkv, Npk/64], v_scale and k_mean [B*Hkv, d]; Npq, Npk = Nq, Nk rounded
 * up to 128.  Other arguments, alignment and error behaviour as for the
 * per-head calls. */
SAGE_API sage_status sage_workspace_layout_gqa(int B, int Hq, int Hkv, int Nq, int Nk, int d, int mode,
                                               sage_ws_layout* out);
SAGE_API sage_status sage_quantize_qkv_gqa(const void* q, const void* k, const void* v, int dtype, int B, int Hq,
                                           int Hkv, int Nq, int Nk, int d, int smooth_q, int mode, void* ws,
                                           size_t ws_bytes, sage_stream_t stream);
SAGE_API sage_status sage_attn_quantized_gqa(const void* ws, size_t ws_bytes, void* out, int dtype, int B, int Hq,
                                             int Hkv, int Nq, int Nk, int d, int causal, int smooth_q, int mode,
                                             sage_stream_t stream);
SAGE_API sage_status sage_attn_fwd_gqa(const void* q, const void* k, const void* v, void* out, int B, int Hq, int Hkv,
                                       int Nq, int Nk, int d, int causal, int mode, int dtype, int smooth_q, void* ws,
                                       size_t ws_bytes, sage_stream_t stream);

/* Q smoothed per block of 128 query rows instead of per slice.  The
 * SageAttention2 abstract smooths Q by subtracting its channel mean but fixes
 * no granularity for that mean; these calls take one mean per 128-row block
 * (the attention's query tile), which follows Q where its offset drifts
 * along the sequence.  Per slice and block b (rows 128b .. min(N, 128b+128)):
 *   mean_b[c] = (sum over the block's 64-row chunks, in order, of the
 *               sequential fp32 sum of the chunk) / (valid rows of the block);
 *   the block's Q codes and 32-row granule scales as in sage_quantize_qkv,
 *   after subtracting mean_b;
 *   bias_b[j] = fma chain over c, in order, of mean_b[c] * (k - k_mean)[j, c]
 *   for every key j < N (0 for padded keys); query row i adds the row of its
 *   own block, bias_{i/128}.
 * K, V and everything else as in sage_quantize_qkv / sage_attn_quantized with
 * smooth_q = 1.  INT8/FP8 modes only (SAGE_MODE_NVFP4 returns
 * SAGE_ERR_UNSUPPORTED).  Workspace layout (sage_workspace_layout_blocksmooth):
 * the per-head layout with q_mean f32 [BH, Npad/128, d] and q_bias f32
 * stored key-tile-major, [BH, Npad/128 key tiles, Npad/128 blocks, 128]:
 * block b's bias at key j is element ((bh * Npad/128 + j/128) * Npad/128 +
 * b) * 128 + j % 128.  The bias takes 4 * Npad^2 / 128 bytes per slice (32
 * MiB at N = 32768) and Npad^2 * d / 128 fp32 multiply-adds on the CUDA
 * cores (1/256 of the attention's tensor-core operations, run at a small
 * fraction of their rate): on a B200 a quantize + attention step takes 7 %
 * (B1 H12 N32760 d128, FP16 accumulator) to 17 % (B1 H32 N8192 d128 causal)
 * longer than with per-slice smoothing.  Other arguments,
 * alignment and error behaviour as for the per-head calls. */
SAGE_API sage_status sage_workspace_layout_blocksmooth(int B, int H, int N, int d, int mode, sage_ws_layout* out);
SAGE_API sage_status sage_quantize_qkv_blocksmooth(const void* q, const void* k, const void* v, int dtype, int B,
                                                   int H, int N, int d, int mode, void* ws, size_t ws_bytes,
                                                   sage_stream_t stream);
SAGE_API sage_status sage_attn_quantized_blocksmooth(const void* ws, size_t ws_bytes, void* out, int dtype, int B,
                                                     int H, int N, int d, int causal, int mode, sage_stream_t stream);
SAGE_API sage_status sage_attn_fwd_blocksmooth(const void* q, const void* k, const void* v, void* out, int B, int H,
                                               int N, int d, int causal, int mode, int dtype, void* ws,
                                               size_t ws_bytes, sage_stream_t stream);

/* Parity helper: the INT32 tile S = Q^ K^T of query tile `q_tile` and key tile
 * `k_tile` (128 x 128) of slice `bh`, computed by the same tensor-core path as
 * the attention kernel (kind::i8 MMA, accumulator in TMEM).  out: device
 * int32 [128, 128], row = query.  INT8 modes only.  ws_bytes: at least
 * sage_ws_layout.scratch, as for sage_attn_quantized. */
SAGE_API sage_status sage_debug_qk_s32(const void* ws, size_t ws_bytes, int B, int H, int N, int d, int bh, int q_tile,
                              int k_tile, int32_t* out, sage_stream_t stream);

/* Parity helper of the NVFP4 mode (SageAttention3 abstract): one 128x128
 * tile S[i][j] = sum_c (q_ic * sq_i,c/16) (k_jc * sk_j,c/16) of query tile
 * q_tile and key tile k_tile of slice bh, computed from the workspace's
 * packed e2m1 codes and ue4m3 block scales by the tensor-core path the
 * NVFP4 attention uses (tcgen05.cp of the scale atoms into TMEM, tcgen05.mma
 * kind::mxf4nvf4, FP32 accumulator); global scales are not applied.
 * out: device float [128, 128], row = query.  NVFP4 workspace, d = 128. */
SAGE_API sage_status sage_debug_fp4_s(const void* ws, size_t ws_bytes, int B, int H, int N, int d, int bh,
                                      int q_tile, int k_tile, float* out, sage_stream_t stream);

/* Test helper for the failure path: launches one thread that waits on a
 * barrier nothing completes.  The bounded wait gives up after about 2 s, sets
 * the workspace error word, and the kernel returns; the CUDA context stays
 * usable.  A following sage_check() returns SAGE_ERR_TIMEOUT.  Uses only the
 * error word at offset 0 of `ws` (>= 4 bytes, 1024-byte aligned). */
SAGE_API sage_status sage_debug_timeout_probe(void* ws, size_t ws_bytes, sage_stream_t stream);

/* Tensor-core rate probe, the denominator of the library's roofline
 * fractions (the pages measure instruction speedups in the SageAttention2++
 * summary, Sec. 2.2, Table 1: FP8 with an FP16 accumulator against FP8 with
 * an FP32 one).  Launches `ctas` CTAs (one per SM: each allocates 512 TMEM
 * columns) that each issue `iters` x 4 back-to-back tcgen05.mma of one kind,
 * M = 128, N = 256, on operand tiles resident in shared memory, and returns
 * in *ops (may be NULL) the operation count 2*M*N*K summed over all of them.
 * The caller times the launch (events on `stream`) and divides.  kind: one of
 * the SAGE_PROBE_* values.  iters <= 2^20; keep one launch under a second
 * (the completion wait is bounded at 2 s and reports SAGE_ERR_TIMEOUT through
 * sage_check).  Uses only the error word at offset 0 of `ws`. */
enum { SAGE_PROBE_I8 = 0, SAGE_PROBE_F8_F32ACC = 1, SAGE_PROBE_F8_F16ACC = 2, SAGE_PROBE_BF16 = 3, SAGE_PROBE_FP4 = 4 };
SAGE_API sage_status sage_probe_mma_rate(int kind, int ctas, int iters, void* ws, size_t ws_bytes, double* ops,
                                         sage_stream_t stream);

/* Synchronize `stream`, then read and clear the workspace error word.
 * Returns SAGE_ERR_TIMEOUT if a kernel gave up a wait, SAGE_ERR_CUDA on a
 * CUDA error, else SAGE_OK. */
SAGE_API sage_status sage_check(void* ws, size_t ws_bytes, sage_stream_t stream);

/* Message for the calling thread's last non-OK status ("" if none). */
SAGE_API const char* sage_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_H_ */
