/*
 * q4gemv -- group-quantised weight x activation products for single-user LLM
 * decode on NVIDIA B200 (sm_100a).
 *
 * The operation.  Single-user decode of a dense ~27B hybrid model streams every
 * low-bit weight once per generated token, so its speed is set by how fast the
 * weight bytes leave HBM ("Fit != Speed": wiselychen guide "Qwen3.8-27B
 * measured: RTX 3090/4090/5090/PRO 6000/DGX Spark/Mac", section "Before
 * deploying: weights, KV cache, memory bandwidth"; bs178.com llamAmpere post,
 * "Why it is this fast", part two).  The weights are 4-bit integers ("INT4",
 * four bits instead of sixteen: jdon.com "Two RTX 3090s, 105 tok/s", section
 * "27 billion parameters into 24 GB"), with 8-bit integers for the sensitive
 * attention projections and the output head (bs178.com post, part two), and
 * 16-bit activations ("W4A16": jdon.com page, section "Schools of
 * quantisation").  The pages give no bit layout; this library reads the formats
 * as: groups of 32 consecutive k, one fp16 scale per group, symmetric (no zero
 * point), q4 in [-8, 7], q8 in [-127, 127].
 *
 *   W[n][k] = s[n][k/32] * q[n][k]                  (N x K)
 *   y[m][n] = sum_k W[n][k] * x[m][k]               m < M <= 4, x bf16, y fp32
 *
 * M = 1 is plain decode; M = 4 is one verification pass over three drafted
 * tokens plus one (multi-token-prediction speculative decoding with depth 3:
 * bs178.com post, part four).
 *
 * Conventions for every entry point:
 *   - Return value: Q4_OK (0) or a negative Q4_ERR_* code; q4_last_error()
 *     then returns a message for the calling thread.
 *   - Argument errors are detected on the host, synchronously, before any
 *     launch; nothing is launched when a call fails.
 *   - "device" pointers are CUDA device (or managed) memory owned by the
 *     caller; "host" pointers are ordinary host memory owned by the caller.
 *   - Device work is asynchronous on the caller's stream (a cudaStream_t passed
 *     as void*; NULL is the legacy default stream).  No entry point except
 *     layer_stack_create / layer_stack_destroy / q4_workspace_check allocates,
 *     frees or synchronises.
 *   - There is no CPU fallback: without a usable sm_100a device the GPU entry
 *     points fail with Q4_ERR_CUDA.
 *
 * ---------------------------------------------------------------------------
 * Canonical (interchange) layout -- the input of q4_pack_weights:
 *   q4:     uint8 [N][K/2]; element k of a row is in byte k/2, low nibble for
 *           even k; 4-bit two's complement (-8..7).
 *   q8:     int8  [N][K].
 *   scales: uint16 [N][K/32], IEEE binary16 bits.
 *   x:      uint16 [M][K], bfloat16 bits, row-major (leading dimension K).
 *   y:      float  [M][N], row-major (leading dimension N); overwritten.
 *
 * Kernel-native packed layout -- the output of q4_pack_weights:
 *   Rows are cut into T = ceil(N/32) tiles of 32 rows.  Each tile is cut along
 *   K into C chunks: q4 chunks cover 64 k (two groups), C = ceil(K/64); q8
 *   chunks cover 32 k (one group), C = K/32.  Chunk (t, c) is CB bytes at
 *   offset (t*C + c)*CB, CB = 1152 (q4) or 1088 (q8), so each tile, and the
 *   whole tensor, is one contiguous run in memory order t, c.
 *   A chunk is two 512-byte code blocks, h = 0, 1 (rows 32t + 16h .. +15),
 *   then the scales of its groups.  Code block h is 32 slots of 16 bytes,
 *   slot L = 4*gi + ti (gi in 0..7, ti in 0..3), each four little-endian
 *   32-bit words.  With R = 32t + 16h + gi and R' = R + 8:
 *   q4: word j = 2G + e (G, e in {0,1}) holds eight nibbles; nibble i (bits
 *       4i..4i+3) is u = q + 8 of row (i odd ? R' : R), column
 *       64c + 32G + 8ti + 4e + 2*((i>>1)&1) + (i>>2).
 *       Scales (at byte 1024): 8 entries of 16 bytes; entry gi holds the
 *       fp16 scales s(r, 2c + g) at position 4h + 2up + g for the rows
 *       r = 32t + 16h + gi + 8up (h, up, g in {0,1}).
 *   q8: word j = 2e + f holds four bytes; byte b (bits 8b..8b+7) is
 *       u = q + 128 of row (b odd ? R' : R), column 32c + 8ti + 4e + 2f + (b>>1).
 *       Scales (at byte 1024): 8 entries of 8 bytes; entry gi holds s(r, c)
 *       at position 2h + up for r = 32t + 16h + gi + 8up.
 *   q5 / q6 (bits = 5, 6; K % 64 == 0; canonical codes int8 [N][K] with q in
 *       [-16, 15] / [-32, 31]; a width between q4 and q8 for tensors that
 *       need more precision, as the bs178 post's recipe upgrades some tensors
 *       to 5 and 6 bits): the q4 chunk geometry, CB = 1408 (q5) or 1664 (q6).
 *       u = q + 16 (q5) or q + 32 (q6).  The code blocks hold the low nibble
 *       u & 15 at the q4 nibble's place.  The high bits u >> 4 of lane L's
 *       values follow at byte 1024: q5, 8 bytes at 1024 + 8L (32-bit word h
 *       for half h); q6, 16 bytes at 1024 + 16L (word 2h + (j >> 1)).  The
 *       value in nibble i of code word j (tensor-core register r = i & 3,
 *       half-word e = i >> 2) has its high bit(s) at bit
 *         16e + S + (r odd ? 8 : 4),
 *       S = {-4, -3, -2, -1, 4, 5, 6, 7}[2j + (r >> 1)] (q5, one bit) or
 *       S = {-4, -2, 4, 6}[2 (j & 1) + (r >> 1)] (q6, two bits), so one shift
 *       of the word by S brings a register pair's bits to the mantissa bits
 *       the decode needs.  Scales: the q4 placement, at byte 1280 (q5) or 1536
 *       (q6).  q5 / q6 products run in stream-mode stacks.
 *   Padding rows (>= N) and padding groups (>= K/32) hold q = 0 and scale 0.
 *   This places, for one warp, exactly the operands of bf16 m16n8k16 tensor-core
 *   products: slot L of block h is lane L's A fragment for the 16-row half h,
 *   and every word decodes to bf16 pairs with one mask-and-or per pair.  The
 *   packed buffer must be 16-byte aligned.
 * ---------------------------------------------------------------------------
 */
#ifndef Q4GEMV_H
#define Q4GEMV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define Q4_API __attribute__((visibility("default")))
#else
#define Q4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define Q4_OK 0
#define Q4_ERR_INVALID_ARG (-1)      /* null pointer, bits not 4/8, M outside 0..4 */
#define Q4_ERR_SHAPE (-2)            /* K % 32 != 0, negative sizes, sizes too large */
#define Q4_ERR_ALIGN (-3)            /* packed / x / workspace not 16-byte aligned, y not 4-byte */
#define Q4_ERR_BUFFER_TOO_SMALL (-4) /* output or workspace smaller than required */
#define Q4_ERR_CUDA (-5)             /* a CUDA call failed (message has the CUDA error) */
#define Q4_ERR_TIMEOUT (-6)          /* a bounded device wait gave up (see q4_workspace_check) */
#define Q4_ERR_UNSUPPORTED (-7)      /* no sm_100 device, or a request this library does not serve */

/* Message of the last failing call on this thread ("" if none). */
Q4_API const char* q4_last_error(void);

/* Bytes of the packed layout for an N x K tensor of `bits` (4, 5, 6 or 8); 0
 * when bits is not one of them, N or K is negative, K % 32 != 0, or (5 and 6
 * bits) K % 64 != 0.
 * Weight-stream bytes are the algorithmic N*K/2 + N*K/16 (q4) or
 * N*K + N*K/16 (q8); the packed size adds only the row and group padding. */
Q4_API size_t q4_packed_bytes(int bits, int64_t N, int64_t K);

/* Offline repack (host -> host), once per tensor, not per token.  Reads the
 * canonical q (uint8 [N][K/2] for bits=4, int8 [N][K] for bits=8) and fp16
 * scales [N][K/32]; writes the packed layout into `out` (out_bytes >=
 * q4_packed_bytes).  A pure byte and bit permutation plus the q -> q+8 / q+128
 * offset; bit-exact inverse: q4_unpack_weights.  The same call packs q8
 * (bits = 8) and q5 / q6 (bits = 5, 6: canonical int8 [N][K]; a code outside
 * the width's range is INVALID_ARG).  Errors: INVALID_ARG, SHAPE,
 * BUFFER_TOO_SMALL. */
Q4_API int q4_pack_weights(int bits, const void* canon_q, const uint16_t* scales_fp16, int64_t N, int64_t K,
                           void* out, size_t out_bytes);

/* The same repack on the device: canonical q and scales in device memory,
 * packed bytes written to `out` (device, 16-byte aligned, out_bytes >=
 * q4_packed_bytes), asynchronously on `stream`.  Produces exactly the bytes
 * q4_pack_weights produces.  Errors: INVALID_ARG, SHAPE, ALIGN,
 * BUFFER_TOO_SMALL, CUDA. */
Q4_API int q4_pack_weights_device(int bits, const void* canon_q, const uint16_t* scales_fp16, int64_t N, int64_t K,
                                  void* out, size_t out_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Offline quantiser: bf16 weights -> canonical codes and fp16 scales (the
 * input of q4_pack_weights).  Round to nearest, group 32 along K, symmetric
 * (no zero point).  The pages name 4-bit and 8-bit formats and say that a
 * quantiser's grouping and scale computation matter (jdon.com "Two RTX 3090s,
 * 105 tok/s", section "Schools of quantisation"; bs178.com llamAmpere post,
 * "Why it is this fast", part two) but give no recipe; this one fixes every
 * rounding step, so host and device produce the same bits.  Per group of 32
 * values w (fp32, exact from bf16):
 *   ABSMAX:      s32 = max|w| / qmax   (qmax 7 for q4, 127 for q8), IEEE fp32 division
 *   SIGNED_MAX:  s32 = w_m / -8        (q4 only; w_m the first value of largest
 *                                       magnitude, which then gets the code -8)
 *   s16 = fp16 of s32, round to nearest even, saturated to +-65504; s = s16 as fp32
 *   q   = 0 if s == 0, else clamp(rint(w / s), lo, hi): IEEE division, ties to
 *         even; [lo, hi] = [-7, 7] (ABSMAX q4), [-8, 7] (SIGNED_MAX), [-127, 127] (q8)
 * ABSMAX never uses the q4 code -8; SIGNED_MAX uses all sixteen.  Weights must
 * be finite.  Outputs: canonical q (q4: uint8 [N][K/2], low nibble = even k;
 * q8: int8 [N][K]) and scales (fp16 bits [N][K/32]).
 * -------------------------------------------------------------------------*/
#define Q4_QUANT_ABSMAX 0
#define Q4_QUANT_SIGNED_MAX 1

/* Host: w_bf16 [N][K] in host memory, outputs in host memory.  Errors:
 * INVALID_ARG (bits, mode, null), SHAPE (K % 32), ALIGN (2-byte w, scales). */
Q4_API int q4_quantize(int bits, int mode, const uint16_t* w_bf16, int64_t N, int64_t K, void* canon_q_out,
                       uint16_t* scales_out);

/* Device: the same computation, every pointer device memory (w 16-byte and
 * codes 8-byte aligned), asynchronous on `stream`; bit-identical to
 * q4_quantize.  Errors: as q4_quantize, plus CUDA. */
Q4_API int q4_quantize_device(int bits, int mode, const uint16_t* w_bf16, int64_t N, int64_t K, void* canon_q_out,
                              uint16_t* scales_out, void* stream);

/* Inverse of q4_pack_weights (host -> host): writes canonical q and scales.
 * Padding is dropped.  packed_bytes must be >= q4_packed_bytes. */
Q4_API int q4_unpack_weights(int bits, const void* packed, size_t packed_bytes, int64_t N, int64_t K,
                             void* canon_q_out, uint16_t* scales_out);

/* ---------------------------------------------------------------------------
 * NVFP4 weights (the 4-bit format the pages name for Blackwell engines:
 * wiselychen.com guide, section "RTX 5090 32GB", SGLang / vLLM + NVFP4; the
 * format's published definition).  Blocks of 16 values along K; each value an
 * FP4 E2M1 code (sign, 2 exponent bits with bias 1, 1 mantissa bit: 0, 0.5,
 * 1, 1.5, 2, 3, 4, 6 and negatives), each block one FP8 E4M3 scale (sign, 4
 * exponent bits with bias 7, 3 mantissa bits, subnormals, S.1111.111 = NaN),
 * the tensor one fp32 scale t:  w[n][k] = t * e4m3(s[n][k/16]) * e2m1(c[n][k]).
 * Canonical layout: codes uint8 [N][K/2] (element k in byte k/2, low nibble
 * for even k), scales uint8 [N][K/16] (E4M3 bits).  K % 64 == 0.
 * Packed layout: T = ceil(N/32) tiles x C = K/64 chunks of 1152 bytes, in
 * memory order t, c, then 16 bytes holding t (float, then zeros).  Chunk (t,c)
 * covers rows 32t .. 32t+31, columns 64c .. 64c+63:
 *   byte 512h + 16L + 4j + r (L = 4gi + ti; j = 2G + e; h, G, e in {0,1};
 *   r in 0..3; gi in 0..7; ti in 0..3) holds the codes of row
 *   32t + 16h + gi + 8(r & 1), columns 64c + 32G + 8ti + 4e + 2(r >> 1) + {0,1}
 *   (low nibble the lower column);
 *   byte 1024 + 8(2gi + b) + 4h + 2G + up (b, up in {0,1}) holds the scale of
 *   row 32t + 16h + gi + 8up, block 4c + 2G + b.
 * Padding rows hold code 0 and scale 0.  The code bytes are those of the q4
 * layout's nibbles for the same tensor-core register, two per byte.
 * -------------------------------------------------------------------------*/
#define Q4_FMT_NVFP4 16 /* q4_stack_entry.bits value of an NVFP4 product (stream mode only) */

/* Packed bytes of an N x K NVFP4 tensor (chunks plus the 16-byte trailer);
 * 0 when N or K is negative or K % 64 != 0. */
Q4_API size_t q4_nvfp4_packed_bytes(int64_t N, int64_t K);

/* Host -> host repack.  Errors: INVALID_ARG (null), SHAPE, BUFFER_TOO_SMALL. */
Q4_API int q4_pack_nvfp4(const uint8_t* codes, const uint8_t* scales, float tensor_scale, int64_t N, int64_t K,
                         void* out, size_t out_bytes);

/* Inverse of q4_pack_nvfp4 (host -> host); padding is dropped. */
Q4_API int q4_unpack_nvfp4(const void* packed, size_t packed_bytes, int64_t N, int64_t K, uint8_t* codes_out,
                           uint8_t* scales_out, float* tensor_scale_out);

/* The same repack on the device (all pointers device memory, out 16-byte
 * aligned), asynchronous on `stream`; the same bytes as q4_pack_nvfp4.
 * Errors: as q4_pack_nvfp4, plus ALIGN and CUDA. */
Q4_API int q4_pack_nvfp4_device(const uint8_t* codes, const uint8_t* scales, float tensor_scale, int64_t N,
                                int64_t K, void* out, size_t out_bytes, void* stream);

/* Debug decoder: the weights the product kernels multiply, through the same
 * in-register conversion, as fp32 w_out [N][K] (device): the exact fp16
 * product e4m3 * e2m1, times t in fp32.  Errors: INVALID_ARG, SHAPE, ALIGN,
 * CUDA. */
Q4_API int q4_nvfp4_dequant_device(const void* packed, int64_t N, int64_t K, float* w_out, void* stream);

/* ---------------------------------------------------------------------------
 * Speculative decoding around the M = 4 product (MTP draft / verify).  The
 * bs178.com llamAmpere post ("Why it is this fast", part four) drafts three
 * tokens with the model's multi-token-prediction head, checks them with one
 * pass of the main model, and keeps each drafted token with probability
 * min(1, p/q) (p the main model's probability of the token, q the draft
 * head's), so the output is distributed as plain generation; the draft head
 * projects onto a vocabulary map of 65,536 of the ~248K tokens, the main model
 * onto all of them.  At the first rejected position the emitted token is drawn
 * from max(0, p - q) normalised; when every draft is kept one more token is
 * drawn from the main model's next distribution (the standard speculative
 * sampling step the post's equivalence claim needs).
 *   dist(l, T) = softmax(l / T) (T > 0), computed in fp32 on the device;
 *   a draw from weights w with a uniform u in [0, 1) is the first index whose
 *   running sum exceeds u * sum(w).
 *   T = 0 is greedy: a draft is kept iff it is the first maximum of the main
 *   model's logits, and the emitted correction / bonus is that maximum.
 * The random numbers are inputs (device arrays of uniforms in [0, 1)), so a
 * step is reproducible and can be captured in a CUDA graph.  Logits may hold
 * -inf (masked tokens, probability 0); every row needs one finite logit, and
 * NaN logits give undefined tokens.  Results are bitwise reproducible run to
 * run (fixed reduction orders).  All pointers are device memory, 4-byte
 * aligned; calls are asynchronous on `stream`.
 * -------------------------------------------------------------------------*/
#define Q4_SPEC_MAX_DRAFT 15

/* Row gather (vocabulary-mapped draft head): dst row r = src row rows[r],
 * row_bytes bytes each (e.g. canonical q4 codes K/2, q8 codes K, fp16 scales
 * K/16), for r < n_rows; a rows[r] outside [0, n_src) gives a zero row.  Pack
 * the gathered codes and scales with q4_pack_weights_device.  Errors: SHAPE,
 * INVALID_ARG, ALIGN (rows), UNSUPPORTED, CUDA. */
Q4_API int q4_gather_rows_device(const void* src, int64_t row_bytes, int64_t n_src, const int32_t* rows,
                                 int64_t n_rows, void* dst, void* stream);

/* One draft token: z fp32 [n_map] (the draft head's logits over the mapped
 * rows), vmap int32 [n_map] (mapped row -> token id), u [1].  Writes the drawn
 * mapped row, its token vmap[row] and q = dist(z, T)[row] (1 when greedy).
 * Errors: SHAPE (n_map < 1), INVALID_ARG (T < 0, NaN or inf; null), ALIGN,
 * UNSUPPORTED, CUDA. */
Q4_API int q4_spec_draft(const float* z, int64_t n_map, const int32_t* vmap, float temperature, const float* u,
                         int32_t* row_out, int32_t* token_out, float* q_out, void* stream);

/* Verify n_draft drafted tokens (0..Q4_SPEC_MAX_DRAFT).
 *   target  fp32 [n_draft + 1][V]: the main model's logits at the drafted
 *           positions and the one after them (the M = n_draft + 1 product of
 *           the output head);
 *   drafts  fp32 [n_draft][n_map]: the draft head's logits of each draft;
 *   vmap    int32 [n_map], inv_map int32 [V] (token -> mapped row, -1 if
 *           unmapped; entries outside [0, n_map) count as unmapped);
 *   rows    int32 [n_draft]: the drafted mapped rows (from q4_spec_draft);
 *   u       fp32 [2 n_draft + 1]: keep uniforms, correction uniforms, bonus
 *           uniform;
 *   out     int32 [3 n_draft + 3]: out[0] = a, the number of leading drafts
 *           kept; out[1 .. a] their tokens; out[a + 1] the correction (a <
 *           n_draft) or bonus token; out[a + 2 .. n_draft + 1] = -1.  Then,
 *           per position j: out[n_draft + 2 + j] = 1 if draft j passed its
 *           own test (j < n_draft), and out[2 n_draft + 2 + j] = the draw of
 *           position j (correction or bonus; -1 where the draft was kept).
 *           Positions after the first rejection are evaluated too; only the
 *           first a + 1 tokens are the step's output.
 * Two launches: one cluster of 8 CTAs per position, then one small kernel.
 * Errors: INVALID_ARG (n_draft, temperature, null), SHAPE, ALIGN,
 * UNSUPPORTED, CUDA. */
Q4_API int q4_spec_verify(const float* target, int64_t V, const float* drafts, int64_t n_map, const int32_t* vmap,
                          const int32_t* inv_map, const int32_t* rows, int n_draft, float temperature,
                          const float* u, int32_t* out, void* stream);

/* Bytes of device workspace q4_gemv / q8_gemv need for this shape on the
 * current device.  The workspace holds a status word, the per-warp parts of
 * tiles split between warps (tagged 64-bit words, a region of fixed size per
 * device) and one reserved 4-byte word per 32-row tile.  It must be zero-filled before its first use; every
 * completed call leaves the status word and the split-tile words zero again,
 * so one workspace serves any sequence of stream-ordered calls, of any shapes
 * and M, whose requirements it meets.  Calls that may run concurrently need
 * separate workspaces.  Returns 0 for invalid arguments. */
Q4_API size_t q4_gemv_workspace_bytes(int bits, int64_t N, int64_t K, int M);

/* y = W x for packed q4 weights (device), bf16 x [M][K] (device, 16-byte
 * aligned), fp32 y [M][N] (device, overwritten).  M in 0..4; M = 0 or N = 0
 * is a no-op; K = 0 writes y = 0.  Asynchronous on `stream`; launches one
 * kernel; deterministic (bitwise-identical y for identical inputs and device).
 * Errors: INVALID_ARG, SHAPE, ALIGN, BUFFER_TOO_SMALL (workspace), CUDA.
 * A device-side wait that gives up is reported by q4_workspace_check. */
Q4_API int q4_gemv(const void* packed, int64_t N, int64_t K, const uint16_t* x, int M, float* y, void* workspace,
                   size_t workspace_bytes, void* stream);

/* The same product for packed q8 weights. */
Q4_API int q8_gemv(const void* packed, int64_t N, int64_t K, const uint16_t* x, int M, float* y, void* workspace,
                   size_t workspace_bytes, void* stream);

/* q4_gemv for callers that cannot allocate device memory where they run the
 * product: plug-ins inside a host application that owns the device memory
 * budget (its own pool or allocator, none of it handed to them), and
 * latency-critical loops that must not call cudaMalloc, which can synchronise
 * the whole device.  The pages describe no such entry point; it has no
 * counterpart there.
 * Same product, arguments and errors as q4_gemv, without the workspace: the
 * split-tile scratch is a file-scope device array of 4 MiB that every GPU
 * loading the library holds until the process exits.  Shapes whose scratch
 * does not fit (more than about 14 million rows on a 148-SM device) are
 * rejected with Q4_ERR_UNSUPPORTED before any device work.  Allocates and
 * frees nothing.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress, with that device current); make that first
 * call before any stream capture.  Each call clears the array's status word
 * and the split-tile words its kernel uses with two asynchronous memsets on
 * `stream` before its kernel.  All calls share the one array, which keeps the last call's
 * contents: calls that may overlap on the GPU (different streams without
 * ordering between them) race and give undefined results.  A device wait
 * that gives up is not reported by this entry point. */
Q4_API int q4_gemv_noalloc(const void* packed, int64_t N, int64_t K, const uint16_t* x, int M, float* y,
                           void* stream);

/* Synchronises `stream`, then reads and clears the workspace's status word.
 * Returns Q4_OK, or Q4_ERR_TIMEOUT when a kernel that used this workspace gave
 * up a bounded wait since the last check (that call's y is then undefined);
 * in that case the whole workspace is zero-filled again before returning. */
Q4_API int q4_workspace_check(void* workspace, size_t workspace_bytes, void* stream);

/* Upper bound, in nanoseconds, of every device-side wait the library's kernels
 * make (on the arrival of their own bulk copies).  Default 2e9.  Applies to
 * launches and stack captures made after the call.  0 restores the default. */
Q4_API int q4_set_wait_timeout_ns(uint64_t ns);

/* Debug decode on the device: runs the kernels' in-register dequantisation on
 * every packed word and writes the integers q (int8 [N][K], device) and the
 * scales (uint16 [N][K/32], device).  Both decodes the kernels use (to bf16
 * and to fp16) run; an element where they disagree is written as -128, a
 * value neither format holds.  Used to check that in-register unpack is
 * bit-exact against the canonical weights. */
Q4_API int q4_unpack_device(int bits, const void* packed, int64_t N, int64_t K, int8_t* q_out, uint16_t* scales_out,
                            void* stream);

/* Self-test of the bounded device wait: launches one kernel that waits, with
 * the library's wait routine and a limit of timeout_ns, on a barrier that
 * nothing completes, then reports.  *status_out (host) receives 1 when the
 * wait gave up as designed, 0 if it (wrongly) succeeded.  Synchronous. */
Q4_API int q4_selftest_wait_timeout(uint64_t timeout_ns, int* status_out);

/* ---------------------------------------------------------------------------
 * The 64-layer weight stream of one decode step.  A model with 64 layers (16
 * gated-attention, 48 Gated DeltaNet: wiselychen guide, section "Before
 * deploying") reads every projection once per token; engines capture the
 * decode step in a CUDA graph (wiselychen guide, section "RTX 5090 32GB",
 * "SGLang/vLLM + NVFP4").  layer_stack_create captures the listed products, in
 * order, once; layer_stack_run replays them on a stream.
 * -------------------------------------------------------------------------*/
typedef struct q4_stack_entry {
  int bits;            /* 4 or 8, or Q4_FMT_NVFP4 (packed by q4_pack_nvfp4) */
  int64_t N, K;        /* weight shape */
  const void* packed;  /* device, packed layout */
  const uint16_t* x;   /* device, bf16 [M][K] */
  float* y;            /* device, fp32 [M][N] */
} q4_stack_entry;

typedef struct q4_stack q4_stack;

#define Q4_STACK_NO_PDL 1 /* graph mode, launched without programmatic dependent launch */
#define Q4_STACK_GRAPH 2  /* graph mode: one kernel per product, captured as a CUDA graph */
#define Q4_STACK_INDEPENDENT 4 /* stream mode: the caller asserts no product reads another's output */
#define Q4_STACK_ORDERED 32    /* ordered persistent mode */

/* Validates every entry and prepares the stack on the current device.
 * flags == 0 is graph mode (measured faster than the ordered mode on the
 * 257-product decode stream: 3.87 against 5.74 ms).
 * Ordered mode (Q4_STACK_ORDERED): one cooperative kernel, one CTA per SM,
 * runs the whole list; each product's weights are streamed exactly as by
 * q4_gemv / q8_gemv (bitwise-equal outputs), the bulk-copy rings prefetch the
 * next product's weights while the current one finishes, and a grid-wide
 * barrier between products guarantees that every output of a product is
 * written before any of the next product's activations are read -- the
 * ordering of a stream of one launch per product.
 * Stream mode (Q4_STACK_INDEPENDENT): for products that do not read each
 * other's outputs (the activations are inputs of the step, not outputs of an
 * earlier product).  One kernel treats the concatenated products
 * as a single work-split problem: every warp streams one contiguous range
 * across product boundaries with no synchronisation, so the HBM stream never
 * pauses between products.  At M >= 2 (q4 / q8 lists with four chunks per
 * stage) the products are run in groups, one such launch each, formed so
 * that every group's activations fit in shared memory beside its weight
 * stages (products whose activations fit nowhere form one group that
 * carries them with the weights); layer_stack_launches counts them.  Before it, a small kernel prepares each distinct
 * activation tensor: when a power of two 2^s makes every x * 2^-s exactly
 * representable in fp16, the products of that tensor run on that fp16 copy
 * (a shorter decode; outputs scaled back by 2^s, exactly), otherwise on x in
 * bf16.  Outputs agree with q4_gemv / q8_gemv within the product tolerance
 * (tiles may be split at other places, and fp16 sums round differently).
 * Both persistent modes need every product non-empty with an even number of
 * chunks per tile; other lists use graph mode.  Stream mode also needs every
 * q4 K to be a multiple of 64; otherwise the ordered mode is used.  A list
 * not eligible for the persistent modes takes graph mode.
 * NVFP4 products (bits = Q4_FMT_NVFP4) run in stream mode only: a list holding
 * one needs flags == Q4_STACK_INDEPENDENT and every product eligible for it,
 * else UNSUPPORTED.  They decode each code byte and scale pair in one
 * conversion and accumulate a whole tile on the tensor cores (the decoded
 * weights are exact in fp16 and bf16); t multiplies the tile sums.
 * Graph mode (Q4_STACK_GRAPH, or Q4_STACK_NO_PDL): the products are launched in
 * order, each as its own kernel, and captured once as a CUDA graph; with PDL
 * each kernel prefetches its first weight tiles while its predecessor
 * finishes and reads x only after the predecessor has completed.
 * Either mode allocates a library-owned workspace (and, persistent, the entry
 * table); the caller's buffers must outlive the stack.
 * Errors: as q4_gemv, plus CUDA for allocation or capture failures and
 * UNSUPPORTED if the persistent kernel cannot be resident on every SM. */
Q4_API int layer_stack_create(const q4_stack_entry* entries, int n_entries, int M, int flags, q4_stack** out);

/* Runs the products on `stream`: one cooperative kernel launch (ordered
 * mode), the activation preparation and one kernel launch (stream mode), or
 * one cudaGraphLaunch (graph mode).  Asynchronous. */
Q4_API int layer_stack_run(q4_stack* stack, void* stream);

/* Synchronises `stream` and reports a bounded wait that gave up during the
 * stack's runs since the last check (Q4_ERR_TIMEOUT), as q4_workspace_check. */
Q4_API int layer_stack_check(q4_stack* stack, void* stream);

/* Number of kernel launches one layer_stack_run makes. */
Q4_API int layer_stack_launches(const q4_stack* stack);

/* ---------------------------------------------------------------------------
 * A dependent decode chain: products whose activations come from the outputs
 * of earlier products through the steps that sit between them in a decoder
 * layer, all captured once as a CUDA graph with programmatic dependent launch
 * (each kernel starts its prologue -- a product its first weight copies --
 * while the one before it finishes, and reads its input only after that one
 * has completed).  The pages name the layer structure (64 layers: 16 gated
 * attention, 48 Gated DeltaNet: wiselychen guide, section "Before deploying")
 * but not the steps; the plain textbook forms are used:
 *   Q4_OP_RESIDUAL_RMSNORM: h <- h + in (in may be NULL: h unchanged), or,
 *       with bits = 1, h <- in (the residual stream starts from `in`);
 *       out = bf16( h / sqrt(mean_k h_k^2 + 1e-6) * gamma )  per row, gamma
 *       bf16 [N] or NULL for 1; h fp32 [M][N] in `resid`, updated in place
 *   Q4_OP_SWIGLU: out = bf16( silu(g) * u ), silu(z) = z / (1 + e^-z), with
 *       in = fp32 [M][2N] holding g = in[:, :N] and u = in[:, N:]
 *   Q4_OP_PRODUCT: out (fp32 [M][N]) = W in, W packed (bits 4 or 8, N x K),
 *       in bf16 [M][K] -- q4_gemv / q8_gemv
 * bf16 rounding is to nearest, ties to even.  The attention / DeltaNet mixer
 * is not part of the chain: its output enters as an input buffer.
 * -------------------------------------------------------------------------*/
#define Q4_OP_PRODUCT 0
#define Q4_OP_RESIDUAL_RMSNORM 1
#define Q4_OP_SWIGLU 2

typedef struct q4_chain_op {
  int kind;            /* Q4_OP_* */
  int bits;            /* product: 4 or 8; else ignored */
  int64_t N, K;        /* product: weight shape; RMSNORM: row length; SWIGLU: output row length */
  const void* packed;  /* product: packed weights (16-byte aligned); RMSNORM: gamma (bf16 [N]) or NULL */
  const void* in;      /* see above (device) */
  void* out;           /* see above (device) */
  float* resid;        /* RMSNORM: residual stream h (fp32 [M][N], device); else NULL */
} q4_chain_op;

/* Q4_CHAIN_PERSISTENT: the whole chain as ONE cooperative kernel launch
 * instead of a graph of one kernel per op.  Every product is split between
 * all warps of the GPU as a one-product stream-mode stack splits it (at
 * M <= 2 its output is bitwise that stack's on the same activations); the
 * weight copies run ahead across ops.  No fence, atomic or grid barrier sits
 * between one product and the next: every value another warp reads is
 * written as a 64-bit word holding it and a tag (run, op), which the reader
 * polls (bounded).  A split tile is summed by the warp holding its first
 * chunk; a step's elementwise part (residual add; silu(gate) * up) runs in
 * the owners of the product before it, and every CTA then finishes the step
 * for itself (mean square, bf16 activations, fp16 when exact) into its
 * shared-memory copy of the next product's activations.  Activations of a
 * product that no op writes (the mixer outputs) are prepared once at the
 * start of the launch and copied into shared memory while the op before runs.
 * The steps' outputs are bitwise those of q4_residual_rmsnorm / q4_swiglu on
 * the same inputs.  Needs: M in 1..4; products q4 or q8 with K a multiple of
 * 256 / 128 (M <= 2) or 128 / 64 (M >= 3), N > 0; steps with N % 8 == 0 and a
 * 16-byte aligned out, RMSNorm rows of at most 16,384 values; no op writing
 * bytes that an earlier (or the same) op reads, no two ops writing the same
 * bytes except RMSNorm ops sharing one residual stream (same pointer and N),
 * no op reading a residual stream through `in`; M rows of the largest
 * activation tensor (2 bytes a value) within the shared memory beside the
 * weight rings (M = 4: 139,264 bytes, a 17,408-value row).  Otherwise
 * Q4_ERR_UNSUPPORTED with the reason.  A wait that gives up sets the status
 * word (layer_stack_check returns Q4_ERR_TIMEOUT and clears the workspace). */
#define Q4_CHAIN_PERSISTENT 8
/* Q4_CHAIN_GRAPH: the graph of one kernel per op (programmatic dependent
 * launch).  Without either flag, layer_chain_create builds the graph, the
 * form measured faster on the 64-layer decode chain at M = 1 and M = 4
 * (4.08 / 4.61 ms against 4.41 / 7.83 ms for the single launch). */
#define Q4_CHAIN_GRAPH 16

/* Validates the ops and captures them, in order, on the current device.
 * flags: Q4_STACK_NO_PDL launches the graph without programmatic dependent
 * launch; Q4_CHAIN_PERSISTENT, Q4_CHAIN_GRAPH as above.
 * The returned stack runs with layer_stack_run, is checked with
 * layer_stack_check and freed with layer_stack_destroy.  Errors: as
 * layer_stack_create (INVALID_ARG for an unknown kind, a null or misaligned
 * buffer: fp32 4-byte, bf16 2-byte). */
Q4_API int layer_chain_create(const q4_chain_op* ops, int n_ops, int M, int flags, q4_stack** out);

/* The chain's two steps as single asynchronous calls on `stream` (the same
 * kernels the chain captures).  q4_residual_rmsnorm: h (fp32 [M][N]) <- h + y
 * (y may be NULL) or, when set != 0, h <- y; x (bf16 [M][N]) = the
 * normalised h times gamma (bf16 [N], or NULL for 1).  q4_swiglu: x (bf16
 * [M][N]) from y_gu (fp32 [M][2N]).  M in 1..4; errors as layer_chain_create. */
Q4_API int q4_residual_rmsnorm(float* h, const float* y, const uint16_t* gamma, uint16_t* x, int64_t N, int M,
                               int set, void* stream);
Q4_API int q4_swiglu(const float* y_gu, uint16_t* x, int64_t N, int M, void* stream);

/* Frees the graph and the workspace.  NULL is ignored. */
Q4_API void layer_stack_destroy(q4_stack* stack);

#ifdef __cplusplus
}
#endif

#endif /* Q4GEMV_H */
