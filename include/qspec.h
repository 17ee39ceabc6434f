/*
 * qspec.h - C ABI of the shared-INT4 QSpec hot path on B200 (sm_100a).
 *
 * The method (QSpec: Speculative Decoding with Complementary Quantization
 * Schemes, abstract) serves ONE set of 4-bit weights through two linear-layer
 * modes: a W4A4 drafting mode (weights and activations both 4-bit) and a
 * W4A16 verifying mode (4-bit weights, 16-bit activations).  The explainer
 * essay on the same paper (paragraph 4) states that the two modes share the
 * underlying quantized weights and differ in how activations are handled;
 * every GEMM entry point below therefore takes the same `wq`/`ws` buffers.
 * Each draft-verify round ends with the speculative accept / residual
 * resample step (SpecQuant review, paragraph 5: "the usual Leviathan rule").
 *
 * Conventions shared by all entry points
 *  - Pointers are DEVICE pointers owned by the caller unless stated
 *    otherwise.  The library never allocates or frees device memory; scratch
 *    space is the caller's `workspace`, sized with qspec_workspace_size().
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and returns after enqueueing its kernels.
 *  - 16-bit floating point buffers are passed as uint16_t bit patterns:
 *    bf16 for activations, IEEE fp16 for weight scales.
 *  - Arguments are validated on the host before anything is launched; a
 *    failed check returns a status and launches nothing.  Launch failures
 *    return QSPEC_ERR_CUDA.  Faults seen by a kernel (a bounded wait that ran
 *    out, a draft token outside the vocabulary) are recorded in a status
 *    word at the start of the workspace; read it with
 *    qspec_workspace_status().
 *  - Device buffers read by TMA (x, wq, and the workspace) must be 16-byte
 *    aligned; all buffers must be at least 16-byte aligned.
 *  - The device must be compute capability 10.0 (B200, sm_100a), else
 *    QSPEC_ERR_UNSUPPORTED_DEVICE.
 *  - Inputs must be finite.
 */
#ifndef QSPEC_H_
#define QSPEC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum qspec_status {
  QSPEC_OK = 0,
  QSPEC_ERR_INVALID_ARG = 1,        /* a size, alignment or pointer check failed */
  QSPEC_ERR_UNSUPPORTED_DEVICE = 2, /* current device is not sm_100 */
  QSPEC_ERR_CUDA = 3,               /* a CUDA runtime call or launch failed */
  QSPEC_ERR_WORKSPACE_TOO_SMALL = 4,
  QSPEC_ERR_TIMEOUT = 5,            /* a kernel's bounded wait ran out (device status) */
  QSPEC_ERR_BAD_INPUT = 6           /* a kernel saw invalid data, e.g. a draft token >= vocab */
} qspec_status;

/*
 * GEMM flags.
 *  QSPEC_GEMM_WEIGHTS_READY: `wq` and `ws` are not being written by any work
 *    that may still be running when this call's kernels start (typically:
 *    the weights were quantized or copied once, and that work has been waited
 *    for).  The GEMM kernels are launched as programmatic dependents of the
 *    preceding kernel on the stream; with this flag they stream the packed
 *    weights and scales into shared and tensor memory while that kernel is
 *    still finishing, and wait for it only where they read activations or
 *    write anything.  Without the flag the weights are read only after the
 *    preceding kernel has completed.  Results are identical either way.
 * Other bits are reserved and must be zero.
 */
#define QSPEC_GEMM_WEIGHTS_READY 1u
/*
 *  QSPEC_GEMM_FUSED_QUANT (drafting modes, m <= 32; ignored otherwise): the
 *    GEMM kernel quantizes the activations itself instead of a separate
 *    per-token pre-pass kernel: the epilogue warps of CTA c quantize token
 *    rows c, c + grid, ... into the workspace and count them done, and every
 *    CTA's activation producer waits (bounded) for all rows before loading
 *    them.  Same codes, scales and results as without the flag.  Measured on
 *    B200 it is slower than the pre-pass (the cross-CTA hand-off costs about
 *    what the kernel boundary does), so it is not the default.
 */
#define QSPEC_GEMM_FUSED_QUANT 2u
/*
 *  QSPEC_GEMM_TEST_STALL: a test hook for the failure path, not for normal
 *    use.  The GEMM's weight producer first waits, for 10 ms at most, on a
 *    barrier that nothing signals; the wait runs out and every CTA gives up
 *    exactly as on a real stall: it raises its abort flag, sets the device
 *    status word, stops every role at its next wait, lets the copies it has
 *    issued land, frees its tensor memory and returns.  `y` is left
 *    incomplete; qspec_workspace_status() then returns QSPEC_ERR_TIMEOUT and
 *    readies the workspace for the next call.
 */
#define QSPEC_GEMM_TEST_STALL 0x100u

/* Operation ids for qspec_workspace_size(). */
enum {
  QSPEC_OP_QUANTIZE_WEIGHTS = 0,
  QSPEC_OP_QUANT_ACT = 1,
  QSPEC_OP_GEMM_W4A4 = 2,
  QSPEC_OP_GEMM_W4A16 = 3,
  QSPEC_OP_SPEC_ACCEPT = 4,
  QSPEC_OP_GEMM_W4A8 = 5
};

/*
 * Offline weight quantization, run once per model (QSpec abstract: both
 * stages reuse the same quantized weights, "without retraining").
 * Recipe (the pages give none; this is the library's definition): for output
 * channel n and group g of `group` consecutive input channels,
 *   s = max|w| / 7 (fp32), s_h = fp16(s) (round to nearest even),
 *   q = clamp(rint(w / s_h), -8, 7) (fp32 division, ties to even; q = 0 if s_h = 0).
 *  w   [n][k] fp32, row-major.
 *  wq  [n][k/2] bytes out: byte j of a row holds k = 2j in its low nibble and
 *      k = 2j+1 in its high nibble, two's complement.
 *  ws  [n][ldg] fp16 bit patterns out, ldg = k/group rounded up to a multiple
 *      of 8 (rows start on 16-byte boundaries, so the GEMMs fetch scale tiles
 *      with TMA); entry [n][g] is s_h of group g for g < k/group, the padding
 *      entries are written as zero.  16-byte aligned.
 * Requires n >= 1, group in {64, 128}, k a multiple of group.
 */
qspec_status qspec_quantize_weights(const float* w, int64_t n, int64_t k, int32_t group,
                                    uint8_t* wq, uint16_t* ws, void* stream);

/*
 * Per-token activation quantization of the W4A4 drafting mode (explainer
 * essay, paragraph 2: W4A4 quantizes both weights and activations).
 * For each row m: a = max_k |x|, s_a = a / 7, inv = 7 / a (fp32 divisions),
 *   q = clamp(rint(x * inv), -8, 7) (product rounded to fp32); a zero row gives 0.
 *  x   [m][k] bf16.
 *  xq  [m][k/2] bytes out, same nibble order as wq.
 *  xs  [m] fp32 out: s_a.
 * Requires m >= 1, k >= 8, k a multiple of 8.
 */
qspec_status qspec_quant_act(const uint16_t* x, int64_t m, int64_t k, uint8_t* xq, float* xs,
                             void* stream);

/*
 * Glue between chained linear layers (the synthetic draft-verify round runs
 * the same layers back to back, each on the previous one's output): writes
 * x[i][j] = bf16(y[i][j]) (round to nearest even) for i < m, j < k.
 *  y   [m][ldy] fp32, the previous layer's output; its first k columns are read.
 *  x   [m][k] bf16 bit patterns out.
 * Requires m >= 1, k >= 8 and a multiple of 8, ldy >= k and a multiple of 4,
 * y and x 16-byte aligned.  Launched as a programmatic dependent of the
 * preceding kernel on the stream (it reads y only after that kernel has
 * completed), so the kernel after it may launch while it waits.
 */
qspec_status qspec_cast_bf16(const float* y, int64_t m, int64_t ldy, int64_t k, uint16_t* x,
                             void* stream);

/*
 * W4A4 drafting GEMM: y = x . deq(wq, ws)^T with the activations quantized
 * per token first (QSpec abstract: "low-precision joint quantization for
 * fast drafting").  Per group g, acc[m][n][g] = sum_{k in g} qa[m][k] qw[n][k]
 * is computed exactly on the int8 tensor cores (int32), and
 *   y[m][n] = s_a[m] * sum_g s_h[n][g] * acc[m][n][g]   (fp32 arithmetic).
 *  x        [m][k] bf16.
 *  wq, ws   as produced by qspec_quantize_weights for [n][k] weights (ws with
 *           its padded row stride); both 16-byte aligned.
 *  y        [m][n] fp32 out.
 *  workspace  device scratch of at least
 *           qspec_workspace_size(QSPEC_OP_GEMM_W4A4, m, n, k, group, 0, 0, 0)
 *           bytes; it must be zero-filled before its first use, and every
 *           call that completes leaves it ready for the next one.
 *  dbg_acc  optional (may be NULL): [m][n][k/group] int32 out, the per-group
 *           integer accumulators.
 *  flags    0 or QSPEC_GEMM_WEIGHTS_READY (see above).
 * Requires m, n >= 1, group in {64, 128}, k a multiple of 128, and fewer than
 * 2^22 work units ceil(m / T) * ceil(n / 128) * (k / 128), where the token
 * tile T is m rounded up to a multiple of 16 for m <= 96, else 128.
 */
qspec_status qspec_gemm_w4a4(const uint16_t* x, int64_t m, int64_t k, const uint8_t* wq,
                             const uint16_t* ws, int64_t n, int32_t group, float* y,
                             void* workspace, size_t workspace_bytes, int32_t* dbg_acc,
                             uint32_t flags, void* stream);

/*
 * W4A8 drafting variant: the W4A4 GEMM with 8-bit per-token activation codes
 * (a higher-precision draft activation; the SpecQuant abstract builds INT4 /
 * FP8 / FP16 model copies, and the QSpec page ties draft quality to how the
 * activations are quantized).  For each row m: a = max_k |x|,
 * s_a = a / 127, inv = 127 / a (fp32 divisions), qa = clamp(rint(x * inv),
 * -128, 127); per group g, acc[m][n][g] = sum_{k in g} qa[m][k] qw[n][k]
 * (exact, int32), y[m][n] = s_a[m] * sum_g s_h[n][g] * acc[m][n][g].
 * Same weights, arguments, requirements and workspace layout as
 * qspec_gemm_w4a4 (workspace sized for QSPEC_OP_GEMM_W4A8).
 */
qspec_status qspec_gemm_w4a8(const uint16_t* x, int64_t m, int64_t k, const uint8_t* wq,
                             const uint16_t* ws, int64_t n, int32_t group, float* y,
                             void* workspace, size_t workspace_bytes, int32_t* dbg_acc,
                             uint32_t flags, void* stream);

/*
 * The drafting GEMMs on a chained layer's fp32 output: the activations are
 * x[i][j] = bf16(xf[i][j]) (round to nearest even) for i < m, j < k, rounded
 * as the per-token quantizer reads them, so no separate bf16 copy (and no
 * qspec_cast_bf16 launch) is needed between layers.  The result is
 * bit-identical to qspec_cast_bf16 followed by qspec_gemm_w4a4 (resp. _w4a8).
 *  xf   [m][ldx] fp32, 16-byte aligned; its first k columns are read.
 *  ldx  row stride in elements: ldx >= k, a multiple of 4.
 * Other arguments, workspace size (QSPEC_OP_GEMM_W4A4 resp. _W4A8) and
 * errors as for qspec_gemm_w4a4; QSPEC_GEMM_FUSED_QUANT is not accepted here.
 */
qspec_status qspec_gemm_w4a4_f32in(const float* xf, int64_t ldx, int64_t m, int64_t k,
                                   const uint8_t* wq, const uint16_t* ws, int64_t n, int32_t group,
                                   float* y, void* workspace, size_t workspace_bytes,
                                   int32_t* dbg_acc, uint32_t flags, void* stream);
qspec_status qspec_gemm_w4a8_f32in(const float* xf, int64_t ldx, int64_t m, int64_t k,
                                   const uint8_t* wq, const uint16_t* ws, int64_t n, int32_t group,
                                   float* y, void* workspace, size_t workspace_bytes,
                                   int32_t* dbg_acc, uint32_t flags, void* stream);

/*
 * W4A16 verifying GEMM: y = x . deq(wq, ws)^T with bf16 activations and the
 * same packed weights as the drafting mode (QSpec abstract: "high-precision
 * weight-only quantization for accurate verification").  deq = q * s_h is
 * applied exactly: the integer codes enter the bf16 tensor cores unchanged
 * and each group's fp32 partial sum is scaled by s_h[n][g].
 *  Arguments as for qspec_gemm_w4a4 (workspace sized for QSPEC_OP_GEMM_W4A16).
 */
qspec_status qspec_gemm_w4a16(const uint16_t* x, int64_t m, int64_t k, const uint8_t* wq,
                              const uint16_t* ws, int64_t n, int32_t group, float* y,
                              void* workspace, size_t workspace_bytes, uint32_t flags,
                              void* stream);

/*
 * Speculative accept / residual resample for a batch of sequences (SpecQuant
 * review, paragraph 5; the rule of "Fast Inference from Transformers via
 * Speculative Decoding" and "Accelerating Large Language Model Decoding with
 * Speculative Sampling").  For sequence b and draft position i < gamma with
 * draft token x:  accept iff u_acc[b][i] * q[b][i][x] < p[b][i][x] (exact).
 * n = first rejected position, or gamma.  The new token is drawn from
 * r = max(0, p[b][n] - q[b][n]) if n < gamma, else from p[b][gamma], by the
 * fixed-point inverse CDF F_j = floor(r_j 2^62), C_j = sum_{i<=j} F_i,
 * token = min{ j : C_j > floor(u_res[b] * C_{V-1}) }; if C_{V-1} = 0 the draw
 * uses p[b][n] instead, and the token is -1 if that row is empty as well.
 *  p          [batch][gamma+1][vocab] fp32 target probabilities (rows sum to <= ~1).
 *  q          [batch][gamma][vocab] fp32 draft probabilities.
 *  draft      [batch][gamma] int32 draft tokens.
 *  u_acc      [batch][gamma] fp32 uniforms in [0, 1).
 *  u_res      [batch] fp32 uniforms in [0, 1).
 *  n_accepted [batch] int32 out.
 *  tokens     [batch][gamma+1] int32 out: accepted draft tokens, then the new
 *             token, then -1 padding.
 *  workspace  optional (NULL or >= qspec_workspace_size(QSPEC_OP_SPEC_ACCEPT,...)
 *             bytes): receives the device status word.  A draft token outside
 *             [0, vocab) is treated as rejected and reported as BAD_INPUT there.
 * Requires 1 <= batch <= 65535, 1 <= gamma <= 16, 4 <= vocab <= 409600, vocab % 4 == 0.
 */
qspec_status qspec_spec_accept(const float* p, const float* q, const int32_t* draft,
                               const float* u_acc, const float* u_res, int32_t batch,
                               int32_t gamma, int32_t vocab, int32_t* n_accepted,
                               int32_t* tokens, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * Greedy verification for a batch of sequences (SpecQuant review, paragraph
 * 5: a draft that matches in full is kept and the first mismatch is replaced
 * by the target model's own choice).  The target's choice at position i is
 * t_i = argmax_j p[b][i][j], ties to the lowest index; draft position i is
 * accepted while draft[b][i] == t_i; n = first mismatch (gamma if none); the
 * new token is t_n.  Only rows 0..n of p are read.
 *  p          [batch][gamma+1][vocab] fp32 target scores (probabilities or
 *             logits: only their order matters); finite.
 *  draft      [batch][gamma] int32 draft tokens.
 *  n_accepted [batch] int32 out.
 *  tokens     [batch][gamma+1] int32 out: accepted draft tokens, then t_n,
 *             then -1 padding.
 *  workspace  optional, as for qspec_spec_accept: a draft token outside
 *             [0, vocab) never matches and is reported as BAD_INPUT there.
 * Requires 1 <= batch <= 65535, 1 <= gamma <= 16, 4 <= vocab <= 409600, vocab % 4 == 0,
 * p 16-byte aligned.
 */
qspec_status qspec_spec_accept_greedy(const float* p, const int32_t* draft, int32_t batch,
                                      int32_t gamma, int32_t vocab, int32_t* n_accepted,
                                      int32_t* tokens, void* workspace, size_t workspace_bytes,
                                      void* stream);

/*
 * The KV cache shared by the drafting and the verifying stage.
 * QSpec page, abstract: the two stages reuse the KV cache as well as the
 * weights.  The page gives no layout or rule; the ones taken here:
 *  - one cache per layer, K and V each [batch][h_kv][l_max][head_dim] bf16
 *    (device, caller-owned), head_dim = 128;
 *  - `lens` (device int32 [batch]): the number of valid positions of each
 *    sequence at the start of the round; only qspec_kv_commit changes it;
 *  - a pass over t_new new tokens per sequence (drafting pass j: t_new = 1,
 *    offset = j; the verifying pass: t_new = gamma + 1, offset = 0, which
 *    overwrites the drafted entries with the verifier's) first appends the
 *    tokens' keys and values at positions lens[b] + offset + t, then runs the
 *    attention, in which token (b, t) sees positions 0 .. lens[b] + offset + t;
 *  - after the accept step, qspec_kv_commit advances lens[b] by
 *    n_accepted[b] + 1 (the accepted drafts plus the verifier's token); the
 *    entries past it are rolled back simply by being overwritten later.
 * Token rows come from the fused QKV projection (a GEMM output): row
 * b * t_new + t of `qkv` (fp32, row stride ld_qkv floats, a multiple of 4,
 * at least (h_q + 2 h_kv) * 128) holds the h_q query heads, then the h_kv
 * key heads, then the h_kv value heads, 128 columns each.  Query head h reads
 * KV head h / (h_q / h_kv); t_new * (h_q / h_kv) must be at most 32.
 * Asynchronous on `stream`.  Host-side argument errors return
 * QSPEC_ERR_INVALID_ARG and launch nothing; a position outside the cache
 * (from the device-side lengths) is skipped and reported as
 * QSPEC_ERR_BAD_INPUT through qspec_workspace_status on `workspace`
 * (optional for append and commit: NULL, or >= 256 zeroed bytes).
 */

/* Writes the t_new new keys and values of every sequence, rounded to bf16
 * (nearest even), at positions lens[b] + offset + t. */
qspec_status qspec_kv_append(const float* qkv, int64_t ld_qkv, int32_t batch, int32_t t_new,
                             int32_t h_q, int32_t h_kv, int32_t head_dim, const int32_t* lens,
                             int32_t offset, uint16_t* k_cache, uint16_t* v_cache, int32_t l_max,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Decode attention over the shared cache (call after qspec_kv_append of the
 * same tokens):  out[b*t_new + t][h*128 + i] = sum_j w_j v_j[i],
 * w = softmax_j(q . k_j / sqrt(128)) over j = 0 .. lens[b] + offset + t, with
 * q the token's query head h (fp32, as given), k_j, v_j the cached entries of
 * KV head h / (h_q / h_kv).  Scores, weights and sums in fp32.
 *  ctx_max    a bound on lens[b] + offset + t_new for every b, at most l_max
 *             and 32768: it sizes the launch (one CTA per 256 keys); a
 *             sequence past it gets zero output and QSPEC_ERR_BAD_INPUT.
 *  out        fp32, row stride ld_out >= h_q * 128.
 *  workspace  >= qspec_attn_workspace_size(...) bytes, 16-byte aligned, zeroed
 *             before its first use; every call that completes leaves it ready
 *             for the next.  Calls sharing one workspace must not overlap.
 * The result does not depend on the order in which the CTAs finish. */
qspec_status qspec_attn_decode(const float* qkv, int64_t ld_qkv, int32_t batch, int32_t t_new,
                               int32_t h_q, int32_t h_kv, int32_t head_dim, const int32_t* lens,
                               int32_t offset, const uint16_t* k_cache, const uint16_t* v_cache,
                               int32_t l_max, int32_t ctx_max, float* out, int64_t ld_out,
                               void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace qspec_attn_decode needs (0 for invalid arguments). */
size_t qspec_attn_workspace_size(int32_t batch, int32_t t_new, int32_t h_q, int32_t h_kv,
                                 int32_t head_dim, int32_t ctx_max);

/* lens[b] += n_accepted[b] + 1 for every sequence (device arrays); a count
 * that is negative or would pass l_max leaves lens[b] unchanged and is
 * reported as QSPEC_ERR_BAD_INPUT. */
qspec_status qspec_kv_commit(int32_t* lens, const int32_t* n_accepted, int32_t batch,
                             int32_t l_max, void* workspace, size_t workspace_bytes, void* stream);

/*
 * W4A16 verifying GEMM that allocates nothing and takes no workspace.
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory at the point of the call: a plugin
 * hosted by an application that owns all device memory and permits no
 * allocation outside its own pools, or a latency-critical path that must not
 * enter the allocator (cudaMalloc/cudaFree may synchronise the device).
 * Call it from ordinary host code: CUDA forbids CUDA calls inside a host
 * function enqueued on a stream, and this entry point makes several.
 * Computes exactly what qspec_gemm_w4a16 computes, with its scratch held in a
 * file-scope device array of QSPEC_STATIC_SCRATCH_BYTES (16 MiB) that every
 * GPU loading this library keeps until the process exits.
 *  - The first call on a device looks up the array's device address (with
 *    that device current) and keeps it for the life of the process; make
 *    that first call before any stream capture, and do not use this entry
 *    point on a device after cudaDeviceReset() on it.
 *  - Every call shares the one array: calls that overlap on the GPU (on
 *    different streams, or from different threads) race and must not be
 *    issued.  Each call clears the split-tile tickets with an asynchronous
 *    memset on `stream` (so the GEMM cannot start streaming weights before
 *    the preceding kernel ends, as it can on the workspace path); nothing
 *    else needs to start at zero.
 *  - Device faults (a wait that ran out) are recorded in the array's status
 *    word, which stays set until qspec_gemm_w4a16_noalloc_status() reads it.
 *  - Shapes whose scratch would exceed the array (for example m > 96 on a
 *    148-SM B200) return QSPEC_ERR_WORKSPACE_TOO_SMALL and launch nothing.
 *  - Calls no cudaMalloc, cudaFree or other allocating routine.
 * Arguments as for qspec_gemm_w4a16, without workspace.
 */
#define QSPEC_STATIC_SCRATCH_BYTES (16u << 20)
qspec_status qspec_gemm_w4a16_noalloc(const uint16_t* x, int64_t m, int64_t k, const uint8_t* wq,
                                      const uint16_t* ws, int64_t n, int32_t group, float* y,
                                      uint32_t flags, void* stream);

/*
 * Device status of qspec_gemm_w4a16_noalloc on the current device, without
 * allocating: synchronizes `stream`, reads the built-in array's status word,
 * clears it (and, after a timeout, the split-tile tickets) and returns
 * QSPEC_OK, QSPEC_ERR_TIMEOUT or QSPEC_ERR_BAD_INPUT (QSPEC_ERR_CUDA if the
 * read failed).  QSPEC_OK if no such call has run on the device.
 */
qspec_status qspec_gemm_w4a16_noalloc_status(void* stream);

/* Bytes of workspace an operation needs on the current device (0 = none).
 * Unused size arguments are ignored.  Returns 0 for invalid arguments too. */
size_t qspec_workspace_size(int32_t op, int64_t m, int64_t n, int64_t k, int32_t group,
                            int32_t batch, int32_t gamma, int32_t vocab);

/* Synchronizes `stream`, reads the device status word at the start of
 * `workspace`, clears it, and returns QSPEC_OK, QSPEC_ERR_TIMEOUT or
 * QSPEC_ERR_BAD_INPUT (or QSPEC_ERR_CUDA if the read itself failed).  After
 * a timeout (which only a GEMM reports) it also clears the split-tile
 * tickets the stopped call may have left taken, so the workspace is ready
 * for the next call. */
qspec_status qspec_workspace_status(void* workspace, void* stream);

/* Version of this ABI (3: adds QSPEC_GEMM_TEST_STALL, qspec_gemm_w4a8, qspec_cast_bf16,
 * qspec_spec_accept_greedy and qspec_gemm_w4a16_noalloc_status; 4: adds
 * qspec_gemm_w4a4_f32in and qspec_gemm_w4a8_f32in; 5: adds qspec_kv_append,
 * qspec_attn_decode, qspec_attn_workspace_size and qspec_kv_commit). */
#define QSPEC_ABI_VERSION 5
int32_t qspec_abi_version(void);

/* Static, human-readable name of a status code. */
const char* qspec_status_string(qspec_status status);

#ifdef __cplusplus
}
#endif

#endif /* QSPEC_H_ */
