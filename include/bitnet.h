/*
 * bitnet.h -- C ABI of libbitnet.so, the BitNet b1.58 BitLinear hot path
 * for NVIDIA B200 (sm_100a).
 *
 * The library quantises latent weights to ternary values with a per-tensor
 * absmean scale, packs them at 2 bits per weight, quantises activations to
 * int8 per token with an absmax scale (optionally after an RMSNorm gain), and
 * computes y = (x_q . W_q^T) * gamma * s_x with hand-written CUDA kernels:
 * a packed-ternary GEMV for a few tokens and a tcgen05 int8 tensor-core GEMM
 * for many tokens.
 *
 * Sources of the operations (page title and section):
 *   - "Key Technologies Enabling the BitNET Family", Advanced Quantization
 *     Methodologies: ternary weights by absmean quantisation, 8-bit
 *     activations by per-token absmax quantisation; Architectural
 *     Innovations: BitLinear layers, RMSNorm, no bias terms.
 *   - "BitNet / Ternary / Binary -- Les LLMs 1-bit" (brain.gartu.xyz),
 *     section "Apercu de l'entrainement d'un BitLinear": beta = mean|w|,
 *     w_q = clamp(round(w / (beta + 1e-8)), -1, 1), y = F.linear(x, w_q).
 *   - "BitNet Technical Notes" (afondiel.github.io), System Design and the
 *     Appendix glossary: 2 bits per ternary weight.
 *   - Hacker News thread on the b1.58 paper: a ternary dot product is the
 *     sum of activations at +1 weights minus the sum at -1 weights;
 *     activations are int8 at inference.
 *
 * Conventions for every call:
 *   - Matrices are row-major.  W and W_q are [N, K] (out-features x in-
 *     features, the nn.Linear convention); x, x_q are [M, K]; y is [M, N].
 *   - Every tensor pointer is a DEVICE pointer owned by the caller; the
 *     library never allocates, frees or keeps caller memory.  Scratch space
 *     comes from a caller-supplied workspace (see bitnet_workspace_bytes).
 *   - Pointers to tensors must be 16-byte aligned (BITNET_ERR_ALIGN).
 *   - K must be a positive multiple of 16; M, N >= 1; M, N, K < 2^31 and
 *     N*K < 2^39 (BITNET_ERR_SHAPE).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  The returned status reports argument errors and
 *     launch errors only.  Errors found on the device (a watchdog expiry,
 *     invalid codes) are recorded in the workspace's status word and read
 *     with bitnet_get_error().
 *   - Rounding: round-to-nearest-even everywhere (torch.round semantics).
 *   - There is no CPU fallback: without a usable sm_100 device every compute
 *     call returns BITNET_ERR_UNSUPPORTED.
 */
#ifndef BITNET_H
#define BITNET_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *bitnet_stream_t;   /* same type as cudaStream_t */

typedef enum bitnet_status {
    BITNET_OK = 0,
    BITNET_ERR_NULL = 1,          /* a required pointer is NULL */
    BITNET_ERR_SHAPE = 2,         /* a size is out of range or K % 16 != 0 */
    BITNET_ERR_ALIGN = 3,         /* a tensor pointer is not 16-byte aligned */
    BITNET_ERR_DTYPE = 4,         /* unknown dtype code */
    BITNET_ERR_UNSUPPORTED = 5,   /* no sm_100 device, or a forced path that cannot run */
    BITNET_ERR_CUDA = 6,          /* a CUDA runtime call failed */
    BITNET_ERR_TIMEOUT = 7,       /* a device-side wait ran past its limit */
    BITNET_ERR_WORKSPACE = 8,     /* workspace NULL, too small or misaligned */
    BITNET_ERR_VALUE = 9          /* invalid ternary value or 2-bit code */
} bitnet_status;

/* dtype codes for activations and outputs */
#define BITNET_F32 0
#define BITNET_BF16 1

/* path codes for the *_ex calls */
#define BITNET_PATH_AUTO 0
#define BITNET_PATH_GEMV 1        /* CUDA-core packed-ternary GEMV, M <= 4 */
#define BITNET_PATH_TC 2          /* tcgen05 int8 tensor-core GEMM, any M */

/* ------------------------------------------------------------------------
 * Workspace.  A caller-owned device buffer, 256-byte aligned.  Its first
 * 256 bytes hold the device status word; zero them once before first use
 * (bitnet_workspace_init).  Calls sharing one workspace must be ordered
 * on one stream.
 * ------------------------------------------------------------------------ */

/* Bytes needed by bitnet_linear / bitnet_linear_q for an M x K x N call
 * (covers every smaller call with the same or smaller M*K and M). */
size_t bitnet_workspace_bytes(int64_t M, int64_t K, int64_t N);

/* Bytes needed by bitnet_quant_weights for an N x K weight. */
size_t bitnet_quant_weights_workspace_bytes(int64_t N, int64_t K);

/* Zero the status word of a workspace (asynchronous on stream). */
bitnet_status bitnet_workspace_init(void *ws, size_t ws_bytes, bitnet_stream_t stream);

/* Synchronise `stream`, read the workspace status word and clear it.
 * Returns BITNET_OK, BITNET_ERR_TIMEOUT or BITNET_ERR_VALUE recorded by an
 * earlier call, or BITNET_ERR_CUDA if the synchronisation failed. */
bitnet_status bitnet_get_error(void *ws, bitnet_stream_t stream);

const char *bitnet_status_str(bitnet_status s);

/* ------------------------------------------------------------------------
 * Weight preparation (offline, once per weight tensor).
 * ------------------------------------------------------------------------ */

/* Absmean ternarisation ("Key Technologies ...", Advanced Quantization
 * Methodologies; "BitNet / Ternary / Binary", BitLinear forward):
 *   gamma  = mean over all N*K entries of |W|: the exact real sum of |W|
 *            rounded to binary64, divided by N*K in binary64, rounded to
 *            binary32 (deterministic, independent of launch shape);
 *   W_q    = clamp(rint(W / (gamma + eps)), -1, 1) in binary32, with
 *            gamma + eps rounded to binary32 before one IEEE division.
 * W: [N, K] binary32, finite.  Wq: [N, K] int8 output, or NULL to compute
 * gamma only.  gamma: one binary32 on the device (output).  eps: 1e-8 in
 * the pages.  ws: at least bitnet_quant_weights_workspace_bytes(N, K). */
bitnet_status bitnet_quant_weights(const float *W, int64_t N, int64_t K, float eps,
                                   int8_t *Wq, float *gamma,
                                   void *ws, size_t ws_bytes, bitnet_stream_t stream);

/* The ternarisation step alone with a given gamma (device pointer):
 * W_q = clamp(rint(W / (*gamma + eps)), -1, 1).  Same layout as above. */
bitnet_status bitnet_ternarise(const float *W, int64_t N, int64_t K, const float *gamma,
                               float eps, int8_t *Wq, bitnet_stream_t stream);

/* 2-bit pack ("BitNet Technical Notes", 2 bits per ternary weight).
 * Layout (this library's; the pages fix none):
 *   code c = q + 1  (0 -> -1, 1 -> 0, 2 -> +1; code 3 is invalid);
 *   row n occupies bytes [n*K/4, (n+1)*K/4) of Wp, so Wp is [N, K/4] uint8;
 *   the row is a sequence of little-endian 32-bit groups, one per 16
 *   weights; in group g, weight k = 16g + 4s + j (s, j in 0..3) sits at
 *   bits [8j + 2s, 8j + 2s + 1].  Thus (group >> 2s) & 0x03030303 gives the
 *   codes of weights 16g+4s .. 16g+4s+3 as four bytes in k order.
 * Wq: [N, K] int8 with values in {-1, 0, 1}.  Entries outside that set are
 * stored as code 3, counted into *n_invalid (device uint32, may be NULL,
 * accumulated, not cleared), and make later calls compute with code 3
 * (weight +2).  Wp: [N, K/4] uint8 output. */
bitnet_status bitnet_pack(const int8_t *Wq, int64_t N, int64_t K, uint8_t *Wp,
                          uint32_t *n_invalid, bitnet_stream_t stream);

/* Inverse of bitnet_pack (for tests and inspection).  Code 3 decodes to 0
 * and is counted into *n_invalid (device uint32, may be NULL). */
bitnet_status bitnet_unpack(const uint8_t *Wp, int64_t N, int64_t K, int8_t *Wq,
                            uint32_t *n_invalid, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * BitNet b1 binary weights ("BitNet / Ternary / Binary -- Les LLMs 1-bit",
 * BitNet b1 (binaire): every weight of the BitLinear layer is exactly +1
 * or -1).  The pages give no binarisation rule; this library reads it as
 * the sign with ties to +1 and the absmean scale of the ternary case.
 * ------------------------------------------------------------------------ */

/* beta = mean|W| exactly as gamma in bitnet_quant_weights (same workspace
 * and errors), and W_b = +1 where W >= 0, else -1 (NaN gives -1).
 * Wb: [N, K] int8 output or NULL (beta only); beta: device binary32. */
bitnet_status bitnet_quant_weights_b1(const float *W, int64_t N, int64_t K, int8_t *Wb,
                                      float *beta, void *ws, size_t ws_bytes,
                                      bitnet_stream_t stream);

/* 1-bit pack: K % 32 == 0; group g of row n is the little-endian uint32 at
 * byte n*K/8 + 4g; weight k = 32g + 4s + j (s in 0..7, j in 0..3) is bit
 * 8j + s, 1 for +1 and 0 for -1.  Values other than +-1 are stored as 0
 * and counted into *n_invalid (device uint32, may be NULL, accumulated).
 * Wp: [N, K/8] uint8 output. */
bitnet_status bitnet_pack_b1(const int8_t *Wb, int64_t N, int64_t K, uint8_t *Wp,
                             uint32_t *n_invalid, bitnet_stream_t stream);

/* Inverse of bitnet_pack_b1: every bit pattern is valid. */
bitnet_status bitnet_unpack_b1(const uint8_t *Wp, int64_t N, int64_t K, int8_t *Wb,
                               bitnet_stream_t stream);

/* BitLinear forward with 1-bit weights: as bitnet_linear, with
 *   acc[m,n] = sum_k x_q[m,k] * W_b[n,k] = 2 sum_{W_b = +1} x_q - sum_k x_q
 *   y[m,n]   = (float)acc[m,n] * (beta * s_x[m]).
 * K % 128 == 0 (else BITNET_ERR_SHAPE).  M = 1 runs the fused streaming
 * GEMV (up to K = 79872; beyond, the tensor-core path); larger M the
 * quantiser then the tensor-core GEMM.  Wp: [N, K/8] (bitnet_pack_b1).
 * ws: bitnet_workspace_bytes(M, K, N) bytes. */
bitnet_status bitnet_linear_b1(const void *x, int x_dtype, int64_t M, int64_t K,
                               const uint8_t *Wp, int64_t N, const float *beta,
                               const float *rms_gain, float rms_eps,
                               void *y, int y_dtype, void *ws, size_t ws_bytes,
                               bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * Base-3 packing: five ternary weights per byte (3^5 = 243 <= 256), about
 * 1.6 bits per weight ("Key Technologies ... BitNET Family", Memory
 * Efficiency: 0.4 GB for the 2B model; Hacker News thread on "2 bits
 * instead of 1.58").  A decode format: one token per call.  K % 16 == 0, as
 * everywhere in this library (K need not be a multiple of 20 or 80).
 * Layout (this library's): a row takes bitnet_t3_row_bytes(K) =
 * ceil(K/80) * 16 bytes; byte j of the little-endian uint32 group g holds
 * sum_i c(20g + 4i + j) 3^i (i = 0..4) with codes c = q + 1; weights past K
 * code as 1 (q = 0).
 * ------------------------------------------------------------------------ */
int64_t bitnet_t3_row_bytes(int64_t K);

/* Pack Wq [N, K] int8 in {-1, 0, 1} into Wp [N, bitnet_t3_row_bytes(K)].
 * Values outside {-1, 0, 1} are stored as code 1 and counted into
 * *n_invalid (device uint32, may be NULL, accumulated). */
bitnet_status bitnet_pack_t3(const int8_t *Wq, int64_t N, int64_t K, uint8_t *Wp,
                             uint32_t *n_invalid, bitnet_stream_t stream);

/* Inverse of bitnet_pack_t3; a byte above 242 is invalid: its five weights
 * read as 0 and it is counted into *n_invalid (may be NULL). */
bitnet_status bitnet_unpack_t3(const uint8_t *Wp, int64_t N, int64_t K, int8_t *Wq,
                               uint32_t *n_invalid, bitnet_stream_t stream);

/* BitLinear forward of ONE token (x [1, K]) with base-3 packed weights:
 * y[n] exactly as bitnet_linear would give with the same ternary weights.
 * The streaming GEMV decodes the base-3 digits in registers; it bounds K
 * at 57600 (BITNET_ERR_UNSUPPORTED beyond: this format has no tensor-core
 * path).  ws: bitnet_workspace_bytes(1, K, N) bytes. */
bitnet_status bitnet_linear_t3(const void *x, int x_dtype, int64_t K,
                               const uint8_t *Wp, int64_t N, const float *gamma,
                               const float *rms_gain, float rms_eps,
                               void *y, int y_dtype, void *ws, size_t ws_bytes,
                               bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * Per-call path.
 * ------------------------------------------------------------------------ */

/* Per-token absmax int8 quantisation ("Key Technologies ...", Advanced
 * Quantization Methodologies), with an optional RMSNorm gain
 * (Architectural Innovations: RMSNorm, no bias).  For each row m:
 *   t_k  = x_k * g_k            (t = x when rms_gain is NULL)
 *   a    = max(max_k |t_k|, 1e-5)
 *   x_q  = clamp(rint(t_k * (127 / a)), -128, 127)       (never -128)
 *   s_x  = a / 127                                  (no gain), or
 *   s_x  = r * a / 127, r = 1 / sqrt(mean_k x_k^2 + rms_eps)  (with gain;
 *          r and the product in binary64, s_x rounded to binary32).
 * The gain's row factor r cancels inside the codes, so x_q does not depend
 * on r and is exact; r only scales s_x.
 *   x_sum = sum_k x_q (exact int32).
 * x: [M, K] binary32 (x_dtype BITNET_F32) or bfloat16 (BITNET_BF16).
 * rms_gain: [K] binary32 or NULL.  xq: [M, K] int8; x_scale: [M] binary32;
 * x_sum: [M] int32 or NULL.  All outputs on the device. */
bitnet_status bitnet_quant_act(const void *x, int x_dtype, int64_t M, int64_t K,
                               const float *rms_gain, float rms_eps,
                               int8_t *xq, float *x_scale, int32_t *x_sum,
                               bitnet_stream_t stream);

/* BitLinear forward: quantise x per token (as bitnet_quant_act, with the
 * optional fused RMSNorm gain), contract with the packed ternary weights
 * and rescale:
 *   acc[m,n] = sum_k x_q[m,k] * W_q[n,k]          (exact int32)
 *   y[m,n]   = (float)acc[m,n] * (gamma * s_x[m])  (binary32, then rounded
 *              to bfloat16 when y_dtype is BITNET_BF16).
 * ("BitNet / Ternary / Binary", F.linear(x, w_q) with the two quantiser
 * scales undone.)  No bias.
 * Wp: [N, K/4] packed weights (bitnet_pack).  gamma: device binary32.
 * y: [M, N] of y_dtype.  ws: bitnet_workspace_bytes(M, K, N) bytes.
 * Small M runs one fused kernel (quantise + GEMV); larger M runs the
 * quantiser then the tensor-core GEMM.  The fused kernel holds the
 * quantised activations and one packed weight row per ring slot in shared
 * memory, which bounds K at 48128 (M = 1), 39936 (M = 2) and 29696
 * (M = 3, 4) for 2-bit weights; beyond that the automatic choice takes the
 * tensor-core path, which has no K bound. */
bitnet_status bitnet_linear(const void *x, int x_dtype, int64_t M, int64_t K,
                            const uint8_t *Wp, int64_t N, const float *gamma,
                            const float *rms_gain, float rms_eps,
                            void *y, int y_dtype, void *ws, size_t ws_bytes,
                            bitnet_stream_t stream);

/* bitnet_linear with an explicit path (BITNET_PATH_*).  BITNET_PATH_GEMV
 * with M > 4, or with K beyond the fused kernel's bound (see
 * bitnet_linear), returns BITNET_ERR_UNSUPPORTED. */
bitnet_status bitnet_linear_ex(const void *x, int x_dtype, int64_t M, int64_t K,
                               const uint8_t *Wp, int64_t N, const float *gamma,
                               const float *rms_gain, float rms_eps,
                               void *y, int y_dtype, void *ws, size_t ws_bytes,
                               int path, bitnet_stream_t stream);

/* Contraction and rescale on pre-quantised activations (bitnet_quant_act
 * outputs).  x_sum may be NULL (recomputed on the device).  acc: [M, N]
 * int32 export of the exact accumulator, or NULL.  y may be NULL when only
 * acc is wanted.  path: BITNET_PATH_*. */
bitnet_status bitnet_linear_q(const int8_t *xq, const float *x_scale, const int32_t *x_sum,
                              int64_t M, int64_t K, const uint8_t *Wp, int64_t N,
                              const float *gamma, void *y, int y_dtype, int32_t *acc,
                              void *ws, size_t ws_bytes, int path, bitnet_stream_t stream);

/* Feed-forward down projection with the ReLU^2 gate fused into the input
 * quantiser ("Key Technologies ...", Architectural Innovations: squared
 * ReLU activations in the feed-forward layers, no bias):
 *   t_k = (max(gate_k, 0) * max(gate_k, 0)) * up_k   (binary32, one rounding
 *         per operation, in that order; NaN gate counts as 0)
 * then t is quantised and contracted exactly as x in bitnet_linear (with
 * the optional RMSNorm gain applied to t), and
 *   y[m,n] = resid[m,n] + (float)acc[m,n] * (gamma * s_x[m])   (binary32
 *            sum of the rounded product, then y_dtype)
 * when resid (the block's residual stream, [M, N] of y_dtype) is given,
 * else y as in bitnet_linear.  gate, up: [M, K] of x_dtype (the gate and up
 * projections' outputs).  resid may alias y.  Same workspace as
 * bitnet_linear.  The residual add is this library's reading of a
 * Transformer feed-forward block; the pages name only the gate. */
bitnet_status bitnet_linear_relu2(const void *gate, const void *up, int x_dtype, int64_t M, int64_t K,
                                  const uint8_t *Wp, int64_t N, const float *gamma,
                                  const float *rms_gain, float rms_eps, const void *resid,
                                  void *y, int y_dtype, void *ws, size_t ws_bytes,
                                  bitnet_stream_t stream);

/* bitnet_quant_act of the ReLU^2 gate t = max(gate, 0)^2 * up (as in
 * bitnet_linear_relu2): codes, scales and code sums of t. */
bitnet_status bitnet_quant_act_relu2(const void *gate, const void *up, int x_dtype, int64_t M, int64_t K,
                                     const float *rms_gain, float rms_eps,
                                     int8_t *xq, float *x_scale, int32_t *x_sum,
                                     bitnet_stream_t stream);

/* One problem of a grouped GEMV call. */
typedef struct bitnet_gemv_problem {
    const void *x;          /* [M, K] activations of the call's x_dtype, device */
    const uint8_t *Wp;      /* [N, K/4] packed weights (bitnet_pack), device */
    const float *gamma;     /* device binary32 weight scale */
    const float *rms_gain;  /* [K] RMSNorm gain, device, or NULL (no norm) */
    void *y;                /* [M, N] output of the call's y_dtype, device */
    int64_t K, N;
} bitnet_gemv_problem;

/* Several independent BitLinear forwards with the same token count M <= 4
 * in ONE launch: each problem is computed exactly as bitnet_linear would
 * (quantise its x, contract with its weights, rescale by its gamma), but the
 * packed weights of all problems are streamed as one contiguous byte range
 * split evenly over the GPU, so the memory system never idles between calls.
 * Problems whose x and rms_gain pointers (and K) equal the previous
 * problem's reuse its quantised activations: fused Q|K|V or up|gate
 * projections ("Key Technologies ...", Architectural Innovations: BitLinear
 * layers of one block share their input).  The problems' outputs must not
 * overlap each other's inputs.
 * problems: host array of `count` entries (1 <= count <= 256), read during
 * the call only.  Every K must be a multiple of 64, and the largest K at
 * most the fused kernel's bound (bitnet_linear: 48128 at M = 1, 39936 at
 * M = 2, 29696 at M = 3, 4); otherwise BITNET_ERR_UNSUPPORTED.  ws: at
 * least bitnet_workspace_bytes(1, 16, 1) bytes (status word only). */
bitnet_status bitnet_linear_grouped(const bitnet_gemv_problem *problems, int count, int64_t M,
                                    int x_dtype, float rms_eps, int y_dtype,
                                    void *ws, size_t ws_bytes, bitnet_stream_t stream);

/* bitnet_quant_weights for callers that cannot allocate device memory and
 * so cannot provide its workspace: code running under CUDA stream capture
 * (where allocation is not allowed), or a host framework that owns the
 * device memory pool and gives extensions no allocator.  Same arguments and
 * results as bitnet_quant_weights (gamma and W_q are identical), minus the
 * workspace.  The pages have no counterpart: this is an interface choice.
 *   - Scratch: a 256 KiB array inside the library, resident on every GPU
 *     that loads it until the process exits.  Nothing is allocated or freed.
 *   - Limit: N*K <= 2048 * 2^24 (about 3.4e10); larger returns
 *     BITNET_ERR_SHAPE.
 *   - The first call on each device looks up the array's device address
 *     (with that device current); make that first call before any stream
 *     capture.
 *   - All calls share the one array, which keeps the last call's contents;
 *     every entry a call reads is written earlier in the same call, so
 *     nothing needs clearing.  Calls that overlap on the GPU (other streams,
 *     or other threads) race on it: order them on one stream.
 *   - Non-finite W is not reported (there is no workspace status word). */
bitnet_status bitnet_quant_weights_noalloc(const float *W, int64_t N, int64_t K, float eps,
                                           int8_t *Wq, float *gamma, bitnet_stream_t stream);

/* bitnet_linear_grouped for BitNet b1 weights (bitnet_pack_b1, Wp [N, K/8],
 * gamma = beta), one token (M = 1), K % 128 == 0, K <= 79872: each problem
 * is computed exactly as bitnet_linear_b1. */
bitnet_status bitnet_linear_grouped_b1(const bitnet_gemv_problem *problems, int count, int x_dtype,
                                       float rms_eps, int y_dtype, void *ws, size_t ws_bytes,
                                       bitnet_stream_t stream);

/* bitnet_linear_grouped for base-3 packed weights (bitnet_pack_t3), one
 * token (M = 1), K <= 57600: each problem is computed exactly as
 * bitnet_linear_t3. */
bitnet_status bitnet_linear_grouped_t3(const bitnet_gemv_problem *problems, int count, int x_dtype,
                                       float rms_eps, int y_dtype, void *ws, size_t ws_bytes,
                                       bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * Failure detection.
 * ------------------------------------------------------------------------ */

/* Device-side wait limit, in microseconds, used by every bounded wait of
 * the tensor-core pipeline (default 2,000,000).  A wait that runs past it
 * records BITNET_ERR_TIMEOUT in the workspace status word and the kernel
 * returns after releasing what it holds.  Process-wide setting. */
bitnet_status bitnet_set_wait_limit_us(uint32_t limit_us);

/* Launch a one-CTA kernel that waits on a barrier nothing will complete,
 * with a limit of limit_us microseconds.  It exercises the watchdog path:
 * afterwards bitnet_get_error(ws) returns BITNET_ERR_TIMEOUT. */
bitnet_status bitnet_watchdog_selftest(void *ws, size_t ws_bytes, uint32_t limit_us,
                                       bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * Diagnostics.
 * ------------------------------------------------------------------------ */

/* The launch plan the streaming GEMV (bitnet_linear at small M,
 * bitnet_linear_grouped, and the b1 and base-3 forms) would use for a
 * grouped call of `count` problems (1 <= count <= 256) of sizes K[i] x N[i]
 * with M tokens, on a device described by `sms` (multiprocessor count) and
 * `smem_optin` (opt-in shared memory per block, bytes).  Pure host
 * computation: it reads no device and launches nothing, so it also runs
 * without a GPU.  It is an interface choice of this library; the pages have
 * no counterpart.
 *   bits: 2 (bitnet_pack), 1 (bitnet_pack_b1) or 3 (bitnet_pack_t3).
 *   prequant: nonzero for pre-quantised activations (bitnet_linear_q).
 *   shape: host array of 5, or NULL: {grid (CTAs), dynamic shared-memory
 *          bytes per CTA, activation buffers (1 or 2), ring slots per
 *          consumer warp (1 or 2), bytes per slot}.
 *   rows, task: host arrays of `count`, or NULL: rows per chunk and the
 *          contraction task of each problem.
 * K, N, M follow the library's shape rules (BITNET_ERR_SHAPE otherwise).
 * Returns BITNET_ERR_UNSUPPORTED when no plan fits the shared memory, which
 * is when the calls above fall back or fail as their comments say. */
bitnet_status bitnet_debug_stream_plan(const int64_t *K, const int64_t *N, int count, int64_t M, int bits,
                                       int prequant, int sms, int smem_optin,
                                       int64_t *shape, int32_t *rows, int32_t *task);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_H */
