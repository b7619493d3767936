/*
 * bitlinear.h -- C ABI of libbitlinear.so, the BitNet b1.58 BitLinear forward
 * for NVIDIA B200 (sm_100a).
 *
 * The operation follows the Falcon-Edge blog (Falcon-LLM team, "Falcon-Edge:
 * a series of powerful, universal and fine-tunable 1.58bit language models";
 * section "Falcon-Edge, a series of universal models"), whose listings define
 *   activation_norm_quant(x):  s_x = 127 / max(max_k |x|, 1e-5) per token,
 *                              q = clamp(round(x * s_x), -128, 127)
 *   _weight_quant(w):          s_w = 1 / max(mean |w|, 1e-5) over the tensor,
 *                              u = clamp(round(w * s_w), -1, 1)
 *   BitLinear.forward(x):      y = F.linear(q, u) / (s_x * s_w) (+ bias)
 * Weights are ternary {-1, 0, 1} ("The Era of 1-bit LLMs", TL;DR) and are
 * stored in 2 bits each ("BitNet: inference framework for 1-bit LLMs",
 * GeekNews, Hacker News comments section).
 *
 * Numerics (identical to the CPU oracle that the tests compare against):
 *   - bf16 inputs widen exactly to float32; scales, x*s_x and w*s_w are
 *     float32 round-to-nearest; round() is round-half-to-even;
 *   - mean |w| is the exact sum over the whole tensor divided by N*K and
 *     rounded once to float32 (independent of summation order);
 *   - the contraction is exact in int32 (|acc| <= 127*K);
 *   - d = s_x*s_w (float32), y32 = float(acc) / d (float32, correctly
 *     rounded), y32 += float(bias) if a bias is given, y = bf16_rne(y32).
 *     float(acc) is exact while |acc| < 2^24 (always for K <= 132104), and
 *     rounds to nearest even beyond that.
 *   The flag BITLINEAR_BF16_FAITHFUL switches to the rounding of a bf16
 *   module instead (see its definition below).
 *
 * Conventions for every entry point:
 *   - Shapes: x is [M, K] row-major, W is [N, K] (nn.Linear [out, in]),
 *     y is [M, N].  K must be a positive multiple of 64 and at most 2^19;
 *     0 <= M <= 2^23 and 1 <= N <= 2^23 (BITLINEAR_ERR_SHAPE otherwise).
 *     M == 0 is a no-op that returns BITLINEAR_OK.
 *   - bf16 values travel as their uint16_t bit patterns.
 *   - Every pointer argument is a DEVICE pointer unless its name ends in
 *     _host.  Device pointers must be 16-byte aligned (BITLINEAR_ERR_ALIGN
 *     otherwise).  All buffers are owned by the caller; the library
 *     allocates nothing and keeps no data between calls (it caches
 *     per-device facts: compute capability, SM count, kernel attributes;
 *     bitlinear_forward_noalloc has its own fixed scratch array).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work
 *     is enqueued on it and the call returns without synchronising, except
 *     where stated.  Calls on different streams with distinct workspaces
 *     may run concurrently.
 *   - Argument errors are detected on the host before anything is enqueued.
 *     A failed launch returns BITLINEAR_ERR_CUDA.  Device-side bounded waits
 *     that give up (never expected in normal operation) set a bit in the
 *     workspace status word; read it with bitlinear_check_status.
 *   - Inputs must be finite; the result for Inf/NaN inputs is unspecified.
 *   - The GPU must be compute capability 10.0 (B200); otherwise
 *     BITLINEAR_ERR_DEVICE.
 *
 * Packed weight layout (the pages leave it open; this is the library's):
 * the code u + 1 in {0, 1, 2} of each weight takes 2 bits; row n of the
 * packed matrix is K/4 bytes = K/16 little-endian uint32 words; word g of a
 * row holds k = 16g + 4i + j in bits 8j + 2i .. 8j + 2i + 1 (byte j, bit
 * pair i), so that (word >> 2i) & 0x03030303 gives the codes of four
 * consecutive k in byte lanes.  Code 3 never occurs.
 */
#ifndef BITLINEAR_H_
#define BITLINEAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BITLINEAR_OK = 0,
  BITLINEAR_ERR_NULL = -1,      /* a required pointer is NULL */
  BITLINEAR_ERR_SHAPE = -2,     /* M < 0, N < 1, K < 64 or K % 64 != 0, or too large */
  BITLINEAR_ERR_ALIGN = -3,     /* a device pointer is not 16-byte aligned */
  BITLINEAR_ERR_WORKSPACE = -4, /* workspace NULL or smaller than required */
  BITLINEAR_ERR_CUDA = -5,      /* a CUDA runtime call or launch failed */
  BITLINEAR_ERR_TIMEOUT = -6,   /* a device-side bounded wait gave up */
  BITLINEAR_ERR_DEVICE = -7     /* the current GPU is not sm_100 */
} bitlinear_status;

/* Human-readable name of a status code (static storage; never NULL). */
const char* bitlinear_status_string(int status);

/* ABI version, (major << 16) | minor. */
int bitlinear_version(void);

/* Bytes of the packed weight matrix: N * K / 4. */
size_t bitlinear_packed_bytes(int64_t N, int64_t K);

/* Workspace bytes needed by bitlinear_pack_weights (exponent-binned exact
 * sums, the mean, and the status word).  Independent of the shape. */
size_t bitlinear_pack_workspace_bytes(int64_t N, int64_t K);

/* Workspace bytes needed by bitlinear_forward and bitlinear_forward_debug
 * for this shape: the status word, s_x [M], the row sums [M] and the int8
 * activations [M, K].  Returns 0 for an invalid shape. */
size_t bitlinear_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Workspace bytes needed by bitlinear_forward_host: the above plus device
 * staging for x [M, K] and y [M, N].  Returns 0 for an invalid shape. */
size_t bitlinear_host_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Weight ternarisation and 2-bit packing (_weight_quant followed by the
 * storage packing that BitLinear.forward's unpack_weights undoes).
 *   w        [N, K] float32, finite
 *   packed   [N, K/4] uint8 out (bitlinear_packed_bytes)
 *   w_scale  [1] float32 out: s_w = 1 / max(mean|w|, 1e-5); stays on the
 *            device so that packing and the forward need no host sync
 *   w_mean   [1] float32 out, the exactly rounded mean |w|; may be NULL
 *   ws       workspace of bitlinear_pack_workspace_bytes bytes; its
 *            contents on entry do not matter
 * N * K must be below 2^39 (the exact sum's 64-bit exponent bins stay
 * below 2^64; no GPU holds a float32 tensor of that size). */
int bitlinear_pack_weights(const float* w, int64_t N, int64_t K, uint8_t* packed,
                           float* w_scale, float* w_mean, void* ws, size_t ws_bytes,
                           void* stream);

/* Per-token activation quantisation (activation_norm_quant).
 *   x          [M, K] bf16
 *   xq         [M, K] int8 out
 *   x_scale    [M] float32 out, s_x
 *   xq_rowsum  [M] int32 out, sum_k xq (used by the contraction engines);
 *              may be NULL */
int bitlinear_quant_act(const uint16_t* x, int64_t M, int64_t K, int8_t* xq, float* x_scale,
                        int32_t* xq_rowsum, void* stream);

/* The BitLinear forward: y = BitLinear(x) with packed ternary weights.
 *   x         [M, K] bf16
 *   packed_w  [N, K/4] uint8 from bitlinear_pack_weights
 *   w_scale   [1] float32 (device) from bitlinear_pack_weights
 *   bias      [N] bf16, or NULL for no bias
 *   y         [M, N] bf16 out
 *   ws        workspace of at least bitlinear_workspace_bytes(M, N, K);
 *             its contents on entry do not matter
 * M <= 16 runs the decode engine: one kernel that quantises x, streams
 * the packed weights through warp-level int8 MMA and applies the epilogue.
 * M > 16 runs the prefill engine: an activation-quantisation kernel, then a
 * tcgen05 int8 GEMM with accumulators in tensor memory and the epilogue. */
int bitlinear_forward(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w,
                      int64_t N, const float* w_scale, const uint16_t* bias, uint16_t* y,
                      void* ws, size_t ws_bytes, void* stream);

/* Flags of bitlinear_forward_ex. */
#define BITLINEAR_WEIGHTS_RESIDENT 1u
/*   packed_w, w_scale and bias were completely written before the operation
 *   enqueued on `stream` just ahead of this call started -- e.g. weights
 *   packed once at load time.  The decode engine may then start streaming
 *   them while that operation is still finishing (programmatic dependent
 *   launch), which overlaps consecutive layers.  Never set it when the
 *   previous operation on the stream writes packed_w, w_scale or bias. */

#define BITLINEAR_BF16_FAITHFUL 2u
/*   Compute as the listings do on a bfloat16 module (Falcon-Edge blog,
 *   section "Falcon-Edge, a series of universal models", activation_norm_quant
 *   and BitLinear.forward): every tensor op rounds to bf16, s_x =
 *   bf16(bf16(1 / max(a, 1e-5)) * 127) (PyTorch's evaluation of 127.0 / t),
 *   q = round(bf16(x * s_x)), y = bf16(bf16(acc) / bf16(bf16(s_w) * s_x)),
 *   then bf16(y + bias).  Without it, every step is float32 with one rounding
 *   to bf16 at the end. */

/* bitlinear_forward with flags (0 = identical to bitlinear_forward). */
int bitlinear_forward_ex(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w, int64_t N,
                         const float* w_scale, const uint16_t* bias, uint16_t* y, unsigned flags, void* ws,
                         size_t ws_bytes, void* stream);

/* Several BitLinear layers that read the same input in one call -- q/k/v,
 * or gate/up (BitLinear.forward of the Falcon-Edge blog, once per layer):
 * the input is quantised once and the layers' weights stream through one
 * launch of the decode engine (M <= 16) or one GEMM (M > 16).
 *   packed_w    [N, K/4] uint8: the layers' packed matrices stacked row-wise
 *               (pack layer g into rows [row_g, row_g + group_rows[g]) with
 *               bitlinear_pack_weights, its scale into w_scales[g])
 *   group_rows  host array [groups] of row counts, each >= 1; N = their sum
 *   groups      1 .. BITLINEAR_MAX_GROUPS
 *   w_scales    [groups] float32 (device), s_w of each layer
 *   bias        [N] bf16 (the layers' biases stacked) or NULL
 *   y           [M, N] bf16 out: layer g's outputs are the columns
 *               [row_g, row_g + group_rows[g])
 *   flags, ws   as for bitlinear_forward_ex with this N.
 * Each output equals the one bitlinear_forward gives for that layer alone. */
#define BITLINEAR_MAX_GROUPS 8
int bitlinear_forward_grouped(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w,
                              const int64_t* group_rows, int groups, const float* w_scales, const uint16_t* bias,
                              uint16_t* y, unsigned flags, void* ws, size_t ws_bytes, void* stream);

/* The contraction and epilogue of the forward on activations that
 * bitlinear_quant_act has already quantised (so that several weight
 * matrices that read the same input -- q/k/v, gate/up -- quantise it once).
 *   xq [M, K] int8, x_scale [M] float32 and xq_rowsum [M] int32 as written
 *   by bitlinear_quant_act; packed_w, w_scale, bias, y as for
 *   bitlinear_forward; ws: at least 256 bytes (only the status word is
 *   used).  This call does not reset the status word. */
int bitlinear_forward_q8(const int8_t* xq, const float* x_scale, const int32_t* xq_rowsum, int64_t M,
                         int64_t K, const uint8_t* packed_w, int64_t N, const float* w_scale,
                         const uint16_t* bias, uint16_t* y, void* ws, size_t ws_bytes, void* stream);

/* bitlinear_forward_debug with flags (BITLINEAR_BF16_FAITHFUL or 0). */
int bitlinear_forward_debug_ex(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w,
                               int64_t N, const float* w_scale, const uint16_t* bias, uint16_t* y,
                               int8_t* xq, float* x_scale, int32_t* acc, float* y32, int engine,
                               unsigned flags, void* ws, size_t ws_bytes, void* stream);

/* bf16 export of packed ternary weights, for loading them into a plain bf16
 * linear layer (Falcon-Edge blog, section "Falcon-Edge, a series of universal
 * models": the state-dict loop param_value = u / param_scale stored as
 * bfloat16).  w_bf16[n, k] = bf16_rne(float32(u[n, k] / s_w)); zeros are +0.
 *   packed_w  [N, K/4] uint8 from bitlinear_pack_weights
 *   w_scale   [1] float32 (device), s_w
 *   w_bf16    [N, K] bf16 out (16-byte aligned), row-major
 * Same shape rules as bitlinear_forward; no workspace. */
int bitlinear_dequant_weights(const uint8_t* packed_w, int64_t N, int64_t K, const float* w_scale,
                              uint16_t* w_bf16, void* stream);

/* bitlinear_forward with intermediate outputs, for parity tests.  Same
 * kernels; each extra output may be NULL:
 *   xq [M, K] int8, x_scale [M] float32, acc [M, N] int32 (the exact
 *   contraction sum_k q*u), y32 [M, N] float32 (before the bf16 rounding).
 * engine: 0 = automatic (as bitlinear_forward), 1 = force the decode
 * engine (requires M <= 16), 2 = force the prefill engine. */
int bitlinear_forward_debug(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w,
                            int64_t N, const float* w_scale, const uint16_t* bias, uint16_t* y,
                            int8_t* xq, float* x_scale, int32_t* acc, float* y32, int engine,
                            void* ws, size_t ws_bytes, void* stream);

/* bitlinear_forward with HOST activations and output: copies x_host to the
 * device (through the workspace), runs the forward, copies y back to
 * y_host and synchronises the stream before returning.  The weights,
 * w_scale and bias stay device-resident.  ws must hold
 * bitlinear_host_workspace_bytes(M, N, K).  Pinned host memory gives the
 * fastest copies; pageable memory works. */
int bitlinear_forward_host(const uint16_t* x_host, int64_t M, int64_t K, const uint8_t* packed_w,
                           int64_t N, const float* w_scale, const uint16_t* bias,
                           uint16_t* y_host, void* ws, size_t ws_bytes, void* stream);

/* bitlinear_forward_host without the final synchronisation, with flags:
 * the copies and kernels are only enqueued on `stream`.  y_host holds the
 * result once the stream reaches that point (synchronise it, or an event
 * recorded after the call).  x_host must stay unchanged until then.  With
 * pinned host memory the copies are asynchronous, so consecutive calls
 * overlap their copies with the previous calls' kernels.  Pageable memory
 * falls back to synchronous copies.  Each call in flight needs its own
 * workspace. */
int bitlinear_forward_host_async(const uint16_t* x_host, int64_t M, int64_t K, const uint8_t* packed_w,
                                 int64_t N, const float* w_scale, const uint16_t* bias, uint16_t* y_host,
                                 unsigned flags, void* ws, size_t ws_bytes, void* stream);

/* bitlinear_forward for callers that cannot allocate device memory (code
 * running inside someone else's CUDA-graph capture, server plugins given no
 * allocator, paths that must never allocate).  It takes no workspace: the
 * library uses one fixed device array of BITLINEAR_NOALLOC_SCRATCH_BYTES
 * bytes, held by every GPU that loads the library until the process exits.
 * It is an interface convenience; the BitLinear definition it computes is
 * the one bitlinear_forward follows.
 *   - Returns BITLINEAR_ERR_WORKSPACE when bitlinear_workspace_bytes(M, N, K)
 *     exceeds that fixed size (roughly M * K <= 16 MiB), and
 *     BITLINEAR_ERR_SHAPE for an invalid shape; other arguments and errors
 *     as for bitlinear_forward.
 *   - All calls share the array: calls that overlap on the GPU (on
 *     different streams or from racing host threads) race and corrupt each
 *     other.  Serialise them, e.g. on one stream.
 *   - The first call on a device looks up the array's device address on that
 *     device (make the device current first); make that first call before
 *     any stream capture.  The address is cached for the device's primary
 *     context: do not use this entry point after a cudaDeviceReset in the
 *     same process.
 *   - A device-side wait that gives up is recorded in the scratch array's
 *     status word; read it with bitlinear_noalloc_check_status.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
#define BITLINEAR_NOALLOC_SCRATCH_BYTES (16u << 20)
int bitlinear_forward_noalloc(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w, int64_t N,
                              const float* w_scale, const uint16_t* bias, uint16_t* y, void* stream);

/* bitlinear_check_status for the fixed scratch array of
 * bitlinear_forward_noalloc on the current device: reads and clears its
 * status word (synchronises `stream`).  Returns BITLINEAR_OK, or
 * BITLINEAR_ERR_TIMEOUT if a device-side bounded wait of a noalloc call gave
 * up since the last reset (each noalloc call resets it when it starts).  It
 * is an interface convenience, like bitlinear_forward_noalloc. */
int bitlinear_noalloc_check_status(void* stream);

/* Reads and clears the status word of a workspace (synchronises
 * `stream`).  bitlinear_pack_weights, bitlinear_forward, _debug and _host
 * reset the word when they start; bitlinear_forward_q8 does not.  Returns
 * BITLINEAR_OK, or BITLINEAR_ERR_TIMEOUT if a device-side bounded wait gave
 * up since the last reset.  `ws_bytes` is the size the calls were given. */
int bitlinear_check_status(const void* ws, size_t ws_bytes, void* stream);

/* ---- Tensor-parallel K-split (row-parallel) pieces -------------------------
 *
 * BitLinear.forward and _weight_quant (Falcon-Edge blog, section
 * "Falcon-Edge, a series of universal models") reduce over whole tensors:
 * s_x takes each token's absmax over all of K, and s_w takes mean |w| over the
 * whole weight matrix.  When x and W are split along K over several GPUs
 * (rank r holds x[:, K_r] and W[:, K_r]), these calls plus three exchanges
 * reproduce the unsplit forward bit for bit:
 *   packing:  bitlinear_absmean_bins on each shard -> all-reduce SUM of the
 *             uint64 bins (exact integers) -> bitlinear_pack_weights_from_bins
 *             on each shard with the summed bins and the total element count;
 *   forward:  bitlinear_act_absmax -> all-reduce MAX of the [M] floats ->
 *             bitlinear_forward_partial (int32 partial sums over K_r) ->
 *             all-reduce SUM of the int32 [M, N] partials (exact) ->
 *             bitlinear_epilogue_sum; or, with peer access, pass every rank's
 *             partial sums to bitlinear_epilogue_sum, which adds them as it
 *             reads them.
 * Each exchange is exact and independent of order, so every rank gets the
 * same bits as the unsplit call. */

/* Number of exponent bins of the exact sum of |w|. */
#define BITLINEAR_ABSMEAN_BINS 320

/* The exact sum of |w| over this shard as integer exponent bins:
 * sum |w| = sum_e bins[e] * 2^(max(e,1) - 150).  The bins of several shards
 * add (as uint64) to the bins of their union.
 *   w     [N, K] float32, finite (N * K below 2^39)
 *   bins  [BITLINEAR_ABSMEAN_BINS] uint64 out (device), overwritten */
int bitlinear_absmean_bins(const float* w, int64_t N, int64_t K, uint64_t* bins, void* stream);

/* bitlinear_pack_weights for one shard of a larger weight matrix: s_w and
 * the exact mean come from `bins` -- the bins of all shards added -- and
 * n_total, the element count of the whole matrix (>= N * K, below 2^39);
 * the codes of this shard are then packed with that s_w.  Other arguments
 * as for bitlinear_pack_weights. */
int bitlinear_pack_weights_from_bins(const float* w, int64_t N, int64_t K, const uint64_t* bins, int64_t n_total,
                                     uint8_t* packed, float* w_scale, float* w_mean, void* ws, size_t ws_bytes,
                                     void* stream);

/* Each token's max_k |x[m, k]| over this x (one K-shard of the row), as
 * float32 (exact: bf16 widens exactly).
 *   x       [M, K] bf16
 *   absmax  [M] float32 out (device) */
int bitlinear_act_absmax(const uint16_t* x, int64_t M, int64_t K, float* absmax, void* stream);

/* The contraction of one K-shard: x is quantised with s_x = 127 / max(a,
 * 1e-5) from the whole row's absmax a (the all-reduced output of
 * bitlinear_act_absmax), and contracted with this shard's packed weights.
 *   x        [M, K] bf16, this shard's columns
 *   absmax   [M] float32 (device), absmax over the whole K
 *   packed_w [N, K/4] uint8, this shard's packed columns
 *   acc      [M, N] int32 out: sum over this shard's k of q * u (exact)
 *   flags    0, or BITLINEAR_BF16_FAITHFUL for the bf16 module's s_x and q
 *            (give the same flag to bitlinear_epilogue_sum)
 *   ws       workspace of bitlinear_workspace_bytes(M, N, K) bytes
 * Same shape rules and engines as bitlinear_forward. */
int bitlinear_forward_partial(const uint16_t* x, int64_t M, int64_t K, const float* absmax, const uint8_t* packed_w,
                              int64_t N, int32_t* acc, unsigned flags, void* ws, size_t ws_bytes, void* stream);

/* The epilogue on partial sums: acc = partials[0] + ... + partials[n-1]
 * (int32, exact), then y = bf16(acc / (s_x * s_w) (+ bias)) with s_x from
 * absmax, as the forward does (flags: 0 or BITLINEAR_BF16_FAITHFUL).
 *   partials  host array of nparts (1 .. BITLINEAR_MAX_PARTS) device
 *             pointers, each [M, N] int32; they may point into other GPUs'
 *             memory through peer access (plain loads only).  Every partial
 *             sum must be complete before this call's kernel starts.
 *   absmax    [M] float32 (device), the tokens' absmax over the whole K
 *   w_scale   [1] float32 (device); bias [N] bf16 or NULL; y [M, N] bf16 out
 *   acc_out   [M, N] int32 out, the summed accumulators, or NULL */
#define BITLINEAR_MAX_PARTS 8
int bitlinear_epilogue_sum(const int32_t* const* partials, int nparts, int64_t M, int64_t N, const float* absmax,
                           const float* w_scale, const uint16_t* bias, uint16_t* y, int32_t* acc_out,
                           unsigned flags, void* stream);

/* Measurement utility, not part of the method (the pages have no
 * counterpart): enqueues a kernel that runs the int8 tensor cores alone at
 * full rate -- one CTA per SM, `iters` x 4 back-to-back tcgen05.mma kind::i8
 * of 128 x 256 x 32 on zero operands -- so that the caller can time it with
 * CUDA events and derive the GPU's dense int8 rate:
 *   int8 ops = 2 * 128 * 256 * 32 * 4 * iters * (*grid).
 *   iters   1 .. 2^24
 *   grid    host out: the number of CTAs launched (the SM count)
 *   ws      at least 256 bytes of device memory: its first word is a status
 *           word (bitlinear_check_status reads it) */
int bitlinear_measure_i8_peak(int iters, int* grid, void* ws, size_t ws_bytes, void* stream);

/* Test hook for the failure path of the device-side waits.  While it is on
 * (on != 0), every forward launched by this process -- bitlinear_forward and
 * its variants, both engines -- makes one wait on a barrier that nothing
 * signals, with a 1 ms limit instead of the usual 1 s for its main-loop
 * waits.  That wait gives up, the kernel stops its main loop, lets every copy
 * and tensor-core operation already started finish (those drains keep the
 * 1 s limit), sets BITLINEAR_ERR_TIMEOUT in the status word and exits; y is
 * then left unspecified.  No fault, trap or hang is involved: the context
 * stays usable and the next forward after switching the hook off is normal.
 * Process-wide and not meant for production use.  Returns the previous
 * setting (0 or 1). */
int bitlinear_test_force_timeout(int on);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H_ */
