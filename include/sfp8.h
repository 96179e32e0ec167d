/*
 * sfp8 -- row-wise scaled 2:4 sparse FP8 linear layer for B200 (sm_100a).
 *
 * C ABI of libsfp8.so.  Plain pointers and sizes only; no C++ or framework
 * types cross this boundary.  Every pointer argument named *device* must be
 * device memory of the current CUDA device; the caller owns every buffer.
 *
 * The operation (page "Add CUTLASS-based row-wise scaled sparse FP8 kernel",
 * pytorch/ao pull request 1671, items 1, 3 and 4):
 *
 *     y[m, n] = s_a[m] * s_w[n] * sum_k A_q[m, k] * W_q[n, k]  (+ bias[n])
 *
 * where A_q, s_a come from dynamic per-row FP8 quantisation of the
 * activation, and W_q, s_w from the same quantisation of a 2:4-pruned weight
 * that is then stored compressed (kept values + 2-bit index metadata).
 *
 * Conventions shared by all entry points:
 *  - Asynchronous: work is enqueued on `stream` (a cudaStream_t; NULL means
 *    the legacy default stream).  Nothing is synchronised.
 *  - Validation errors are returned synchronously before anything is
 *    launched: null pointers, unsupported shapes or dtypes, misalignment,
 *    a too-small workspace, a device that is not sm_100.  A failed launch
 *    returns SFP8_ERR_CUDA.  No exception crosses the ABI.
 *  - Device-side failures (a pipeline wait that ran out its time limit) are
 *    recorded in a per-device status word; read it with
 *    sfp8_read_device_status() after synchronising.
 *  - Reentrant: independent calls may run concurrently on different streams
 *    as long as they do not share an output or a workspace.
 *  - Deterministic: the same inputs give bit-identical outputs, run to run.
 *  - Empty problems (rows, m or n equal to 0) return SFP8_OK and launch
 *    nothing, except where an entry point states an output for them
 *    (sfp8_quantize_rowwise with cols == 0 and sfp8_quantize_tensorwise
 *    with numel == 0 write the guard scale).
 *  - Strides (ld) are in elements.  Row-major everywhere.
 *
 * Typical use (one layer, W [n, k] bf16, k % 128 == 0):
 *   once:     packed <- sfp8_compressed_bytes(n, k) bytes, s_w <- n floats;
 *             sfp8_prepare_weight_24(W, SFP8_BF16, n, k, k, SFP8_E4M3, packed, s_w, st);
 *             ws <- sfp8_sparse_linear_quant_workspace_bytes(m, n, k) bytes, zeroed
 *             (sfp8_workspace_clear);
 *   per call: sfp8_sparse_linear_quant(x, SFP8_BF16, k, SFP8_E4M3, a_q, s_a, m,
 *                                      packed, SFP8_E4M3, s_w, n, k, bias, y,
 *                                      ws, ws_bytes, st);
 *   optional: sfp8_sparse_linear_search + sfp8_sparse_linear_set_algo to pick
 *             the work split for a token count (before sizing ws).
 *
 * The compressed weight is one packed buffer (kept values and index
 * metadata interleaved per 128 x 128 tile) rather than separate values and
 * metadata buffers, so that one copy brings a tile's operands on chip;
 * sfp8_compressed_values_bytes / sfp8_compressed_meta_bytes give the sizes
 * of the two parts inside it.
 */
#ifndef SFP8_H_
#define SFP8_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SFP8_OK = 0,
  SFP8_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad enum  */
  SFP8_ERR_UNSUPPORTED_SHAPE = 2,  /* e.g. k not a multiple of 128           */
  SFP8_ERR_MISALIGNED = 3,         /* a base pointer or stride not aligned   */
  SFP8_ERR_UNSUPPORTED_DTYPE = 4,  /* dtype not accepted by this entry point */
  SFP8_ERR_ARCH = 5,               /* current device is not sm_100           */
  SFP8_ERR_WORKSPACE = 6,          /* workspace missing or too small         */
  SFP8_ERR_CUDA = 7,               /* a CUDA runtime/driver call failed      */
  SFP8_ERR_TIMEOUT = 8,            /* a device-side wait hit its time limit  */
  SFP8_ERR_DEVICE_CHECK = 9        /* a device-side consistency check failed */
} sfp8_status;

typedef enum {
  SFP8_BF16 = 0,
  SFP8_F16 = 1,
  SFP8_F32 = 2,
  SFP8_E4M3 = 3,  /* OCP e4m3 ("e4m3fn"): max 448, no infinities   */
  SFP8_E5M2 = 4   /* OCP e5m2: max 57344                          */
} sfp8_dtype;

/* Bits of the device status word. */
#define SFP8_DEVICE_TIMEOUT     0x1u  /* a bounded mbarrier wait gave up     */
#define SFP8_DEVICE_CHECK_FAIL  0x2u  /* a device-side check failed          */

/* Version of the compressed-weight layout written by sfp8_compress_24. */
#define SFP8_LAYOUT_VERSION 3

/*
 * Dynamic row-wise FP8 quantisation (the activation path of item 4; also
 * used once on the pruned weight).  For each row r of x:
 *     amax     = max_c |x[r, c]|                     (fp32, exact)
 *     s        = max(amax, 1e-12f) / FP8_MAX         (IEEE fp32 division)
 *     q[r, c]  = RNE_satfinite_fp8(x[r, c] / s)      (IEEE fp32 division,
 *                                                      then one rounding)
 * FP8_MAX = 448 (E4M3) or 57344 (E5M2).  Overflow saturates; the sign of a
 * value that rounds to zero is kept.  NaN/Inf inputs are outside the
 * contract.
 *
 *  x       device, [rows, cols] of x_dtype (BF16, F16 or F32), row stride
 *          ld_x >= cols elements; 16-byte aligned base, ld_x*size 16-byte
 *          multiple.
 *  q       device, [rows, cols] bytes (q_dtype E4M3 or E5M2), row stride
 *          cols; 16-byte aligned.
 *  scales  device, [rows] float32 (s above); 4-byte aligned.
 *  cols % 16 == 0 (cols may be 0: scales are then the guard scale).
 */
sfp8_status sfp8_quantize_rowwise(const void* x, sfp8_dtype x_dtype,
                                  int64_t rows, int64_t cols, int64_t ld_x,
                                  void* q, sfp8_dtype q_dtype, float* scales,
                                  void* stream);

/*
 * How sfp8_quantize_tensorwise finds the global amax (page "[float8nocompile]
 * Add alternate Triton kernels for FP8 conversion which use atomic_max-based
 * algo instead of reduction-based algo", pytorch/ao pull request 1455,
 * Summary and review): REDUCE writes one partial maximum per block and
 * reduces them; ATOMIC folds every block's maximum into one word with an
 * atomic max, so it needs no buffer sized by the block count.  A maximum is
 * exact in any order: both modes give the same bits.
 */
typedef enum {
  SFP8_AMAX_REDUCE = 0,
  SFP8_AMAX_ATOMIC = 1
} sfp8_amax_mode;

/*
 * Workspace bytes of sfp8_quantize_tensorwise on the current device:
 * 64 for ATOMIC, 64 + 16 * (number of SMs) for REDUCE; 0 for an unknown mode.
 */
size_t sfp8_quantize_tensorwise_workspace_bytes(sfp8_amax_mode mode);

/*
 * Tensor-wise (one scale) FP8 quantisation of a contiguous tensor of numel
 * elements -- the row-wise rule above with the whole tensor as the one row:
 *     amax  = max_i |x[i]|                        (fp32, exact)
 *     s     = max(amax, 1e-12f) / FP8_MAX          (IEEE fp32 division)
 *     q[i]  = RNE_satfinite_fp8(x[i] / s)          (IEEE fp32 division,
 *                                                   then one rounding)
 * One launch (a cooperative grid: both sweeps over x, the amax between them
 * through a grid barrier in the workspace).
 *
 *  x       device, numel elements of x_dtype (BF16, F16 or F32), contiguous,
 *          16-byte aligned.  Any numel >= 0 (numel == 0 writes the guard
 *          scale 1e-12f / FP8_MAX).
 *  q       device, numel bytes (q_dtype E4M3 or E5M2), 16-byte aligned.
 *  scale   device, one float32 (s above), written.
 *  workspace  device, >= sfp8_quantize_tensorwise_workspace_bytes(mode)
 *          bytes, 16-byte aligned, zero before its first use (e.g. by
 *          sfp8_workspace_clear); every call leaves it ready for the next.
 *          Calls that share a workspace must not overlap on the GPU; clear
 *          it again after a call that reported a device error.
 * A barrier wait that runs out its time limit sets SFP8_DEVICE_TIMEOUT and
 * leaves q unwritten.
 */
sfp8_status sfp8_quantize_tensorwise(const void* x, sfp8_dtype x_dtype, int64_t numel,
                                     void* q, sfp8_dtype q_dtype, float* scale,
                                     sfp8_amax_mode mode, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * 2:4 magnitude pruning along the row (the weight preparation that the
 * page's "sparsify/quantize method" performs before quantisation): in every
 * group of four consecutive elements keep the two of largest |w| (-0.0 is
 * zero; ties to the lower index) and write +0.0 in the other two.  Kept
 * elements are copied bit for bit.
 *
 *  w       device, [rows, cols] of dtype (BF16, F16 or F32), row stride ld;
 *          16-byte aligned base, ld*size 16-byte multiple.
 *  out     device, [rows, cols] of dtype, row stride cols, 16-byte aligned.
 *          May not alias w unless ld == cols (then in-place is allowed).
 *  cols % 16 == 0.
 */
sfp8_status sfp8_prune_24(const void* w, sfp8_dtype dtype, int64_t rows,
                          int64_t cols, int64_t ld, void* out, void* stream);

/*
 * Size of the compressed (packed) weight for an [n, k] FP8 weight
 * (k % 128 == 0): n_pad * k * 5/8 bytes with n_pad = ceil(n / 128) * 128.
 */
int64_t sfp8_padded_rows(int64_t n);
size_t sfp8_compressed_bytes(int64_t n, int64_t k);

/*
 * The two parts of that buffer (item 1's converter emits kept values and
 * index metadata): sfp8_compressed_values_bytes = n_pad * k / 2 bytes of
 * kept codes and sfp8_compressed_meta_bytes = n_pad * k / 8 bytes of index
 * nibbles; for k % 128 == 0 their sum is sfp8_compressed_bytes.  The two
 * parts are not separate buffers: every 128 x 128 tile stores its 8192 value
 * bytes and then its 2048 metadata bytes (layout below), so that one
 * contiguous copy brings a tile's operands into shared memory.  Both return
 * 0 for a negative n or k.
 */
size_t sfp8_compressed_values_bytes(int64_t n, int64_t k);
size_t sfp8_compressed_meta_bytes(int64_t n, int64_t k);

/*
 * 2:4 compression of an FP8 weight (item 1's converter, with item 3's rule
 * that -0.0 is a zero).  Per group g of four codes along k: keep the two of
 * largest magnitude (ties to the lower index; -0.0 ranks as 0), emit the two
 * source codes unchanged, lower index first, and the index nibble
 * i0 | (i1 << 2).
 *
 * Layout (version 3): one buffer of 10240-byte tiles; tile t = nt*(k/128)+kt
 * covers weight rows 128*nt .. 128*nt+127 and k columns 128*kt .. 128*kt+127
 * and starts at byte 10240*t:
 *   bytes 0 .. 8191: kept values.  Row r of the tile at byte 64*r holds the
 *           row's 64 kept codes (two per group, lower index first) as four
 *           16-byte chunks, chunk c at position c ^ ((r >> 1) & 3).
 *   bytes 8192 .. 10239: index metadata.  Row r at byte 8192 + 16*r; byte b
 *           holds the nibble of group 32*kt + 2b in bits 0..3 and of group
 *           32*kt + 2b + 1 in bits 4..7.
 *   Rows n..n_pad-1: value 0x00 and nibble 0x4 everywhere.
 * (One tile is exactly what one k step of the GEMM needs in shared memory,
 * values already in the tensor core's 64-byte-swizzled form, so the GEMM
 * streams the weight with one contiguous copy per pipeline stage.)
 *
 *  w_q     device, [n, k] FP8 codes (w_dtype E4M3 or E5M2), row stride k,
 *          16-byte aligned.  NaN codes are outside the contract.
 *  packed  device, sfp8_compressed_bytes(n, k) bytes, 16-byte aligned.
 */
sfp8_status sfp8_compress_24(const void* w_q, sfp8_dtype w_dtype, int64_t n,
                             int64_t k, void* packed, void* stream);

/*
 * The whole weight preparation in one pass: sfp8_prune_24, then
 * sfp8_quantize_rowwise (one scale per weight row n), then sfp8_compress_24,
 * with the same results bit for bit (item 4's preparation of the weight at
 * quantisation time, item 1's compressed format) but one read of w and no
 * intermediate buffers.
 *
 *  w       device, [n, k] of w_dtype (BF16, F16 or F32), row stride ld_w >= k
 *          elements; 16-byte aligned base, ld_w*size a 16-byte multiple.
 *          Finite values (NaN/Inf are outside the contract).
 *  q_dtype E4M3 or E5M2: the FP8 format of the compressed codes.
 *  packed  device, sfp8_compressed_bytes(n, k) bytes, 16-byte aligned;
 *          the layout of sfp8_compress_24.
 *  s_w     device, [n] float32 (the row scales), 4-byte aligned.
 *  k % 128 == 0, k > 0; n >= 0 (n == 0: nothing is launched).
 * Validation errors return with nothing launched; buffers must not overlap.
 */
sfp8_status sfp8_prepare_weight_24(const void* w, sfp8_dtype w_dtype, int64_t n,
                                   int64_t k, int64_t ld_w, sfp8_dtype q_dtype,
                                   void* packed, float* s_w, void* stream);

/*
 * Inverse of sfp8_compress_24 (a checking aid): writes the dense [n, k]
 * codes, 0x00 in dropped slots.  w_q 16-byte aligned, row stride k.
 * An invalid nibble sets SFP8_DEVICE_CHECK_FAIL in the device status word.
 */
sfp8_status sfp8_decompress_24(const void* packed, int64_t n, int64_t k,
                               void* w_q, void* stream);

/*
 * Workspace for sfp8_sparse_linear on the current device (split-K partial
 * sums and per-tile counters); 0 when the chosen work split needs none.  The
 * counters part must be zero before the first call that uses a workspace;
 * every call leaves it zero again (clear it again after a call that reported
 * a device error).  sfp8_workspace_clear zeroes a workspace on a stream.
 */
size_t sfp8_sparse_linear_workspace_bytes(int64_t m, int64_t n, int64_t k);
sfp8_status sfp8_workspace_clear(void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * The sparse FP8 linear (item 1's operator; the four e4m3/e5m2 operand
 * pairs of the page's per-dtype files are run-time choices here):
 *     y[m, n] = bf16_RNE( acc[m, n] * s_a[m] * s_w[n] + bias[n] )
 * with acc[m, n] = sum over kept slots of dec(A_q[m, k]) * dec(W_q[n, k]),
 * accumulated in fp32 by the sm_100 sparse tensor cores.
 *
 *  a_q     device, [m, k] FP8 codes (a_dtype E4M3 or E5M2), row stride k,
 *          16-byte aligned.
 *  s_a     device, [m] float32.
 *  packed  device, from sfp8_compress_24 for an [n, k] weight of w_dtype
 *          (E4M3 or E5M2).
 *  s_w     device, [n] float32.
 *  bias    device, [n] bf16, or NULL for none.
 *  y       device, [m, n] bf16, row stride n.
 *  workspace  device, >= sfp8_sparse_linear_workspace_bytes(m, n, k) bytes
 *          (may be NULL when that is 0), 16-byte aligned, counters zero.
 *  k % 128 == 0, k > 0; m, n >= 0.
 *
 * The call is launched as a programmatic dependent of the preceding kernel on
 * the stream: it streams the first weight tiles before waiting for that
 * kernel to finish, and reads a_q, s_a, bias only after.  So `packed` and
 * `s_w` must not be written by a kernel that lets its dependents launch
 * early (none of this library's kernels writes them that way).
 */
sfp8_status sfp8_sparse_linear(const void* a_q, sfp8_dtype a_dtype,
                               const float* s_a, int64_t m,
                               const void* packed, sfp8_dtype w_dtype,
                               const float* s_w, int64_t n, int64_t k,
                               const void* bias, void* y, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * Work-split selection ("algorithms") of the sparse linear.  The page "Add
 * CUTLASS-based row-wise scaled sparse FP8 kernel" (pytorch/ao pull request
 * 1671) leaves "a meaningful config selection" as future work, and the page
 * "Add algorithm search to FP8 sparse linear benchmark" (pytorch/ao #4432)
 * threads an algorithm id through the sparse matmul and finds the fastest
 * one per shape with a search call.  Here an algorithm is one work split of
 * the GEMM for a shape (m, n, k): the kernel (one CTA per tile, or CTA pairs
 * sharing a 256-row tile), the token-tile width, the k steps per pipeline
 * stage, the weight tiles per CTA and the whole-tile / stream-K split.
 * Algorithm 0 is the built-in rule; the list depends on the shape and the
 * device's SM count.  Every algorithm computes the same y up to the fp32
 * summation order (within the tolerance of sfp8_sparse_linear; each one is
 * deterministic).
 */

/* Number of algorithms for (m, n, k) on the current device (0 for an
 * unsupported shape). */
int sfp8_sparse_linear_algo_count(int64_t m, int64_t n, int64_t k);

/* Description of one algorithm: info[0..7] = {pair kernel (0/1), tokens per
 * tile, k steps per stage, weight tiles per CTA, whole tiles (1) or
 * stream-K (0), activation resident in shared memory (0/1), pipeline stages,
 * CTAs launched (pairs: at most; the count is capped at launch by the
 * co-resident clusters)}. */
sfp8_status sfp8_sparse_linear_algo_info(int64_t m, int64_t n, int64_t k, int algo,
                                         int32_t* info);

/* The same list for a device of num_sms SMs without touching any device (a
 * host-only query, e.g. to inspect plans offline): the count, and
 * info[0..11] = {pair kernel, tokens per tile, k steps per stage, weight
 * tiles per CTA, whole tiles, resident activation, stages, CTAs, producer
 * warps, dynamic shared memory bytes, workspace bytes, token tiles}. */
int sfp8_sparse_linear_plan_count(int64_t m, int64_t n, int64_t k, int num_sms);
sfp8_status sfp8_sparse_linear_plan_info(int64_t m, int64_t n, int64_t k, int num_sms,
                                         int algo, int64_t* info);

/* Workspace bytes of one algorithm, and the most over all algorithms of the
 * shape (what sfp8_sparse_linear_search needs). */
size_t sfp8_sparse_linear_algo_workspace_bytes(int64_t m, int64_t n, int64_t k, int algo);
size_t sfp8_sparse_linear_search_workspace_bytes(int64_t m, int64_t n, int64_t k);

/* sfp8_sparse_linear with an explicit algorithm (0 <= algo < count, else
 * SFP8_ERR_INVALID_ARG); arguments otherwise as sfp8_sparse_linear, the
 * workspace sized by sfp8_sparse_linear_algo_workspace_bytes. */
sfp8_status sfp8_sparse_linear_algo(const void* a_q, sfp8_dtype a_dtype,
                                    const float* s_a, int64_t m,
                                    const void* packed, sfp8_dtype w_dtype,
                                    const float* s_w, int64_t n, int64_t k,
                                    const void* bias, void* y, int algo,
                                    void* workspace, size_t workspace_bytes,
                                    void* stream);

/*
 * Times every algorithm of the shape on the caller's buffers and returns the
 * fastest in *best_algo (times_us[i], when given, receives algorithm i's
 * median time in microseconds for i < times_len).  Each algorithm runs once
 * untimed, then `reps` (1..64) times, each launch bracketed by CUDA events on
 * `stream`; when `flush` is given, flush_bytes of it are overwritten before
 * every timed launch (a buffer larger than L2 makes each launch read its
 * operands from HBM).  Synchronous: it waits for the stream.  y and the
 * workspace (>= sfp8_sparse_linear_search_workspace_bytes) are overwritten,
 * and the workspace is left zeroed only in the parts the last algorithm
 * used -- clear it before giving it to sfp8_sparse_linear.  Not for use
 * inside a stream capture.
 */
sfp8_status sfp8_sparse_linear_search(const void* a_q, sfp8_dtype a_dtype,
                                      const float* s_a, int64_t m,
                                      const void* packed, sfp8_dtype w_dtype,
                                      const float* s_w, int64_t n, int64_t k,
                                      const void* bias, void* y, void* workspace,
                                      size_t workspace_bytes, void* flush,
                                      size_t flush_bytes, int reps, int* best_algo,
                                      float* times_us, int times_len, void* stream);

/*
 * The shape-keyed table of the current device: after
 * sfp8_sparse_linear_set_algo(m, n, k, a) with a > 0, sfp8_sparse_linear,
 * sfp8_sparse_linear_quant, sfp8_sparse_linear_noalloc and their workspace
 * queries use algorithm a for exactly that (m, n, k); a <= 0 removes the
 * entry (back to the built-in rule).  Query workspace sizes after setting.
 * Thread-safe; the table lives until the process exits.
 * sfp8_sparse_linear_get_algo returns the entry (0 when none).
 */
sfp8_status sfp8_sparse_linear_set_algo(int64_t m, int64_t n, int64_t k, int algo);
int sfp8_sparse_linear_get_algo(int64_t m, int64_t n, int64_t k);

/*
 * Workspace for sfp8_sparse_linear_quant: sfp8_sparse_linear's for these
 * sizes, plus, when the GEMM keeps the activation resident and m is below its
 * token tile (decode with fewer than 16 tokens), a staging area of tile-high
 * codes that the quantiser writes besides a_q and the GEMM reads as whole
 * rows.
 */
size_t sfp8_sparse_linear_quant_workspace_bytes(int64_t m, int64_t n, int64_t k);

/*
 * The layer's forward in one call: dynamic row-wise quantisation of the
 * activation (exactly sfp8_quantize_rowwise: page "Add CUTLASS-based
 * row-wise scaled sparse FP8 kernel", items 1 and 4) followed by the sparse
 * linear (exactly sfp8_sparse_linear), on `stream`.  Two forms, with the same
 * results bit for bit (a_q, s_a and y):
 *   chained  the row-wise quantiser, then the GEMM as its programmatic
 *            dependent (its weight stream starts while the activation is
 *            being quantised);
 *   fused    (where sfp8_sparse_linear_quant_fusable(m, n, k): at most 16
 *            tokens and the activation resident in one token tile) ONE
 *            kernel: every CTA of the GEMM quantises the m rows itself into
 *            shared memory while its weight streams in, and the codes and
 *            scales are also written to a_q and s_a.
 * sfp8_sparse_linear_quant runs the chained form, the faster of the two on
 * B200 at every fusable shape measured (1 to 16 tokens, k = 4096,
 * n = 14336: 8.5-8.9 us against 10.3-15.4 us per step); _chained and _fused
 * force one form (the fused one returns SFP8_ERR_UNSUPPORTED_SHAPE where it
 * does not apply).
 *
 *  x       device, [m, ld_x] bf16 / fp16 / fp32 activation, 16-byte aligned,
 *          ld_x >= k, ld_x * element size a multiple of 16.
 *  a_dtype SFP8_E4M3 or SFP8_E5M2: the activation's FP8 format.
 *  a_q     device, [m, k] u8, written (the quantised activation).
 *  s_a     device, [m] float32, written (its row scales).
 *  packed, w_dtype, s_w, n, k, bias, y: as for sfp8_sparse_linear.
 *  workspace  >= sfp8_sparse_linear_quant_workspace_bytes(m, n, k) bytes,
 *          zero before the first call (left zero by every call).
 *  x's span (rows 0..m-1 at stride ld_x) must not overlap a_q, s_a or y (the
 *  kernels read x while they write those); with n > 0 an overlap is refused
 *  with SFP8_ERR_INVALID_ARG before anything is launched.
 *
 * Returns the first failing status of the two steps (validation of both
 * before anything is launched where the arguments allow).  With n == 0 only
 * the activation is quantised.
 */
sfp8_status sfp8_sparse_linear_quant(const void* x, sfp8_dtype x_dtype, int64_t ld_x,
                                     sfp8_dtype a_dtype, void* a_q, float* s_a, int64_t m,
                                     const void* packed, sfp8_dtype w_dtype,
                                     const float* s_w, int64_t n, int64_t k,
                                     const void* bias, void* y, void* workspace,
                                     size_t workspace_bytes, void* stream);
sfp8_status sfp8_sparse_linear_quant_fused(const void* x, sfp8_dtype x_dtype, int64_t ld_x,
                                           sfp8_dtype a_dtype, void* a_q, float* s_a, int64_t m,
                                           const void* packed, sfp8_dtype w_dtype,
                                           const float* s_w, int64_t n, int64_t k,
                                           const void* bias, void* y, void* workspace,
                                           size_t workspace_bytes, void* stream);
sfp8_status sfp8_sparse_linear_quant_chained(const void* x, sfp8_dtype x_dtype, int64_t ld_x,
                                             sfp8_dtype a_dtype, void* a_q, float* s_a,
                                             int64_t m, const void* packed, sfp8_dtype w_dtype,
                                             const float* s_w, int64_t n, int64_t k,
                                             const void* bias, void* y, void* workspace,
                                             size_t workspace_bytes, void* stream);

/*
 * 1 when sfp8_sparse_linear_quant_fused accepts (m, n, k) on the current
 * device (the work split of the shape, from the table or the built-in rule,
 * keeps a 16-token activation tile resident), else 0 (also for invalid sizes
 * and without a device).  Host-only query.
 */
int sfp8_sparse_linear_quant_fusable(int64_t m, int64_t n, int64_t k);

/*
 * The layer's forward from host memory to host memory in one call: on
 * `stream`, the copy of x_host into the device staging buffer x_dev, then
 * exactly sfp8_sparse_linear_quant on it, then the copy of y_dev into y_host.
 * For the end-to-end path of a caller that holds its activations on the
 * host; with page-locked host buffers the copies are asynchronous like the
 * rest (pageable buffers work, and make the copies synchronous).
 *
 *  x_host  host, [m, k] of x_dtype, contiguous.
 *  x_dev   device, [m, k] of x_dtype, contiguous, 16-byte aligned (staging).
 *  y_dev   device, [m, n] bf16 (as y of sfp8_sparse_linear).
 *  y_host  host, [m, n] bf16, contiguous, written.
 *  Everything else as for sfp8_sparse_linear_quant (ld_x = k).  All
 *  arguments are validated before anything is enqueued.
 */
sfp8_status sfp8_sparse_linear_quant_host(const void* x_host, void* x_dev, sfp8_dtype x_dtype,
                                          sfp8_dtype a_dtype, void* a_q, float* s_a,
                                          int64_t m, const void* packed, sfp8_dtype w_dtype,
                                          const float* s_w, int64_t n, int64_t k,
                                          const void* bias, void* y_dev, void* y_host,
                                          void* workspace, size_t workspace_bytes,
                                          void* stream);

/*
 * Size of the scratch buffer built into the library for
 * sfp8_sparse_linear_noalloc (per device that loads the library).
 */
#define SFP8_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * sfp8_sparse_linear for callers that cannot allocate device memory.
 *
 * The pages have no counterpart of this entry point; it exists for callers
 * that may not allocate at call time -- code replayed from a pre-built CUDA
 * graph, runtimes whose allocator forbids cudaMalloc after start-up, or hosts
 * that give the library nothing but its inputs and outputs.  It computes the
 * same result as sfp8_sparse_linear (same kernel, same work split, so the
 * same bits) but takes no workspace: the split-K scratch is a fixed
 * SFP8_NOALLOC_SCRATCH_BYTES buffer compiled into the library, one per
 * device, held until the process exits.  It calls no cudaMalloc/cudaFree or
 * other allocating routine.
 *
 *  - Arguments, layouts and alignment as for sfp8_sparse_linear, minus the
 *    workspace.
 *  - Size limit: problems whose sfp8_sparse_linear_workspace_bytes(m, n, k)
 *    exceeds SFP8_NOALLOC_SCRATCH_BYTES are rejected with SFP8_ERR_WORKSPACE
 *    before anything is launched (on a 148-SM B200 this admits any n and k
 *    for m <= 32 and for m >= 512, which need at most 4.8 MB and no scratch;
 *    between them it depends on the work split chosen for n and k).  That
 *    statement describes the built-in work split.  An entry stored with
 *    sfp8_sparse_linear_set_algo for (m, n, k) is used by this call too; its
 *    scratch is checked against SFP8_NOALLOC_SCRATCH_BYTES in the same way,
 *    so a stream-K entry may be rejected with SFP8_ERR_WORKSPACE for a shape
 *    that the built-in split would have admitted.
 *  - The first call on a device looks up the buffer's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    outside any stream capture.
 *  - All calls on a device share the one buffer, which keeps the previous
 *    call's contents; each call clears the counters it needs (an async
 *    memset on `stream`).  Calls that overlap on the GPU -- on different
 *    streams, or on one stream inside concurrently replayed graphs -- race
 *    on the buffer and give wrong results; serialise them.
 */
sfp8_status sfp8_sparse_linear_noalloc(const void* a_q, sfp8_dtype a_dtype,
                                       const float* s_a, int64_t m,
                                       const void* packed, sfp8_dtype w_dtype,
                                       const float* s_w,
                                       int64_t n, int64_t k, const void* bias,
                                       void* y, void* stream);

/*
 * Test of the failure path (no counterpart on the pages): launches one
 * thread that waits, with the same bounded wait as every pipeline of this
 * library, on a barrier that nothing completes.  After the wait limit (about
 * a second) it sets SFP8_DEVICE_TIMEOUT in the status word and returns; no
 * fault, nothing left in flight, the context stays usable.  Read and clear
 * the word with sfp8_read_device_status afterwards.
 */
sfp8_status sfp8_selftest_timeout(void* stream);

/*
 * Reads (and with clear != 0, resets) the current device's status word.
 * Synchronises the device first.  *flags receives SFP8_DEVICE_* bits.
 * Returns SFP8_ERR_TIMEOUT / SFP8_ERR_DEVICE_CHECK when such a bit is set,
 * SFP8_OK otherwise.
 */
sfp8_status sfp8_read_device_status(uint32_t* flags, int clear);

/*
 * The status of the last device-side work on the current device, without
 * clearing it: synchronises the device, then returns SFP8_ERR_TIMEOUT when
 * a bounded wait gave up, SFP8_ERR_DEVICE_CHECK when a device-side check
 * failed, SFP8_ERR_CUDA when the device cannot be read, SFP8_OK otherwise.
 * Same word as sfp8_read_device_status (use that one to clear it).
 */
sfp8_status sfp8_last_device_status(void);

const char* sfp8_status_string(sfp8_status s);
int sfp8_layout_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SFP8_H_ */
