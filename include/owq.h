/*
 * owq.h -- C ABI of the OWQ mixed-precision weight-only matmul for NVIDIA B200 (sm_100a).
 *
 * The operation (OWQ, Lee et al., arXiv:2306.02272; pages: "OWQ: Outlier-Aware Weight
 * Quantization for Efficient Fine-Tuning and Inference of Large Language Models",
 * paperlayer.ai, items "Weak-column selection" (paper p.4), "Real-device acceleration"
 * (paper "Acceleration on Real Device", p.6) and "Storage Methods" (appendix §2,
 * pp.10-11)):
 *
 *     y[m, i] = sum_j W_hat[i, j] x[m, j]  +  sum_t W_weak[i, t] x[m, idx[t]]
 *
 * W is N x K (N output channels, K input channels; y = x W^T as in a PyTorch Linear).
 * The dense part W_hat is stored as 3- or 4-bit codes q with an fp16 scale s and an fp16
 * integral zero point z per (output row, group of `group` consecutive input columns):
 * W_hat = fp16_rn(s * (q - z)).  The k "weak" columns listed in idx stay in fp16 (W_weak,
 * N x k) and their codes in the dense matrix are q = z, so the dense part is exactly 0
 * there (the latency-favoured, zero-filled layout).
 *
 * Conventions for every call:
 *   - fp16 values are passed as their IEEE binary16 bit patterns (uint16_t).
 *   - Every data pointer is a DEVICE pointer on the current CUDA device, owned by the
 *     caller, unless the comment says "host".  The library never frees caller memory.
 *   - Every call is asynchronous on `stream` (NULL = the legacy default stream) unless
 *     its comment says it synchronises.
 *   - On any error nothing is launched and no output is written; the return value says
 *     why.  Arguments are validated on the host before any launch.
 *   - Shapes: K is a multiple of 128 (the packed block), 128 <= K <= 65536, 1 <= N <= 2^20.
 *     group is K (per output channel) or 128.  bits is 3 or 4.  0 <= k <= K, k <= 1024.
 *   - Alignment: every device pointer is 16-byte aligned (OWQ_ERR_ALIGN otherwise).
 */
#ifndef OWQ_H_
#define OWQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int owq_status_t;
#define OWQ_OK            0
#define OWQ_ERR_NULL      1   /* a required pointer is NULL                                 */
#define OWQ_ERR_SHAPE     2   /* N, K, M, T or k outside the ranges above                    */
#define OWQ_ERR_BITS      3   /* bits not 3 or 4                                             */
#define OWQ_ERR_GROUP     4   /* group neither K nor 128                                     */
#define OWQ_ERR_INDEX     5   /* idx not strictly ascending or outside [0, K)                */
#define OWQ_ERR_ALIGN     6   /* a device pointer is not 16-byte aligned                      */
#define OWQ_ERR_CUDA      7   /* a CUDA runtime call or a launch failed                       */
#define OWQ_ERR_TIMEOUT   8   /* a bounded device-side wait gave up (see owq_device_status)    */
#define OWQ_ERR_NOMEM     9   /* a device or host allocation failed                           */
#define OWQ_ERR_HANDLE    10  /* the layer handle is NULL or not one this library made         */
#define OWQ_ERR_DEVICE    11  /* no CUDA device, or the device is not sm_100                   */
#define OWQ_ERR_ARG       12  /* an argument outside its documented set (owq_debug_inject)      */
#define OWQ_ERR_BOUNDS    13  /* debug-bounds build: a device index check failed (owq_device_status) */

/* Failures owq_debug_inject can arm. */
#define OWQ_INJECT_NONE         0
#define OWQ_INJECT_GEMV_TAG     1
#define OWQ_INJECT_GEMM_ARRIVE  2
#define OWQ_INJECT_BOUNDS       3

/* Opaque handle of one packed layer; owns the device buffers owq_pack allocated. */
typedef struct owq_layer_s* owq_layer_t;
/* Same object as cudaStream_t. */
typedef struct CUstream_st* owq_stream_t;

/*
 * owq_quantize -- the OWQ quantiser on the GPU: weak-column selection, then min-max RTN
 * of the dense columns.  Pages: "Weak-column selection" (paper p.4; the score combines
 * a column's perturbation norm with its Hessian diagonal) and the min-max RTN quantiser
 * named in "OWQ -- paper by Lee et al. (2023) -- summary and ideas", Key points.
 *   lambda_j = sum_t X[t, j]^2                        (fp64, t ascending)
 *   W_hat0   = min-max RTN of W over all columns
 *   sens_j   = lambda_j * sum_i (W[i,j] - W_hat0[i,j])^2   (fp64, i ascending)
 *   idx      = the k largest sens_j (ties: lower j), stored ascending
 *   codes/scales/zeros = min-max RTN with the idx columns excluded from each range and
 *              coded q = z;  w_weak[i, t] = W[i, idx[t]] (bit copy).
 * RTN per (row, group), fp32, round-half-to-even: mn = min(0, min w), mx = max(0, max w)
 * over the dense columns ([-1, 1] if mn == mx or if the fp16 scale would be 0);
 * s = fp16(fp32(mx - mn) / (2^bits - 1)); z = clamp(rint(-mn / s)); q = clamp(rint(w / s) + z).
 * In:  W  fp16 N x K row-major; X fp16 T x K row-major (calibration tokens), 1 <= T <= 2^20.
 * Out: codes uint8 N x K; scales, zeros fp16 N x (K / group); idx int32 k; w_weak fp16 N x k.
 * Allocates and frees its own device scratch (stream-ordered; about 20 K + 8 N K / group
 * bytes).  Deterministic: the same inputs give bit-identical outputs.
 */
owq_status_t owq_quantize(const uint16_t* W, const uint16_t* X, int N, int K, int T,
                          int bits, int group, int k,
                          uint8_t* codes, uint16_t* scales, uint16_t* zeros,
                          int32_t* idx, uint16_t* w_weak, owq_stream_t stream);

/*
 * owq_quantize_noalloc -- owq_quantize without any device allocation.  (The paper has no
 * counterpart: this is a deployment variant of the same computation.)
 * For callers that cannot let a library allocate GPU memory -- serving processes that
 * reserve nearly all device memory up front for their own pool (a library cudaMalloc would
 * fail or fragment it) and processes that forbid allocation after start-up.  Same arguments,
 * outputs and results (bit-identical) as owq_quantize, but its scratch lives in a static
 * device array sized for K <= OWQ_NOALLOC_MAX_K columns (25 bytes per column, 1 MB), which
 * every GPU that loads this library keeps until the process exits.  K above that limit
 * returns OWQ_ERR_SHAPE and launches nothing.  Every call made outside a stream capture
 * looks up the array's device address in the current context (cudaGetSymbolAddress) and
 * caches it per device; a call inside a capture uses that cache, so the first call on a
 * device must come before any stream capture (a capture before it returns OWQ_ERR_CUDA).
 * The address belongs to the context current at the lookup: after cudaDeviceReset, or in
 * another context on the same device, make one call outside a capture first.  All calls share the one array: calls that can overlap on the
 * GPU (unordered streams) race on it and must be serialised by the caller.  No state carries
 * over between calls (each kernel fully writes what it later reads).  Calls no cudaMalloc,
 * cudaFree or other allocating routine.
 */
#define OWQ_NOALLOC_MAX_K 40960
owq_status_t owq_quantize_noalloc(const uint16_t* W, const uint16_t* X, int N, int K, int T,
                                  int bits, int group, int k,
                                  uint8_t* codes, uint16_t* scales, uint16_t* zeros,
                                  int32_t* idx, uint16_t* w_weak, owq_stream_t stream);

/*
 * owq_search_params -- the truncation-aware 2-D grid search of the quantisation parameters
 * that OWQ runs before OPTQ ("Low-precision quantization", paper "Quantization
 * Configuration Search", pp.4-5: a search over step size and zero point with nearest rounding
 * and truncation, which may shrink the range below min-max).  The pages give no grid; per
 * (row, group), over the group's dense (non-idx) columns w (fp16 -> fp32):
 *   mn = min(0, min w), mx = max(0, max w)  ([-1, 1] if mn == mx);
 *   candidates: alpha in {1.00, 0.98, ..., 0.50} (alpha_i = fp32(1 - 0.02 i)) and every
 *   integer z in [0, 2^bits - 1];  s = fp16_rn(fp32(fp32(mx - mn) * alpha) / (2^bits - 1))
 *   (a candidate whose s is 0 is skipped);
 *   error = sum over the dense columns in ascending order of (w - fp16_rn(s (q - z)))^2, fp64,
 *   q = clamp(rint(w / s) + z, 0, 2^bits - 1) in fp32 (round half to even);
 *   the first minimum in the order (alpha descending, z ascending) wins; if every s is 0,
 *   s = fp16(2 / (2^bits - 1)) and z = 2^(bits-1).
 * In:  W fp16 N x K; idx int32 k (device; strictly ascending in [0, K); may be NULL if k == 0).
 * Out: scales, zeros fp16 N x (K / group) (fully overwritten; zeros integral).
 * Synchronises `stream` once (idx validated on the host: OWQ_ERR_INDEX); one kernel, a CTA
 * per (row, group) and a thread per candidate.  No scratch.  Deterministic.
 */
owq_status_t owq_search_params(const uint16_t* W, int N, int K, int bits, int group,
                               const int32_t* idx, int k, uint16_t* scales, uint16_t* zeros,
                               owq_stream_t stream);

/*
 * owq_optq -- OPTQ with the weak columns moved last, the dense quantiser the paper runs after
 * the parameter search ("Low-precision quantization", paper p.4: column-by-column quantisation
 * whose error each step compensates on the columns not yet quantised; the weak columns come
 * last, are never quantised, and keep their compensated fp16 values; "Layer-wise Quantization
 * and Hessian", p.3: each row's error is dW H dW^T).
 *   H = X^T X + damp * mean(diag(X^T X)) * I                 (fp64; damp = 0.01 is OPTQ's usual)
 *   order = the dense (non-idx) columns ascending, then the idx columns ascending;
 *   for each dense column j in that order, with F the columns from j on and M = (H over F)^-1:
 *     q = clamp(rint(fp32(w_j) / s) + z, 0, 2^bits - 1)  (the (s, z) of j's group, given);
 *     w_hat = fp16_rn(s (q - z));  w_F\j -= (w_j - w_hat) / M[j][j] * M[j][F\j];  w_j = w_hat.
 *   M is kept exact from step to step by the Schur-complement identity of the inverse of a
 *   principal submatrix (one fp64 Gauss-Jordan inversion of H first); all arithmetic is fp64.
 * In:  W fp16 N x K; X fp16 T x K (calibration tokens; 1 <= T <= 2^20); idx int32 k (device,
 *      strictly ascending); scales, zeros fp16 N x (K / group) (e.g. from owq_search_params);
 *      0 <= damp (H must be positive definite: with damp = 0, T >= K is needed).
 * Out: codes uint8 N x K (the weak columns get their group's zero point, so the result can
 *      go straight to owq_pack); w_weak fp16 N x k (the compensated weak columns).
 * Allocates K*K + N*K doubles (+ small) of stream-ordered scratch, freed before it returns;
 * synchronises `stream` once (idx is validated on the host).  Offline: 2 K + 2 (K - k) kernel
 * launches; about 0.5 s for a 4096 x 4096 layer.  Deterministic.
 */
owq_status_t owq_optq(const uint16_t* W, const uint16_t* X, int N, int K, int T, int bits,
                      int group, const int32_t* idx, int k, const uint16_t* scales,
                      const uint16_t* zeros, double damp, uint8_t* codes, uint16_t* w_weak,
                      owq_stream_t stream);

/*
 * owq_quantize_optq -- the paper's dense quantiser, end to end ("Weak-column selection",
 * "Low-precision quantization", pp.4-5): the weak columns of owq_quantize (lambda, all-column
 * RTN perturbation, sensitivity, top k), then owq_search_params over the dense columns, then
 * owq_optq with those parameters.  Same arguments and outputs as owq_quantize plus damp;
 * scales/zeros are the searched ones, codes and w_weak those of OPTQ (w_weak holds the
 * compensated weak columns).  Synchronises `stream` (idx validation of the two later steps).
 */
owq_status_t owq_quantize_optq(const uint16_t* W, const uint16_t* X, int N, int K, int T,
                               int bits, int group, int k, double damp,
                               uint8_t* codes, uint16_t* scales, uint16_t* zeros,
                               int32_t* idx, uint16_t* w_weak, owq_stream_t stream);

/*
 * owq_pack -- build a layer handle in the packed, latency-favoured layout ("Storage
 * Methods", appendix §2: a full low-precision matrix, zero-filled at the weak columns,
 * plus a separate fp16 block of the weak columns).
 * In:  codes uint8 N x K (values < 2^bits; the codes of the idx columns are ignored and
 *      stored as z); scales, zeros fp16 N x (K / group) (zeros integral in [0, 2^bits-1]);
 *      idx int32 k (device; strictly ascending in [0, K)); w_weak fp16 N x k row-major.
 *      idx and w_weak may be NULL when k == 0.
 * Out: *out = a new handle.  The handle owns copies of everything; the inputs may be
 *      freed once this call returns.
 * Packed format of one 128-code block of a row (4 * bits little-endian uint32 words):
 *   codes 2p, 2p+1 form pair p (p = 0..63); the block is four chunks of `bits` words and
 *   chunk q holds the pairs p = 4j + q (j = 0..15).  Pair j of a chunk sits at a slot
 *   (word, offset): the even code at bit `offset`, the odd code at bit 16 + offset of
 *   that word.  bits = 4: word 2(j/8) + j%2, offset 4((j%8)/2).  bits = 3: slots
 *   (0,0) (1,0) (0,3) (1,3) (0,6) (1,6) (0,9) (1,9) (0,12) (1,12) (2,6) D (2,3) (2,12)
 *   (2,0) (2,9) for j = 0..15, where D (j = 11) keeps bit e of its even / odd code in
 *   bit 15 / 31 of word e.  (A tensor-core lane's operand fragment of a block is exactly
 *   one chunk.)  The handle stores the blocks of each 16-row tile block-major (rows padded
 *   to a multiple of 16 with zero words) and, for the decode kernel, tile-major copies of
 *   the weak block and of the (scale, zero) pairs plus a split-tile workspace (2 KB per
 *   16-row tile and per extra CTA that may share it: one for most layers, N/16 * 2 KB).
 * Synchronises `stream` twice: once to copy idx to the host and validate it (OWQ_ERR_INDEX,
 * before anything is allocated), and once at the end, so that the host-side tables it uploads
 * outlive their copies.
 */
owq_status_t owq_pack(const uint8_t* codes, int N, int K, int bits, int group,
                      const uint16_t* scales, const uint16_t* zeros,
                      const int32_t* idx, int k, const uint16_t* w_weak,
                      owq_stream_t stream, owq_layer_t* out);

/*
 * The storage-favoured form ("Storage Methods", appendix §2, pp.10-11: the low-precision
 * matrix without the zero-filled weak columns, b + (16 - b) k / K bits per weight instead of
 * b + 16 k / K; using it costs an index remap).  The pages give only the bit counts.  The
 * stream used here: per row, the codes of the K - k dense (non-weak) columns in column order
 * as one little-endian bit stream of `bits` bits per code -- code p of the row at bits
 * [p*bits, p*bits + bits), bit b of the stream being bit b%32 of uint32 word b/32 -- padded
 * with zero bits to W = ceil((K - k) * bits / 32) words per row; rows are consecutive
 * (N x W uint32, row-major).  For a dense column j the stream position is p = j - #{t : idx[t]
 * < j}.
 */

/* owq_storage_words -- W, the uint32 words per row of the storage-favoured stream (host
 * call, no device work).  OWQ_ERR_SHAPE / OWQ_ERR_BITS for shapes outside the ranges above. */
owq_status_t owq_storage_words(int K, int bits, int k, int* words_per_row);

/*
 * owq_storage_pack -- codes (uint8 N x K, values < 2^bits) -> the storage-favoured stream
 * `words` (uint32 N x W, fully overwritten).  The codes of the idx columns are dropped.
 * idx: int32 k (device; strictly ascending in [0, K); may be NULL when k == 0).
 * Synchronises `stream` once (idx is copied to the host and validated: OWQ_ERR_INDEX), then
 * launches one kernel (a thread per output word).
 */
owq_status_t owq_storage_pack(const uint8_t* codes, int N, int K, int bits,
                              const int32_t* idx, int k, uint32_t* words, owq_stream_t stream);

/*
 * owq_storage_unpack -- the inverse: the storage-favoured stream `words` (uint32 N x W) ->
 * codes (uint8 N x K, fully overwritten) with each weak column set to its group's zero point
 * (the zero-filled codes the latency layout stores; zeros fp16 N x (K / group), integral).
 * Synchronises `stream` once (idx validated on the host), then launches one kernel.
 */
owq_status_t owq_storage_unpack(const uint32_t* words, int N, int K, int bits, int group,
                                const int32_t* idx, int k, const uint16_t* zeros,
                                uint8_t* codes, owq_stream_t stream);

/*
 * owq_pack_storage -- build a layer handle from the storage-favoured stream: the stream is
 * repacked on the GPU into the latency-favoured layout of owq_pack (same handle, same
 * products, bit-identical to owq_pack of the unpacked codes).  Arguments as owq_pack, with
 * `words` (uint32 N x W) in place of the codes.  Allocates an N x K byte code buffer for the
 * duration of the call and frees it before returning; synchronises `stream`.
 */
owq_status_t owq_pack_storage(const uint32_t* words, int N, int K, int bits, int group,
                              const uint16_t* scales, const uint16_t* zeros,
                              const int32_t* idx, int k, const uint16_t* w_weak,
                              owq_stream_t stream, owq_layer_t* out);

/*
 * owq_gemv -- decode product for 1 <= M <= 16 tokens ("Real-device acceleration",
 * paper p.6: low-bit dense product plus fp16 weak columns on the activation channels
 * selected on the fly).  One kernel, one wave of one 16-warp CTA per SM: every warp
 * streams an equal share of the layer's (16-row tile, 128-code block) units through its
 * own shared-memory ring (bulk copies), lifts each code pair into an exact fp16x2 value with
 * one AND, multiplies on the tensor cores (m16n8k16, fp32 accumulation), applies scale and
 * zero point per row segment, and adds the weak columns (gathered activations x fp16 block)
 * in the same pass; a row tile shared by several warps is summed by the warp holding its
 * last unit.  One fp16 rounding of each output.
 * In:  x fp16 M x K row-major.   Out: y fp16 M x N row-major (fully overwritten).
 * Every call writes the handle's split-tile workspace and call counter: calls on one
 * handle must be ordered (one stream, or events between streams); calls on different
 * handles may overlap.  Bounded device waits: on a timeout (see owq_gemm) y is undefined.
 */
owq_status_t owq_gemv(owq_layer_t layer, const uint16_t* x, uint16_t* y, int M,
                      owq_stream_t stream);

/*
 * owq_gemv_multi -- `count` independent decode products in ONE launch (layers that
 * read their inputs before any of them writes, e.g. q/k/v of one attention block).
 * layers, xs, ys are HOST arrays of `count` entries; xs[i] is M x K_i and ys[i] is
 * M x N_i (device).  All layers must share bits; 1 <= count <= 16; a handle may appear
 * only once (OWQ_ERR_HANDLE).  Output buffers must not overlap inputs of another entry.
 */
owq_status_t owq_gemv_multi(const owq_layer_t* layers, const uint16_t* const* xs,
                            uint16_t* const* ys, int count, int M, owq_stream_t stream);

/*
 * owq_gemm -- prefill product for any M >= 1 (tuned for M >= 64): TMA-staged packed tiles,
 * dequantised in registers into tensor memory (the A operand of tcgen05 MMA, B = the
 * activations in shared memory) with fp32 accumulators in tensor memory; the weak block and the weak activations (gathered by a small kernel into the
 * handle's scratch) run as extra K-steps into the same accumulator.  Same semantics and
 * layouts as owq_gemv; M <= 65536.  Bounded device waits: on a timeout the kernel abandons
 * its tile, sets the device status word and this call's later owq_device_status returns
 * OWQ_ERR_TIMEOUT (y is then undefined).  The first call on a handle builds its tensor
 * maps on the host: first calls from several host threads on one handle must be
 * serialised.  The handle's scratch (M * k_ld * 2 bytes of weak activations; when
 * owq_gemm_plan splits K, also a workspace of fp32 partial sums) grows on the first call that
 * needs more, which must not be inside a stream capture: there a too-small weak-activation
 * scratch gives OWQ_ERR_NOMEM (a too-small partial-sum workspace: the call runs unsplit).
 * Split outputs are the fp32 partials added in split order, then rounded once: repeated calls
 * give identical bits.  Calls on one handle must be ordered (same stream, or synchronised):
 * they share that scratch.
 */
owq_status_t owq_gemm(owq_layer_t layer, const uint16_t* x, uint16_t* y, int M,
                      owq_stream_t stream);

/*
 * owq_gemm_plan -- the launch shape owq_gemm takes for an N x K layer, M tokens, on a device
 * with `sms` SMs (host only; no device, no handle).  Tiles are 128 weight rows x `tile_tokens`
 * tokens (64 for M <= 64, 128 for M <= 256, else 256).  With fewer tiles than SMs every tile
 * is split over K; with a short last wave the row tiles of the last few token tiles are split
 * over K instead (the "tail"), to run on the SMs the whole tiles leave idle.  Either way a
 * reduction kernel adds the fp32 partials in split order.
 * Out: plan[0] tile_tokens, plan[1] K splits of every tile (1: none), plan[2] token tiles in
 *      the tail (0: none), plan[3] K splits of each tail tile (1: none).
 * Errors: OWQ_ERR_NULL (plan NULL), OWQ_ERR_SHAPE (N, K outside owq_pack's ranges, M outside
 * 1..65536), OWQ_ERR_ARG (sms < 1).
 */
owq_status_t owq_gemm_plan(int N, int K, int M, int sms, int plan[4]);

/*
 * owq_weak_grad -- weak column tuning: gradient of a loss with respect to the layer's fp16
 * weak block ("PEFT with Weak Column Tuning", paper p.5, and "WCT-based fine-tuning",
 * p.7: only the weak columns are trained, the packed low-bit matrix stays frozen).
 *   dw_weak[i][t] = sum_m dy[m][i] * x[m][idx[t]]
 * In:  x fp16 M x K row-major (the layer's forward input), dy fp16 M x N row-major (the
 *      gradient of its output); 1 <= M <= 65536.
 * Out: dw_weak fp32 N x k row-major (fully overwritten; may be NULL when k == 0, and then
 *      nothing is launched).  A dense N x k x M contraction on the tensor cores (mma.sync
 *      m16n8k16, fp16 products exact in fp32, fp32 accumulation): a small kernel gathers
 *      x[:, idx] into the handle's scratch, the product kernel splits the tokens over CTAs when
 *      the output alone would not fill the GPU, and a last kernel adds the splits in split
 *      order, so repeated calls give identical bits.  The scratch (M * k rounded up to 32 fp16,
 *      plus splits * N * k fp32) grows on the first call that needs more, which must be outside
 *      a stream capture; inside one, or when N is not a multiple of 8, a CUDA-core kernel that
 *      needs no scratch runs instead (same result up to fp32 rounding).  Calls on one handle
 *      must be ordered (they share the scratch).  No waits.
 * Device pointers, 16-byte aligned (OWQ_ERR_ALIGN); asynchronous on `stream`.
 */
owq_status_t owq_weak_grad(owq_layer_t layer, const uint16_t* x, const uint16_t* dy,
                           float* dw_weak, int M, owq_stream_t stream);

/*
 * owq_input_grad -- weak column tuning: the gradient the frozen layer passes to its input
 * (same pages; earlier layers' weak columns need it), the transposed product
 *   dx[m][j] = sum_i dy[m][i] * W_eff[i][j],
 * W_eff = the dequantised matrix except at the weak columns, which take their fp16 values from
 * the weak block.  Read straight from the packed layout (no W_hat in memory), fp32
 * accumulation, one fp16 rounding of each output.  Two paths:
 *  - M <= 16, or N not a multiple of 8: 16 tokens per pass (mma.sync m16n8k16); the exact
 *    integers q - z times dy * s carried as an fp16 pair (high part + residual), i.e. the
 *    unrounded s (q - z) like the decode product (each weight within half an fp16 spacing of
 *    W_hat = fp16_rn(s (q - z))).  The rows of a 128-column block are split over up to 8 CTAs
 *    of one thread-block cluster whose fp32 sums are added in a fixed order through distributed
 *    shared memory: no workspace, allowed inside a stream capture.
 *  - M > 16 and N % 8 == 0: the 5th-generation tensor cores (tcgen05.mma, accumulator and the
 *    A operand W_hat^T in tensor memory, dy by TMA) multiply W_hat = fp16_rn(s (q - z)) itself,
 *    bit-exact per weight; the weak columns come out exactly 0 there (their codes hold q = z)
 *    and a second kernel then writes dx[:, idx] = dy W_weak (mma.sync).  With fewer output
 *    tiles than SMs the rows are split over CTAs: fp32 partials in the handle's prefill
 *    workspace (and the weak pass's in the weak-gradient scratch), grown on the first call that
 *    needs more, which must be outside a stream capture (inside one: a single split, slower,
 *    same result); the splits are added in split order.  Calls on one handle must be ordered.
 * Both paths: with a single nonzero dy (1.0) per token the output row is W_eff's row bit for
 * bit; repeated calls give identical bits.  Waits are bounded (OWQ_ERR_TIMEOUT through
 * owq_device_status).
 * In:  dy fp16 M x N row-major; 1 <= M <= 65536.  Out: dx fp16 M x K row-major (fully
 *      overwritten).  Device pointers, 16-byte aligned; asynchronous on `stream`.
 */
owq_status_t owq_input_grad(owq_layer_t layer, const uint16_t* dy, uint16_t* dx, int M,
                            owq_stream_t stream);

/*
 * owq_dequant -- test hook: write W_hat = fp16_rn(s * (q - z)) (N x K fp16, 0 at the weak
 * columns) and, if codes is not NULL, the unpacked codes (N x K uint8).
 */
owq_status_t owq_dequant(owq_layer_t layer, uint16_t* w_hat, uint8_t* codes,
                         owq_stream_t stream);

/* Shape of a layer (host outputs; any may be NULL). */
owq_status_t owq_layer_info(owq_layer_t layer, int* N, int* K, int* bits, int* group, int* k);

/* Bytes of the layer's data, per part (host outputs; any may be NULL): packed codes
 * N*K*bits/8, scales+zeros 4*N*K/group, weak block 2*N*k, index list 4*k.  (The handle also
 * keeps the working copies described at owq_pack.) */
owq_status_t owq_layer_bytes(owq_layer_t layer, size_t* packed, size_t* scales_zeros,
                             size_t* weak, size_t* index);

/* Release a layer (stream-ordered on the stream given to owq_pack). NULL is a no-op. */
owq_status_t owq_layer_free(owq_layer_t layer);

/* Synchronises the current device (cudaDeviceSynchronize), then returns and clears its device
 * status word (OWQ_OK, or OWQ_ERR_TIMEOUT if a bounded wait of any call on this device gave up
 * since the last query, or OWQ_ERR_BOUNDS, first, if a check of the debug-bounds build failed).
 * The debug-bounds build (libowq_b200_bounds.so, compiled with -DOWQ_DEBUG_BOUNDS; owq_version
 * ends in "+debug-bounds") checks the kernels' data-dependent indices before each access -- the
 * weak index list in every gather and scatter, the storage stream positions -- and skips an
 * access that fails (writing 0 or nothing), so an indexing fault reports here instead of
 * faulting the GPU.  The default build compiles the checks out.  The word is per device, not per handle: a bounded wait gives up
 * inside a kernel, which has no way to name the handle of the call that launched it, and the
 * kernels of every handle on a device write the same word.  The whole device is synchronised
 * because the failed call may sit on any stream; call this between steps, not on a hot path. */
owq_status_t owq_device_status(void);

/*
 * owq_debug_inject -- test hook for the bounded-wait error path (host only, process-wide,
 * not thread-safe).  Arms one injected failure, consumed by the next call of its kind:
 *   OWQ_INJECT_GEMV_TAG     next owq_gemv / owq_gemv_multi: the partial sums of row tiles that
 *                           are split across CTAs are published under a tag no reader accepts,
 *                           so each cross-CTA wait runs out and its tile is not written (a
 *                           layer whose tiles all stay inside one CTA has no such wait);
 *   OWQ_INJECT_GEMM_ARRIVE  next owq_gemm: one dequantisation thread of every CTA skips its
 *                           arrival for its first K step, so the MMA issuer's wait runs out,
 *                           then the producer's and the dequantisation threads' waits.
 * wait_cycles (>= 1) bounds every device wait of that call, in SM clock cycles (otherwise the
 * bound is 4e9 cycles, about 2 s).  The kernel records the timeout in the device status
 * word, leaves y undefined, lets its own bulk copies land, frees its tensor memory and
 * returns: the next owq_device_status returns OWQ_ERR_TIMEOUT and the context stays usable.
 *   OWQ_INJECT_BOUNDS       debug-bounds build only (OWQ_ERR_ARG otherwise; wait_cycles ignored):
 *                           the next owq_input_grad that takes the many-token path on a handle
 *                           with weak columns stores token 0 of weak slot 0 one row of K past
 *                           its column; the bounds check skips that store and the next
 *                           owq_device_status returns OWQ_ERR_BOUNDS (dx[0][idx[0]] is then
 *                           undefined, every other output as without the injection).
 * OWQ_INJECT_NONE disarms (wait_cycles ignored).  Errors: OWQ_ERR_ARG for an unknown `what`
 * or wait_cycles < 1.
 */
owq_status_t owq_debug_inject(int what, long long wait_cycles);

/* Static, human-readable name of a status code. */
const char* owq_status_string(owq_status_t status);

/* Library version as "major.minor.patch" (static string). */
const char* owq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* OWQ_H_ */
