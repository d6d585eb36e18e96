/*
 * gptq.h -- C ABI of the B200 GPTQ layer solver (libgptq.so).
 *
 * The library turns one linear layer's weights W (out x in) and its
 * calibration activations X (in x tokens) into 2/3/4/8-bit group-quantized
 * integer codes with one scale and one zero per group, the act-order
 * permutation and g_idx.  Three calls make one layer solve:
 *
 *   gptq_hessian_accumulate  S += X X^T            (once per calibration chunk)
 *   gptq_prepare_hinv        H = 2 S / n, dead-channel fix, dampening,
 *                            act-order permutation, U = upper Cholesky
 *                            factor of H^-1
 *   gptq_quantize_layer      the blocked column sweep with error
 *                            compensation, group quantization and packing
 *
 * and, around them: gptq_dequantize_layer (codes back to weights),
 * gptq_export_checkpoint (the outputs in the loaders' checkpoint layout),
 * gptq_quantize_layer_noalloc (quantize on a fixed library scratch),
 * gptq_workspace_bytes / gptq_validate_config (host-side sizing and checks)
 * and gptq_selftest_wait_timeout (the bounded-wait failure path).
 *
 * What is computed follows the GPTQ pages: "gptq" glossary page (Method and
 * Algorithm: layer-wise, Hessian from calibration data, quantize each weight
 * in order and compensate the error with H^-1; Group quantization), "Using
 * AutoGPTQ in Practice" (Hessian computation, Cholesky factorization, group
 * quantization; Key Parameters: bits, group_size, desc_act, damp_percent),
 * "gptq" agent-skill page (Group-wise quantization: own scale and zero per
 * group; group_size -1 = per column) and the AutoGPTQ artifact page (2/3/4/8
 * bits, symmetric and asymmetric schemes, config validation).
 *
 * Conventions for every call
 *   - Pointers named "device" are CUDA device (or managed) memory owned by the
 *     caller; the library never keeps them after the call returns and never
 *     allocates device memory itself: scratch space is the caller's
 *     workspace, sized by gptq_workspace_bytes().
 *   - stream is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Work is enqueued on it; only gptq_prepare_hinv and
 *     gptq_selftest_wait_timeout wait for it.
 *   - Matrices are row-major unless stated otherwise; leading dimensions are
 *     in elements.
 *   - Every call returns a gptq_status_t.  Nothing aborts or traps.  On an
 *     error, gptq_last_error() returns a message for the calling thread.
 *   - The kernels are built for sm_100a only; on any other device the calls
 *     return GPTQ_ERR_UNSUPPORTED.  There is no CPU fallback.
 */
#ifndef GPTQ_B200_H
#define GPTQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GPTQ_ABI_VERSION 1

typedef enum gptq_status {
  GPTQ_OK = 0,
  GPTQ_ERR_INVALID_ARG = 1,  /* rejected on the host before any launch        */
  GPTQ_ERR_NOT_PD = 2,       /* damped Hessian has no Cholesky factor          */
  GPTQ_ERR_NONFINITE = 3,    /* NaN or Inf met in S                            */
  GPTQ_ERR_WORKSPACE = 4,    /* workspace missing, misaligned or too small     */
  GPTQ_ERR_CUDA = 5,         /* a CUDA runtime call failed (message says which)*/
  GPTQ_ERR_TIMEOUT = 6,      /* a bounded device-side wait gave up             */
  GPTQ_ERR_UNSUPPORTED = 7   /* valid request this build does not implement    */
} gptq_status_t;

typedef enum gptq_dtype {
  GPTQ_F16 = 0,
  GPTQ_BF16 = 1,
  GPTQ_F32 = 2
} gptq_dtype_t;

/*
 * Quantization settings, the fields of the pages' BaseQuantizeConfig
 * ("gptq" agent-skill page, Quantization configurations; "Using AutoGPTQ in
 * Practice", Key Parameters) plus the symmetric flag (AutoGPTQ artifact page)
 * and the lazy-batch width.
 *   bits          2, 3, 4 or 8.
 *   group_size    -1 (one group per output row) or a positive divisor of in.
 *                 This build also needs group_size >= 8 and either
 *                 128 % group_size == 0 or group_size % 128 == 0 (else
 *                 GPTQ_ERR_UNSUPPORTED).
 *   sym           0: asymmetric grid over [min(0, min w), max(0, max w)],
 *                    zero = rint(-lo / scale);
 *                 1: symmetric, scale = 2 max|w| / maxq, zero = (maxq+1)/2.
 *   desc_act      1: process columns by decreasing diag(H) (ActOrder).
 *   damp_percent  >= 0, finite: damp_percent * mean(diag H) is added to the
 *                 diagonal.
 *   block_size    > 0; with group_size != -1 it must divide group_size or be
 *                 a multiple of it.  It is the lazy-batch width: it changes
 *                 only the order of floating-point rounding, never the
 *                 result in exact arithmetic.  This build validates it and
 *                 always batches 128 columns (the width its kernels are
 *                 built around).
 * maxq = 2^bits - 1.  code = clamp(rint(w / scale) + zero, 0, maxq), the
 * division and rint in IEEE float32 (round half to even).
 * Layer size limits of this build: 1 <= in <= 32768, 0 <= out <= 65535
 * (larger layers return GPTQ_ERR_UNSUPPORTED).
 */
typedef struct gptq_config {
  int32_t bits;
  int32_t group_size;
  int32_t sym;
  int32_t desc_act;
  float damp_percent;
  int32_t block_size;
} gptq_config_t;

/* GPTQ_ABI_VERSION of the loaded library. */
int gptq_abi_version(void);

/* Number of CUDA kernels this library has launched in this process, over
 * all calls and threads (a diagnostic: callers can count the launches of a
 * region by differencing two reads). */
uint64_t gptq_kernel_launches(void);

/* Message for the last error on the calling thread ("" if none).  The
 * pointer stays valid until the thread's next gptq_* call. */
const char* gptq_last_error(void);

/* Host-only check of a configuration for a layer of out x in (the pages'
 * config validator, AutoGPTQ artifact page).  out may be 0. */
gptq_status_t gptq_validate_config(const gptq_config_t* cfg, int64_t out,
                                   int64_t in);

/* Bytes of device workspace that gptq_prepare_hinv (out = 0) or both
 * gptq_prepare_hinv and gptq_quantize_layer (out > 0) need for a layer of
 * out x in.  Returns 0 for invalid sizes.  The workspace must be 256-byte
 * aligned; its contents need no initialisation and are not preserved. */
size_t gptq_workspace_bytes(int64_t out, int64_t in, const gptq_config_t* cfg);

/*
 * S += X X^T: accumulate the Gram matrix of one chunk of calibration tokens
 * ("gptq" glossary page, Algorithm (1): the Hessian comes from calibration
 * data).
 *   S        device fp32, in x in, row-major.  Only the upper triangle with
 *            the diagonal (S[i][j], j >= i) is read and written; the strictly
 *            lower triangle is left untouched.  Zero it before the first
 *            chunk.  (S, n) is additive: chunks may come in any number of
 *            calls, and a saved (S, n) resumes accumulation.
 *   in       channels, >= 1.
 *   X        device, in x tokens, element type xt, row stride ldx >= tokens
 *            (row i = channel i, tokens contiguous).  Read only.
 *   tokens   >= 0; 0 is a no-op.
 *   n_accum  host pointer or NULL; *n_accum += tokens on success.
 * fp16/bf16 X with a 16-byte aligned base and (ldx * 2) % 16 == 0 runs on the
 * tensor cores (exact products, fp32 accumulation, drained into S every 32768
 * tokens so the accumulation error stays below 5e-5 relative for any token
 * count); fp32 X and other layouts run on CUDA cores in fp32.  Asynchronous.
 * Accumulation order is fixed for a given (in, tokens, device), so repeated
 * calls give identical S.
 */
gptq_status_t gptq_hessian_accumulate(float* S, int64_t in, const void* X,
                                      gptq_dtype_t xt, int64_t tokens,
                                      int64_t ldx, int64_t* n_accum,
                                      void* stream);

/*
 * From the accumulated S (upper triangle) and token count n:
 *   H = 2 S / n;  dead channels (H_ii == 0) get H_ii = 1;
 *   perm = stable descending argsort of diag(H) if desc_act, else identity
 *          ("Using AutoGPTQ in Practice", Key Parameters, desc_act);
 *   H += damp_percent * mean(diag H) * I (same section, damp_percent);
 *   U = upper Cholesky factor of (H[perm][:, perm])^-1, i.e. U upper
 *       triangular with positive diagonal and U^T U = H_perm^-1 ("Using
 *       AutoGPTQ in Practice": Cholesky factorization).
 * Outputs (device, caller-owned):
 *   U     fp32 in x in, COLUMN-major: element (i, j) of U at U[j*in + i].
 *         Entries with i > j are written as 0.
 *   perm  int32[in]: perm[p] = original column processed at position p.
 *   dead  uint8[in], by original column: 1 if the channel never fired.
 * ws / ws_bytes: workspace from gptq_workspace_bytes(0, in, cfg) or larger.
 * Waits for the stream once, to read the device status word:
 *   GPTQ_ERR_NONFINITE if S holds NaN/Inf, GPTQ_ERR_NOT_PD if a pivot of the
 *   factorisation is not positive, GPTQ_ERR_TIMEOUT if a bounded device wait
 *   gave up.  Only bits/group_size/sym/block_size are not used here.
 */
gptq_status_t gptq_prepare_hinv(const float* S, int64_t n, int64_t in,
                                const gptq_config_t* cfg, float* U,
                                int32_t* perm, uint8_t* dead, void* ws,
                                size_t ws_bytes, void* stream);

/*
 * The column sweep ("gptq" glossary page, Algorithm (2): for each weight in
 * order, quantize it, compute the error, adjust the remaining weights with
 * H^-1), in processing order perm, with one scale/zero per group of
 * group_size consecutive processed columns ("gptq" agent-skill page,
 * Group-wise quantization).  For processed column j of row r:
 *   at a group start, scale/zero from the group's current (updated) weights;
 *   q = clamp(rint(w / scale) + zero, 0, maxq);   deq = scale * (q - zero);
 *   e = (w - deq) / U[j][j];   w[r][c] -= e * U[j][c] for all later c.
 * Inputs (device): W out x in, element type wt, row stride ldw >= in, not
 *   modified (dead columns are zeroed in the library's working copy);
 *   U, perm, dead as written by gptq_prepare_hinv.
 * Outputs (device, caller-owned; NULL allowed where marked):
 *   codes    int32 out x in, original column order (NULL: skipped).
 *   qweight  uint32 [out][in*bits/32]: row r's codes in original column
 *            order as an LSB-first stream of bits-wide fields in
 *            little-endian words (fields may straddle words).  Needs
 *            (in*bits) % 32 == 0 (NULL: skipped).
 *   scales   fp32 [out][ngroups], ngroups = in/group_size or 1 for -1;
 *            group index in processing order.
 *   zeros    int32 [out][ngroups], same indexing.
 *   g_idx    int32[in]: group of original column c (0 for group_size -1).
 *   loss     fp32[out] or NULL: sum over columns of e^2 for each row (the
 *            quadratic error (W - deq) H (W - deq)^T with the damped H).
 * ws / ws_bytes: workspace from gptq_workspace_bytes(out, in, cfg).
 * Asynchronous.  out == 0 is a no-op.  Inside the call, every kernel is an
 * ordinary launch on the caller's stream (the gathers, one cooperative
 * launch for the sweep and its updates, the inverse permutation and the
 * packing), so the call's work is ordered after everything already queued
 * on the stream and before everything queued after it.
 * The call returns before its kernels run, so a failure inside them (a
 * bounded device-side wait that gave up: GPTQ_ERR_TIMEOUT) is not in its
 * return value: it is raised in the status word at the start of ws, which
 * gptq_workspace_status(ws, ws_bytes, stream) reads back once the stream has
 * finished the call.
 */
gptq_status_t gptq_quantize_layer(const void* W, gptq_dtype_t wt, int64_t out,
                                  int64_t in, int64_t ldw, const float* U,
                                  const int32_t* perm, const uint8_t* dead,
                                  const gptq_config_t* cfg, int32_t* codes,
                                  uint32_t* qweight, float* scales,
                                  int32_t* zeros, int32_t* g_idx, float* loss,
                                  void* ws, size_t ws_bytes, void* stream);

/*
 * Device-side status of the last gptq_prepare_hinv or gptq_quantize_layer
 * call that used workspace ws.  Each of those calls clears a 32-bit status
 * word at the start of ws on its stream before its first kernel; its kernels
 * only ever raise flags in it.  This call waits for stream, reads the word
 * and returns:
 *   GPTQ_ERR_TIMEOUT    a bounded device-side wait gave up (the call's
 *                       outputs are incomplete);
 *   GPTQ_ERR_NONFINITE  S held NaN or Inf (prepare);
 *   GPTQ_ERR_NOT_PD     a pivot of the factorisation was not positive
 *                       (prepare);
 *   GPTQ_OK             none of these.
 * Pass the stream the call was made on (or one ordered after it).  ws must
 * be 256-byte aligned and ws_bytes >= 256.  gptq_prepare_hinv already
 * returns this status itself; for gptq_quantize_layer this call is the only
 * way to see it.
 */
gptq_status_t gptq_workspace_status(const void* ws, size_t ws_bytes,
                                    void* stream);

/*
 * Dequantize: Wq[r][c] = scales[r][g] * (code[r][c] - zeros[r][g]) with
 * g = g_idx[c], the inverse of the group quantizer ("gptq" agent-skill page,
 * Group-wise quantization; "gptq" glossary page: weights stored as low-bit
 * codes with a scale and zero point per group).  The product is formed in
 * fp32 and rounded once to wt.
 * Inputs (device, as written by gptq_quantize_layer): qweight uint32
 *   [out][in*bits/32] (LSB-first fields, original column order); scales fp32
 *   and zeros int32 [out][ngroups]; g_idx int32[in], 16-byte aligned.
 * Output (device, caller-owned): Wq, out x in, element type wt, row stride
 *   ldw >= in.
 * Needs in % 8 == 0 and (in * bits) % 32 == 0 (GPTQ_ERR_UNSUPPORTED
 * otherwise).  Asynchronous.  out == 0 is a no-op.
 */
gptq_status_t gptq_dequantize_layer(const uint32_t* qweight,
                                    const float* scales, const int32_t* zeros,
                                    const int32_t* g_idx, int64_t out,
                                    int64_t in, int bits, int ngroups,
                                    void* Wq, gptq_dtype_t wt, int64_t ldw,
                                    void* stream);

/*
 * Export: the solver's outputs rewritten in the checkpoint layout of the
 * GPTQ loaders ("AutoGPTQ" artifact page, Why AutoGPTQ Matters: the GPTQ
 * format that ExLlamaV2 and vLLM load; "gptq" agent-skill page, Marlin:
 * quantized models saved and loaded in it).  The pages print no bit layout;
 * the one written here stores every tensor input-dimension-major:
 *   qweight_t uint32 [in*bits/32][out]: column o is row o's codes in
 *             original column order as an LSB-first stream of bits-wide
 *             fields (fields may straddle words) -- the transpose of the
 *             qweight gptq_quantize_layer writes.  Needs (in*bits) % 32 == 0.
 *   qzeros    uint32 [ngroups][out*bits/32]: row g is the LSB-first stream,
 *             along the output dimension, of (zeros[o][g] - zero_offset)
 *             mod 2^bits.  Needs (out*bits) % 32 == 0.  zero_offset 1 is
 *             the convention of the format's first version (readers add 1
 *             back; a zero of 0 wraps to 2^bits - 1, which such a reader
 *             cannot tell from 2^bits - 1); 0 stores the zeros as they are.
 *   scales_h  float16 bits (uint16) [ngroups][out]: scales^T rounded to
 *             nearest, ties to even (values above 65504 become infinity).
 * g_idx needs no rewrite: the loaders read the int32[in] that
 * gptq_quantize_layer writes.
 * Inputs (device, as written by gptq_quantize_layer): qweight uint32
 *   [out][in*bits/32], scales fp32 and zeros int32 [out][ngroups].
 * Outputs (device, caller-owned, not aliasing the inputs): any may be NULL
 *   to skip it; each requested output needs its input non-NULL.
 * Errors: GPTQ_ERR_INVALID_ARG for bits outside {2, 3, 4, 8}, sizes outside
 * the limits, ngroups outside [1, in], zero_offset outside {0, 1} or a
 * missing input; GPTQ_ERR_UNSUPPORTED for the divisibility rules above.
 * Asynchronous.  out == 0 or no requested output is a no-op.
 */
gptq_status_t gptq_export_checkpoint(const uint32_t* qweight,
                                     const float* scales, const int32_t* zeros,
                                     int64_t out, int64_t in, int bits,
                                     int ngroups, int zero_offset,
                                     uint32_t* qweight_t, uint32_t* qzeros,
                                     uint16_t* scales_h, void* stream);

/*
 * Diagnostic with no counterpart in the method: every wait inside this
 * library's kernels (pipeline barriers, copy completion, grid barriers) is
 * bounded and, when it gives up, raises GPTQ_ERR_TIMEOUT through a status
 * word instead of hanging or trapping.  This call runs that path on purpose:
 * one thread waits on a barrier that nothing ever completes, gives up after
 * limit_ns nanoseconds (1 .. 2e9), and the call returns GPTQ_ERR_TIMEOUT.
 * The device stays usable afterwards.  Synchronises the stream.
 */
gptq_status_t gptq_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/*
 * Diagnostic with no counterpart in the method: the sweep decides each code
 * from x / scale rounded to nearest, computed without a divide (a
 * reciprocal and two fma corrections, Markstein's method).  This call checks
 * that quotient against the IEEE division on n pseudo-random pairs drawn from
 * seed (a quarter with random magnitudes, the rest within 8 units in the last
 * place of a half-integer multiple of the scale).  *checked receives the
 * pairs inside the method's range (the sweep takes an exact fallback
 * outside it), *mismatches those whose quotient differed in any bit.
 * Synchronises the stream.
 */
gptq_status_t gptq_selftest_quotient(uint64_t n, uint64_t seed, uint64_t* checked, uint64_t* mismatches,
                                     void* stream);

/* Size of the fixed device scratch used by gptq_quantize_layer_noalloc:
 * 32 MiB, enough for layers up to 1024 x 1024. */
#define GPTQ_STATIC_SCRATCH_BYTES ((size_t)32 << 20)

/*
 * gptq_quantize_layer without a caller workspace and without allocating.
 * The GPTQ paper has no counterpart to this call: it is a convenience of
 * this library.  It is meant for callers that cannot allocate device memory
 * at the moment they quantize: code running inside an allocator callback or
 * an out-of-memory handler (allocating there would re-enter the allocator),
 * code that must not add the device-wide synchronisation that cudaFree
 * implies, and processes whose device memory is already fully claimed by a
 * caching allocator.  Nothing inside this call runs cudaMalloc, cudaFree or
 * any other routine that allocates device memory.
 *
 * Arguments, outputs and results are those of gptq_quantize_layer, without
 * ws / ws_bytes.  Instead the call uses one static device array of
 * GPTQ_STATIC_SCRATCH_BYTES bytes (256-byte aligned) that the library's
 * device code carries; it exists once per device, from when that code is
 * loaded on the device.
 *
 * Limit: a layer whose quantize workspace needs more than
 * GPTQ_STATIC_SCRATCH_BYTES is rejected with GPTQ_ERR_WORKSPACE before any
 * work is queued; gptq_last_error() gives the bytes needed.  Such layers
 * need gptq_quantize_layer with a caller workspace.
 *
 * Device and setup: the call works on the calling thread's current device;
 * stream must belong to it.  The first call on each device (more precisely,
 * on each CUDA context of a device: after cudaDeviceReset the next call sets
 * up again) is the set-up.  It looks up the scratch's address with
 * cudaGetSymbolAddress, which creates the device's primary context if the
 * thread has none yet, and makes the driver load every kernel the call can
 * launch.  Loading device code reserves device memory inside the driver, so
 * make the first call on each device outside the situations this entry point
 * is for (allocator callbacks, out-of-memory handlers) and before any stream
 * capture begins; gptq_quantize_layer_noalloc_status also does the set-up
 * and can serve as that first call.  Later calls on the same context read
 * the cached address and load nothing.
 *
 * Device-side status: as for gptq_quantize_layer, a failure inside the
 * kernels is raised in a status word, here at the start of the static
 * scratch; gptq_quantize_layer_noalloc_status(stream) reads it back.
 *
 * Zero state: no byte of the scratch has to start at zero.  Each call clears
 * the scratch's 256-byte status header itself, on stream, before its first
 * kernel, and writes every other scratch byte before reading it.
 *
 * Overlapping calls race: all calls on one device share the one scratch.
 * Two calls whose device work overlaps in time (from two host threads, or on
 * two streams with no ordering between them) corrupt each other's scratch and
 * both results are undefined.  Order them: issue them on one stream, or make
 * the later stream wait on an event recorded after the earlier call.  The
 * call is asynchronous, so the scratch stays in use until stream has
 * finished the call's work.
 */
gptq_status_t gptq_quantize_layer_noalloc(const void* W, gptq_dtype_t wt,
                                          int64_t out, int64_t in, int64_t ldw,
                                          const float* U, const int32_t* perm,
                                          const uint8_t* dead,
                                          const gptq_config_t* cfg,
                                          int32_t* codes, uint32_t* qweight,
                                          float* scales, int32_t* zeros,
                                          int32_t* g_idx, float* loss,
                                          void* stream);

/*
 * gptq_workspace_status for gptq_quantize_layer_noalloc: waits for stream
 * and returns the device-side status of the last noalloc call on the
 * current device (GPTQ_OK or GPTQ_ERR_TIMEOUT), read from the status word at
 * the start of the static scratch.  Like that call, it has no counterpart in
 * the GPTQ paper.  On a device with no earlier noalloc call it performs the
 * set-up and returns GPTQ_OK.
 */
gptq_status_t gptq_quantize_layer_noalloc_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_H */
