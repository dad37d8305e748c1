/*
 * tq.h -- C ABI of libtq, a B200 (sm_100a) implementation of the TurboQuant
 * hot path: online rotate -> Lloyd-Max -> 1-bit QJL quantisation of key
 * vectors, and unbiased inner-product estimation (attention logits, top-k)
 * against the packed codes.
 *
 * Sources for what each call computes (web pages on TurboQuant):
 *   [p2]  airosetta.com, "Google TurboQuant KV compression":
 *         section "第一階段：PolarQuant" (random rotation from the QR of a
 *         Gaussian matrix, Beta coordinate law, per-coordinate Lloyd-Max with a
 *         precomputed codebook, dequantise = table lookup + inverse rotation)
 *         and section "第二階段：QJL" (1-bit sign sketch of the residual,
 *         unbiased inner-product estimator, O(d) per vector).
 *   [p1]  mooersco.com news article, section 1.1 (rotation preserves the L2
 *         norm; the key is multiplied by the rotation matrix) and 2.2 (4-bit
 *         logits on GPU are memory-bandwidth bound).
 *   [p5]  zhengruan.com news, "第一步 / 第二步" (precomputed codebook; one bit
 *         for the residual direction combined with the full-precision query).
 *
 * Conventions (all calls):
 *   - Device pointers are caller-owned CUDA device memory; the library never
 *     frees them.  Host pointers are marked "host".
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous on `stream`: the returned status covers argument
 *     validation and the launch; the kernels' own bounded waits report into a
 *     per-context status word read by tq_check_device_status().
 *   - A context is immutable after tq_init and may be used from several
 *     streams at once; calls that share output buffers must be ordered by
 *     the caller.
 *   - Errors never abort the process.  TQ_ERR_ARG: a null pointer, a negative
 *     or inconsistent size, a misaligned pointer.  TQ_ERR_UNSUPPORTED: a shape
 *     the kernels do not cover.  TQ_ERR_CUDA: a CUDA runtime error (the
 *     message is kept in tq_last_cuda_error()).  TQ_ERR_RANGE: a quantised
 *     key's norm did not fit in fp16 (reported through the context's status
 *     word, see tq_check_device_status, since the kernels run asynchronously).
 *
 * Packed layout (one row per key; the pages fix no layout, only "no
 * per-block constants"):  b' = bits - 1.  The layout has dp and mp slots, d
 * and m rounded up to multiples of 64 (equal to d and m when they are
 * multiples of 64); in the formulas below d and m stand for dp and mp, and
 * the code slots j >= d and sign slots i >= m of the true sizes are zero.
 *   payload row = 4 quarter chunks q = 0..3 of 2 (b' d/64 + m/64) bytes.
 *   Chunk q holds rotated coordinates j = q d/4 + 4r + e (r < d/16, e < 4) as
 *   little-endian 16-bit halfwords: the b' code halfwords of each unit
 *   u = 0..d/64-1 (unit u = r in [4u, 4u+4)), then one sign halfword per unit
 *   of 16 sign coordinates.  "Nibble e" of a halfword is bits 4e..4e+3.
 *     b'=1: H0 nibble e bit i              = code(4u+i, e)
 *     b'=2: Hi nibble e bits 0-1 / 2-3     = code(4u+2i, e) / code(4u+2i+1, e)
 *     b'=3: Hi nibble e bits 0-2 (i<3)     = code(4u+i, e);  bit 3 = bit i of code(4u+3, e)
 *     signs: H nibble e bit i              = [ (S r)_{q m/4 + 4(4u+i) + e} >= 0 ]
 *   norms: two fp16 per key, (||k||, ||r||), round to nearest even.
 *   Rows of a cache are ordered [B][Hkv][S]; row bytes = dp b'/8 + mp/8.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tq_ctx tq_ctx;

typedef enum {
  TQ_OK = 0,
  TQ_ERR_ARG = 1,
  TQ_ERR_UNSUPPORTED = 2,
  TQ_ERR_CUDA = 3,
  TQ_ERR_NOMEM = 4,
  TQ_ERR_WORKSPACE = 5,
  TQ_ERR_DEVICE = 6,
  TQ_ERR_RANGE = 7
} tq_status;

typedef enum { TQ_F32 = 0, TQ_BF16 = 1 } tq_dtype;

/* Build the data-oblivious parameters of one quantizer and upload them to
 * the current CUDA device ([p2] stage 1: a rotation from the QR factor of a
 * Gaussian matrix and a precomputed Lloyd-Max codebook; [p2] stage 2: a
 * Gaussian JL matrix).  R (d x d) is the orthogonal factor, with a positive triangular
 * diagonal, of a d x d Gaussian drawn from Philox4x32-10 stream 0 of `seed`;
 * P (m x d) is drawn from stream 1 and the JL matrix applied to the residual
 * is S = P R; the codebook has 2^(bits-1) Lloyd-Max levels for the law of one
 * coordinate of a random unit vector in R^d.  m = d.
 * d: multiple of 8, 64 <= d <= 256.  bits: 2..4 (1..3 Lloyd-Max bits + 1 QJL bit).
 * *out receives a library-owned context; release it with tq_free.
 * Errors: TQ_ERR_ARG (out == NULL), TQ_ERR_UNSUPPORTED (d, bits), TQ_ERR_CUDA. */
tq_status tq_init(int d, int bits, uint64_t seed, tq_ctx** out);

/* As tq_init with an explicit JL row count m (multiple of 8, 64 <= m <= 256) and the
 * first Philox stream used (G from stream_base, P from stream_base + 1).
 * m = 0 selects the MSE-only variant ([p2] stage 1 alone): the same rotation
 * and codebook, no sign sketch (rows hold only the b' = bits - 1 code bits),
 * and the estimator is its first term n16 sum_j c[idx_j] (Rq)_j.
 * Errors: as tq_init; TQ_ERR_UNSUPPORTED also for m outside {0} u [64, 256]
 * or not a multiple of 8. */
tq_status tq_init_ex(int d, int bits, int m, uint64_t seed, uint32_t stream_base, tq_ctx** out);

/* Host only, no GPU needed: the fp64 tables tq_init_ex builds for these
 * arguments (R d*d, P m*d, c 2^(bits-1), t 2^(bits-1)-1; host pointers, any
 * may be NULL).  Errors: TQ_ERR_UNSUPPORTED for the shapes tq_init_ex
 * refuses. */
tq_status tq_host_tables(int d, int bits, int m, uint64_t seed, uint32_t stream_base, double* R, double* P,
                         double* c, double* t);

/* Release a context (NULL is ignored).  Must not race with calls using it. */
void tq_free(tq_ctx* ctx);

/* Sizes: d, bits, m and the packed payload bytes per key (host out-params,
 * any may be NULL).  Errors: TQ_ERR_ARG (ctx == NULL). */
tq_status tq_info(const tq_ctx* ctx, int* d, int* bits, int* m, int* row_bytes);

/* Copy the fp64 master tables to host memory for inspection: R (d*d,
 * row-major), P (m*d), codebook levels c (2^(bits-1)) and boundaries t
 * (2^(bits-1) - 1), ascending, on the unit-sphere scale.  Host pointers;
 * any may be NULL.  Errors: TQ_ERR_ARG (ctx == NULL). */
tq_status tq_export_tables(const tq_ctx* ctx, double* R, double* P, double* c, double* t);

/* Quantise n keys ([p2] stages 1 and 2): per key k (row i of `keys`, leading
 * dimension ld elements) compute n = ||k||, u = R k / n, the Lloyd-Max cell
 * index of every u_j, the residual r = k - n R^T c[idx], the sign bits
 * [(S r)_i >= 0] and fp16(n), fp16(||r||), and write them in the packed
 * layout.  keys: device, dtype TQ_F32 or TQ_BF16, 16-byte aligned, ld >= d and
 * ld a multiple of 8.  payload: device, n * row_bytes bytes.  norms: device,
 * n * 2 fp16 values.  A zero key gets codes 0, all sign bits 1, norms 0.
 * A key whose norm rounds past the fp16 range (||k|| >= 65520, or a key with
 * non-finite entries) is stored with an infinite (or NaN) norm, and the
 * kernel sets the range bit of the context's status word:
 * tq_check_device_status then returns TQ_ERR_RANGE.  Such a row must not be
 * scored (its logits are inf or NaN).
 * n == 0 is a no-op.
 * Errors: TQ_ERR_ARG (ctx NULL; n < 0; a NULL buffer; dtype; ld < d or not a
 * multiple of 8; keys or payload not 16-byte aligned, norms not 4-byte
 * aligned); TQ_ERR_CUDA. */
tq_status tq_quantize(const tq_ctx* ctx, const void* keys, tq_dtype dtype, int64_t n, int64_t ld,
                      uint8_t* payload, uint16_t* norms, void* stream);

/* Reconstruct n keys from the packed layout ([p2] stage 1: look up the
 * codebook and rotate back): out[i] = n16 R^T c[idx] when full == 0, plus the
 * QJL term sqrt(pi/2)/m rho16 S^T sigma when full != 0 (then <q, out[i]>
 * equals the inner-product estimate).  out: device fp32, n * d.
 * Errors: TQ_ERR_ARG (ctx NULL; n < 0; a NULL buffer; payload or norms not
 * 2-byte aligned, out not 4-byte aligned); TQ_ERR_CUDA. */
tq_status tq_dequantize(const tq_ctx* ctx, const uint8_t* payload, const uint16_t* norms, int64_t n,
                        int full, float* out, void* stream);

/* Workspace bytes tq_logits needs for B*Hq query heads (prepared queries);
 * 0 for invalid arguments (ctx NULL, a size <= 0, Hq not a multiple of Hkv). */
size_t tq_logits_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv);

/* Decode attention logits against a packed KV cache ([p2] stage 2
 * estimator; [p1] 2.2 memory-bound logits):
 *   out[b, h, s] = scale * ( n16 sum_j c[idx_j] (R q)_j
 *                            + sqrt(pi/2)/m rho16 sum_i sigma_i (S q)_i )
 * for q = q[b, h], key row (b, h / (Hq/Hkv), s).
 * q: device fp32 [B, Hq, d].  payload/norms: device, rows [B, Hkv, S].
 * out: device fp32 [B, Hq, S].  Hq must be a multiple of Hkv.
 * workspace: device, >= tq_logits_workspace_bytes, 256-byte aligned.
 * B = 0 or Hq = 0 is a no-op.
 * Errors: TQ_ERR_ARG (ctx NULL; a negative size; Hkv = 0 or Hq not a
 * multiple of Hkv; a NULL buffer; payload not 16-byte aligned, norms, q or
 * out not 4-byte aligned; workspace NULL or misaligned); TQ_ERR_WORKSPACE
 * (workspace_bytes too small); TQ_ERR_CUDA. */
tq_status tq_logits(const tq_ctx* ctx, const float* q, int B, int Hq, int Hkv, int64_t S,
                    const uint8_t* payload, const uint16_t* norms, float scale, float* out,
                    void* workspace, size_t workspace_bytes, void* stream);

/* Size of the library-owned scratch array used by tq_logits_noalloc. */
#define TQ_NOALLOC_SCRATCH_BYTES (1u << 20)

/* tq_logits without a caller workspace and without any allocation.  The
 * pages have no counterpart to this call: it exists for callers that cannot
 * allocate device memory where they compute logits, for instance an engine
 * that has handed its whole device-memory budget to its own pool, or a
 * latency-critical decode loop in which a cudaMalloc (which may synchronise
 * the device) is not acceptable.  It computes exactly what tq_logits
 * computes, with the same arguments minus the workspace.
 * Scratch: one static device array of TQ_NOALLOC_SCRATCH_BYTES bytes in
 * libtq, present on every GPU that loads the library until the process
 * exits.  The call allocates nothing and frees nothing.  The first call on a
 * device looks up the array's device address (once per device, with that
 * device current), so make that first call before any stream capture.
 * Every call shares the array and it keeps the last call's contents; nothing
 * in it has to start at zero (each call rewrites all it reads).  Calls whose
 * kernels overlap on the GPU (for example on two streams) race on the array:
 * order them.
 * The looked-up address belongs to the device's context at that time: after
 * a cudaDeviceReset of the device, do not call this entry point on it again.
 * Errors: as tq_logits; TQ_ERR_ARG also when the current device is not ctx's
 * device; TQ_ERR_WORKSPACE when tq_logits_workspace_bytes for (B, Hq, Hkv)
 * exceeds TQ_NOALLOC_SCRATCH_BYTES (about 500 (batch, KV head) groups of up
 * to 4 query heads each). */
tq_status tq_logits_noalloc(const tq_ctx* ctx, const float* q, int B, int Hq, int Hkv, int64_t S,
                            const uint8_t* payload, const uint16_t* norms, float scale, float* out,
                            void* stream);

/* Workspace bytes of tq_attend (per-chunk partial sums); 0 for invalid
 * arguments. */
size_t tq_attend_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int64_t S);

/* Decode attention output over a quantised value cache (the value path;
 * mooersco.com sections 1.2-1.3: the softmax of the logits weights the
 * values, and the output is recovered from the compressed values).  The
 * values are rows of ctx's packed layout ([B][Hkv][S], quantised with
 * tq_quantize under their own context); each enters through its unbiased
 * reconstruction v_hat = n16 R^T c[idx] + sqrt(pi/2)/m rho16 S^T sigma (the
 * first term only when ctx->m = 0):
 *   out[b, h] = sum_s softmax(logits[b, h, :])_s v_hat[b, h / (Hq/Hkv), s].
 * logits: device fp32 [B, Hq, S], already scaled (for instance tq_logits'
 * output).  out: device fp32 [B, Hq, d].  S = 0 gives zeros.
 * Hq / Hkv <= 8 (TQ_ERR_UNSUPPORTED otherwise).
 * workspace: device, 256-byte aligned, >= tq_attend_workspace_bytes.
 * B = 0 or Hq = 0 is a no-op.
 * Errors: TQ_ERR_ARG (ctx NULL; a negative size; Hkv = 0 or Hq not a
 * multiple of Hkv; a NULL buffer; payload not 16-byte aligned, norms, logits
 * or out not 4-byte aligned; workspace NULL or misaligned);
 * TQ_ERR_UNSUPPORTED; TQ_ERR_WORKSPACE; TQ_ERR_CUDA. */
tq_status tq_attend(const tq_ctx* ctx, const float* logits, int B, int Hq, int Hkv, int64_t S,
                    const uint8_t* payload, const uint16_t* norms, float* out, void* workspace,
                    size_t workspace_bytes, void* stream);

/* Workspace bytes tq_topk needs for nq queries against n database rows; 0
 * for invalid arguments. */
size_t tq_topk_workspace_bytes(const tq_ctx* ctx, int64_t nq, int64_t n, int k);

/* Inner-product top-k over a packed database (vector search, [p2] "GloVe
 * recall@1@k, near-zero indexing time"): for every query the k rows with the
 * largest estimate (same estimator as tq_logits with scale 1), ordered by
 * score descending and id ascending on ties.  Candidates are selected with
 * the fast estimator and re-scored in fp64 before the final order.
 * q: device fp32 [nq, d]; ids: device int64 [nq, k]; scores: device fp32
 * [nq, k].  1 <= k <= 256, k <= n.
 * Errors: TQ_ERR_ARG (a null or misaligned pointer: payload 16 bytes, norms,
 * q and scores 4, ids 8, workspace 256; k out of range); TQ_ERR_WORKSPACE
 * when workspace_bytes < tq_topk_workspace_bytes; TQ_ERR_CUDA. */
tq_status tq_topk(const tq_ctx* ctx, const float* q, int64_t nq, const uint8_t* payload,
                  const uint16_t* norms, int64_t n, int k, int64_t* ids, float* scores,
                  void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Channel split: fractional bit rates such as 2.5 bits per channel
 * (the rom4ai.github.io note "TurboQuant: Online Vector Quantization with
 * Near-Optimal Distortion Rate" sizes the cache at 3.5 bits per channel;
 * mooersco.com section 2.1 lists a 2.5-bit setting; zhengruan.com reports a
 * small quality loss at 2.5 bits).
 * The pages do not say how a fractional rate is reached; this library's
 * reading: per KV head, the channels are split into a high-variance group and
 * a low-variance group (mooersco.com FAQ: unrotated channel variances differ
 * by orders of magnitude), each group is quantised as its own vector with its
 * own context (rotation, JL matrix, codebook, bit width), and the estimate of
 * <q, k> is the sum of the two groups' estimates, since
 * <q, k> = <q_hi, k_hi> + <q_lo, k_lo> for the same split of q and k.
 * 2.5 bits per channel at d = 128: 64 channels at bits = 3 plus 64 at 2.
 *
 * A split holds, per KV head h, a channel order perm[h][0 .. d-1] (d =
 * hi.d + lo.d): group coordinate p < hi.d of head h is key channel
 * perm[h][p] of the high group, coordinate hi.d + p is channel
 * perm[h][hi.d + p] of the low group.  It starts as the identity order.
 * Keys are [B][Hkv][S][d] rows (row-major, contiguous); each group is stored
 * in its own context's packed layout, rows in the same [B][Hkv][S] order.
 * ------------------------------------------------------------------------ */
typedef struct tq_split tq_split;

/* A split for Hkv KV heads between the contexts hi and lo (same device, the
 * current one; hi.d + lo.d <= 512).  The contexts must outlive the split.
 * Library-owned; release with tq_split_free.  The tensor-core quantizer
 * covers hi.d = lo.d = hi.m = lo.m = 64 with bf16 keys; other shapes run on
 * CUDA cores.  Synchronises the device (uploads the identity order).
 * Errors: TQ_ERR_ARG (out NULL; hi or lo NULL; Hkv < 1; contexts of
 * different devices or not of the current one); TQ_ERR_UNSUPPORTED
 * (hi.d + lo.d > 512); TQ_ERR_NOMEM, TQ_ERR_CUDA. */
tq_status tq_split_create(const tq_ctx* hi, const tq_ctx* lo, int Hkv, tq_split** out);
void tq_split_free(tq_split* sp);

/* Workspace bytes of tq_split_plan (fp64 partial sums); 0 when sp is NULL. */
size_t tq_split_plan_workspace_bytes(const tq_split* sp);

/* Choose the channel order from keys [B][Hkv][S][d] (fp32 or bf16, device):
 * per KV head, the hi.d channels of largest variance over the head's B S
 * keys, ties to the lower channel index, in ascending channel order, then
 * the other channels in ascending order.  With no keys (B S = 0) every
 * variance is 0 and the order is the identity.  Asynchronous on `stream`;
 * workspace: device, 8-byte aligned, >= tq_split_plan_workspace_bytes.
 * Errors: TQ_ERR_ARG (sp NULL; B or S negative; dtype; keys NULL with
 * B S > 0 or not aligned to its element; workspace NULL or misaligned);
 * TQ_ERR_WORKSPACE; TQ_ERR_CUDA. */
tq_status tq_split_plan(tq_split* sp, const void* keys, tq_dtype dtype, int B, int64_t S, void* workspace,
                        size_t workspace_bytes, void* stream);

/* Set (host perm, [Hkv][d], each row a permutation of 0..d-1, else
 * TQ_ERR_ARG) or read (host out-param) the channel order.  Both synchronise
 * the device. */
tq_status tq_split_set_plan(tq_split* sp, const int32_t* perm);
tq_status tq_split_get_plan(const tq_split* sp, int32_t* perm);

/* Quantise keys [B][Hkv][S][d] (device, fp32 or bf16, 16-byte aligned): the
 * high group of every row with hi into payload_hi / norms_hi (B Hkv S rows of
 * hi's layout), the low group with lo into payload_lo / norms_lo.  Each group
 * is quantised exactly as tq_quantize quantises a key of that group's
 * channels.  A group norm outside the fp16 range sets the range bit of hi's
 * status word (tq_check_device_status on hi).  B S = 0 is a no-op.
 * Errors: TQ_ERR_ARG (sp NULL; B or S negative; dtype; a NULL buffer; keys
 * or payloads not 16-byte aligned, norms not 4-byte aligned); TQ_ERR_CUDA. */
tq_status tq_split_quantize(const tq_split* sp, const void* keys, tq_dtype dtype, int B, int64_t S,
                            uint8_t* payload_hi, uint16_t* norms_hi, uint8_t* payload_lo, uint16_t* norms_lo,
                            void* stream);

/* Workspace bytes of tq_split_logits; 0 for invalid arguments. */
size_t tq_split_logits_workspace_bytes(const tq_split* sp, int B, int Hq);

/* Decode logits against a split cache: out[b, h, s] = scale (estimate of the
 * high group + estimate of the low group), each group's estimate as in
 * tq_logits with the query's channels gathered by the split of its KV head
 * h / (Hq / Hkv).  q: device fp32 [B, Hq, d]; out: device fp32 [B, Hq, S];
 * workspace: device, 256-byte aligned.  B = 0 or Hq = 0 is a no-op.
 * Errors: as tq_logits (the split's Hkv in place of the argument). */
tq_status tq_split_logits(const tq_split* sp, const float* q, int B, int Hq, int64_t S, const uint8_t* payload_hi,
                          const uint16_t* norms_hi, const uint8_t* payload_lo, const uint16_t* norms_lo,
                          float scale, float* out, void* workspace, size_t workspace_bytes, void* stream);

/* Merge of per-shard top-k lists (a database split by rows over several
 * devices or calls, each shard searched with tq_topk; airosetta.com "Google
 * TurboQuant" on vector search): scores and ids are device arrays
 * [parts][nq][k] as tq_topk returns them (ids local to their shard);
 * first_rows (host, parts entries) gives each shard's first global row.  Per
 * query, out_ids / out_scores (device [nq][k]) receive the k best candidates
 * by score descending and global id ascending, ids made global.  Each shard
 * must hold at least k rows.  1 <= parts <= 64, parts * k <= 4096
 * (TQ_ERR_UNSUPPORTED above).  Candidates are ordered by their fp32 scores:
 * two rows whose exact scores round to one fp32 value are ordered by id, which
 * can differ from a single tq_topk call over the whole database only at such
 * near-ties.  Needs no context. */
tq_status tq_topk_merge(const float* scores, const int64_t* ids, const int64_t* first_rows, int parts, int64_t nq,
                        int k, int64_t* out_ids, float* out_scores, void* stream);

/* Status word bits (tq_check_device_status). */
#define TQ_STATUS_QUANTIZE_WAIT 0x1u   /* the tensor-core quantizer gave up a bounded wait */
#define TQ_STATUS_SEARCH_WAIT 0x2u     /* the tensor-core search gave up a bounded wait */
#define TQ_STATUS_RANGE 0x4u           /* a quantised key's norm was not finite in fp16 */

/* Read (and clear) the context's device status word after synchronising the
 * stream: 0 when every kernel finished its bounded waits and every stored
 * norm was finite; otherwise the TQ_STATUS_* bits of what happened since the
 * last check.  Returns TQ_ERR_DEVICE when a wait bit is set, else
 * TQ_ERR_RANGE when the range bit is set, else TQ_OK (word: host, may be
 * NULL).  Errors: TQ_ERR_ARG (ctx NULL), TQ_ERR_CUDA. */
tq_status tq_check_device_status(const tq_ctx* ctx, void* stream, uint32_t* word);

/* Test hook for the failure path of the bounded waits: the number of SM
 * clock cycles each bounded wait of the tensor-core quantizer (tq_quantize
 * on d = 128) spins before it gives up; 0 restores the default (about 2 s).
 * A wait that gives up makes every role of the kernel leave its loop (the
 * copies and MMAs already issued are drained with the default budget before
 * the block exits), the rows of that call are left incomplete, and the
 * context's status word gets TQ_STATUS_QUANTIZE_WAIT, so that
 * tq_check_device_status returns TQ_ERR_DEVICE; the context stays usable.
 * With a budget of a few cycles the first wait that is not satisfied at once
 * gives up.  Not for production use; must not race with calls on ctx.
 * Errors: TQ_ERR_ARG (ctx NULL, cycles < 0). */
tq_status tq_set_wait_budget(tq_ctx* ctx, int64_t cycles);

const char* tq_strerror(tq_status s);
const char* tq_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* TQ_H_ */
