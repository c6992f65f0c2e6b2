/*
 * tq.h - C ABI of the TurboQuant compressed-KV library for NVIDIA B200 (sm_100a).
 *
 * The library compresses transformer key/value cache vectors in two stages and
 * runs decode attention directly on the packed cache:
 *
 *   keys   : n = ||k||, u = k/n, y = Pi u (random orthogonal rotation),
 *            idx = Lloyd-Max cell of each y_j, r = y - c[idx], gamma = ||r||,
 *            1-bit QJL signs s = [S r >= 0], packed codes + signs + fp16 (n, gamma)
 *   values : groups of 32 coordinates, min/max uniform codes at 2, 3 or 4 bits,
 *            fp16 (scale, min) per group
 *   decode : qr = Pi q, sq = S qr; logit_t = scale * n_t * (<qr, c[idx_t]>
 *            + sqrt(pi/2)/m * gamma_t * <sq, s_t>); online softmax over the cache;
 *            output = sum_t p_t * (min + scale * code_t) / sum_t p_t
 *
 * Sources (web pages about TurboQuant):
 *   - "turboquant-pytorch" skill card, section "Что делает": rotation +
 *     Lloyd-Max + one-bit QJL residual correction; attention scores computed
 *     straight from the compressed keys (TurboQuantProd).
 *   - discosf.com TurboQuant news item, section "一句话看懂": the four steps
 *     (rotation, Lloyd-Max with pre-generated codebooks, QJL sign bits, value
 *     group quantization with four 2-bit values per byte); decode runs in fused
 *     kernels on the compressed cache.
 *   - tproger.ru "TurboQuant неделю спустя", section "Реализации TurboQuant":
 *     the dense O(d^2) rotation is slow; a Walsh-Hadamard transform is O(d log d).
 *
 * Conventions for every call:
 *   - All device buffers belong to the caller. The library allocates device
 *     memory only inside tq_codebook_load (its own tables, freed by tq_free).
 *   - Device pointers must be 16-byte aligned, else TQ_EINVAL.
 *   - Calls are asynchronous on the given CUDA stream (a cudaStream_t passed as
 *     void*, NULL = legacy default stream). Only tq_codebook_load synchronizes.
 *   - Unsupported sizes or bit widths return TQ_EUNSUPPORTED; CUDA launch or
 *     runtime errors return TQ_ECUDA (tq_last_error() has the CUDA message).
 *   - No function throws; no function calls exit() or abort().
 *
 * Packed formats (little-endian, one record per vector, records contiguous):
 *   k_codes  [n_vec][lm_bits*d/8] u8  code j in bits [lm_bits*j, lm_bits*j+lm_bits)
 *                                     of the record, least significant bit first
 *   k_signs  [n_vec][m/8]         u8  sign bit i = bit i%8 of byte i/8, 1 <=> (S r)_i >= 0
 *   k_norms  [n_vec][2]           u16 fp16 bit patterns (n, gamma), round-to-nearest-even
 *   v_codes  [n_vec][v_bits*d/8]  u8  same stream layout as k_codes
 *   v_params [n_vec][d/32][2]     u16 fp16 (scale, min) per group of 32 coordinates
 * A zero key is stored as all-zero bytes.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_EINVAL = 1,        /* bad pointer, alignment, size or argument combination */
  TQ_EUNSUPPORTED = 2,  /* d, bit width, m or group size outside what is built */
  TQ_ECUDA = 3,         /* a CUDA runtime call or kernel launch failed */
  TQ_ENOMEM = 4         /* device or host allocation failed (tq_codebook_load only) */
} tq_status;

typedef enum { TQ_F32 = 0, TQ_BF16 = 1 } tq_dtype;

typedef enum {
  TQ_ROT_HADAMARD = 0,  /* Pi = H_d diag(sigma) / sqrt(d), applied as sign flip + FWHT */
  TQ_ROT_HAAR = 1       /* Pi = dense Haar orthogonal matrix (d x d) */
} tq_rot;

/* Method parameters. Every array is HOST memory and is copied by
 * tq_codebook_load; the caller may free it afterwards.
 *   d              head dimension: 64, 128 or 256
 *   k_lm_bits      Lloyd-Max bits per key coordinate: 1 to 7 (a key then costs
 *                  k_lm_bits + 1 bits per coordinate with its QJL sign); a lane's
 *                  codes must fit one 32-bit word, k_lm_bits * d / 32 <= 32 (so at
 *                  most 4 bits at d = 256); 4 bits and more run on the CUDA-core kernels
 *   qjl_m          rows of the QJL matrix S: a multiple of 32, at most 256; or 0 for
 *                  keys without the QJL stage (Lloyd-Max codes only, the MSE-optimal
 *                  first stage): no sign bytes (k_signs may be NULL), gamma is still
 *                  stored, and scores and decompressed keys use the codes alone
 *   v_bits         value bits: 2, 3 or 4 (3-bit codes straddle 32-bit words and run on
 *                  the CUDA-core value kernels; keys still take the tensor-core ones)
 *   v_group        value group size: 32
 *   rot            rotation kind
 *   centroids      2^k_lm_bits ascending fp32 centroids of the Lloyd-Max codebook
 *   boundaries     2^k_lm_bits - 1 ascending fp32 cell boundaries; coordinate y
 *                  gets code #{k : y >= boundaries[k]}
 *   hadamard_signs d entries, each +1 or -1 (TQ_ROT_HADAMARD; ignored otherwise)
 *   haar           d*d row-major orthogonal matrix Pi in fp64, y = Pi u (TQ_ROT_HAAR)
 *   qjl_S          m*d row-major fp32 matrix S (i.i.d. N(0,1) draws); NULL if m = 0 */
typedef struct {
  int d;
  int k_lm_bits;
  int qjl_m;
  int v_bits;
  int v_group;
  tq_rot rot;
  const float* centroids;
  const float* boundaries;
  const signed char* hadamard_signs;
  const double* haar;
  const float* qjl_S;
} tq_params;

typedef struct tq_ctx tq_ctx;

/* Load a codebook, rotation and QJL matrix onto the current CUDA device.
 * Pre-generated codebooks are part of the method (discosf news item,
 * "一句话看懂" step 2); tq_lloyd_max_codebook below produces them.
 * Validates the parameters (TQ_EINVAL / TQ_EUNSUPPORTED), allocates the
 * context's device tables (TQ_ENOMEM), uploads them on `stream` and
 * synchronizes that stream once. On success *out owns the tables until
 * tq_free. The context is bound to the device that was current here. */
tq_status tq_codebook_load(const tq_params* params, void* stream, tq_ctx** out);

/* Release a context and its device tables. NULL is a no-op. The caller must
 * make sure no work using the context is still running. */
void tq_free(tq_ctx* ctx);

/* Static, human-readable name of a status code. Never NULL. */
const char* tq_status_string(tq_status status);

/* Message of the last failing call on this thread ("" if none). */
const char* tq_last_error(void);

/* HOST ONLY (no GPU needed). Lloyd-Max codebook of one coordinate of a uniform
 * random unit vector in R^d (the law of every rotated coordinate), with 2^bits
 * levels: centroids at cell means, boundaries at centroid midpoints, iterated
 * in fp64 to convergence and rounded to fp32. The skill card ("turboquant-
 * pytorch", "Что делает") builds these codebooks with scipy; this is a
 * self-contained solver. Writes 2^bits centroids and 2^bits - 1 boundaries.
 * d in [4, 4096], bits in [1, 7]; else TQ_EINVAL. */
tq_status tq_lloyd_max_codebook(int d, int bits, float* centroids, float* boundaries);

/* HOST ONLY. Haar-distributed orthogonal matrix from a d x d row-major matrix
 * of i.i.d. N(0,1) draws: Q of its QR factorisation with R's diagonal made
 * positive (Householder, fp64). Writes d*d row-major doubles to pi_out.
 * d in [1, 1024]; TQ_EINVAL on NULL pointers or a rank-deficient input. */
tq_status tq_haar_from_gaussian(int d, const double* gaussian, double* pi_out);

/* Compress n_vec keys and/or values (prefill / append path).
 *   k, v      device [n_vec][d] of `dtype` (fp32 or bf16); either may be NULL to
 *             skip that half (its output pointers are then ignored)
 *   k_codes, k_signs, k_norms, v_codes, v_params: device outputs, formats above
 * Each output record is written in full. n_vec = 0 returns TQ_OK before any
 * pointer is examined (NULL buffers are fine then).
 * Keys follow TurboQuantProd (skill card, "Что делает"; discosf steps 1-3),
 * values the group quantizer (discosf step 4). */
tq_status tq_compress_kv(const tq_ctx* ctx, const void* k, const void* v, tq_dtype dtype,
                         int64_t n_vec, uint8_t* k_codes, uint8_t* k_signs, uint16_t* k_norms,
                         uint8_t* v_codes, uint16_t* v_params, void* stream);

/* tq_compress_kv with a slot map: vector i's records go to row slot[i] of the output
 * arrays instead of row i. This appends new tokens to a growing cache in place (slots
 * after each sequence's last token) and fills paged layouts (slots inside pages). The
 * arrays hold n_rows records; rows not named by the map are not touched.
 *   slot    device int64 [n_vec], 8-byte aligned; distinct entries in [0, n_rows).
 *           An entry outside that range is not written and sets the context's device
 *           error word (tq_check_device then returns TQ_EINVAL).
 * Other arguments, ownership and errors as tq_compress_kv; NULL slot is TQ_EINVAL. */
tq_status tq_compress_kv_slots(const tq_ctx* ctx, const void* k, const void* v, tq_dtype dtype,
                               int64_t n_vec, const int64_t* slot, int64_t n_rows, uint8_t* k_codes,
                               uint8_t* k_signs, uint16_t* k_norms, uint8_t* v_codes,
                               uint16_t* v_params, void* stream);

/* Bytes of device workspace tq_decode_attention needs for this shape (split-K
 * partials and prepared queries). Returns 0 for invalid arguments. */
size_t tq_decode_workspace_bytes(const tq_ctx* ctx, int batch, int hq, int hkv, int64_t max_len);

/* One decode step of attention over a packed cache (skill card, "Что делает":
 * scores straight from the compressed keys without dequantizing them; discosf
 * "一句话看懂": fused decode kernels on the compressed cache).
 *   q         device [batch][hq][d], fp32 or bf16 (q_dtype)
 *   seq_lens  device int32 [batch] valid cache lengths (<= max_len), or NULL for
 *             max_len everywhere; a length of 0 yields a zero output row
 *   max_len   tokens per (sequence, KV head) slot in the packed arrays
 *   packed    k_codes ... v_params laid out [batch][hkv][max_len][record]
 *   hq        a multiple of hkv; query head h reads KV head h / (hq / hkv)
 *   softmax_scale  logit scale; 0 selects 1/sqrt(d)
 *   scores    NULL, or device fp32 [batch][hq][max_len] receiving the scaled
 *             logits of valid positions (others untouched)
 *   out       device fp32 [batch][hq][d]
 *   workspace device scratch of at least tq_decode_workspace_bytes(...) bytes
 * At d = 128 with 1- to 3-bit Lloyd-Max codes of a codebook symmetric about zero,
 * 2- to 4-bit values and at most 8 query heads per KV head, a tensor-core decode runs
 * (tq_set_decode_kernel); it carries p * scale (p < 4) as f16 operands, so value-group
 * scales must stay below 16376 (values spanning less than 49000 at 2 bits). Other
 * shapes run the CUDA-core decode. With seq_lens, the mma.sync decode (the default for
 * codes with the QJL stage) spreads only the tokens present over the SMs, reading the
 * lengths on the device, so a batch of varied lengths costs the tokens it holds; the
 * workspace is sized for max_len either way.
 * Returns TQ_EINVAL if the workspace is too small or any pointer is misaligned. */
tq_status tq_decode_attention(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int batch, int hq,
                              int hkv, const int32_t* seq_lens, int64_t max_len,
                              const uint8_t* k_codes, const uint8_t* k_signs,
                              const uint16_t* k_norms, const uint8_t* v_codes,
                              const uint16_t* v_params, float softmax_scale, float* scores,
                              float* out, void* workspace, size_t workspace_bytes, void* stream);

/* tq_decode_attention over a paged cache: the packed arrays hold n_pages pages of
 * page_size consecutive records, each page belonging to one (sequence, KV head), in
 * any order (filled e.g. by tq_compress_kv_slots).
 *   block_table  device int32 [batch][hkv][max_pages], 16-byte aligned: the page that
 *                holds tokens [j page_size, (j+1) page_size) of (sequence b, KV head h)
 *                is block_table[(b hkv + h) max_pages + j]; only entries of blocks below
 *                the sequence's length are read. An entry outside [0, n_pages) sets the
 *                device error word (tq_check_device returns TQ_EINVAL) and reads page 0.
 *   page_size    tokens per page, a positive multiple of 512 (a whole number of every
 *                decode kernel's tiles)
 *   max_pages    block-table entries per (sequence, KV head), >= ceil(max_len / page_size)
 * max_len bounds seq_lens and sizes the scores rows; the workspace is the one
 * tq_decode_workspace_bytes gives for the same shape. Other arguments and errors as
 * tq_decode_attention. */
tq_status tq_decode_attention_paged(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int batch,
                                    int hq, int hkv, const int32_t* seq_lens, int64_t max_len,
                                    const int32_t* block_table, int64_t page_size,
                                    int64_t max_pages, int64_t n_pages, const uint8_t* k_codes,
                                    const uint8_t* k_signs, const uint16_t* k_norms,
                                    const uint8_t* v_codes, const uint16_t* v_params,
                                    float softmax_scale, float* scores, float* out,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* tq_decode_attention that also returns each row's log-partition, for a sequence
 * whose tokens are split over several GPUs (or several caches): every part decodes
 * its own token range and the parts are combined by tq_merge_attention. The pages
 * describe decode over one cache (skill card, "Что делает"); the split is an exact
 * identity of that softmax over the union of disjoint ranges (output = sum_r
 * e^{lse_r} out_r / sum_r e^{lse_r}), the log-sum-exp merge the split-K decode
 * already applies to its chunks.
 *   out  device fp32 [batch][hq][d]: attention over this cache's valid tokens only
 *   lse  device fp32 [batch][hq], float-aligned: log sum_t exp(scaled logit_t) over
 *        the same tokens (natural log); -inf where the length is 0 (out row zero)
 * Other arguments, layouts and errors as tq_decode_attention; lse must not be NULL. */
tq_status tq_decode_attention_partial(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int batch,
                                      int hq, int hkv, const int32_t* seq_lens, int64_t max_len,
                                      const uint8_t* k_codes, const uint8_t* k_signs,
                                      const uint16_t* k_norms, const uint8_t* v_codes,
                                      const uint16_t* v_params, float softmax_scale, float* scores,
                                      float* out, float* lse, void* workspace, size_t workspace_bytes,
                                      void* stream);

/* Combine n_parts attention results over disjoint token ranges of the same rows
 * (e.g. one tq_decode_attention_partial per GPU, gathered into one buffer) into
 * the attention over all their tokens.
 *   outs   device fp32: part r's outputs [rows][d] start at outs + r * outs_stride
 *   lses   device fp32: part r's log-partitions [rows] start at lses + r * lses_stride
 *          (-inf marks an empty range, which gets weight 0)
 *   out    device fp32 [rows][d]: sum_r w_r out_r / sum_r w_r with w_r = exp(lse_r - max lse);
 *          a row whose parts are all empty gets zeros
 *   lse    NULL, or device fp32 [rows]: the merged log-partition (for merging again)
 * Strides are in floats and must be at least rows * d and rows; all pointers float-
 * aligned; out and lse must not overlap the inputs. Returns TQ_EINVAL for bad sizes
 * or pointers, TQ_ECUDA if the launch fails; rows = 0 is a no-op. */
tq_status tq_merge_attention(const float* outs, int64_t outs_stride, const float* lses,
                             int64_t lses_stride, int n_parts, int64_t rows, int d, float* out,
                             float* lse, void* stream);

/* Synchronize `stream`, then read and clear the context's device error word.
 * Kernels never spin without a bound: a wait for a staged copy that does not
 * complete in time sets this word, abandons the rest of its work and exits, so
 * the CUDA context stays usable. Returns TQ_ECUDA (with tq_last_error() saying
 * which wait) if any call since the last check hit such a timeout, TQ_EINVAL if a
 * slot or page index was out of range, TQ_OK otherwise. */
tq_status tq_check_device(const tq_ctx* ctx, void* stream);

/* Decode attention that allocates nothing and takes no workspace. The pages describe
 * no such call; this entry point exists for callers that cannot allocate device
 * memory: a plugin that is handed only input and output pointers by its host
 * application, a serving loop that must not call cudaMalloc once running (the
 * allocation can synchronize the device and stall other streams), or a runtime
 * without a caching allocator.
 * Same arguments, layouts and results as tq_decode_attention, minus workspace.
 * The scratch is a fixed device array of tq_decode_static_scratch_capacity()
 * bytes (32 MiB) inside this library; every GPU that loads the library holds one
 * until the process exits. A shape whose workspace (tq_decode_workspace_bytes)
 * exceeds it returns TQ_EUNSUPPORTED with the sizes in tq_last_error().
 * Every call looks up the array's device address in the current CUDA context
 * (cudaGetSymbolAddress, with the context's device current; nothing is cached, so
 * a context created after a device reset, or one the caller made current itself,
 * is served its own copy). The first call in a context loads the library's device
 * code there: make that first call before any stream capture. All calls on a device share the one array and it keeps
 * the last call's contents: every byte a call reads is written earlier in the
 * same call, but calls whose work overlaps on the GPU (different streams, or
 * host threads without ordering) race on it and must be serialized.
 * The context must belong to the current device. */
tq_status tq_decode_attention_static(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int batch,
                                     int hq, int hkv, const int32_t* seq_lens, int64_t max_len,
                                     const uint8_t* k_codes, const uint8_t* k_signs,
                                     const uint16_t* k_norms, const uint8_t* v_codes,
                                     const uint16_t* v_params, float softmax_scale, float* scores,
                                     float* out, void* stream);

/* Bytes of the fixed scratch array tq_decode_attention_static uses (no GPU needed). */
size_t tq_decode_static_scratch_capacity(void);

/* Instrumentation: when `start` and `stop` (cudaEvent_t passed as void*) are
 * non-NULL, every later call on this context records `start` on its stream
 * right before its main kernel (the compression kernel of tq_compress_kv, the
 * split-K attention kernel of tq_decode_attention) and `stop` right after it,
 * so a caller can time that kernel alone with cudaEventElapsedTime. NULL for
 * both disables it. Not thread-safe with concurrent calls on the same context. */
tq_status tq_set_profile_events(tq_ctx* ctx, void* start, void* stop);

/* Which decode attention kernel family a context uses. Every family computes the
 * same results within the decode tolerance; they differ in speed and coverage.
 *   TQ_DECODE_AUTO      the fastest family that supports the shape (default)
 *   TQ_DECODE_TCGEN05   key scores on the 5th-generation tensor cores (tcgen05, digit
 *                       sums in tensor memory), value sums on warp-level MMAs: d = 128,
 *                       m = 128 or 0, 1- to 3-bit codes of a symmetric codebook, 2- or
 *                       4-bit values, at most 8 query heads per KV head
 *   TQ_DECODE_MMA       warp-level tensor-core MMAs (mma.sync) over the packed bits:
 *                       d = m = 128, 1- to 3-bit codes of a symmetric codebook, 2- or
 *                       4-bit values, at most 8 query heads per KV head
 *   TQ_DECODE_CUDA_CORE the generic kernels: every shape the library accepts */
typedef enum {
  TQ_DECODE_AUTO = 0,
  TQ_DECODE_TCGEN05 = 1,
  TQ_DECODE_MMA = 2,
  TQ_DECODE_CUDA_CORE = 3
} tq_decode_kernel;

/* Select the decode kernel family for later decode calls on this context (all of
 * tq_decode_attention, _paged, _partial and _static). A family that does not support
 * a call's shape makes that call return TQ_EUNSUPPORTED; TQ_DECODE_AUTO never does.
 * The workspace size (tq_decode_workspace_bytes) depends on the family: query it
 * after selecting. Not thread-safe with concurrent calls on the same context. */
tq_status tq_set_decode_kernel(tq_ctx* ctx, tq_decode_kernel kernel);

/* The family a decode call with these head counts would run on this context, or -1
 * if the selected family does not support the shape (no GPU work). */
int tq_decode_kernel_for(const tq_ctx* ctx, int hq, int hkv);

/* Decompress n_vec packed keys and/or values to fp32 [n_vec][d] (debug / parity;
 * not on the hot path). Keys: x = n Pi^T (c[idx] + sqrt(pi/2)/m * gamma * S^T s).
 * Values: min + scale * code. Pass NULL for the half to skip. */
tq_status tq_decompress(const tq_ctx* ctx, const uint8_t* k_codes, const uint8_t* k_signs,
                        const uint16_t* k_norms, const uint8_t* v_codes, const uint16_t* v_params,
                        int64_t n_vec, float* k_out, float* v_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
