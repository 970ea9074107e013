/*
 * tq.h -- C ABI of libtq.so: data-oblivious vector quantization of KV-cache and
 * embedding vectors (TurboQuant / PolarQuant / QJL style) on NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page title and section:
 *  [TQ6x]  "Google TurboQuant: 6x KV-cache compression" (ebisuda.net),
 *          sections "Stage 1: PolarQuant (MSE-optimal compression)" and
 *          "Stage 2: QJL residual correction (1 bit)".
 *  [DEEP]  "TurboQuant / PolarQuant / QJL technical deep dive" (gemilab.net),
 *          sections "KV cache basics", "PolarQuant: Cartesian to polar", "QJL",
 *          "GPU kernel optimisation".
 *  [HAKU]  "TurboQuant: redefining AI efficiency with extreme compression"
 *          (hakusoku.com), sections "PolarQuant", "QJL: zero-overhead 1-bit
 *          compression", "Impact on high-dimensional vector search".
 *  [POLAR] "PolarQuant explainer" (aibr.jp), sections 1 and 3 (the recursive
 *          polar transform and its angle codebooks).
 *  [FRAC]  "Fractal KV-cache archive" (gist.science), section "Problem
 *          statement" (amortised O(1) append to a growing cache).
 *
 * Conventions for every entry point:
 *  - Return value: TQ_OK (0) or a TQ_E* status; nothing is thrown across the ABI.
 *    On error, tq_last_error() returns a message for the calling host thread.
 *  - "device" pointers are CUDA device (or managed) memory owned by the caller;
 *    "host" pointers are ordinary host memory owned by the caller. The library
 *    never frees caller memory and allocates nothing in hot calls (encode,
 *    append, score, attention, search); scratch is the caller's `workspace`.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Device work is
 *    enqueued asynchronously; no hot call synchronises. Errors the GPU detects
 *    (cache overflow, bounded-wait timeouts) are OR-ed into a per-handle
 *    device error word that tq_last_status() reads.
 *  - Sizes: d % 32 == 0, 32 <= d <= 4096; MSE bits in 1..4 (0 for QJL-only
 *    rows); QJL m % 32 == 0.
 *
 * Packed layout (one row per vector, caller-allocated, rows contiguous):
 *  - codes: ceil(d * b / 8) bytes, b = MSE bits. LSB-first contiguous: bit t of
 *    index j is bit (j*b + t) of the row read as a little-endian bitstream.
 *    Index j is the Lloyd-Max cell of rotated coordinate j, ascending order.
 *  - signs (prod handles): m / 8 bytes, bit j = 1 iff projection j of the
 *    residual is >= 0.
 *  - norms: one per row, fp32 or fp16 (tq_set_norm_dtype); rnorms: fp16.
 *  - QJL-only rows (tq_create_prod with bits = 1): no codes (codes_B = 0) and
 *    no rnorms; signs of the projections of the whole vector, and its norm.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---- */
#define TQ_OK 0
#define TQ_EINVAL 1          /* bad argument (null pointer, size, dtype, alignment) */
#define TQ_ENOMEM 2          /* allocation failed (tq_create* only)                 */
#define TQ_ECUDA 3           /* a CUDA runtime call failed (incl. no device)        */
#define TQ_ECAPACITY 4       /* tq_append: a sequence is full (len[b] == L_cap)     */
#define TQ_ETIMEOUT 5        /* a bounded device wait gave up                       */
#define TQ_EUNSUPPORTED 6    /* valid but unsupported shape (e.g. d % 32 != 0)      */

/* ---- element types ---- */
#define TQ_F32 0
#define TQ_F16 1
#define TQ_BF16 2

typedef struct tq_handle tq_handle; /* opaque; owns Pi, S, S Pi^T and the codebook on the device */

/* One quantized cache (K or V) of B sequences x Hkv heads x L_cap slots.
 * All pointers are device pointers, row-major in the order [B][Hkv][L_cap]
 * (then the packed row). codes/signs rows must start on 16-byte boundaries
 * (base pointers 16-byte aligned); norms/rnorms 4-byte aligned.
 * signs and rnorms are NULL for MSE-only handles; codes and rnorms may be NULL
 * for QJL-only handles (they are not read). */
typedef struct tq_cache {
  uint8_t* codes;   /* [B][Hkv][L_cap][codes_B]                  */
  uint8_t* signs;   /* [B][Hkv][L_cap][signs_B] or NULL           */
  void* norms;      /* [B][Hkv][L_cap], fp32 or fp16 (handle's)   */
  void* rnorms;     /* [B][Hkv][L_cap], fp16, or NULL             */
  int64_t L_cap;    /* slots per (sequence, head)                 */
} tq_cache;

/* ---------------------------------------------------------------------------
 * Host-only math (no GPU needed; used by tq_create and exported for tests).
 * ------------------------------------------------------------------------ */

/* Lloyd-Max codebook for one rotated coordinate of a unit vector in R^d:
 * continuous k-means on the density proportional to (1 - t^2)^((d-3)/2) on
 * [-1, 1] [TQ6x Stage 1]. Writes 2^bits ascending centroids and 2^bits - 1
 * boundaries (midpoints) to host arrays. 3 <= d <= 65536, 1 <= bits <= 8. */
int tq_codebook_host(int d, int bits, double* centroids, double* bounds);

/* Lloyd-Max codebook of the level-`level` angle of the recursive polar transform of
 * a uniform direction [POLAR sections 1, 3]: level 1 is uniform on (-pi, pi] (the
 * uniform grid); level l >= 2 has density proportional to
 * (sin psi cos psi)^(2^(l-1) - 1) on [0, pi/2]. 2^bits ascending centroids and
 * 2^bits - 1 midpoint boundaries (host arrays). 1 <= level <= 16, 1 <= bits <= 8. */
int tq_polar_codebook_host(int level, int bits, double* centroids, double* bounds);

/* Seeded rotation Pi (d x d, row-major, y = Pi u) = Q of a Householder QR of a
 * Gaussian matrix G with diag(R) > 0 [TQ6x Stage 1], and the QJL matrix S
 * (m x d, row-major; may be NULL when m == 0) [DEEP QJL]. G then S are filled
 * row-major from one SplitMix64 + Box-Muller stream started at `seed`.
 * Pi and S are host arrays of d*d and m*d doubles. */
int tq_rotation_host(int d, int m, uint64_t seed, double* Pi, double* S);

/* ---------------------------------------------------------------------------
 * Handles
 * ------------------------------------------------------------------------ */

/* MSE-only handle: b = bits per coordinate, norms stored as fp32 by default.
 * Builds the codebook and Pi on the host (fp64) and uploads device copies.
 * Needs the current CUDA device; *out is NULL on failure. */
int tq_create(int d, int bits, uint64_t seed, tq_handle** out);

/* Prod handle [TQ6x Stage 2]: `bits` total per coordinate = (bits - 1) MSE bits
 * + one QJL sign per projection, qjl_m projections (m % 32 == 0, m <= 1024).
 * Norms default to fp16; residual norms are always fp16. 1 <= bits <= 5; d <= 128.
 * bits = 1 makes QJL-only rows [HAKU "QJL: zero-overhead 1-bit compression"]:
 * no MSE stage, the signs of S x (sign(0) = +1) and ||x||, which weighs the
 * signs where a prod row uses its residual norm. */
int tq_create_prod(int d, int bits, int qjl_m, uint64_t seed, tq_handle** out);

/* Recursive polar transform handle [POLAR sections 1 and 3; HAKU "PolarQuant"]:
 * y = Pi x / ||x|| (Pi as tq_create's for `seed`), then log2(d) levels: level 1
 * pairs (y_2i, y_2i+1) into a radius and an angle atan2(y_2i+1, y_2i) in (-pi, pi],
 * each further level pairs the previous radii (angle in [0, pi/2]); every angle
 * is bucketized against its level's Lloyd-Max codebook (tq_polar_codebook_host),
 * bits_level1 bits at level 1 and bits_upper at every other level (each 1..4).
 * d a power of two, 32 <= d <= 256. Norms fp32 by default.
 * Row layout: the level fields one after the other, level 1 first, each index
 * LSB-first in its level's width; codes_B = 16 * ceil(total bits / 128), pad
 * bits 0. Works with tq_encode, tq_append and tq_score (s = ||x|| <Pi q, y_hat>,
 * y_hat the unit vector rebuilt from the centroids); other hot calls return
 * TQ_EUNSUPPORTED for polar handles. */
int tq_create_polar(int d, int bits_level1, int bits_upper, uint64_t seed, tq_handle** out);

/* Levels and widths of a polar handle (TQ_EINVAL for other handles). */
int tq_polar_info(const tq_handle* h, int* nlevels, int* bits_level1, int* bits_upper);

/* Host copies (fp64) of level `level`'s (1-based) centroids and boundaries. */
int tq_get_polar_codebook(const tq_handle* h, int level, double* centroids, double* bounds);

/* Storage type of the per-vector norm: TQ_F32 or TQ_F16. */
int tq_set_norm_dtype(tq_handle* h, int dtype);

/* Frees the handle's device and host memory. NULL is ignored. Must not be
 * called while work that uses the handle is still running on a stream. */
void tq_destroy(tq_handle* h);

/* Handle parameters: dimension, MSE bits, QJL projections (0 for MSE-only),
 * norm dtype. Any output pointer may be NULL. */
int tq_get_info(const tq_handle* h, int* d, int* bits_mse, int* qjl_m, int* norm_dtype);

/* Per-vector strides in bytes of the codes and signs rows (signs_B = 0 for
 * MSE-only handles). */
int tq_code_bytes(const tq_handle* h, int* codes_B, int* signs_B);

/* Host copies (fp64) of the codebook: 2^b centroids and 2^b - 1 boundaries
 * (TQ_EINVAL for polar handles: tq_get_polar_codebook). */
int tq_get_codebook(const tq_handle* h, double* centroids, double* bounds);

/* Host copies (fp64) of Pi (d*d) and, if S != NULL and the handle is prod, S (m*d). */
int tq_get_rotation(const tq_handle* h, double* Pi, double* S);

/* ---------------------------------------------------------------------------
 * Hot path
 * ------------------------------------------------------------------------ */

/* Encode n vectors [TQ6x Stage 1 and 2; DEEP "PolarQuant", "QJL"]:
 * norm = ||x||, y = Pi x / norm, index_j = #{i : bound_i < y_j}, bit-pack;
 * prod handles also write signs of S r, r = x - norm * Pi^T c[index], and ||r||
 * (QJL-only handles: signs of S x and the norm; codes and rnorms may be NULL).
 *  x      device [n][d] of x_dtype (TQ_F32 / TQ_F16 / TQ_BF16), 16-byte aligned
 *  codes  device [n][codes_B];  signs device [n][signs_B] (prod) or NULL
 *  norms  device [n] of the handle's norm dtype;  rnorms device [n] fp16 (prod) or NULL
 * n == 0 is a no-op. A zero vector gets norm 0 and index 2^(b-1) - 1. */
int tq_encode(const tq_handle* h, const void* x, int x_dtype, int64_t n,
              uint8_t* codes, uint8_t* signs, void* norms, void* rnorms, void* stream);

/* Test hook: packs indices idx (device uint8 [n][d], each < 2^b) into codes
 * (device [n][codes_B]) with the layout above. TQ_EINVAL for QJL-only handles. */
int tq_pack_indices(const tq_handle* h, const uint8_t* idx, int64_t n, uint8_t* codes, void* stream);

/* Streaming append of one token per (sequence, head) [TQ6x Stage 1: online
 * arrival with a fixed codebook; FRAC "Problem statement": O(1) append]:
 * encodes x_new (device [B][Hkv][d], x_dtype) into slot len[b] of `cache` for
 * every head, then, if `advance` != 0, increments len[b] (device int32 [B]).
 * A K and a V cache sharing one len array: append K with advance = 0, then V
 * with advance = 1 on the same stream. A full sequence (len[b] >= L_cap) is
 * skipped and TQ_ECAPACITY is recorded in the handle's error word. */
int tq_append(const tq_handle* h, const void* x_new, int x_dtype, int B, int Hkv,
              const tq_cache* cache, int32_t* len, int advance, void* stream);

/* Workspace sizes (bytes) for the calls below; 0 is never returned for a valid call.
 * tq_attn_workspace_bytes is the recommended size: for 3-bit prod caches of 256 MB and
 * more it includes a [B][Hq][L_cap] fp32 scores buffer for the two-kernel attention
 * (scores, then values); tq_attn_decode and tq_decode_step accept any workspace of at
 * least the size without it and then run the single-kernel attention. */
size_t tq_score_workspace_bytes(const tq_handle* hk, int B, int Hq);
size_t tq_attn_workspace_bytes(const tq_handle* hk, const tq_handle* hv, int B, int Hq, int Hkv,
                               int64_t L_cap);
size_t tq_search_workspace_bytes(const tq_handle* h, int nq, int64_t n, int k);

/* Inner-product scores of full-precision queries against a quantized key cache
 * [HAKU "QJL": precise query vs low-bit data; TQ6x Stage 2]:
 *   s = norm * <Pi q, c[index]>  (+ rnorm * sqrt(pi/2)/m * <S q, 2 sigma - 1> for prod;
 *   QJL-only keys: s = norm * sqrt(pi/2)/m * <S q, 2 sigma - 1>; polar keys:
 *   s = norm * <Pi q, y_hat> folded up the transform tree [POLAR section 3], Hq/Hkv <= 8).
 *  q        device fp32 [B][Hq][d];  Hq % Hkv == 0; query head h reads KV head h / (Hq/Hkv)
 *  k, len   key cache and device int32 [B] lengths (0 <= len[b] <= L_cap)
 *  logits   device fp32 [B][Hq][L_cap]; entries i < len[b] are written, the rest untouched
 *  workspace device scratch of tq_score_workspace_bytes(hk, B, Hq) bytes, 16-byte aligned */
int tq_score(const tq_handle* hk, const float* q, int B, int Hq, int Hkv,
             const tq_cache* k, const int32_t* len, float* logits,
             void* workspace, size_t ws_bytes, void* stream);

/* Fused GQA decode attention over quantized K and V [DEEP "Scaled dot-product
 * attention"; TQ6x Stage 1 and 2]: out = softmax(scale * s) V_hat per query
 * head, s from tq_score's formula with hk, V_hat the dequantized values of hv
 * (prod V adds the QJL back-projection rnorm sqrt(pi/2)/m S^T (2 sigma - 1);
 * QJL-only V is that back-projection alone, with the norm in place of rnorm).
 *  q        device [B][Hq][d] fp32 (q_dtype TQ_F32) or bf16 (TQ_BF16)
 *  k, v     caches of hk and hv (same d; any bits/prod mix)
 *  out      device fp32 [B][Hq][d]; a sequence with len[b] == 0 gets zeros
 *  workspace device scratch of tq_attn_workspace_bytes(hk, hv, B, Hq, Hkv, L_cap) bytes
 *           (see the workspace sizes above for the smaller size that is also accepted) */
int tq_attn_decode(const tq_handle* hk, const tq_handle* hv, const void* q, int q_dtype,
                   int B, int Hq, int Hkv, const tq_cache* k, const tq_cache* v,
                   const int32_t* len, float scale, float* out,
                   void* workspace, size_t ws_bytes, void* stream);

/* Same computation, arguments and results as tq_attn_decode, minus the
 * workspace. The pages have no counterpart to this call; it exists for callers
 * that cannot allocate device memory at call time -- e.g. a plugin inside an
 * inference engine that is handed only its input and output buffers, or a
 * serving loop whose allocator is frozen after start-up. The split-K scratch
 * comes from a fixed 4 MiB array compiled into libtq.so (every GPU that loads
 * the library holds it until the process exits); nothing is allocated.
 *  - A shape whose minimum attention workspace (without the two-kernel scores
 *    buffer) exceeds 4 MiB is rejected with TQ_EINVAL (e.g. B*Hq*nsplit*(d+m+2)*4
 *    bytes of partial sums too large).
 *  - B == 0 returns TQ_OK without touching any buffer, as tq_attn_decode does.
 *  - The first call on a device looks up the array's device address with that
 *    device current; make that first call before any stream capture. The
 *    address belongs to the device's primary context: after cudaDeviceReset
 *    it is stale (as is every handle), so the library must not be used again
 *    in that process.
 *  - All calls share the one array and nothing in it needs to start at zero
 *    (every call rewrites what it reads). Calls that overlap on the GPU (other
 *    streams, other host threads) race on it: serialise them. */
int tq_attn_decode_noalloc(const tq_handle* hk, const tq_handle* hv, const void* q, int q_dtype,
                           int B, int Hq, int Hkv, const tq_cache* k, const tq_cache* v,
                           const int32_t* len, float scale, float* out, void* stream);

/* One whole decode step in three launches: append the new key and value of every
 * (sequence, KV head) at slot len[b] (as tq_append on hk and hv), attend over the
 * len[b] + 1 tokens (as tq_attn_decode), then advance len[b] by one. Same results
 * as tq_append(hk, k_new, .., advance 0), tq_append(hv, v_new, .., advance 1) and
 * tq_attn_decode called in that order; the query rotation runs in the same launch
 * as the appends, and len[b] is advanced by the last launch, after every read of it.
 * [Google TurboQuant "Stage 1", "Stage 2"; gemilab "Scaled dot-product attention";
 * gist.science "Problem statement": O(1) append to a growing cache]
 *  k_new, v_new  device [B][Hkv][d] of x_dtype (16-byte aligned)
 *  len           device int32 [B]; a sequence already at L_cap is not appended
 *                (TQ_ECAPACITY is recorded in hk's error word), attends over its
 *                L_cap tokens and keeps len[b] == L_cap
 *  other arguments as tq_attn_decode; needs d <= 128 and m <= 128 for both handles.
 *  Calls sharing len or a cache must be stream-ordered. */
int tq_decode_step(const tq_handle* hk, const tq_handle* hv, const void* q, int q_dtype,
                   const void* k_new, const void* v_new, int x_dtype, int B, int Hq, int Hkv,
                   const tq_cache* k, const tq_cache* v, int32_t* len, float scale, float* out,
                   void* workspace, size_t ws_bytes, void* stream);

/* Top-k inner-product search over n packed database vectors [HAKU "Impact on
 * high-dimensional vector search"]: for each of nq queries (device fp32 [nq][d])
 * the k largest estimated scores norm * <Pi q, c[index]> (MSE handles),
 * ordered by score, equal scores by lower index. codes device [n][codes_B],
 * norms device [n] (handle's dtype). idx device int64 [nq][k], score device
 * fp32 [nq][k]. 1 <= k <= 64, k <= n. */
int tq_search_topk(const tq_handle* h, const float* q, int nq, const uint8_t* codes,
                   const void* norms, int64_t n, int k, int64_t* idx, float* score,
                   void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Kernel timer (tracing; off by default, no cost when off)
 * ------------------------------------------------------------------------ */

/* While enabled, every kernel launched by the library is bracketed by two CUDA
 * events recorded on the launching stream (events come from a pool owned by
 * the library). Kernels are named "encode", "advance_len", "pack", "qprep",
 * "score", "attn_split", "attn_combine", "search", "topk_merge".
 * tq_timer_enable(0) stops recording; recorded events are kept until read. */
int tq_timer_enable(int on);

/* Synchronises the recorded events of kernel `name` (NULL = all kernels), adds
 * their elapsed times in milliseconds to *ms and the number of launches to
 * *launches, and forgets them (forget = 0 keeps them: event pairs captured
 * into a CUDA graph are re-recorded by every replay and can be read again
 * after each one). Either output may be NULL. */
int tq_timer_read(const char* name, double* ms, int* launches, int forget);

/* Synchronises `stream`, then returns and clears the handle's device error word
 * (TQ_OK if nothing was recorded), or TQ_ECUDA if the stream reported an error. */
int tq_last_status(const tq_handle* h, void* stream);

/* Self-test of the device-side failure path. One thread of one CTA waits on a shared-memory
 * barrier that no thread and no copy will complete, giving up after `limit` polls (each poll
 * may suspend for at most about 20 us), and then records a wait timeout in h's device error
 * word exactly as the kernels do when a copy or a release never arrives. The next
 * tq_last_status(h) returns TQ_ETIMEOUT and clears the word; the CUDA context stays usable.
 *  limit  1 .. 65536 (TQ_EINVAL otherwise). Asynchronous on `stream`. */
int tq_selftest_wait_timeout(const tq_handle* h, int limit, void* stream);

/* Message for the last failed call on this host thread ("" if none). */
const char* tq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
