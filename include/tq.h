/*
 * tq.h -- C ABI of libtq, a B200 (sm_100a) implementation of the TurboQuant
 * hot path: online vector quantization (Q_MSE, Q_prod) and inner-product
 * estimation over the compressed vectors, including fused decode attention
 * over a compressed KV cache.
 *
 * Sources (titles of the pages the method is taken from):
 *   [NOTES] "[2026 ICLR] TurboQuant: Online Vector Quantization with
 *           Near-optimal Distortion Rate", blog notes: eq. (1)-(4), Lemma 1,
 *           residual definition, Q_prod estimator and definition.
 *   [EXPL]  TurboQuant interactive explainer (Traditional-Chinese copy):
 *           §3 rotation, §4 Beta marginal, §5 Lloyd-Max, §6 TurboQuant-MSE,
 *           §7 shrinkage, §8 QJL and TurboQuant-prod, §0.9 randomized Hadamard.
 *   [PYT]   "turboquant-pytorch" skill page: Core API, Pattern 1.
 *   [FVQ]   FastVQ README: sign-flipped Hadamard backend, padding.
 *
 * Conventions for every entry point:
 *   - All tensor arguments are caller-owned DEVICE pointers unless stated
 *     otherwise; the library never frees them.  A tq_params handle owns its
 *     own small device tables (S, dense Pi) and is freed by tq_params_destroy.
 *   - All device work is enqueued asynchronously on `stream` (a cudaStream_t
 *     passed as void*; NULL = legacy default stream).  No entry point
 *     synchronizes the device except tq_params_create/destroy, tq_sync_check.
 *   - Arguments are validated before any launch; a failed check returns an
 *     error status and enqueues nothing.  No entry point aborts, prints or
 *     throws; CUDA launch errors are reported as TQ_ERR_CUDA.
 *   - Nothing on the hot path allocates memory: ops that need scratch take a
 *     caller-supplied workspace whose size is returned by the matching
 *     *_workspace_size query.  Workspace must be 256-byte aligned.
 *   - Device pointers must be 16-byte aligned.
 *
 * Bit layouts of the compressed vectors:
 *   TQ_LAYOUT_ROW: per vector, k bit-planes (plane p = bit p of the code
 *     index, p = 0 least significant), each ceil(d_pad/32) uint32 words; bit
 *     i of word w of a plane holds coordinate 32*w + i.  A row is
 *     k * ceil(d_pad/32) words.  QJL sign words use the same order over the m
 *     rows of S (bit = 1 <=> (S r)_i >= 0).
 *   TQ_LAYOUT_BLOCK32: vectors are grouped in blocks of 32 consecutive
 *     vectors of one segment; a block is k * d_pad uint32 words, word
 *     (p * d_pad + j) holds bit p of coordinate j's index for the 32 vectors,
 *     bit t <-> vector 32*b + t of the segment.  Missing vectors of a ragged
 *     last block have zero bits.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned buffer, ...  */
  TQ_ERR_UNSUPPORTED = 2, /* valid request outside the supported shapes      */
  TQ_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed      */
  TQ_ERR_TIMEOUT = 4,     /* a device-side bounded wait expired               */
  TQ_ERR_INTERNAL = 5,    /* solver did not converge, or another bug          */
  TQ_ERR_WORKSPACE = 6    /* workspace missing or smaller than required      */
} tq_status;

typedef enum { TQ_F32 = 0, TQ_F16 = 1, TQ_BF16 = 2 } tq_dtype;
typedef enum { TQ_ROT_HADAMARD = 0, TQ_ROT_DENSE = 1 } tq_rot;
typedef enum { TQ_MODE_MSE = 0, TQ_MODE_PROD = 1, TQ_MODE_MSE_UNBIASED = 2 } tq_mode;
typedef enum { TQ_LAYOUT_ROW = 0, TQ_LAYOUT_BLOCK32 = 1 } tq_layout;
/* Storage flag OR'ed into the mode of tq_params_create (TQ_MODE_PROD only):
 * residual norms rho are stored as IEEE fp16 (round to nearest even), as in
 * [PYT] Pattern 4's memory formula ("1 float16 per vector").  Every rnorms /
 * krnorms argument of such a handle then points to uint16_t storage with
 * the same element count (pass the address cast to float*). */
typedef enum { TQ_STORE_RNORM_F16 = 0x100 } tq_store_flag;

typedef struct tq_params tq_params; /* opaque quantizer description */

/* Human-readable name of a status code (static string, never NULL). */
const char* tq_status_string(tq_status s);

/* Library version string (static). */
const char* tq_version(void);

/*
 * tq_build_codebook -- Lloyd-Max codebook of the rotated-coordinate density.
 * [NOTES] Lemma 1 gives the density f(x) = Gamma(d/2)/(sqrt(pi)
 * Gamma((d-1)/2)) (1-x^2)^((d-3)/2) on [-1,1] of one coordinate of a uniform
 * point on S^{d-1}; [NOTES] eq. (4) / [EXPL] §5 the 1-D continuous k-means
 * (Lloyd-Max) problem whose solution is the codebook; [PYT] Core API
 * build_lloyd_max_codebook(dim, bits) -> (boundaries, centroids).
 *   d          dimension of the density (the rotated dimension d_pad), 4..4096
 *   bits       1..4 (2^bits levels)
 *   centroids  HOST float[2^bits], ascending, odd-symmetric
 *   boundaries HOST float[2^bits - 1], midpoints of adjacent centroids
 * Solved on the host in double precision, rounded to fp32.  Returns
 * TQ_ERR_INVALID_ARG on bad sizes/null, TQ_ERR_INTERNAL if Lloyd's iteration
 * does not converge.
 */
tq_status tq_build_codebook(int d, int bits, float* centroids, float* boundaries);

/*
 * tq_make_rotation -- the dense rotation Pi from a Gaussian draw G ([EXPL]
 * §3: QR of an iid N(0,1) d x d matrix, keep the orthogonal factor), made
 * unique as Pi = Q diag(sign(diag R)) so that it is Haar-distributed.
 * Householder QR in double on the host.
 *   d   1..4096;  G  HOST double[d * d] row-major;  Pi HOST float[d * d]
 *   row-major, y = Pi x.
 */
tq_status tq_make_rotation(int d, const double* G, float* Pi);

/*
 * tq_params_create -- describe one quantizer (Q_MSE or Q_prod).
 *   d       vector dimension (1..1536)
 *   bits    total bit budget b per coordinate: Q_MSE uses b-bit codes
 *           (1..4); Q_prod uses (b-1)-bit codes plus one QJL sign per row of
 *           S (b = 2..5) ([EXPL] §8, [NOTES] definition of Q_prod)
 *   mode    TQ_MODE_MSE, TQ_MODE_PROD or TQ_MODE_MSE_UNBIASED.  The last
 *           writes the same b-bit codes as TQ_MODE_MSE but stores, in place
 *           of the norm n = ||x||, EDEN's unbiased per-vector scale
 *           S = ||x||^2 / <Pi x, C[idx]> = n / <y, C[idx]> ([EXPL] prior
 *           work: EDEN's scale, and DRIVE's ||x||^2 / ||Pi x||_1 at b = 1),
 *           0 for a zero vector.  Every Q_MSE decoder (tq_decode, the value
 *           side of tq_decode_attention / tq_decode_step) then reconstructs
 *           S Pi^T C[idx], whose component along x is exactly x and whose
 *           mean over uniformly random rotations is x.  Accepted wherever
 *           TQ_MODE_MSE is.
 *           TQ_MODE_PROD | TQ_STORE_RNORM_F16 stores the residual norms in
 *           fp16 (see tq_store_flag).
 *   rot     TQ_ROT_HADAMARD: Pi = H D / sqrt(d_pad), d_pad = next power of
 *           two >= d (at least 32), the vector zero-padded ([EXPL] §0.9,
 *           [FVQ]); d_pad must be 32..256.
 *           TQ_ROT_DENSE: Pi = Q diag(sign diag R) from the QR of G
 *           ([EXPL] §3); d_pad = d, a multiple of 32.
 *   m       QJL rows (PROD only): multiple of 32, 32..4096; ignored for MSE
 *   signs   HOST int8[d_pad] of +1/-1 (the diagonal of D); HADAMARD only
 *   S       HOST float[m * d_pad] row-major Gaussian draws (PROD only).  The
 *           library keeps S exactly as given (fp32) and also an fp16 copy;
 *           entries that are not fp16-representable make the call fail with
 *           TQ_ERR_INVALID_ARG (draw S in fp16, e.g. N(0,1) rounded to fp16).
 *   G       HOST double[d * d] row-major Gaussian draws; DENSE only
 *   out     receives the handle
 * The codebook is solved here (tq_build_codebook), the dense rotation is
 * factored here (Householder QR in double, stored fp32), and the tables are
 * copied to the current device.  Synchronous.  The handle may be used from
 * any stream on that device; it is read-only after creation.
 */
tq_status tq_params_create(int d, int bits, tq_mode mode, tq_rot rot, int m,
                           const int8_t* signs, const float* S, const double* G,
                           tq_params** out);

/* Free a handle and its device tables (synchronous).  NULL is a no-op. */
tq_status tq_params_destroy(tq_params* p);

/*
 * tq_params_info -- sizes derived from a handle (any pointer may be NULL):
 * d_pad, code bits k, code words per vector (ROW layout), sign words per
 * vector (m/32, 0 for MSE), and m.
 */
tq_status tq_params_info(const tq_params* p, int* d_pad, int* k, int* code_words,
                         int* sign_words, int* m);

/*
 * tq_params_tables -- HOST copies of the fp32 tables the kernels use:
 * centroids [2^k], boundaries [2^k - 1] and, for DENSE, Pi [d * d] row-major
 * (y = Pi x).  Any pointer may be NULL.
 */
tq_status tq_params_tables(const tq_params* p, float* centroids, float* boundaries, float* Pi);

/*
 * tq_encode_mse -- TurboQuant-MSE encode ([NOTES] Q_MSE; [EXPL] §6; [PYT]
 * TurboQuantMSE.quantize / compressors.compress).  Per vector x:
 *   n = ||x||_2 (fp32 accumulation), y = Pi (x / n) (y = 0 if n = 0),
 *   idx_j = #{k : B_k < y_j} (nearest centroid; ties to the lower cell),
 *   codes = bit-packed idx (layout), norms = n.
 *   x       DEVICE, n_vec rows of d elements of dtype `dt`, row stride `ld`
 *           elements (ld >= d; ld * sizeof(dt) a multiple of 16 bytes)
 *   n_vec   number of vectors (0 is allowed and enqueues nothing)
 *   seg_len vectors per segment (0 = one segment of n_vec); n_vec must be a
 *           multiple of seg_len.  Segment s is rows [s*seg_len, (s+1)*seg_len).
 *   seg_cap output slots per segment (0 = seg_len rounded up to 32 for
 *           BLOCK32, seg_len for ROW); >= seg_len, a multiple of 32 for
 *           BLOCK32.  Slot t of segment s is output vector s*seg_cap + t.
 *           Slots >= seg_len are not written.
 *   codes   DEVICE uint32: ROW: [n_seg * seg_cap][k * ceil(d_pad/32)];
 *           BLOCK32: [n_seg * seg_cap / 32][k * d_pad]
 *   norms   DEVICE float[n_seg * seg_cap]
 *   ws      workspace of tq_encode_workspace_size bytes (NULL allowed when 0)
 */
tq_status tq_encode_mse(const tq_params* p, const void* x, tq_dtype dt, int64_t n_vec, int64_t ld,
                        int64_t seg_len, int64_t seg_cap, tq_layout layout, uint32_t* codes,
                        float* norms, void* ws, size_t ws_bytes, void* stream);

/*
 * tq_encode_workspace_size -- scratch bytes tq_encode_mse / tq_encode_prod
 * need for n_vec vectors: 0 for the Hadamard rotation (ws may be NULL); for
 * the dense rotation, room for one chunk of rotated vectors (and of S r).
 */
tq_status tq_encode_workspace_size(const tq_params* p, int64_t n_vec, size_t* bytes);

/*
 * tq_encode_prod -- TurboQuant-prod encode ([NOTES] residual, Q_prod
 * definition; [EXPL] §8; [PYT] TurboQuantProd.compress -> codes, signs,
 * residual_norms).  As tq_encode_mse with (b-1)-bit codes (ROW layout), then
 *   r = y - C[idx] (rotated domain), rho = ||r||_2,
 *   signs_i = [ (S r)_i >= 0 ], i < m, packed ROW order,
 *   rnorms = rho.
 *   codes  DEVICE uint32 [n_seg * seg_cap][k * ceil(d_pad/32)]
 *   signs  DEVICE uint32 [n_seg * seg_cap][m / 32]
 *   norms, rnorms  DEVICE float [n_seg * seg_cap]
 */
tq_status tq_encode_prod(const tq_params* p, const void* x, tq_dtype dt, int64_t n_vec, int64_t ld,
                         int64_t seg_len, int64_t seg_cap, uint32_t* codes, uint32_t* signs,
                         float* norms, float* rnorms, void* ws, size_t ws_bytes, void* stream);

/*
 * tq_decode -- reconstruction ([NOTES] Q_MSE^{-1}: centroids then Pi^T;
 * [EXPL] §8 QJL dequantization; [PYT] dequantize / decompress):
 *   x~ = n Pi^T ( C[idx] + [signs != NULL] kappa rho S^T (2 sigma - 1) ),
 *   kappa = sqrt(pi/2) / m, truncated to the first d coordinates.
 *   codes/norms  as written by the encoders (layout; seg_len/seg_cap as there)
 *   signs/rnorms Q_prod only; NULL gives the Q_MSE part only
 *   out          DEVICE float [n_vec][ldo], ldo >= d
 */
tq_status tq_decode(const tq_params* p, tq_layout layout, const uint32_t* codes,
                    const uint32_t* signs, const float* norms, const float* rnorms, int64_t n_vec,
                    int64_t seg_len, int64_t seg_cap, float* out, int64_t ldo, void* stream);

/*
 * tq_scores -- inner-product estimates of fp32 queries against Q_prod-encoded
 * vectors ([NOTES] unbiased estimator; [EXPL] §8; [PYT]
 * TurboQuantProd.inner_product, asymmetric_attention_scores):
 *   q' = Pi q, u = S q' (once per query),
 *   s[a, t] = n_t ( <q'_a, C[idx_t]> + kappa rho_t <u_a, 2 sigma_t - 1> ).
 *   q       DEVICE float [nq][ldq]
 *   codes/signs/norms/rnorms  ROW layout, n_vec vectors
 *   scores  DEVICE float [nq][n_vec] or NULL (then topk > 0 is required)
 *   topk    0, or 1..32: also return, per query, the top-k scores (desc) and
 *           their vector indices (ties -> lower index) in top_s [nq][topk],
 *           top_i [nq][topk] (int64)
 *   ws      workspace of tq_scores_workspace_size bytes
 */
tq_status tq_scores(const tq_params* kp, const float* q, int64_t nq, int64_t ldq,
                    const uint32_t* codes, const uint32_t* signs, const float* norms,
                    const float* rnorms, int64_t n_vec, float* scores, int topk, float* top_s,
                    int64_t* top_i, void* ws, size_t ws_bytes, void* stream);
tq_status tq_scores_workspace_size(const tq_params* kp, int64_t nq, int64_t n_vec, int topk,
                                   size_t* bytes);

/*
 * tq_decode_attention -- one decode step over a compressed KV cache ([PYT]
 * Pattern 1: scores from compressed keys, softmax, weighted sum of the
 * Q_MSE-reconstructed values), fused: the values are averaged in the rotated
 * domain and Pi_V^T is applied once per output (Pi^T is linear).
 *   kp      Q_prod handle of the keys; vp Q_MSE handle of the values
 *           (TQ_MODE_MSE or TQ_MODE_MSE_UNBIASED); both with the same d and
 *           rotation kind.
 *   q       DEVICE float [L][B][Hq][d] (one query token per head)
 *   Hq, Hkv query / KV heads, Hq a multiple of Hkv; query head h reads KV
 *           head h / (Hq / Hkv); at most 16 query heads per KV head
 *           (TQ_ERR_UNSUPPORTED above).
 *   seq     valid tokens per (layer, batch, kv-head), >= 1
 *   cap     token slots per (layer, batch, kv-head) in the cache, >= seq, a
 *           multiple of 32
 *   scale   softmax scale alpha: p = softmax(alpha * s)
 *   kcodes  DEVICE uint32 [L][B][Hkv][cap][kp code words]   (ROW)
 *   ksigns  DEVICE uint32 [L][B][Hkv][cap][m/32]
 *   knorms, krnorms DEVICE float [L][B][Hkv][cap]
 *   vcodes  DEVICE uint32 [L][B][Hkv][cap/32][k_v * d_pad]   (BLOCK32)
 *   vnorms  DEVICE float [L][B][Hkv][cap]
 *   out     DEVICE float [L][B][Hq][d]
 *   ws      workspace of tq_decode_attention_workspace_size bytes
 */
tq_status tq_decode_attention(const tq_params* kp, const tq_params* vp, const float* q, int L,
                              int B, int Hq, int Hkv, int64_t seq, int64_t cap, float scale,
                              const uint32_t* kcodes, const uint32_t* ksigns, const float* knorms,
                              const float* krnorms, const uint32_t* vcodes, const float* vnorms,
                              float* out, void* ws, size_t ws_bytes, void* stream);
tq_status tq_decode_attention_workspace_size(const tq_params* kp, const tq_params* vp, int L,
                                             int B, int Hq, int Hkv, int64_t seq,
                                             size_t* bytes);

/*
 * tq_decode_attention_noalloc -- tq_decode_attention with no workspace
 * argument and no allocation of any kind.  The pages have no counterpart to
 * this call; it exists for deployment.
 *
 * Some callers cannot call cudaMalloc or otherwise obtain device memory on
 * the decode path: for example a plugin inside an inference engine that owns
 * every byte of the device's memory pool and offers plugins no allocation
 * hook, or a latency-bound decode loop that must never risk the device-wide
 * synchronization an allocation can cause.  This entry point serves them.
 *
 * Its scratch is one file-scope device array of TQ_NOALLOC_SCRATCH_BYTES
 * (32 MiB), part of the library image: every GPU that loads libtq holds it
 * until the process exits.  A call whose tq_decode_attention_workspace_size
 * is larger returns TQ_ERR_WORKSPACE and enqueues nothing.
 *
 * Every call looks up the array's device address in the caller's current
 * device and context (nothing is cached, so the address stays right after
 * cudaDeviceReset or when the caller switches contexts).  The first call in
 * a context may load the library's module into it: make that first call
 * before any stream capture.  Every call shares the same array.  The
 * attention kernels write every scratch byte they later read within the
 * same call (a chunk whose staging wait expires writes an empty partial),
 * so nothing relies on the array's previous contents; but calls that
 * overlap on the GPU (other streams, other host threads) race on the array
 * and corrupt each other's results -- serialize them.
 *
 * Arguments, layouts, results and the other errors are those of
 * tq_decode_attention.
 */
#define TQ_NOALLOC_SCRATCH_BYTES (32u << 20)
tq_status tq_decode_attention_noalloc(const tq_params* kp, const tq_params* vp, const float* q,
                                      int L, int B, int Hq, int Hkv, int64_t seq, int64_t cap,
                                      float scale, const uint32_t* kcodes, const uint32_t* ksigns,
                                      const float* knorms, const float* krnorms,
                                      const uint32_t* vcodes, const float* vnorms, float* out,
                                      void* stream);

/*
 * tq_decode_step -- one serving decode step over a compressed KV cache:
 * append the new token's key and value to every (layer, batch, kv-head)
 * cache at slot `pos`, then attend over the pos + 1 cached tokens
 * ("turboquant-pytorch" skill page, KV Cache Wrapper (TurboQuantKVCache):
 * append_key / append_value as tokens are generated, then attention of a
 * query against all cached keys with MSE-reconstructed values).
 *   k_new, v_new DEVICE [L][B][Hkv][d] of dtype dt (rows 16-byte aligned):
 *           the new token's key and value per (layer, batch, kv-head)
 *   pos     slot of the new token, 0 <= pos < cap; slots 0 .. pos - 1 must
 *           already hold the earlier tokens (e.g. from tq_encode_prod /
 *           tq_encode_mse or earlier steps)
 *   kcodes, ksigns, knorms, krnorms, vcodes, vnorms  the caches of
 *           tq_decode_attention, written at slot pos (in BLOCK32 only bit
 *           pos % 32 of block pos / 32 changes) and then read
 *   q, Hq, Hkv, cap, scale, out  as tq_decode_attention with seq = pos + 1
 *   ws      workspace of tq_decode_step_workspace_size bytes (256-byte
 *           aligned)
 * Everything is enqueued on `stream` in order (key encode, value encode,
 * bit scatter, attention).  Errors: those of tq_decode_attention, and
 * TQ_ERR_INVALID_ARG for pos outside [0, cap) or a bad dtype.
 */
tq_status tq_decode_step(const tq_params* kp, const tq_params* vp, const float* q,
                         const void* k_new, const void* v_new, tq_dtype dt, int L, int B, int Hq,
                         int Hkv, int64_t pos, int64_t cap, float scale, uint32_t* kcodes,
                         uint32_t* ksigns, float* knorms, float* krnorms, uint32_t* vcodes,
                         float* vnorms, float* out, void* ws, size_t ws_bytes, void* stream);
tq_status tq_decode_step_workspace_size(const tq_params* kp, const tq_params* vp, int L, int B,
                                        int Hq, int Hkv, int64_t pos, size_t* bytes);

/*
 * tq_sync_check -- synchronize `stream` and report (then clear) the device
 * error word that kernels set when a bounded wait expires (TQ_ERR_TIMEOUT)
 * or an internal check fails (TQ_ERR_INTERNAL).  When it reports
 * TQ_ERR_TIMEOUT, the outputs of the calls enqueued since the previous check
 * are not valid results: a kernel whose wait expired skipped the rest of its
 * work (an attention chunk then contributes nothing to its heads' outputs).
 */
tq_status tq_sync_check(void* stream);

/*
 * tq_check_wait_expiry -- exercise the bounded-wait helper that every kernel
 * uses on its mbarriers, in both of its forms (polling and suspending): one
 * CTA waits on barriers that nothing ever completes, gives up after
 * `budget_cycles` SM clock cycles (1 .. 2^31) per wait, sets the device error
 * word to TQ_ERR_TIMEOUT and exits, leaving the context usable.  Enqueued on `stream`; the status appears at the next
 * tq_sync_check.  TQ_ERR_INVALID_ARG for a budget outside the range.
 */
tq_status tq_check_wait_expiry(int64_t budget_cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
