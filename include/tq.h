/*
 * tq.h -- C ABI of libtq: TurboQuant-prod / QJL compressed KV cache and decode
 * attention computed directly on the compressed cache, for NVIDIA B200 (sm_100a).
 *
 * Sources of the operations (cited per call below):
 *   [TQ]   TurboQuant KV-cache quantization article (kwkr.cn/news/562855),
 *          sections 二 (three-stage pipeline), 四 (QJL unbiasedness),
 *          五 (two-stage estimator, ProdQuantized), 六 (scoring kernels, store,
 *          ring buffer), 七 (value quantization, known limits).
 *   [AQJL] A-QJL adaptive layer-wise KV compression article
 *          (zingnex.cn/forum/thread/a-qjl-kv): QJL, A-QJL, deployment config.
 *   [NQ]   KV-cache compression article "无需训练即可将大模型的 KV 缓存压缩 33 倍"
 *          (explore.n1n.ai): six-stage pipeline, step 4 (Hadamard rotation).
 *
 * Conventions shared by every call:
 *   - Every call returns an int status (enum tq_status).  On failure a
 *     thread-local message is available from tq_last_error().
 *   - All argument checks happen on the host before any launch; a call that
 *     fails a check launches nothing and writes nothing.
 *   - Device buffers are owned by the caller.  The library never allocates
 *     device memory and never synchronises, except where a call says so.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Work is enqueued on it; results are ready when the stream reaches them.
 *   - A CUDA error seen at launch (or left pending by earlier work) is
 *     returned as TQ_ERR_CUDA.
 *   - No kernel uses a device-side assert or trap.
 *   - Device pointers must be 16-byte aligned unless stated otherwise.
 *   - Supported sizes: head_dim d in {64, 128, 256}; Lloyd-Max bits b1 in
 *     {0 (pure QJL), 1, 2, 3}; sketch dim m a multiple of 32 in [32, 1024];
 *     value bits vbits in {2, 4}; value group g in {16, 32, 64, 128} dividing d;
 *     query heads per KV head G = Hq / Hkv in [1, 8].
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum tq_status {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,   /* a pointer, size or shape is invalid            */
  TQ_ERR_UNSUPPORTED = 2,   /* a valid but unsupported size / bit width        */
  TQ_ERR_CAPACITY = 3,      /* append would exceed the cache capacity          */
  TQ_ERR_CUDA = 4,          /* a CUDA runtime error                            */
  TQ_ERR_NOT_CONVERGED = 5  /* codebook iteration did not converge             */
};

enum tq_dtype { TQ_F32 = 0, TQ_F16 = 1, TQ_BF16 = 2 };

/* Number of tokens per packed block of the cache layout. */
#define TQ_BLOCK_TOKENS 64

/* Message of the last failed call on this thread ("" if none). */
const char* tq_last_error(void);

/* ABI version of this header: 1. */
int tq_version(void);

/*
 * Host-side fault injection for testing callers' error paths: after
 * tq_debug_fail_next(name), the next call of the ABI function `name` on any
 * thread returns TQ_ERR_CUDA with message "injected fault" without launching
 * anything.  name == NULL clears it.  The environment variable TQ_FAULT, read
 * on the first call, has the same effect.
 */
int tq_debug_fail_next(const char* name);

/* ------------------------------------------------------------------------ */
/* Setup: codebook and projections                                          */
/* ------------------------------------------------------------------------ */

/*
 * tq_codebook_build -- Lloyd-Max codebook for one coordinate of a rotated unit
 * vector in dimension d ([TQ] 二: continuous 1-D k-means for the Beta law of
 * the rotated coordinates).  The law is f(t) ~ (1 - t^2)^((d-3)/2) on [-1, 1];
 * the fixed point beta_k = (c_k + c_{k+1})/2, c_k = E[t | cell k] is iterated in
 * float64 from Gaussian quantiles until max |delta c| < 1e-13 max |c|, then
 * made exactly antisymmetric.
 *   d            head dimension, any value in [16, 4096] (not only 64/128/256)
 *   bits         b1 in [1, 4]; 2^bits centroids
 *   centroids    device, float[2^bits], ascending (written)
 *   boundaries   device, float[2^bits - 1], fp32 midpoints (written)
 * SYNCHRONOUS: waits for the stream to read the convergence flag.
 * Errors: INVALID_ARG (null/misaligned pointers, d out of range),
 *         UNSUPPORTED (bits), NOT_CONVERGED, CUDA.
 */
int tq_codebook_build(int d, int bits, float* centroids, float* boundaries, void* stream);

/* Bytes of device workspace tq_make_projections needs for head dimension d. */
size_t tq_projections_workspace_bytes(int d);

/*
 * tq_make_projections -- per-layer random rotation Pi and Gaussian sketch S
 * ([TQ] 二: Pi from a QR factorisation, S Gaussian; [TQ] 六: seed
 * base_seed + stride * layer, i.e. 42 + 7 * layer).  Generator: Philox4x64-10
 * (Salmon et al., SC'11), draw k of a row-major matrix = counter (k,0,0,0),
 * key (seed, stream) with stream 0 for Pi's Gaussian source G and 1 for S;
 * u = ((w >> 11) + 0.5) 2^-53, z = sqrt(-2 ln u0) cos(2 pi u1).
 * Pi = Q diag(sign diag R) for G = QR (Householder, float64); y = Pi u.
 *   Pi      device float[d*d] row-major (written); NULL = pure QJL (no rotation)
 *   S       device float[m*d] row-major (written)
 *   T       device float[m*d] row-major (written): T = S Pi^T, the sketch in
 *           rotated coordinates used by the key quantiser (T = S if Pi == NULL);
 *           may be NULL
 *   workspace / ws_bytes  device scratch of tq_projections_workspace_bytes(d)
 *           bytes (needed only when Pi != NULL)
 * Errors: INVALID_ARG, UNSUPPORTED (d, m), CUDA.
 */
int tq_make_projections(int d, int m, int layer, uint64_t base_seed, uint64_t stride,
                        float* Pi, float* S, float* T, void* workspace, size_t ws_bytes,
                        void* stream);

/*
 * tq_make_projections_hadamard -- the structured rotation ([NQ] the KV-cache
 * compression page "无需训练即可将大模型的 KV 缓存压缩 33 倍", six-stage pipeline,
 * step 4: a Hadamard rotation spreads a vector's energy evenly over the
 * coordinates) in place of the QR one: Pi = H diag(s) / sqrt(d), H the
 * Sylvester Hadamard matrix (entry (r, c) = (-1)^popcount(r & c)), s_c = +1 when
 * the top bit of word 0 of Philox4x64-10 draw c under key (seed, 2) is 0, else
 * -1; every entry is +-fl32(1/sqrt(d)).  S and T = S Pi^T as tq_make_projections
 * (same seed rule, same S).  Pi is orthogonal, so every call that takes Pi and T
 * works unchanged with it; Pi u is a fast Walsh-Hadamard transform of s * u.
 * A cache whose descriptor says rotation = TQ_ROTATION_HADAMARD reads only row 0
 * of Pi (= s / sqrt(d)) where the rotation runs on CUDA cores -- the append of up
 * to 8 tokens per sequence (a decode step), the tile quantiser of shapes without
 * the tensor-core path, and the query preparation of every decode and prefill --
 * and applies Pi u = H (Pi[0,:] * u) as an O(d log d) butterfly; the tensor-core
 * tile quantiser multiplies by the dense Pi.
 *   Pi  device float[d*d] row-major (written)
 *   S   device float[m*d] row-major (written)
 *   T   device float[m*d] row-major (written; may be NULL)
 * No workspace.  Errors: INVALID_ARG, UNSUPPORTED (d, m), CUDA.
 */
int tq_make_projections_hadamard(int d, int m, int layer, uint64_t base_seed, uint64_t stride,
                                 float* Pi, float* S, float* T, void* stream);

/* ------------------------------------------------------------------------ */
/* Quantisation of keys and values (token-major output arrays)              */
/* ------------------------------------------------------------------------ */

/*
 * tq_quantize_keys -- [TQ] 二 / 五: rho = ||x||, y = Pi x / rho,
 * idx_j = #{k : beta_k < y_j} (b1 bits), residual r = x - rho Pi^T c[idx],
 * sign bits [S r >= 0] (computed as [rho T (y - c[idx]) >= 0]), ||r||.
 * b1 == 0 is pure QJL ([AQJL] QJL): bits [S x >= 0] and rho only.
 *   K           device, [n, d] of dtype, row-major
 *   Pi, T       device, from tq_make_projections (Pi unused when b1 == 0; then
 *               T must be S)
 *   centroids, boundaries  device, from tq_codebook_build(d, b1) (unused if b1 == 0)
 *   idx_planes  device uint8[n * b1*d/8]: per key, b1 bit-planes of d bits,
 *               plane p byte j>>3 bit j&7 = bit p of idx_j   (NULL if b1 == 0)
 *   signs       device uint8[n * m/8], bit i at byte i>>3, bit i&7
 *   norm_x      device float[n] (rho)
 *   norm_r      device float[n] (||r||; NULL if b1 == 0)
 * More than 8 keys at head dim 128 or 256 with m a multiple of 32 up to 512 run
 * on the tensor cores (the rotation and sketch products as f16 hi + lo splits,
 * fp32 accumulation); other shapes on a CUDA-core fp32 tile kernel.  Outside
 * d = m = 128 the call takes a per-call operand scratch of 4 d (d [b1 > 0] + m)
 * bytes from a library-owned stream-ordered pool on the current device.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
int tq_quantize_keys(const void* K, int dtype, int64_t n, int d, int b1, int m,
                     const float* Pi, const float* T, const float* centroids,
                     const float* boundaries, uint8_t* idx_planes, uint8_t* signs,
                     float* norm_x, float* norm_r, void* stream);

/*
 * tq_quantize_values -- [TQ] 二 table / 七: min-max group quantisation, per
 * token and per contiguous group of g channels, IEEE fp32 in this order:
 * mn, mx, s = (mx - mn)/(2^vb - 1), code = clamp(rint((v - mn)/s), 0, 2^vb - 1)
 * (round half to even; 0 when s == 0).  Dequantised value: mn + code * s.
 *   V       device [n, d] of dtype
 *   codes   device uint8[n * d*vbits/8], code j at byte (j*vb)>>3, bit (j*vb)&7
 *   scale   device float[n * d/g];  vmin  device float[n * d/g]
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
int tq_quantize_values(const void* V, int dtype, int64_t n, int d, int vbits, int group,
                       uint8_t* codes, float* scale, float* vmin, void* stream);

/* ------------------------------------------------------------------------ */
/* The packed cache                                                          */
/* ------------------------------------------------------------------------ */

typedef struct tq_cache_desc {
  int32_t B;          /* batch (sequences advance together)                  */
  int32_t Hkv;        /* KV heads                                            */
  int32_t d;          /* head dim                                            */
  int32_t b1;         /* Lloyd-Max bits (0 = pure QJL)                       */
  int32_t m;          /* sketch dim                                          */
  int32_t vbits;      /* value bits                                          */
  int32_t group;      /* value group size                                    */
  int32_t W;          /* full-precision ring size, 0..1024                    */
  int64_t capacity;   /* max compressed tokens per (b, kv head)              */
  int32_t dtype;      /* dtype of K, V, Q, the ring and the output           */
  int32_t rotation;   /* TQ_ROTATION_DENSE (0): Pi any orthogonal matrix;
                         TQ_ROTATION_HADAMARD (1): Pi from
                         tq_make_projections_hadamard, applied as a fast
                         Walsh-Hadamard transform where the rotation runs on
                         CUDA cores (see tq_make_projections_hadamard)      */
} tq_cache_desc;

#define TQ_ROTATION_DENSE 0
#define TQ_ROTATION_HADAMARD 1

/*
 * Cache state.  Layout of the device buffer (also defined by the CPU oracle):
 * for each (b, h) a region of ceil(capacity/64) blocks of 64 tokens; a block
 * stores, field after field, the 64 tokens' idx planes (b1*d/8 B each), sign
 * bits (m/8 B), rho (fp32), ||r|| (fp32, absent if b1 == 0), value codes
 * (d*vbits/8 B), value scales (d/g fp32) and value minima (d/g fp32).  The
 * value codes alone are stored by token pairs (tokens 2i, 2i+1 of the block):
 * cut a token's codes (code j at bit (j*vbits) mod 16 of 16-bit half
 * (j*vbits)/16) into halves; with H = g*vbits/16 halves per group and NG = d/g,
 * half gi*H + s of token 2i is the low and that of token 2i+1 the high 16 bits
 * of 32-bit word s*NG + gi of the pair's record (d*vbits/16 words), so that one
 * masked word is a tensor-core operand of two tokens.  After the
 * regions, 256-byte aligned: ring keys [B, Hkv, W, d] then ring values, in dtype.
 * Token t (counting every token ever appended) sits in ring slot t mod W.
 * After each append the ring holds the last min(W, n_total) tokens and every
 * older token is compressed exactly once, in order ([TQ] 六 store and ring).
 */
typedef struct tq_cache {
  tq_cache_desc desc;
  void* base;            /* caller-owned device buffer                        */
  size_t bytes;
  int64_t n_total;       /* tokens appended so far                            */
  int64_t block_bytes, region_bytes, ring_k_off, ring_v_off;
  int32_t token_bytes;
  int32_t o_idx, o_sign, o_rho, o_rnorm, o_vcode, o_vscale, o_vmin;
} tq_cache;

/* Bytes of device memory a cache with this descriptor needs (0 if invalid). */
size_t tq_cache_bytes(const tq_cache_desc* desc);

/*
 * tq_cache_layout -- host only: fill `out` with the layout of a cache with
 * this descriptor (offsets, sizes; base = NULL, n_total = 0).  No CUDA call.
 * Errors: INVALID_ARG, UNSUPPORTED.
 */
int tq_cache_layout(const tq_cache_desc* desc, tq_cache* out);

/*
 * tq_cache_init -- bind a caller-owned device buffer of at least
 * tq_cache_bytes(desc) bytes (256-byte aligned) to `c`, zero it on `stream`,
 * and set n_total = 0.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
int tq_cache_init(tq_cache* c, const tq_cache_desc* desc, void* dev_mem, size_t bytes,
                  void* stream);

/* Compressed / ring token counts of a cache (host values). */
int64_t tq_cache_compressed_tokens(const tq_cache* c);
int64_t tq_cache_ring_tokens(const tq_cache* c);

/*
 * tq_append -- append n_new tokens per (b, kv head) ([TQ] 六: chunked append
 * into a flat cache; recent tokens kept at full precision in a ring).  Tokens
 * leaving the ring and tokens of the chunk older than the last W are quantised
 * (keys as tq_quantize_keys, values as tq_quantize_values) straight into the
 * packed blocks; the last W go to the ring.  Two kernels, in stream order; one
 * at d = m = 128 with b1 >= 1 when the chunk has more than 8 tokens per (b, kv
 * head) and at least W, which writes the ring itself and may start while the
 * previous append's kernel finishes (consecutive chunks overlap).
 *   K, V     device [B, Hkv, n_new, d] of desc.dtype, contiguous
 *   Pi, T, centroids, boundaries  as for tq_quantize_keys
 * Errors: INVALID_ARG, CAPACITY (nothing written), CUDA.
 */
int tq_append(tq_cache* c, const void* K, const void* V, int64_t n_new, const float* Pi,
              const float* T, const float* centroids, const float* boundaries,
              void* stream);

/* ------------------------------------------------------------------------ */
/* Decode attention                                                          */
/* ------------------------------------------------------------------------ */

/* Number of split-K partitions tq_decode_attention uses when num_splits == 0: on
 * the tensor-core paths one wave of CTAs (148 SMs x the CTAs an SM holds) divided
 * among the (b, kv head) units, or twice that when the wave would leave some SMs
 * a whole CTA ahead of others (the most loaded SM's share, about
 * ceil(units s / 148) CTAs of ceil(blocks / s) blocks, at least 5 % smaller);
 * at most the number of 64-token blocks.  tq_decode_workspace_bytes(c, Hq, 0)
 * covers the count at every length up to the capacity. */
int tq_decode_auto_splits(const tq_cache* c, int Hq);

/* Bytes of device workspace for a decode with Hq query heads and num_splits
 * partitions (0 = automatic). */
size_t tq_decode_workspace_bytes(const tq_cache* c, int Hq, int num_splits);

/*
 * tq_decode_attention -- one decode step for every (b, query head)
 * ([TQ] 四-六; [AQJL] QJL).  Logit of compressed token t for query q:
 *   b1 > 0: rho_t <Pi q, c[idx_t]> + ||r_t|| sqrt(pi/2)/m <S q, 2 bits_t - 1>
 *   b1 = 0: rho_t sqrt(pi/2)/m <S q, 2 bits_t - 1>
 * and <q, k_t> exactly for the ring tokens; p = softmax(softmax_scale * logits);
 * out = sum_t p_t v_t with v = mn + code * s for compressed tokens and the exact
 * v for ring tokens.  Query head hq uses KV head hq / (Hq / Hkv) (GQA).
 * The query is rotated forward and sketched once; keys are never dequantised.
 * Three kernels: query preparation, split-K partial attention, combine.
 *   Q        device [B, Hq, d] of desc.dtype
 *   Pi, S    device, from tq_make_projections (Pi unused when b1 == 0)
 *   centroids device, from tq_codebook_build (unused when b1 == 0)
 *   out      device [B, Hq, d] of desc.dtype (written)
 *   logits   device float[B, Hq, n_comp + n_ring] (unscaled logits, compressed
 *            tokens in order then ring tokens oldest first) or NULL
 *   num_splits  0 = automatic
 *   workspace   device, tq_decode_workspace_bytes() bytes
 * With no tokens at all the output is zero.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
int tq_decode_attention(const tq_cache* c, const void* Q, int Hq, float softmax_scale,
                        const float* Pi, const float* S, const float* centroids, void* out,
                        float* logits, int num_splits, void* workspace, size_t ws_bytes,
                        void* stream);

/* The three stages of tq_decode_attention, for callers that time or overlap
 * them separately.  Same arguments and workspace as tq_decode_attention; the
 * preparation stage also takes the softmax scale and the centroids (the
 * tensor-core path folds them into the query-side constants).  When `out` is
 * non-NULL, tq_decode_partial also merges the splits into `out` (on the
 * tensor-core path inside the same kernel), and tq_decode_combine is not
 * needed. */
int tq_decode_prep(const tq_cache* c, const void* Q, int Hq, float softmax_scale,
                   const float* Pi, const float* S, const float* centroids, int num_splits,
                   void* workspace, size_t ws_bytes, void* stream);
int tq_decode_partial(const tq_cache* c, int Hq, float softmax_scale, const float* centroids,
                      float* logits, void* out, int num_splits, void* workspace, size_t ws_bytes,
                      void* stream);
int tq_decode_combine(const tq_cache* c, int Hq, void* out, int num_splits, void* workspace,
                      size_t ws_bytes, void* stream);

/*
 * tq_decode_step -- one decode step with its append: the same result (cache
 * bytes, n_total, out, logits) as tq_append(c, K, V, n_new, Pi, T, centroids,
 * boundaries, stream) followed by tq_decode_attention(c, Q, Hq, softmax_scale,
 * Pi, S, centroids, out, logits, num_splits, workspace, ws_bytes, stream).  The
 * pages keep these as two steps ([TQ] 六: capture the new token, then score);
 * this call is the fused form of a decode loop.  When 1 <= n_new <= min(8, W)
 * and the decode runs on the tensor-core path, it takes two launches: one grid
 * quantises the tokens that leave the ring (each such CTA also writes the
 * incoming token into the ring slot it has just read), writes incoming tokens
 * into empty ring slots, and prepares the queries; then the split-K partial
 * attention merges its splits into `out`.  Otherwise it makes the two calls.
 * Arguments as for tq_append and tq_decode_attention; the workspace is sized for
 * the cache after the append (tq_decode_workspace_bytes of a cache with
 * n_total + n_new tokens; the workspace size does not depend on n_total).
 * K, V, Q and out may also be pinned (page-locked) host memory from
 * cudaHostAlloc / cudaMallocHost on a system with unified addressing, where it is
 * mapped into the device address space at the same pointer: the kernels then
 * read the new tokens and queries and write the output across the host link,
 * with no staging copy (the result is identical; only the latency differs).
 * All checks of both parts are made before anything is launched.
 * Errors: INVALID_ARG, CAPACITY, UNSUPPORTED, CUDA.
 */
int tq_decode_step(tq_cache* c, const void* K, const void* V, int64_t n_new, const void* Q, int Hq,
                   float softmax_scale, const float* Pi, const float* S, const float* T,
                   const float* centroids, const float* boundaries, void* out, float* logits,
                   int num_splits, void* workspace, size_t ws_bytes, void* stream);

/*
 * tq_decode_check -- SYNCHRONOUS: waits for `stream`, then reports whether the
 * last decode that used `workspace` completed its staged loads.  A decode
 * kernel whose bounded wait on a shared-memory load gives up (it never should)
 * skips its work and raises a flag instead of hanging; this call returns
 * TQ_ERR_CUDA when the flag is set, TQ_OK otherwise.  Arguments as for
 * tq_decode_attention; workspace == NULL (ws_bytes ignored) reads the flag of
 * the static scratch of tq_decode_attention_noalloc on the current device.
 */
int tq_decode_check(const tq_cache* c, int Hq, int num_splits, const void* workspace,
                    size_t ws_bytes, void* stream);

/*
 * tq_prefill_attention -- multi-token (chunked prefill) attention: the n new
 * tokens of a chunk attend to the cache BEFORE the chunk is appended.  The pages
 * define the single-token fused decode ([TQ] 六) and note that their hybrid path
 * dequantises the history for everything else ([TQ] 七); this call scores the
 * history on the packed cache with the same estimator instead.  Query i (0-based)
 * of the chunk sees
 *   - the compressed history: the tq_decode_attention logit and v = mn + code * s,
 *   - the ring tokens: exact <q, k> and v,
 *   - the chunk's own tokens 0..i: exact <q, k> and v from K, V (causal),
 * with p = softmax(softmax_scale * logits) and out = sum_t p_t v_t.  The cache is
 * not modified: append the chunk afterwards with tq_append(c, K, V, n, ...).
 *   Q        device [B, n, Hq, d] of desc.dtype (token-major)
 *   K, V     device [B, Hkv, n, d] of desc.dtype (the layout tq_append takes)
 *   Pi, S, centroids  as for tq_decode_attention
 *   out      device [B, n, Hq, d] of desc.dtype (written)
 *   num_splits  partitions of the history (0 = automatic)
 *   workspace   device, tq_prefill_workspace_bytes(c, Hq, n, num_splits) bytes;
 *               it may be reused once the call's stream work has completed
 * Four launches: query preparation (per query token, as a decode), history
 * partials (tensor cores for head dim 128, G = 4, 2-bit values in groups of 32,
 * b1 <= 2; CUDA cores otherwise), the exact segment, and the split merge.
 * Errors: INVALID_ARG (null pointers, n outside 1..65535, small workspace),
 * UNSUPPORTED (head mapping, B * n above 2^24), CUDA.
 */
size_t tq_prefill_workspace_bytes(const tq_cache* c, int Hq, int n, int num_splits);
int tq_prefill_attention(const tq_cache* c, const void* Q, int Hq, int n, const void* K,
                         const void* V, float softmax_scale, const float* Pi, const float* S,
                         const float* centroids, void* out, int num_splits, void* workspace,
                         size_t ws_bytes, void* stream);

/*
 * tq_prefill_check -- SYNCHRONOUS: as tq_decode_check, for the last
 * tq_prefill_attention that used `workspace` (same c, Hq, n, num_splits).
 */
int tq_prefill_check(const tq_cache* c, int Hq, int n, int num_splits, const void* workspace,
                     size_t ws_bytes, void* stream);

/*
 * Context-sharded decode (one exchange step).  A context too long for one GPU
 * can be split by token ranges over several caches (one per GPU: the earlier
 * ranges in caches with W = 0, the range holding the newest tokens with the
 * ring).  Each GPU runs tq_decode_prep + tq_decode_partial (out = NULL) on its
 * shard; the split partials of all shards are gathered (an all-gather over
 * NCCL, outside this library) and merged.  Because the softmax partials
 * (m, l, o) of disjoint token sets merge exactly, the result is the decode of the
 * whole context ([TQ] 六 online softmax).
 *
 * tq_decode_partials_view -- where tq_decode_partial leaves its partials in
 * `workspace` (same c, Hq, num_splits): *part_ml = device float
 * [B*Hq][*splits][2] (m in log2 units of softmax_scale * logit, then l),
 * *part_o = device float [B*Hq][*splits][d] (sum of p v, unnormalised), and
 * *splits = the split count that call uses.  No launch.  Errors: INVALID_ARG,
 * UNSUPPORTED.
 *
 * tq_merge_partials -- out[r] = sum_s 2^(m_rs - M_r) o_rs / sum_s 2^(m_rs - M_r) l_rs
 * with M_r = max_s m_rs (slots with m = -inf are empty; a row with no token gives
 * 0) for part_ml [rows][slots][2] and part_o [rows][slots][d] (device, the
 * layout above with the shards' splits side by side); out device [rows][d] of
 * dtype.  Errors: INVALID_ARG, CUDA.
 */
int tq_decode_partials_view(const tq_cache* c, int Hq, int num_splits, void* workspace,
                            size_t ws_bytes, float** part_ml, float** part_o, int* splits);
int tq_merge_partials(const float* part_ml, const float* part_o, int64_t rows, int slots, int d,
                      int dtype, void* out, void* stream);

/*
 * tq_quantize_check -- SYNCHRONOUS: waits for `stream`, then reports (and
 * clears) the sticky device flag of the batched tensor-core key quantisation
 * (tq_quantize_keys and tq_append with more than 8 tokens, head dim 128 or 256,
 * m a multiple of 32 up to 512).  Those kernels wait, with a bound, for their
 * operand copies and tensor-core products to complete; if a wait gives up (it
 * never should) they stop and set the flag instead of hanging.  Returns TQ_ERR_CUDA when the flag was set,
 * TQ_OK otherwise.  The pages have no counterpart: this is a diagnostic of this
 * library.
 */
int tq_quantize_check(void* stream);

/*
 * tq_decode_attention_noalloc -- the same decode as tq_decode_attention, for
 * callers that cannot allocate device memory or pass a workspace (for example
 * an inference-engine plugin whose host framework owns all device memory and
 * gives plugins no scratch buffer).  The pages have no counterpart: this is a
 * deployment convenience of this library.
 *   Scratch comes from a statically allocated device array of
 *   TQ_NOALLOC_SCRATCH_BYTES (8 MiB), which every GPU that loads the library
 *   holds until the process exits.  The call allocates nothing.
 *   The first call on each device looks up that array's device address
 *   (cudaGetSymbolAddress) with the device current; make that first call
 *   before any stream capture.
 *   All calls share the one array: calls that overlap on the GPU (different
 *   streams, or different host threads on one device) race and must be
 *   serialised by the caller.  Each call overwrites every scratch byte it reads,
 *   so nothing needs clearing between calls.
 *   Arguments as tq_decode_attention, without the workspace.
 *   A kernel whose bounded wait gave up leaves its flag in the static scratch:
 *   tq_decode_check(c, Hq, num_splits, NULL, 0, stream) reads it.
 * Errors: those of tq_decode_attention; UNSUPPORTED when the decode needs more
 *   scratch than TQ_NOALLOC_SCRATCH_BYTES (sized from the split count the decode
 *   takes for the cache's current length: e.g. very large B * Hq); CUDA when
 *   the address lookup fails.
 */
#define TQ_NOALLOC_SCRATCH_BYTES (8u << 20)
int tq_decode_attention_noalloc(const tq_cache* c, const void* Q, int Hq, float softmax_scale,
                                const float* Pi, const float* S, const float* centroids,
                                void* out, float* logits, int num_splits, void* stream);

/* ------------------------------------------------------------------------ */
/* Adaptive per-layer-group sketch dimension ([AQJL] A-QJL, deployment)     */
/* ------------------------------------------------------------------------ */

typedef struct tq_layer_groups {
  int32_t n;          /* number of groups, 1..8                              */
  int32_t bound[8];   /* bound[i], i < n-1: first layer of group i+1          */
  int32_t m[8];       /* sketch dim of group i                               */
} tq_layer_groups;

/*
 * Parse the A-QJL config strings, e.g. boundaries "8,16,24" and sketch dims
 * "512,384,256,192" ([AQJL] deployment: "layer_group_boundaries" and
 * "key_quantization_bits_per_group").  Boundaries must increase; there must be
 * one more sketch dim than boundaries; every m is a multiple of 32 in
 * [32, 1024].  Errors: INVALID_ARG.
 */
int tq_layer_groups_parse(const char* boundaries, const char* sketch_dims, tq_layer_groups* out);

/* Sketch dim of `layer`: m of the group containing it (-1 if g is invalid). */
int tq_m_for_layer(const tq_layer_groups* g, int layer);

/*
 * Sensitivity profile ([AQJL] sensitivity analyser: each layer's key variance
 * on calibration data decides the layer groups and their bit allocation; the
 * pages give no formula, the steps below are this library's reading).
 *
 * tq_key_moments -- out[0] = mean and out[1] = population variance of the n
 * entries of K (device, dtype TQ_F32 / TQ_F16 / TQ_BF16, 16-byte aligned), the
 * statistic of the [AQJL] sensitivity analyser, in one streaming pass.  The
 * entries are summed relative to a shift (the fp32 mean of the first min(n, 32)
 * entries): d = x - c, S1 = sum d and S2 = sum d^2 in fp64 (d and d^2 exact),
 * and variance = S2/n - (S1/n)^2 in fp64, so keys whose mean is large against
 * their spread keep their precision.  `out` is a device
 * double[2]; `workspace` device, tq_key_moments_workspace_bytes() bytes.  The
 * result does not depend on scheduling (fixed-order reductions).
 * Errors: INVALID_ARG, CUDA.
 */
size_t tq_key_moments_workspace_bytes(void);
int tq_key_moments(const void* K, int dtype, int64_t n, double* out, void* workspace,
                   size_t ws_bytes, void* stream);

/*
 * tq_sensitivity_profile -- host only.  From the per-layer key variances
 * layer_var[0..L-1] (host), the A-QJL layer groups: num_groups (1..8, <= L)
 * contiguous groups whose boundaries minimise the summed squared deviation of
 * the variances from their group means (ties: smallest boundaries first), and
 * per-group sketch dims, multiples of 32 in [m_min, m_max], minimising
 * sum_g n_g s_g / m_g (n_g layers, mean variance s_g; the QJL term's variance
 * is proportional to |k|^2 / m, [TQ] 四) under the sign-bit budget
 * sum_g n_g m_g <= L * m_avg (greedy 32-steps, largest decrease per bit first,
 * ties: lower group).  Writes `out` in the form tq_layer_groups_parse gives.
 * Errors: INVALID_ARG (sizes, m range, negative or non-finite variance, budget
 * below L * m_min).
 */
int tq_sensitivity_profile(const double* layer_var, int L, int num_groups, int m_avg, int m_min,
                           int m_max, tq_layer_groups* out);

/*
 * Bounds-checked build (libtq_bounds.so, compiled with -DTQ_DEBUG_BOUNDS; not a
 * method step).  In that build every kernel checks each address it computes from
 * cache geometry, token positions or split ranges against the buffer it belongs
 * to (the cache buffer, the caller's arrays, the workspace); a failing check
 * records its code in a device flag and the access is not made (stores go to a
 * sink, loads read zeros, a bulk copy is skipped and the consumer's bounded wait
 * reports it).  No check traps.
 * tq_debug_bounds_enabled -- 1 in the bounds-checked build, 0 otherwise.
 * tq_debug_bounds_check -- SYNCHRONOUS (device-wide): reads and clears every
 *   kernel file's flag; TQ_ERR_CUDA naming the first failed check's code when one
 *   is set, TQ_OK otherwise (always TQ_OK in the normal build).
 */
int tq_debug_bounds_enabled(void);
int tq_debug_bounds_check(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
