/*
 * tq.h -- C ABI of a B200 (sm_100a) library for TurboQuant KV-cache
 * compression and decode attention on the compressed cache.
 *
 * What the calls compute (citations are the web pages on TurboQuant, by
 * title and section):
 *   - TurboQuant_mse: keep ||x|| as is (HN thread on TurboQuant: the radius
 *     is one number per vector and need not be quantized), rotate x/||x||
 *     with a seeded random orthogonal map, replace every rotated coordinate by
 *     the index of its nearest Lloyd-Max centroid, store only the bit-packed
 *     indices ("TurboQuant của Google: nén KV cache 6 lần", sections "Trick
 *     đầu tiên: xoay ngẫu nhiên trước khi nén" and "Lloyd-Max quantizer").
 *   - TurboQuant_prod: (b-1)-bit MSE code of the same kind, then one QJL sign
 *     bit per coordinate of S r for the residual r, plus ||r||, which makes
 *     the inner-product estimate unbiased (same page, section "Vấn đề của
 *     inner product: bias không phải MSE"; "内存厂商的噩梦来了", 4.2-4.3).
 *   - Decode attention: softmax(q K^T / sqrt(d)) V for one new query per head
 *     over all cached tokens ("I Spent 31 Hours On The Math Behind
 *     Turboquant", section "KV Cache: The problem"), with keys scored by the
 *     asymmetric estimator, a full-precision query against compressed keys
 *     ("内存厂商的噩梦来了", 4.2 and its asymmetric_attention_score).
 *
 * Conventions (all calls):
 *   - Every call returns tq_status.  Arguments are validated before any
 *     launch; a failed check returns a non-OK status, launches nothing and
 *     sets tq_last_error().  A failed launch returns TQ_ECUDA.
 *   - The library allocates no device memory and keeps no global state
 *     (tq_decode_attention_noalloc alone uses a fixed scratch array compiled
 *     into the library).  The caller owns every buffer and the stream;
 *     device calls are asynchronous on the given stream (NULL = the legacy
 *     default stream).
 *   - Outputs must not alias inputs.
 *   - d is 64, 128 or 256.  bits is the total b per coordinate, 1..4.
 *     The MSE part uses b_m = b bits (mse) or b_m = b - 1 bits (prod).
 *   - Packed layout per vector ("record"): codes are an LSB-first bitstream,
 *     index i's bit k at stream bit p = i*b_m + k, byte p >> 3, bit p & 7
 *     (d*b_m/8 bytes); the QJL sketch puts bit k (1 = (S r)_k >= 0) at byte
 *     k >> 3, bit k & 7 (d/8 bytes); norms ||x|| and residual norms ||r|| are
 *     separate fp32 arrays.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
/* A CUDA stream handle (the same object as cudaStream_t). */
typedef struct CUstream_st *tq_stream_t;

typedef enum {
  TQ_OK = 0,
  TQ_EINVAL = 1,        /* bad argument: null pointer, size, alignment, enum */
  TQ_EUNSUPPORTED = 2,  /* valid request this build does not implement */
  TQ_ECUDA = 3,         /* a CUDA runtime call or launch failed */
  TQ_EWORKSPACE = 4,    /* workspace smaller than tq_decode_workspace_bytes */
  TQ_ETIMEOUT = 5       /* a kernel gave up a bounded wait (reported by tq_check) */
} tq_status;

typedef enum { TQ_MSE = 0, TQ_PROD = 1 } tq_variant;

/* TQ_ROT_HADAMARD: Pi = H diag(sigma) / sqrt(d), H the Sylvester Hadamard
 * matrix, sigma the seeded signs ("内存厂商的噩梦来了", the note after the
 * section-4 pseudocode: WHT instead of the dense product); d is 64, 128 or
 * 256.
 * TQ_ROT_DENSE: Pi is a Haar-random d x d orthogonal matrix, the Q factor of
 * the QR decomposition of a seeded Gaussian matrix ("TurboQuant của Google",
 * section "Trick đầu tiên"), passed as tq_quantizer.rot (tq_make_rotation);
 * d is any multiple of 8 from 8 to 256. */
typedef enum { TQ_ROT_HADAMARD = 0, TQ_ROT_DENSE = 1 } tq_rotation;

/* Density the codebook is fitted to: N(0, 1/d) (default), or the exact law
 * C (1 - x^2)^((d-3)/2) of a coordinate of a uniform unit vector
 * ("TurboQuant của Google", section "Trick đầu tiên"). */
typedef enum { TQ_CB_GAUSS = 0, TQ_CB_BETA = 1 } tq_codebook_dist;

typedef enum { TQ_F32 = 0, TQ_BF16 = 1, TQ_F16 = 2 } tq_dtype;

/* One quantizer.  A caller-owned value; the pointers are caller-owned DEVICE
 * memory, filled from tq_make_codebook / tq_make_signs / tq_make_qjl.
 * centroids/thresholds must be exactly as tq_make_codebook writes them
 * (ascending, c_i = -c_{K-1-i}, middle threshold 0): the kernels use the
 * positive half and its mirror image. */
typedef struct {
  int32_t d;
  int32_t bits;            /* total b, 1..4 */
  int32_t variant;         /* tq_variant */
  int32_t rotation;        /* tq_rotation */
  const float *centroids;  /* 2^b_m fp32 (unused when b_m == 0) */
  const float *thresholds; /* 2^b_m - 1 fp32 */
  const int8_t *signs;     /* d entries, each +1 or -1 (Hadamard rotation) */
  const float *qjl_S;      /* d*d fp32 row-major, prod only, else NULL */
  const float *rot;        /* d*d fp32 row-major Pi, 16-byte aligned (dense
                              rotation only, else NULL): y = Pi x */
  const int32_t *channels; /* DEVICE, d entries or NULL: coordinate i of the
                              quantized vector is element channels[i] of the
                              input row (a channel group of a wider head,
                              the outlier-channel split); dense rotation
                              only.  NULL = elements 0..d-1. */
} tq_quantizer;

/* A packed cache: records addressed as
 *   rec(b, h, n) = b*stride_b + h*stride_h + n*stride_n   (in records)
 * codes + rec*code_bytes, qjl + rec*(d/8), norms + rec, rnorms + rec.
 * codes is NULL when b_m == 0; qjl and rnorms are NULL for mse.
 * codes and qjl must be 16-byte aligned; strides may be 0 (a shared cache). */
typedef struct {
  uint8_t *codes;
  uint8_t *qjl;
  float *norms;
  float *rnorms;
  int64_t stride_b, stride_h, stride_n;
} tq_cache_view;

/* ---- host, synchronous, pure ------------------------------------------ */

/* Lloyd-Max codebook for d (a multiple of 8 up to 256) and b_m = bits_mse
 * (1..4): 2^b_m centroids and 2^b_m - 1 thresholds (midpoints), fp32,
 * written to HOST arrays.  Lloyd's
 * alternation runs in double and is rounded once to fp32 ("TurboQuant của
 * Google", section "Lloyd-Max quantizer": computed once, shipped, reused). */
tq_status tq_make_codebook(int32_t d, int32_t bits_mse, tq_codebook_dist dist,
                           float *centroids, float *thresholds);

/* Seeded Rademacher signs sigma (d int8 values, +1/-1, HOST array): +1 when
 * bit 63 of SplitMix64 output i is clear. */
tq_status tq_make_signs(uint64_t seed, int32_t d, int8_t *signs);

/* Seeded QJL matrix S, d x d i.i.d. N(0,1), row-major fp32 HOST array, from
 * Box-Muller on consecutive SplitMix64 output pairs ("TurboQuant của
 * Google", section "Vấn đề của inner product": QJL's random projection). */
tq_status tq_make_qjl(uint64_t seed, int32_t d, float *S);

/* Seeded dense rotation Pi (d x d fp32, row-major, HOST array), d a
 * multiple of 8 from 8 to 256: G = the seeded Gaussian matrix of
 * tq_make_qjl's generator in double (unrounded), G = Q R by Householder
 * reflections in double, Q's columns negated where R's diagonal is negative
 * (R then has a positive diagonal, which makes Q Haar-distributed),
 * Pi = Q rounded once to fp32 ("TurboQuant của Google", section "Trick đầu
 * tiên": the rotation is the Q of a Gaussian matrix's QR). */
tq_status tq_make_rotation(uint64_t seed, int32_t d, float *rot);

/* Bytes of one record's codes (d*b_m/8) and QJL sketch (d/8 or 0). */
size_t tq_code_bytes(int32_t d, int32_t bits, int32_t variant);
size_t tq_qjl_bytes(int32_t d, int32_t variant);

/* ---- device, asynchronous on `stream` ---------------------------------- */

/* Encode B*H*N vectors.  Vector (b, h, n) starts at element
 * b*x_stride_b + h*x_stride_h + n*x_stride_n of x (dtype x_dtype, d
 * contiguous elements); x and every stride times the element size must be
 * 16-byte aligned.  Writes codes, norms (and qjl, rnorms for prod) of record
 * (b, h, n) of `out`.  The codes are bit-exact with the canonical fp32
 * procedure: fold-halves sum of squares, sqrt_rn; FWHT stages h = d/2..1 on
 * sigma*x; u = y * fl(1/fl(n*fl(sqrt d))) (0 when n == 0);
 * idx = #{j : u > t_j}.  The QJL projection S r is summed in fp32. */
tq_status tq_encode(const tq_quantizer *q, const void *x, tq_dtype x_dtype,
                    int64_t B, int64_t H, int64_t N, int64_t x_stride_b,
                    int64_t x_stride_h, int64_t x_stride_n,
                    const tq_cache_view *out, tq_stream_t stream);

/* Reconstruct x_hat = ||x|| Pi^T (c[idx] (+ ||r|| sqrt(pi/2)/d S^T sign))
 * for the B*H*N records of `in` into out[B][H][N][d] fp32 (DEVICE)
 * ("内存厂商的噩梦来了", section-4 pseudocode, dequant). */
tq_status tq_dequant(const tq_quantizer *q, const tq_cache_view *in, int64_t B,
                     int64_t H, int64_t N, float *out, tq_stream_t stream);

/* Workspace the decode call needs, in bytes (0 means none).  Depends only
 * on the arguments; the value may change between library versions. */
size_t tq_decode_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv,
                                 int64_t seq_len, int32_t d);

/* Decode attention.  q: [B][Hq][d] (q_dtype, DEVICE).  Query head hq reads
 * kv head hq / (Hq/Hkv).  Cached tokens 0..L_b-1 of batch b are attended
 * with L_b = seq_lens[b] (DEVICE int32 [B], each 0..seq_len; seq_len < 2^31) or seq_len when
 * seq_lens is NULL; no causal mask.  The query is rotated once by the key
 * rotation; scores are
 *   s_j = n_j (<q', c_K[idx_j]> + [prod] ||r_j|| sqrt(pi/2)/d <S q', sign_j>)
 * logits s_j * softmax_scale; values are summed in the value-rotated basis
 * and rotated back once at the end.  out: [B][Hq][d] fp32 (DEVICE); a batch
 * with L_b == 0 gets zeros.  scores_out: optional [B][Hq][seq_len] fp32 of
 * the pre-scale estimator s_j (entries j >= L_b untouched), or NULL.
 * Any valid pair of quantizers with equal d: K and V may each be mse or
 * prod, with either rotation.  Prod values are dequantized as
 * n_j (c_V[idx_j] + ||r_j|| sqrt(pi/2)/d S_V^T sign_j) in the rotated basis.
 * d = 128 with mse values runs on tensor cores (fp16 hi/lo operands, fp32
 * accumulation); every other case runs on CUDA cores in fp32.
 * workspace: DEVICE, at least tq_decode_workspace_bytes(...) bytes, 16-byte
 * aligned, else TQ_EWORKSPACE. */
tq_status tq_decode_attention(const tq_quantizer *kq, const tq_quantizer *vq,
                              const void *q, tq_dtype q_dtype, int32_t B,
                              int32_t Hq, int32_t Hkv, int64_t seq_len,
                              const int32_t *seq_lens, const tq_cache_view *k,
                              const tq_cache_view *v, float softmax_scale,
                              float *out, float *scores_out, void *workspace,
                              size_t workspace_bytes, tq_stream_t stream);

/* One decode step: compress the new token's key and value into the cache,
 * then attend over the cache ("I Spent 31 Hours On The Math Behind
 * Turboquant", section "KV Cache: The problem": each generated token appends
 * its K and V, and the next query attends over all of them).
 * Equivalent to tq_encode(kq, k_new -> k_tail), tq_encode(vq, v_new ->
 * v_tail), then tq_decode_attention(...) with the remaining arguments, with
 * identical results, as one call: the four kernels run as a chain in which
 * each may start while the one before it finishes.
 *   k_new, v_new: [B][Hkv][d] (kv_dtype, DEVICE), element strides
 *                 new_stride_b, new_stride_h (16-byte multiples), unit stride
 *                 along d.
 *   k_tail, v_tail: views of the B x Hkv records that receive them (usually
 *                 token L_b - 1 of k and v, so the new token is attended).
 *   The rest as for tq_decode_attention.  All arguments are validated before
 *   any launch.  The chain's first kernel starts after everything already in
 *   the stream, like any launch; inputs must not be written by later work
 *   until the call's work completes. */
tq_status tq_append_decode_attention(const tq_quantizer *kq, const tq_quantizer *vq,
                                     const void *k_new, const void *v_new, tq_dtype kv_dtype,
                                     int64_t new_stride_b, int64_t new_stride_h,
                                     const tq_cache_view *k_tail, const tq_cache_view *v_tail,
                                     const void *q, tq_dtype q_dtype, int32_t B, int32_t Hq,
                                     int32_t Hkv, int64_t seq_len, const int32_t *seq_lens,
                                     const tq_cache_view *k, const tq_cache_view *v,
                                     float softmax_scale, float *out, float *scores_out,
                                     void *workspace, size_t workspace_bytes, tq_stream_t stream);

/* Decode attention without a caller workspace.  The pages have no
 * counterpart to this call: it exists for callers that cannot allocate
 * device memory at run time, such as a plugin whose enqueue runs inside
 * another engine that owns every device allocation, or a service that
 * forbids cudaMalloc after start-up.  Same arguments, meaning and results
 * as tq_decode_attention, minus the workspace: the scratch it needs lives in
 * a fixed array of TQ_NOALLOC_SCRATCH_BYTES compiled into the library, one
 * copy per GPU that loads the library, kept until the process exits.
 *   - The first call on a device looks up that device's copy of the array
 *     (cudaGetSymbolAddress, with the device current); make that first call
 *     before any stream capture.
 *   - It allocates nothing: no cudaMalloc, no cudaFree, no allocating
 *     library call.
 *   - A problem whose tq_decode_workspace_bytes exceeds
 *     TQ_NOALLOC_SCRATCH_BYTES returns TQ_EWORKSPACE, with the sizes in
 *     tq_last_error().
 *   - All calls share the one array, and it keeps the previous call's
 *     contents.  Every call clears the counters it needs at its start.
 *     Calls whose work overlaps on the GPU (different streams without
 *     ordering between them) race on the array; keep them ordered. */
#define TQ_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
tq_status tq_decode_attention_noalloc(const tq_quantizer *kq, const tq_quantizer *vq,
                                      const void *q, tq_dtype q_dtype, int32_t B,
                                      int32_t Hq, int32_t Hkv, int64_t seq_len,
                                      const int32_t *seq_lens,
                                      const tq_cache_view *k, const tq_cache_view *v,
                                      float softmax_scale, float *out,
                                      float *scores_out, tq_stream_t stream);

/* Decode attention over an outlier-channel split cache ("TurboQuant của
 * Google", the correction in the experiments section: a head's channels in
 * two groups, the outlier channels at a higher bit width).  Each cache is
 * two caches, one per channel group: group 0 of the keys is quantized by
 * kq[0] (its channels list gives the group's head-dim channels), group 1 by
 * kq[1], likewise the values; both groups use the dense rotation and
 * together cover the d = kq[0].d + kq[1].d channels of the head once.
 * Scores are the two groups' asymmetric estimates added,
 *   s_j = est_0(q[ch_0], k_0j) + est_1(q[ch_1], k_1j),
 * the softmax is over all L_b tokens, and each value group is summed in its
 * own rotated basis and rotated back into its channels of out[B][Hq][d].
 * The rest as for tq_decode_attention (q: [B][Hq][d]; GQA; seq_lens;
 * softmax_scale); d <= 256.  workspace: DEVICE, at least
 * tq_decode_split_workspace_bytes(B, Hq, Hkv, seq_len, d) bytes, 16-byte
 * aligned, else TQ_EWORKSPACE.  CUDA cores in fp32: a split over the
 * sequence (blocks of up to 8 query heads by token slices, an online
 * softmax per head) and one merge block per query head. */
size_t tq_decode_split_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int64_t seq_len,
                                       int32_t d);
tq_status tq_decode_attention_split(const tq_quantizer kq[2], const tq_quantizer vq[2],
                                    const void *q, tq_dtype q_dtype, int32_t B, int32_t Hq,
                                    int32_t Hkv, int64_t seq_len, const int32_t *seq_lens,
                                    const tq_cache_view k[2], const tq_cache_view v[2],
                                    float softmax_scale, float *out, void *workspace,
                                    size_t workspace_bytes, tq_stream_t stream);

/* Workspace of tq_search_topk, in bytes (0 when a size is out of range). */
size_t tq_search_workspace_bytes(int32_t n_q, int64_t n_db, int32_t d);

/* Top-k vector search over a packed database ("内存厂商的噩梦来了", section
 * 6.4: TurboQuant as a nearest-neighbour index, database quantized online,
 * full-precision queries).  For each query i (queries: [n_q][d], q_dtype,
 * DEVICE) the k records j < n_db of `db` (record n at n * db->stride_n; the
 * batch and head strides are not used) with the largest estimated inner
 * product
 *   est_j = n_j (<q', c[idx_j]> + [prod] ||r_j|| sqrt(pi/2)/d <S q', sign_j>),
 * q' = Pi q: the decode scores' estimator, computed the same way.  Order:
 * est descending, ties by record index ascending.  top_scores: [n_q][k]
 * fp32, top_index: [n_q][k] int64 (DEVICE); when k > n_db the last k - n_db
 * entries are -inf and -1.  d must be 128 and 1 <= k <= 32; n_db < 2^31.
 * workspace: DEVICE, at least tq_search_workspace_bytes(n_q, n_db, d)
 * bytes, 16-byte aligned, else TQ_EWORKSPACE. */
tq_status tq_search_topk(const tq_quantizer *q, const tq_cache_view *db, int64_t n_db,
                         const void *queries, tq_dtype q_dtype, int32_t n_q, int32_t k,
                         float *top_scores, int64_t *top_index, void *workspace,
                         size_t workspace_bytes, tq_stream_t stream);

/* How the decode's tensor-core split kernel feeds the packed records of a
 * unit-stride cache to its warps, for the whole process (host threads
 * included; calls already enqueued keep the feed they were launched with):
 *   TQ_FEED_REGISTERS (0, the default and the faster one measured on B200):
 *     each warp loads the next chunk's records from global memory straight
 *     into registers while it works on the current one;
 *   TQ_FEED_BULK_STAGED (1): each warp keeps a ring of 2 to 4 shared-memory
 *     slots filled by bulk asynchronous copies (cp.async.bulk, this GPU's
 *     own memory) that complete on one mbarrier per slot, waited on with a
 *     bounded loop (a timeout sets the fault word tq_check reports); the
 *     cache's norm rows must be 16-byte aligned, and a cache or launch that
 *     does not fit it falls back to the register feed.
 * Both compute the same attention ("I Spent 31 Hours On The Math Behind
 * Turboquant", section "KV Cache: The problem"); results agree to rounding.
 * Returns the previous setting, or -1 (setting unchanged) for another value. */
typedef enum { TQ_FEED_REGISTERS = 0, TQ_FEED_BULK_STAGED = 1 } tq_decode_feed;
int32_t tq_set_decode_feed(int32_t feed);

/* Synchronize `stream` and report any asynchronous CUDA error, then read and
 * clear the current GPU's fault word, which the kernels set themselves
 * instead of trapping: TQ_ETIMEOUT when a kernel gave up a bounded wait on
 * data that never arrived (about a second; the outputs of that call are not
 * valid), TQ_ECUDA when a decode launch found its shared-memory layout
 * invalid and wrote nothing.  The word is per GPU, not per stream: it
 * reports every such fault on the device since the last tq_check. */
tq_status tq_check(tq_stream_t stream);

const char *tq_status_string(tq_status s);
/* Message of the last failed call on this host thread ("" if none). */
const char *tq_last_error(void);
const char *tq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
