// Decode attention on the packed TurboQuant cache (sm_100a).
//
// Attention for one new query per head, softmax(q K^T / sqrt(d)) V over all
// cached tokens ("I Spent 31 Hours On The Math Behind Turboquant", section
// "KV Cache: The problem"), with keys scored by the asymmetric estimator: the
// full-precision query against the compressed keys ("内存厂商的噩梦来了",
// section 4.2 and its asymmetric_attention_score):
//   s_j = n_j ( <q', c_K[idx_j]> + [prod] ||r_j|| sqrt(pi/2)/d <S q', sign_j> ),
// q' = Pi_K q the query rotated once.  Values are summed in the value-rotated
// basis, o' = sum_j p_j n_j c_V[idx_j], and rotated back once at the end,
// o = Pi_V^T o'.
//
// Kernel 0 (prep), once per call: rotates every query head (sign flips +
// FWHT, and S q' for prod keys) into the workspace, and for each codebook
// finds a scale s with fp16(s c_k) close to s c_k for every centroid (a
// search over 4096 candidates in [1, 2)) and writes the 256-entry pair table
// entry e -> half2(fp16(s c[e & m]), fp16(s c[(e >> b_m) & m])).
// Kernel 1 (split), persistent: one CTA per SM (12 warps when a kv head has
// <= 4 query heads and the keys are mse, else 8); a warp issues its next
// chunk's key loads as soon as the current keys are scored and its value
// loads once PV is done, and warms L2 with bulk prefetches a window of 4
// chunks ahead.  The work is the flattened space of (unit = batch x kv head
// x group of <= 8 query heads, token) pairs, cut into one equal contiguous
// range per CTA; a range covers one or a few "pieces" (CTA, unit).  When the
// units fit the grid, the host rounds the CTA count down to a multiple of
// the unit count if that idles at most 5% of the SMs, so each CTA stays
// inside one unit.  Per CTA, once: the two pair tables are copied into
// shared memory at address 64 KiB, replicated per lane (entry e, lane l at
// 64 KiB + e*256 + 4l, values at +128) so that table reads never conflict
// on banks and one byte permute forms a lookup's whole address.
// Per piece: the group's rotated queries are split into hi + lo fp16 halves;
// then every warp streams its share of 32-token chunks:
//   * packed K/V words go from HBM straight to registers, one pass;
//   * two adjacent indices (one byte of the bitstream, or a shifted byte for
//     b_m < 4) are one table read -> a half2 of centroids;
//   * scores and PV are mma.m16n8k16 f16 x f16 -> f32: tokens on M for the
//     scores (K-hat [16 tok x 16 dims] x q' [16 dims x 8]), dims on M for PV
//     (V-hat^T [16 dims x 16 tok] x W [16 tok x 8]).  A contraction may
//     permute its summation index as long as both operands agree, so a lane
//     reads contiguous code bytes and q' is laid out to match.  With <= 4
//     query heads per kv head the hi and lo halves of q' (and of the PV
//     weights) share one MMA as columns 0-3 and 4-7; with 5-8 heads they take
//     two MMAs;
//   * QJL bits become +-1 halves with one shift and one LOP3 per pair;
//   * online softmax in base 2 with two running maxima, m over the logits
//     (for the normaliser l) and M over logit + log2 n_V (for the PV weights
//     2^(u - M), which keeps p_j n_j in fp16 range).
// The warps' partials (m, l, M, o') of a piece are merged in shared memory
// and written to workspace slot (unit + CTA index).  Each CTA then bumps its
// unit's counter; the CTA that completes the count merges the unit's slots,
// divides by l and applies Pi_V^T = diag(sigma_V) H / sqrt(d).  No CTA waits
// for another.

#include "../../include/tq.h"
#include "tq_device.cuh"
#include "tq_internal.h"

#include <math.h>

#include <atomic>
#include <mutex>

// Scratch for tq_decode_attention_noalloc: a fixed array in device memory,
// one copy per GPU that loads the library, held until the process exits.
// Host code must not use its name as a device address; the address comes
// from cudaGetSymbolAddress (static_scratch below).
static __device__ __align__(256) unsigned char g_tq_noalloc_scratch[TQ_NOALLOC_SCRATCH_BYTES];

// Faults a kernel detects on its own, one word per GPU (tq::kFault* bits),
// set with atomicOr and read back and cleared by tq_check.
static __device__ unsigned int g_tq_faults;

namespace tq {
namespace {

constexpr int kD = 128;
constexpr int kMaxCtas = 1024;  // persistent CTAs supported (one per SM)
constexpr int kChunk = 32;               // tokens per warp iteration
constexpr int kLutBytes = 256 * 256;     // K and V pair tables, per-lane copies
// Shared-window address of the pair tables.  Entry e, lane l sits at
// kLutAddr + 256 e + 4 l (+128 for the value table): with the tables on a
// 64 KiB boundary, one byte permute of (code byte, lane offset) yields the
// complete shared address of a lookup.
constexpr uint32_t kLutAddr = 0x10000;
constexpr int kPfWin = 4;                // chunks per L2 prefetch window
// The PV weights' reference maximum M moves only when a chunk's maximum of
// logit + log2 n_V passes it by more than kLazy (log2 units); the weights
// then stay below 2^kLazy and most rescales of the accumulators are skipped.
constexpr float kLazy = 8.0f;
constexpr int kPW = kD + 4;              // floats per head in a partial: m, l, M, pad, o'[d]
constexpr int kSlot = 8 * kPW;           // floats per partial slot (8 heads)
constexpr int kScaleCands = 4096;
// workspace layout (floats): [0, 2) scales 1/s_K, 1/s_V; [64, 320) K pair
// table; [320, 576) V pair table; [kHdr, +units * kFragWords) the query
// fragments of every unit; then (units + CTAs) partial slots of kSlot
// floats; then one arrival counter per unit.
constexpr int kHdr = 1024;
// Query fragments of a unit: 64 words per lane, stored as [16][32 lanes][4]
// so that a warp loads 4 words per lane with one coalesced 16-byte load.
// Word w of lane (g8, tig), with q' the unit's rotated queries and
// sel = lo half for PACK lanes g8 >= 4:
//   PACK (<= 4 heads): w = 2s + j      : sel(q'[g8 & 3][32 tig + 4s + 2j, +1])
//                      w = 16 + 2s + j : sel(Sq'[g8 & 3][32 tig + 15 - 2s - j, +16])
//   8 heads          : w = 2s + j / 16 + 2s + j  : hi / lo of q'[g8][32 tig + 4s + 2j, +1]
//                      w = 32 + ... / 48 + ...   : hi / lo of Sq'[g8][32 tig + 15 - 2s - j, +16]
constexpr int kFragWords = 32 * 64;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kKappa = 1.2533141373155003f / (float)kD;  // sqrt(pi/2)/d

struct SplitParams {
  const void *q;
  int q_dtype;
  int B, Hq, Hkv, g, groups;
  int64_t seq_len;
  const int32_t *seq_lens;
  int ctas;
  // keys
  const uint8_t *kc;
  const uint8_t *kj;
  const float *kn;
  const float *kr;
  int64_t ksb, ksh, ksn;
  const float *kcent;
  const int8_t *ksign;
  const float *kS;
  // values
  const uint8_t *vc;
  const float *vn;
  int64_t vsb, vsh, vsn;
  const float *vcent;
  float scale_log2;  // softmax_scale * log2(e)
  float *scores;
  float *ws;
  const uint4 *frag;  // query fragments, kFragWords per unit
  int64_t slot0;      // first float of the partial slots
  unsigned *cnt;      // per-unit arrival counters (zeroed by the prep kernel)
  float *out;
  const int8_t *vsign;
};

struct PrepParams {
  const void *q;
  int q_dtype;
  int nheads;  // B * Hq
  const int8_t *ksign;
  const float *kS;  // prod keys only
  const float *kcent;
  int kbm;
  const float *vcent;
  int vbm;
  float *ws;
  unsigned *cnt;
  int units;
  int Hq, Hkv, g, groups;
  int64_t seq_len;
  const int32_t *seq_lens;
  float *out;
  uint32_t *frag;  // kFragWords per unit
};


// ------------------------------------------------------------------ PTX

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// table entry at shared-window address `addr` (written once, before the
// barrier that precedes every lookup)
__device__ __forceinline__ uint32_t lut(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.b32 %0, [%1];\n" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// fp16 (hi, lo) halves of the pair (a, b): hi = fp16(x), lo = fp16(x - hi)
__device__ __forceinline__ void split_pair(float a, float b, uint32_t &hi, uint32_t &lo) {
  hi = pack_half2(a, b);
  const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hi));
  lo = pack_half2(a - f.x, b - f.y);
}

// hi = fp16(x), lo = fp16(x - hi): x to ~22 significant bits
__device__ __forceinline__ void split_half(float x, float &hi, float &lo) {
  hi = __half2float(__float2half_rn(x));
  lo = x - hi;
}

__device__ __forceinline__ uint32_t pack_hi(float a, float b) {
  float ah, al, bh, bl;
  split_half(a, ah, al);
  split_half(b, bh, bl);
  return pack_half2(ah, bh);
}

__device__ __forceinline__ uint32_t pack_lo(float a, float b) {
  float ah, al, bh, bl;
  split_half(a, ah, al);
  split_half(b, bh, bl);
  return pack_half2(al, bl);
}

// The byte starting `SH` bits up the little-endian word pair (w0, w1), moved
// into byte 1 of the lane's offset (byte 0 = 4*lane, +128 for the value
// table): the entry's byte offset inside the table.
template <int SH>
__device__ __forceinline__ uint32_t lut_addr(uint32_t w0, uint32_t w1, uint32_t laneoff) {
  constexpr int s = SH & 31;
  if constexpr (s % 8 == 0) {
    return __byte_perm(w0, laneoff, 0x7604 | ((s / 8) << 4));
  } else if constexpr (s + 8 <= 32) {
    return __byte_perm(w0 >> s, laneoff, 0x7604);
  } else {
    return __byte_perm(__funnelshift_r(w0, w1, s), laneoff, 0x7604);
  }
}

// pair q (dims 2q, 2q+1) of a BM-bit LSB-first stream held in words W[]
template <int BM, int Q, int NW>
__device__ __forceinline__ uint32_t pair_addr(const uint32_t (&W)[NW], uint32_t laneoff) {
  constexpr int off = 2 * BM * Q;
  constexpr int w = off >> 5;
  constexpr int w1 = (w + 1 < NW) ? w + 1 : w;
  return lut_addr<off>(W[w], W[w1], laneoff);
}

// +-1 half2 from QJL bits (15 - sh, 31 - sh) of w: bit 1 -> +1, bit 0 -> -1
template <int SH>
__device__ __forceinline__ uint32_t qjl_half2(uint32_t w) {
  return ((w << SH) & 0x80008000u) ^ 0xBC00BC00u;
}

template <int BM>
struct VChunk {  // 16 dims of one token: 2*BM bytes
  static constexpr int NW = (2 * BM + 3) / 4;
};

template <int BM>
__device__ __forceinline__ void load_v16(const uint8_t *p, uint32_t (&W)[VChunk<BM>::NW], int g) {
  // bytes [2*BM*g, 2*BM*g + 2*BM) of the record, naturally aligned pieces only
  if constexpr (BM == 4) {
    const uint2 t = __ldg(reinterpret_cast<const uint2 *>(p));
    W[0] = t.x;
    W[1] = t.y;
  } else if constexpr (BM == 2) {
    W[0] = __ldg(reinterpret_cast<const uint32_t *>(p));
  } else if constexpr (BM == 1) {
    W[0] = __ldg(reinterpret_cast<const unsigned short *>(p));
  } else {  // BM == 3: 6 bytes at 6g, 2-byte aligned
    if ((g & 1) == 0) {
      W[0] = __ldg(reinterpret_cast<const uint32_t *>(p));
      W[1] = __ldg(reinterpret_cast<const unsigned short *>(p + 4));
    } else {
      const uint32_t lo = __ldg(reinterpret_cast<const unsigned short *>(p));
      const uint32_t hi = __ldg(reinterpret_cast<const uint32_t *>(p + 2));
      W[0] = lo | (hi << 16);
      W[1] = hi >> 16;
    }
  }
}

template <int BM>
__device__ __forceinline__ void load_k32(const uint8_t *p, uint32_t (&W)[BM > 0 ? BM : 1]) {
  // 4*BM bytes (32 dims) at a 4*BM-aligned offset
  if constexpr (BM == 4) {
    const uint4 t = __ldg(reinterpret_cast<const uint4 *>(p));
    W[0] = t.x;
    W[1] = t.y;
    W[2] = t.z;
    W[3] = t.w;
  } else if constexpr (BM == 2) {
    const uint2 t = __ldg(reinterpret_cast<const uint2 *>(p));
    W[0] = t.x;
    W[1] = t.y;
  } else {
#pragma unroll
    for (int i = 0; i < (BM > 0 ? BM : 1); ++i) W[i] = __ldg(reinterpret_cast<const uint32_t *>(p) + i);
  }
}

// ----------------------------------------------------------- work split

// Length of the units of batch b.
__device__ __forceinline__ int64_t batch_len(const int32_t *seq_lens, int64_t seq_len, int b) {
  if (!seq_lens) return seq_len;
  const int64_t L = seq_lens[b];
  return L < 0 ? 0 : (L > seq_len ? seq_len : L);
}

// Flattened space: units u = (b, kvh, grp) in that order, unit u of batch b
// spans batch_len(b) tokens.  Returns the total; *pb gets the start of batch
// `bq`'s first unit (when bq >= 0).
__device__ __forceinline__ int64_t flat_total(const int32_t *seq_lens, int64_t seq_len, int B, int UH) {
  if (!seq_lens) return (int64_t)B * UH * seq_len;
  int64_t t = 0;
  for (int b = 0; b < B; ++b) t += batch_len(seq_lens, seq_len, b) * UH;
  return t;
}

// CTA c covers [cut(c), cut(c+1)).
__device__ __forceinline__ int64_t cut(int64_t T, int C, int c) {
  return (int64_t)(((uint64_t)T * (uint64_t)c) / (uint64_t)C);  // T * C < 2^64 for any real cache
}

// Unit containing flattened position x (x < T): unit index, its start, length.
__device__ __forceinline__ void locate(const int32_t *seq_lens, int64_t seq_len, int B, int UH, int64_t x,
                                       int *u, int64_t *start, int64_t *len) {
  if (!seq_lens) {
    const int64_t uu = x / seq_len;
    *u = (int)uu;
    *start = uu * seq_len;
    *len = seq_len;
    return;
  }
  int64_t base = 0;
  for (int b = 0; b < B; ++b) {
    const int64_t L = batch_len(seq_lens, seq_len, b);
    const int64_t span = L * UH;
    if (x < base + span) {
      const int64_t r = (x - base) / L;
      *u = b * UH + (int)r;
      *start = base + r * L;
      *len = L;
      return;
    }
    base += span;
  }
  *u = B * UH - 1;
  *start = base;
  *len = 0;
}

// ------------------------------------------------------------- prep kernel

// Index i in [0, kScaleCands) minimising the worst relative fp16 rounding
// error of (1 + i/kScaleCands) * c_k over the K/2 positive centroids (ties ->
// smallest i); then the pair table for that scale.  One 256-thread block.
__device__ void scale_and_table(const float *cent, int bm, float *inv_scale, uint32_t *table) {
  __shared__ uint64_t s_red[8];
  __shared__ float s_c[16];
  const int K = 1 << bm;
  if (threadIdx.x < K) s_c[threadIdx.x] = cent[threadIdx.x];
  __syncthreads();
  float c[8], rc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    c[k] = K / 2 + k < K ? s_c[K / 2 + k] : s_c[K - 1];
    rc[k] = 1.0f / c[k];
  }
  uint64_t best = ~0ull;
  for (int i = threadIdx.x; i < kScaleCands; i += blockDim.x) {
    const float s = 1.0f + (float)i * (1.0f / kScaleCands);
    float worst = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float v = s * c[k];
      worst = fmaxf(worst, fabsf(__half2float(__float2half_rn(v)) - v) * rc[k]);
    }
    const uint64_t key = ((uint64_t)__float_as_uint(worst) << 32) | (uint32_t)i;
    best = key < best ? key : best;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const uint64_t other = __shfl_xor_sync(dev::kFull, best, o);
    best = other < best ? other : best;
  }
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = best;
  __syncthreads();
  uint64_t b = ~0ull;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) b = s_red[w] < b ? s_red[w] : b;
  const float sc = 1.0f + (float)(uint32_t)(b & 0xffffffffu) * (1.0f / kScaleCands);
  const uint32_t m = (uint32_t)K - 1u;
  for (int e = threadIdx.x; e < 256; e += blockDim.x)
    table[e] = pack_half2(sc * s_c[e & m], sc * s_c[(e >> bm) & m]);
  if (threadIdx.x == 0) *inv_scale = 1.0f / sc;
}

// Blocks [0, nheads/2): two query heads each (128 threads per head):
// q' = H(sigma q)/sqrt(d) and q_s = S q'.  The last two blocks: the K and
// V scale and pair table.
__global__ void __launch_bounds__(256) decode_prep_kernel(PrepParams p) {
  // the split kernel may be scheduled now: it waits for this grid to finish
  // (griddepcontrol.wait) before it reads anything written here
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  const int nqb = (p.nheads + 1) / 2;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.units; i += gridDim.x * blockDim.x) p.cnt[i] = 0u;
  if ((int)blockIdx.x >= nqb) {
    if (blockIdx.x == (unsigned)nqb) {
      if (p.kbm > 0) scale_and_table(p.kcent, p.kbm, p.ws + 0, reinterpret_cast<uint32_t *>(p.ws + 64));
      else if (threadIdx.x == 0) p.ws[0] = 1.0f;
    } else {
      scale_and_table(p.vcent, p.vbm, p.ws + 1, reinterpret_cast<uint32_t *>(p.ws + 320));
    }
    return;
  }
  __shared__ float s_q[2][kD], s_qs[2][kD];
  const int half = threadIdx.x >> 7, t = threadIdx.x & 127;
  const int head = blockIdx.x * 2 + half;
  const bool valid = head < p.nheads;
  // a batch with no cached tokens has no work piece: its output is zero
  if (valid && p.seq_lens && batch_len(p.seq_lens, p.seq_len, head / p.Hq) == 0)
    p.out[(int64_t)head * kD + t] = 0.f;
  const int lane = threadIdx.x & 31;
  if ((t >> 5) == 0) {  // one warp per head: 4 dims per lane
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    if (valid) {
      const int64_t qoff = (int64_t)head * kD + lane * 4;
      if (p.q_dtype == TQ_F32) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(p.q) + qoff / 4);
        a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
      } else {
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(static_cast<const char *>(p.q) + qoff * 2));
        if (p.q_dtype == TQ_BF16) {
          a[0] = dev::bf16lo(v.x); a[1] = dev::bf16hi(v.x); a[2] = dev::bf16lo(v.y); a[3] = dev::bf16hi(v.y);
        } else {
          a[0] = dev::f16lo(v.x); a[1] = dev::f16hi(v.x); a[2] = dev::f16lo(v.y); a[3] = dev::f16hi(v.y);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (p.ksign[lane * 4 + i] < 0) a[i] = -a[i];
    }
    dev::fwht<32, 4>(a, lane);
#pragma unroll
    for (int i = 0; i < 4; ++i) s_q[half][lane * 4 + i] = a[i] * 0.08838834764831845f;
  }
  __syncthreads();
  if (valid && p.kS) {
    const float4 *Sk = reinterpret_cast<const float4 *>(p.kS + (size_t)t * kD);
    float acc = 0.f;
#pragma unroll 8
    for (int i = 0; i < kD / 4; ++i) {
      const float4 sv = __ldg(Sk + i);
      acc = fmaf(sv.x, s_q[half][4 * i], acc);
      acc = fmaf(sv.y, s_q[half][4 * i + 1], acc);
      acc = fmaf(sv.z, s_q[half][4 * i + 2], acc);
      acc = fmaf(sv.w, s_q[half][4 * i + 3], acc);
    }
    s_qs[half][t] = acc;
  }
  __syncthreads();
  if (!valid) return;
  // this head's fragment words (the layout of kFragWords above)
  const int b = head / p.Hq, hq = head % p.Hq;
  const int kvh = hq / p.g, grp = (hq % p.g) / 8, hh = (hq % p.g) % 8;
  const int64_t u = ((int64_t)b * p.Hkv + kvh) * p.groups + grp;
  uint32_t *fu = p.frag + u * kFragWords;
  auto put = [&](int ln, int w, uint32_t v) { fu[((w >> 2) * 32 + ln) * 4 + (w & 3)] = v; };
  const float *qv = s_q[half], *sv = s_qs[half];
  if (p.g <= 4) {
    const int ls = t >> 4, w = t & 15, sidx = w >> 1, j = w & 1;
    const int g8 = hh + 4 * (ls >> 2), tig = ls & 3, ln = g8 * 4 + tig;
    const bool lo = g8 >= 4;
    const int d0 = 32 * tig + 4 * sidx + 2 * j;
    put(ln, w, lo ? pack_lo(qv[d0], qv[d0 + 1]) : pack_hi(qv[d0], qv[d0 + 1]));
    if (p.kS) {
      const int e = 32 * tig + 15 - 2 * sidx - j;
      put(ln, 16 + w, lo ? pack_lo(sv[e], sv[e + 16]) : pack_hi(sv[e], sv[e + 16]));
    }
  } else {
    const int tig = t >> 5, w = t & 31, sidx = (w & 15) >> 1, j = w & 1;
    const int ln = hh * 4 + tig;
    const bool lo = w >= 16;
    const int d0 = 32 * tig + 4 * sidx + 2 * j;
    put(ln, w, lo ? pack_lo(qv[d0], qv[d0 + 1]) : pack_hi(qv[d0], qv[d0 + 1]));
    if (p.kS) {
      const int e = 32 * tig + 15 - 2 * sidx - j;
      put(ln, 32 + w, lo ? pack_lo(sv[e], sv[e + 16]) : pack_hi(sv[e], sv[e + 16]));
    }
  }
  // When this grid was launched early after the new tokens' encode (the
  // fused append + decode chain), one thread waits for that grid, so this
  // grid completes after it and the split kernel's wait covers both.  Head 0
  // (block 0, thread 0) always reaches this point.  Without such a launch
  // the wait returns at once.
  if (blockIdx.x == 0 && threadIdx.x == 0) asm volatile("griddepcontrol.wait;\n" ::: "memory");
}

// ------------------------------------------------------------ split kernel

// One lane's loads for the key side of a 32-token chunk: score rows (ms, r)
// are tokens 16 ms + 8 r + g8 of the chunk.  The value norms of the same
// rows ride along (the softmax needs log2 n_V before PV).
template <int KBM, bool KPROD>
struct KBuf {
  uint32_t w[2][2][KBM > 0 ? KBM : 1];
  uint32_t qj[2][2];
  float kn[2][2], kr[2][2], vn[2][2];
};

// The value codes of a chunk: PV tokens (ms, q4) are 16 ms + 2 tig +
// (q4 & 1) + 8 (q4 >> 1), 16 dims [16 g8, 16 g8 + 16) each.
template <int VBM>
struct VBuf {
  uint32_t w[2][4][VChunk<VBM>::NW];
};

// Loads the key side of one chunk with any record strides and nvalid <= 32
// valid tokens (rows past nvalid are masked: norm -1).  Row offsets are
// computed here, so nothing of this path stays live across the main loop.
template <int KBM, bool KPROD>
__device__ __forceinline__ void load_k_slow(KBuf<KBM, KPROD> &c, const SplitParams &p, int64_t krec0, int64_t vrec0,
                                            int nvalid, int tig, int g8) {
  constexpr int KCB = kD * KBM / 8;
#pragma unroll
  for (int ms = 0; ms < 2; ++ms) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int t = 16 * ms + 8 * r + g8;
      const bool ok = t < nvalid;
      const int64_t rec = krec0 + (int64_t)t * p.ksn;
      if constexpr (KBM > 0) {
        if (ok) {
          load_k32<KBM>(p.kc + rec * KCB + tig * (4 * KBM), c.w[ms][r]);
        } else {
#pragma unroll
          for (int i = 0; i < KBM; ++i) c.w[ms][r][i] = 0u;
        }
      }
      if constexpr (KPROD) {
        c.qj[ms][r] = ok ? __ldg(reinterpret_cast<const uint32_t *>(p.kj + rec * (kD / 8)) + tig) : 0u;
        c.kr[ms][r] = ok ? __ldg(p.kr + rec) : 0.f;
      }
      c.kn[ms][r] = ok ? __ldg(p.kn + rec) : -1.f;  // -1 marks a masked row
      c.vn[ms][r] = ok ? __ldg(p.vn + vrec0 + (int64_t)t * p.vsn) : 1.f;
    }
  }
}

// Per-lane pointers of the fast path (unit record strides) at chunk 0 of a
// piece; chunk c adds c * kChunk records.
template <int KBM, bool KPROD, int VBM>
struct FastPtrs {
  const uint8_t *kc;
  const uint32_t *kj;
  const float *kn, *kr, *vn;
  const uint8_t *vc;
};

template <int KBM, bool KPROD, int VBM>
__device__ __forceinline__ FastPtrs<KBM, KPROD, VBM> fast_ptrs(const SplitParams &p, int64_t krec0, int64_t vrec0,
                                                               int tig, int g8) {
  constexpr int KCB = kD * KBM / 8, VCB = kD * VBM / 8;
  FastPtrs<KBM, KPROD, VBM> f;
  const int64_t kr0 = krec0 + g8, vr0 = vrec0 + g8;
  f.kc = p.kc + kr0 * KCB + tig * (4 * KBM);
  f.kj = KPROD ? reinterpret_cast<const uint32_t *>(p.kj + kr0 * (kD / 8)) + tig : nullptr;
  f.kn = p.kn + kr0;
  f.kr = KPROD ? p.kr + kr0 : nullptr;
  f.vn = p.vn + vr0;
  f.vc = p.vc + (vrec0 + 2 * tig) * VCB + g8 * (2 * VBM);
  return f;
}

// Key side of full chunk c through the fast-path pointers.
template <int KBM, bool KPROD, int VBM>
__device__ __forceinline__ void load_k_fast(KBuf<KBM, KPROD> &c, const FastPtrs<KBM, KPROD, VBM> &f, int ci) {
  constexpr int KCB = kD * KBM / 8;
  const int64_t r0 = (int64_t)ci * kChunk;
#pragma unroll
  for (int ms = 0; ms < 2; ++ms) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int t = 16 * ms + 8 * r;
      if constexpr (KBM > 0) load_k32<KBM>(f.kc + (r0 + t) * KCB, c.w[ms][r]);
      if constexpr (KPROD) {
        c.qj[ms][r] = __ldg(f.kj + (r0 + t) * (kD / 32));
        c.kr[ms][r] = __ldg(f.kr + r0 + t);
      }
      c.kn[ms][r] = __ldg(f.kn + r0 + t);
      c.vn[ms][r] = __ldg(f.vn + r0 + t);
    }
  }
}

// Value side of full chunk c through the fast-path pointers.
template <int KBM, bool KPROD, int VBM>
__device__ __forceinline__ void load_v_fast(VBuf<VBM> &c, const FastPtrs<KBM, KPROD, VBM> &f, int ci, int g8) {
  constexpr int VCB = kD * VBM / 8;
  const int64_t r0 = (int64_t)ci * kChunk;
#pragma unroll
  for (int ms = 0; ms < 2; ++ms) {
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4)
      load_v16<VBM>(f.vc + (r0 + 16 * ms + (q4 & 1) + 8 * (q4 >> 1)) * VCB, c.w[ms][q4], g8);
  }
}

// Value side of one chunk with any record strides and nvalid <= 32 valid
// tokens (rows past nvalid read as code 0; their weights are 0).
template <int VBM>
__device__ __forceinline__ void load_v_slow(VBuf<VBM> &c, const SplitParams &p, int64_t vrec0, int nvalid, int g8,
                                            int tig) {
  constexpr int VCB = kD * VBM / 8;
  constexpr int NW = VChunk<VBM>::NW;
#pragma unroll
  for (int ms = 0; ms < 2; ++ms) {
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const int t = 16 * ms + 2 * tig + (q4 & 1) + 8 * (q4 >> 1);
      if (t < nvalid) {
        load_v16<VBM>(p.vc + (vrec0 + (int64_t)t * p.vsn) * VCB + g8 * (2 * VBM), c.w[ms][q4], g8);
      } else {
#pragma unroll
        for (int i = 0; i < NW; ++i) c.w[ms][q4][i] = 0u;
      }
    }
  }
}

// L2 prefetch hint for [ptr, ptr + bytes), shrunk inwards to 16-byte
// boundaries so that every prefetched byte lies inside the range.
__device__ __forceinline__ void prefetch_l2(const void *ptr, int64_t bytes) {
  const uint64_t lo = ((uint64_t)ptr + 15u) & ~(uint64_t)15u;
  const uint64_t hi = ((uint64_t)ptr + (uint64_t)bytes) & ~(uint64_t)15u;
  if (hi > lo)
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(lo), "r"((uint32_t)(hi - lo)) : "memory");
}

// Prefetches the packed records of tokens [j, j + n) of one (batch, kv head)
// slice into L2 (unit record strides only).
template <int KBM, bool KPROD, int VBM>
__device__ __forceinline__ void prefetch_chunk(const SplitParams &p, int64_t kr, int64_t vr, int64_t n) {
  constexpr int KCB = kD * KBM / 8, VCB = kD * VBM / 8;
  if constexpr (KBM > 0) prefetch_l2(p.kc + kr * KCB, n * KCB);
  prefetch_l2(p.vc + vr * VCB, n * VCB);
  prefetch_l2(p.kn + kr, n * 4);
  prefetch_l2(p.vn + vr, n * 4);
  if constexpr (KPROD) {
    prefetch_l2(p.kj + kr * (kD / 8), n * (kD / 8));
    prefetch_l2(p.kr + kr, n * 4);
  }
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Merge the slots of unit u (heads < gh) and write out[b, h0 + hh, :] =
// sigma_V * H (o'/l) / sqrt(d).  The CTA's warps split the work as (head,
// part): warp (hh, part) merges a contiguous share of the slots, 4 dims per
// lane, kMergeBatch slots at a time with an online rescale.  Every load of a
// batch (the slot headers, broadcast to all lanes, and the lane's 4 dims) is
// issued before any is used, so a batch costs one round trip to L2.  The
// parts of a head are then combined through shared memory by one warp,
// which applies the inverse rotation.  CTAs with an empty range never wrote
// their slot and are skipped.  Called by every thread of the CTA.
constexpr int kMergeBatch = 8;

__device__ void merge_unit(const SplitParams &p, const int64_t *cuts, int u, int c0, int c1, int b, int h0,
                           int gh, int warp, int nwarps, int lane, float *s_m) {
  const int n = c1 - c0 + 1;
  const int parts = nwarps / gh;  // gh <= 8 <= nwarps
  // the value rotation's signs for this lane's 4 dims, loaded alongside the
  // slots (byte loads: the sign array carries no alignment promise)
  const int8_t sg0 = p.vsign[lane * 4], sg1 = p.vsign[lane * 4 + 1];
  const int8_t sg2 = p.vsign[lane * 4 + 2], sg3 = p.vsign[lane * 4 + 3];
  if (warp < gh * parts) {
    const int hh = warp % gh, part = warp / gh;
    const int i_lo = part * n / parts, i_hi = (part + 1) * n / parts;
    const float *slots = p.ws + p.slot0 + ((int64_t)u + c0) * kSlot + hh * kPW;
    float m_run = -INFINITY, M_run = -INFINITY, l = 0.f;
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i0 = i_lo; i0 < i_hi; i0 += kMergeBatch) {
      float4 hd[kMergeBatch], v[kMergeBatch];
#pragma unroll
      for (int j = 0; j < kMergeBatch; ++j) {
        const int i = i0 + j;
        const bool live = i < i_hi && cuts[c0 + i + 1] > cuts[c0 + i];
        const float *sl = slots + (int64_t)(live ? i : 0) * kSlot;
        hd[j] = live ? __ldcg(reinterpret_cast<const float4 *>(sl)) : make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
        v[j] = live ? __ldcg(reinterpret_cast<const float4 *>(sl + 4 + lane * 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float mb = m_run, Mb = M_run;
#pragma unroll
      for (int j = 0; j < kMergeBatch; ++j) {
        mb = fmaxf(mb, hd[j].x);
        Mb = fmaxf(Mb, hd[j].z);
      }
      const float ms = mb == -INFINITY ? 0.f : mb, Ms = Mb == -INFINITY ? 0.f : Mb;
      l *= ex2(m_run - ms);
      const float r = ex2(M_run - Ms);
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] *= r;
      m_run = mb;
      M_run = Mb;
#pragma unroll
      for (int j = 0; j < kMergeBatch; ++j) {
        l = fmaf(hd[j].y, ex2(hd[j].x - ms), l);
        const float w = ex2(hd[j].z - Ms);
        a[0] = fmaf(v[j].x, w, a[0]);
        a[1] = fmaf(v[j].y, w, a[1]);
        a[2] = fmaf(v[j].z, w, a[2]);
        a[3] = fmaf(v[j].w, w, a[3]);
      }
    }
    float *mine = s_m + warp * kPW;
    if (lane == 0) {
      mine[0] = m_run;
      mine[1] = l;
      mine[2] = M_run;
    }
    *reinterpret_cast<float4 *>(mine + 4 + lane * 4) = make_float4(a[0], a[1], a[2], a[3]);
  }
  __syncthreads();
  if (warp < gh) {
    const int hh = warp;
    float m_all = -INFINITY, M_all = -INFINITY;
    for (int part = 0; part < parts; ++part) {
      m_all = fmaxf(m_all, s_m[(part * gh + hh) * kPW + 0]);
      M_all = fmaxf(M_all, s_m[(part * gh + hh) * kPW + 2]);
    }
    float *out = p.out + ((int64_t)b * p.Hq + h0 + hh) * kD + lane * 4;
    if (m_all == -INFINITY) {
      *reinterpret_cast<float4 *>(out) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      const float Ms = M_all == -INFINITY ? 0.f : M_all;
      float l = 0.f, a[4] = {0.f, 0.f, 0.f, 0.f};
      for (int part = 0; part < parts; ++part) {
        const float *q = s_m + (part * gh + hh) * kPW;
        l = fmaf(q[1], ex2(q[0] - m_all), l);
        const float w = ex2(q[2] - Ms);
        const float4 v = *reinterpret_cast<const float4 *>(q + 4 + lane * 4);
        a[0] = fmaf(v.x, w, a[0]);
        a[1] = fmaf(v.y, w, a[1]);
        a[2] = fmaf(v.z, w, a[2]);
        a[3] = fmaf(v.w, w, a[3]);
      }
      const float f = ex2(Ms - m_all) / l * 0.08838834764831845f;
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] *= f;
      dev::fwht<32, 4>(a, lane);
      float o4[4];
      o4[0] = sg0 < 0 ? -a[0] : a[0];
      o4[1] = sg1 < 0 ? -a[1] : a[1];
      o4[2] = sg2 < 0 ? -a[2] : a[2];
      o4[3] = sg3 < 0 ? -a[3] : a[3];
      *reinterpret_cast<float4 *>(out) = make_float4(o4[0], o4[1], o4[2], o4[3]);
    }
  }
}

// Largest CTA index c with cuts[c] <= x: the CTA whose range holds x (CTAs
// with empty ranges share their start with the next non-empty one, so the
// largest index is the non-empty one).
__device__ __forceinline__ int cta_of(const int64_t *cuts, int C, int64_t x) {
  int lo = 0, hi = C - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cuts[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int KBM, bool KPROD, int VBM, bool PACK>
__global__ void __launch_bounds__((PACK && !KPROD ? 12 : 8) * 32, 1) decode_split_kernel(SplitParams p) {
  constexpr int kWarps = PACK && !KPROD ? 12 : 8;
  constexpr int kThreads = kWarps * 32;
  constexpr int KW = KBM > 0 ? KBM : 1;
  constexpr int VW = VChunk<VBM>::NW;
  extern __shared__ float4 smem4[];
  char *smem = reinterpret_cast<char *>(smem4);
  // [kLutAddr, +64 KB): the pair tables; then the warps' partials.  The
  // host sizes the allocation to reach past kLutAddr + kLutBytes + partials
  // from any dynamic base at or below kLutAddr.
  const uint32_t dyn_base = static_cast<uint32_t>(__cvta_generic_to_shared(smem4));
  if (dyn_base > kLutAddr) {  // excluded on the host; reported, never silent
    if (threadIdx.x == 0) atomicOr(&g_tq_faults, kFaultSmemLayout);
    return;
  }
  char *s_lut = smem + (kLutAddr - dyn_base);
  float *s_part = reinterpret_cast<float *>(s_lut + kLutBytes);  // [kWarps][8][kPW]
  __shared__ int s_last;
  __shared__ int64_t s_cut[kMaxCtas + 1];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g8 = lane >> 2, tig = lane & 3;
  const int UH = p.Hkv * p.groups;
  const int64_t T = flat_total(p.seq_lens, p.seq_len, p.B, UH);
  const int64_t x0 = cut(T, p.ctas, blockIdx.x), x1 = cut(T, p.ctas, blockIdx.x + 1);
  if (x0 >= x1) return;
  const bool unit = p.ksn == 1 && p.vsn == 1;
  // warm L2 with this warp's first two chunks while the tables are set up
  if (unit && lane == 0) {
    int u;
    int64_t ustart, ulen;
    locate(p.seq_lens, p.seq_len, p.B, UH, x0, &u, &ustart, &ulen);
    const int64_t t0 = x0 - ustart, t1 = min(x1, ustart + ulen) - ustart;
    const int64_t nch = (t1 - t0 + kChunk - 1) / kChunk, pw = (nch + kWarps - 1) / kWarps;
    const int64_t cb = min(nch, (int64_t)warp * pw), ce = min(nch, cb + pw);
    const int b = u / UH, kvh = (u % UH) / p.groups;
    if (cb < ce) {
      const int64_t j = t0 + cb * kChunk;
      prefetch_chunk<KBM, KPROD, VBM>(p, (int64_t)b * p.ksb + (int64_t)kvh * p.ksh + j,
                                      (int64_t)b * p.vsb + (int64_t)kvh * p.vsh + j, min(2 * (int64_t)kChunk, t1 - j));
    }
  }

  for (int c = tid; c <= p.ctas; c += kThreads) s_cut[c] = cut(T, p.ctas, c);
  // Everything above reads only the arguments and the cache; the workspace
  // (tables, query fragments, counters) is written by the prep kernel, which may still be
  // running when this grid starts (programmatic dependent launch).
  asm volatile("griddepcontrol.wait;\n" ::: "memory");

  // ---- once per CTA: the two pair tables (512 words), every load in
  // flight before any store, staged in shared memory, then one copy per lane
  float inv_sK, inv_sV;
  {
    const uint32_t *ktab = reinterpret_cast<const uint32_t *>(p.ws + 64);
    const uint32_t *vtab = reinterpret_cast<const uint32_t *>(p.ws + 320);
    uint32_t *stage = reinterpret_cast<uint32_t *>(s_part);
    static_assert(kThreads >= 256, "two staging loads per thread cover the 512 words");
    const int i0 = tid, i1 = tid + kThreads;
    uint32_t v0 = 0u, v1 = 0u;
    if (i0 < 256) v0 = KBM > 0 ? __ldg(ktab + i0) : 0u;
    else if (i0 < 512) v0 = __ldg(vtab + (i0 - 256));
    if (i1 < 512) v1 = __ldg(vtab + (i1 - 256));
    inv_sK = __ldg(p.ws + 0);
    inv_sV = __ldg(p.ws + 1);
    if (i0 < 512) stage[i0] = v0;
    if (i1 < 512) stage[i1] = v1;
    __syncthreads();
    uint4 *tab = reinterpret_cast<uint4 *>(s_lut);
    for (int i = tid; i < 256 * 16; i += kThreads) {  // 16 uint4 per 256-byte row
      const int e = i >> 4, part = i & 15;
      const uint32_t v = stage[part < 8 ? e : 256 + e];
      tab[i] = make_uint4(v, v, v, v);
    }
  }
  const float sK = 1.0f / inv_sK;
  const float kscale = inv_sK * p.scale_log2;  // logit = raw score * n_K * kscale
  const uint32_t koff = kLutAddr + lane * 4;
  const uint32_t voff = kLutAddr + 128 + lane * 4;
  const bool want_scores = p.scores != nullptr;

  for (int64_t x = x0; x < x1;) {
    int u;
    int64_t ustart, ulen;
    locate(p.seq_lens, p.seq_len, p.B, UH, x, &u, &ustart, &ulen);
    const int64_t t0 = x - ustart;
    const int64_t t1 = min(x1, ustart + ulen) - ustart;
    x = ustart + t1;
    const int b = u / UH;
    const int kvh = (u % UH) / p.groups;
    const int grp = (u % UH) % p.groups;
    const int h0 = kvh * p.g + grp * 8;
    const int gh = min(8, p.g - grp * 8);

    __syncthreads();  // tables ready / the previous piece's shared data consumed

    // ---- B fragments of the unit, written by the prep kernel in this
    // lane's register order.  PACK: column n < 4 is the hi half of head n,
    // n >= 4 the lo half of head n - 4.  Else qf = hi and qf2 = lo of head
    // g8.  Lanes whose head is absent (fewer than 4 or 8 heads) hold zeros.
    uint32_t qf[8][2], qf2[PACK ? 1 : 8][2];
    uint32_t qsf[KPROD ? 8 : 1][2], qsf2[(KPROD && !PACK) ? 8 : 1][2];
    {
      const bool has = (PACK ? (g8 & 3) : g8) < gh;
      const uint4 *fr = p.frag + (int64_t)u * (kFragWords / 4) + lane;
      auto ld4 = [&](int w4) { return has ? __ldg(fr + w4 * 32) : make_uint4(0u, 0u, 0u, 0u); };
      auto put = [](uint32_t (&f)[8][2], int k, uint4 v) {
        f[2 * k][0] = v.x;
        f[2 * k][1] = v.y;
        f[2 * k + 1][0] = v.z;
        f[2 * k + 1][1] = v.w;
      };
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        put(qf, k, ld4(k));
        if constexpr (!PACK) put(qf2, k, ld4(4 + k));
        if constexpr (KPROD) put(qsf, k, ld4((PACK ? 4 : 8) + k));
        if constexpr (KPROD && !PACK) put(qsf2, k, ld4(12 + k));
      }
    }

    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, M_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};

    const int64_t kbase = (int64_t)b * p.ksb + (int64_t)kvh * p.ksh;
    const int64_t vbase = (int64_t)b * p.vsb + (int64_t)kvh * p.vsh;
    // the piece's chunks [0, nch), of which [0, nfull) are full; this warp
    // takes [c_begin, c_end).  A piece is shorter than 2^31 tokens.
    const int nch = (int)((t1 - t0 + kChunk - 1) / kChunk);
    const int nfull = (int)((t1 - t0) / kChunk);
    const int per_warp = (nch + kWarps - 1) / kWarps;
    const int c_begin = min(nch, warp * per_warp);
    const int c_end = min(nch, c_begin + per_warp);
    const FastPtrs<KBM, KPROD, VBM> fp = fast_ptrs<KBM, KPROD, VBM>(p, kbase + t0, vbase + t0, tig, g8);

    KBuf<KBM, KPROD> kb;
    VBuf<VBM> vb;
    // warm L2 up to the end of the first prefetch window
    if (unit && lane == 0 && c_begin + 1 < c_end) {
      const int64_t jp = t0 + (int64_t)(c_begin + 1) * kChunk;
      const int pe = min(c_end, c_begin + kPfWin);
      prefetch_chunk<KBM, KPROD, VBM>(p, kbase + jp, vbase + jp, min((int64_t)(pe - c_begin - 1) * kChunk, t1 - jp));
    }
    if (c_begin < c_end) {
      if (unit && c_begin < nfull) {
        load_k_fast(kb, fp, c_begin);
        load_v_fast(vb, fp, c_begin, g8);
      } else {
        const int64_t j0 = t0 + (int64_t)c_begin * kChunk;
        const int nv = (int)min((int64_t)kChunk, t1 - j0);
        load_k_slow(kb, p, kbase + j0 * p.ksn, vbase + j0 * p.vsn, nv, tig, g8);
        load_v_slow(vb, p, vbase + j0 * p.vsn, nv, g8, tig);
      }
    }
    for (int ci = c_begin; ci < c_end; ++ci) {
      const int cn = ci + 1;
      const bool more = cn < c_end;
      const bool fast_next = unit && cn < nfull;
      // every kPfWin chunks, warm L2 with the window after the next one
      if (unit && lane == 0 && ((ci - c_begin) % kPfWin) == 0 && ci + kPfWin < c_end) {
        const int64_t jp = t0 + (int64_t)(ci + kPfWin) * kChunk;
        const int pe = min(c_end, ci + 2 * kPfWin);
        prefetch_chunk<KBM, KPROD, VBM>(p, kbase + jp, vbase + jp,
                                        min((int64_t)(pe - ci - kPfWin) * kChunk, t1 - jp));
      }
      // -------- scores: rows (ms, r) -> token 32 ci + 16 ms + 8 r + g8
      float sc[2][4];
      float nvl[2][2];  // log2 n_V of the lane's rows
#pragma unroll
      for (int ms = 0; ms < 2; ++ms) {
        const auto &kw = kb.w[ms];
        const auto &qj = kb.qj[ms];
        bool ok[2];
        float fs[2], kr[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          ok[r] = kb.kn[ms][r] >= 0.f;
          fs[r] = kb.kn[ms][r] * kscale;
          kr[r] = KPROD ? kb.kr[ms][r] * (kKappa * sK) : 0.f;  // the table holds s_K c
          nvl[ms][r] = ok[r] ? __log2f(kb.vn[ms][r]) : -INFINITY;
        }
        float cm[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (KBM > 0) {
#define TQ_KSTEP(S)                                                               \
  {                                                                               \
    uint32_t a[4];                                                                \
    a[0] = lut(pair_addr<KBM, 2 * (S), KW>(kw[0], koff));                         \
    a[1] = lut(pair_addr<KBM, 2 * (S), KW>(kw[1], koff));                         \
    a[2] = lut(pair_addr<KBM, 2 * (S) + 1, KW>(kw[0], koff));                     \
    a[3] = lut(pair_addr<KBM, 2 * (S) + 1, KW>(kw[1], koff));                     \
    mma16816(cm, a, qf[S][0], qf[S][1]);                                          \
    if constexpr (!PACK) mma16816(cm, a, qf2[S][0], qf2[S][1]);                   \
  }
          TQ_KSTEP(0) TQ_KSTEP(1) TQ_KSTEP(2) TQ_KSTEP(3)
          TQ_KSTEP(4) TQ_KSTEP(5) TQ_KSTEP(6) TQ_KSTEP(7)
#undef TQ_KSTEP
        }
        float cq[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (KPROD) {
#define TQ_QSTEP(S)                                                               \
  {                                                                               \
    uint32_t a[4];                                                                \
    a[0] = qjl_half2<2 * (S)>(qj[0]);                                             \
    a[1] = qjl_half2<2 * (S)>(qj[1]);                                             \
    a[2] = qjl_half2<2 * (S) + 1>(qj[0]);                                         \
    a[3] = qjl_half2<2 * (S) + 1>(qj[1]);                                         \
    mma16816(cq, a, qsf[S][0], qsf[S][1]);                                        \
    if constexpr (!PACK) mma16816(cq, a, qsf2[S][0], qsf2[S][1]);                 \
  }
          TQ_QSTEP(0) TQ_QSTEP(1) TQ_QSTEP(2) TQ_QSTEP(3)
          TQ_QSTEP(4) TQ_QSTEP(5) TQ_QSTEP(6) TQ_QSTEP(7)
#undef TQ_QSTEP
        }
        // raw score = main + kappa gamma s_K qjl (the table holds s_K c)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float s = cm[i];
          if constexpr (KPROD) s = fmaf(kr[i >> 1], cq[i], s);
          if constexpr (PACK) s += __shfl_xor_sync(dev::kFull, s, 2);  // hi + lo columns
          cm[i] = s;
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
#pragma unroll
          for (int c = 0; c < 2; ++c) sc[ms][2 * r + c] = ok[r] ? cm[2 * r + c] * fs[r] : -INFINITY;
        }
        if (want_scores) {
#pragma unroll
          for (int r = 0; r < 2; ++r) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const int head = PACK ? 2 * (tig & 1) + c : 2 * tig + c;
              if (ok[r] && head < gh && (!PACK || tig < 2)) {
                const int64_t j = t0 + (int64_t)ci * kChunk + 16 * ms + 8 * r + g8;
                p.scores[((int64_t)b * p.Hq + h0 + head) * p.seq_len + j] =
                    cm[2 * r + c] * (kb.kn[ms][r] * inv_sK);
              }
            }
          }
        }
      }
      // the key registers are free: start the next chunk's key loads
      if (more) {
        if (fast_next) {
          load_k_fast(kb, fp, cn);
        } else {
          const int64_t jn = t0 + (int64_t)cn * kChunk;
          load_k_slow(kb, p, kbase + jn * p.ksn, vbase + jn * p.vsn, (int)min((int64_t)kChunk, t1 - jn), tig, g8);
        }
      }

      // -------- online softmax, per head column c
      float wgt[2][4];
      float aM[2];
      bool moved = false;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float mx = fmaxf(fmaxf(sc[0][c], sc[0][2 + c]), fmaxf(sc[1][c], sc[1][2 + c]));
        float Mx = fmaxf(fmaxf(sc[0][c] + nvl[0][0], sc[0][2 + c] + nvl[0][1]),
                         fmaxf(sc[1][c] + nvl[1][0], sc[1][2 + c] + nvl[1][1]));
#pragma unroll
        for (int o = 4; o <= 16; o <<= 1) {
          mx = fmaxf(mx, __shfl_xor_sync(dev::kFull, mx, o));
          Mx = fmaxf(Mx, __shfl_xor_sync(dev::kFull, Mx, o));
        }
        const float mn = fmaxf(m_run[c], mx);
        const float Mn = Mx > M_run[c] + kLazy ? Mx : M_run[c];
        const float ms_ = mn == -INFINITY ? 0.f : mn;
        const float Ms_ = Mn == -INFINITY ? 0.f : Mn;
        const float al = ex2(m_run[c] - ms_);
        aM[c] = ex2(M_run[c] - Ms_);
        moved |= Mn != M_run[c];
        m_run[c] = mn;
        M_run[c] = Mn;
        float ls = 0.f;
#pragma unroll
        for (int ms = 0; ms < 2; ++ms) {
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float t = sc[ms][2 * r + c];
            ls += ex2(t - ms_);
            wgt[ms][2 * r + c] = ex2(t + nvl[ms][r] - Ms_);
          }
        }
        l_run[c] = fmaf(l_run[c], al, ls);
      }
      if (__any_sync(dev::kFull, moved)) {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          acc[mt][0] *= aM[0];
          acc[mt][1] *= aM[1];
          acc[mt][2] *= aM[0];
          acc[mt][3] *= aM[1];
        }
      }

      // -------- PV: for each 16-token half, B = W^T via movmatrix
#pragma unroll
      for (int ms = 0; ms < 2; ++ms) {
        uint32_t b0, b1, b2 = 0u, b3 = 0u;
        {
          uint32_t h01, l01, h23, l23;
          split_pair(wgt[ms][0], wgt[ms][1], h01, l01);
          split_pair(wgt[ms][2], wgt[ms][3], h23, l23);
          if constexpr (PACK) {
            // lanes tig < 2 carry the hi halves (columns 0-3), tig >= 2 the lo
            const bool lo = tig >= 2;
            b0 = movmatrix_trans(lo ? l01 : h01);
            b1 = movmatrix_trans(lo ? l23 : h23);
          } else {
            b0 = movmatrix_trans(h01);
            b1 = movmatrix_trans(h23);
            b2 = movmatrix_trans(l01);
            b3 = movmatrix_trans(l23);
          }
        }
        const auto &vw = vb.w[ms];
        if constexpr (VBM == 4) {
          // cross-nibble bytes: (token a, dim) | (token b, dim) << 4
          uint32_t x0[2][2], x1[2][2];
#pragma unroll
          for (int pr = 0; pr < 2; ++pr) {
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              const uint32_t wa = vw[2 * pr][w], wb = vw[2 * pr + 1][w];
              x0[pr][w] = (wa & 0x0F0F0F0Fu) | ((wb << 4) & 0xF0F0F0F0u);
              x1[pr][w] = ((wa >> 4) & 0x0F0F0F0Fu) | (wb & 0xF0F0F0F0u);
            }
          }
#define TQ_VSTEP4(MT)                                                             \
  {                                                                               \
    uint32_t a[4];                                                                \
    a[0] = lut(pair_addr<4, MT, 2>(x0[0], voff));                           \
    a[1] = lut(pair_addr<4, MT, 2>(x1[0], voff));                           \
    a[2] = lut(pair_addr<4, MT, 2>(x0[1], voff));                           \
    a[3] = lut(pair_addr<4, MT, 2>(x1[1], voff));                           \
    mma16816(acc[MT], a, b0, b1);                                                 \
    if constexpr (!PACK) mma16816(acc[MT], a, b2, b3);                            \
  }
          TQ_VSTEP4(0) TQ_VSTEP4(1) TQ_VSTEP4(2) TQ_VSTEP4(3)
          TQ_VSTEP4(4) TQ_VSTEP4(5) TQ_VSTEP4(6) TQ_VSTEP4(7)
#undef TQ_VSTEP4
        } else {
#define TQ_VSTEP(MT)                                                              \
  {                                                                               \
    const uint32_t h0_ = lut(pair_addr<VBM, MT, VW>(vw[0], voff));          \
    const uint32_t h1_ = lut(pair_addr<VBM, MT, VW>(vw[1], voff));          \
    const uint32_t h2_ = lut(pair_addr<VBM, MT, VW>(vw[2], voff));          \
    const uint32_t h3_ = lut(pair_addr<VBM, MT, VW>(vw[3], voff));          \
    uint32_t a[4];                                                                \
    a[0] = __byte_perm(h0_, h1_, 0x5410);                                         \
    a[1] = __byte_perm(h0_, h1_, 0x7632);                                         \
    a[2] = __byte_perm(h2_, h3_, 0x5410);                                         \
    a[3] = __byte_perm(h2_, h3_, 0x7632);                                         \
    mma16816(acc[MT], a, b0, b1);                                                 \
    if constexpr (!PACK) mma16816(acc[MT], a, b2, b3);                            \
  }
          TQ_VSTEP(0) TQ_VSTEP(1) TQ_VSTEP(2) TQ_VSTEP(3)
          TQ_VSTEP(4) TQ_VSTEP(5) TQ_VSTEP(6) TQ_VSTEP(7)
#undef TQ_VSTEP
        }
      }
      // the value registers are free: start the next chunk's value loads
      if (more) {
        if (fast_next) {
          load_v_fast(vb, fp, cn, g8);
        } else {
          const int64_t jn = t0 + (int64_t)cn * kChunk;
          load_v_slow(vb, p, vbase + jn * p.vsn, (int)min((int64_t)kChunk, t1 - jn), g8, tig);
        }
      }
    }

    // ---- warp totals: l over the 8 row groups; PACK: hi + lo columns of acc
#pragma unroll
    for (int c = 0; c < 2; ++c) {
#pragma unroll
      for (int o = 4; o <= 16; o <<= 1) l_run[c] += __shfl_xor_sync(dev::kFull, l_run[c], o);
    }
    if constexpr (PACK) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[mt][i] += __shfl_xor_sync(dev::kFull, acc[mt][i], 2);
      }
    }

    // ---- CTA merge of the warps' partials for this piece
    {
      float *wp = s_part + (size_t)warp * 8 * kPW;
      if (PACK ? tig < 2 : true) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int hh = 2 * tig + c;
          if (g8 == 0) {
            wp[hh * kPW + 0] = m_run[c];
            wp[hh * kPW + 1] = l_run[c];
            wp[hh * kPW + 2] = M_run[c];
          }
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            // C row g8 -> dim 16 g8 + 2 mt, row g8 + 8 -> dim 16 g8 + 2 mt + 1
            wp[hh * kPW + 4 + 16 * g8 + 2 * mt] = acc[mt][c];
            wp[hh * kPW + 4 + 16 * g8 + 2 * mt + 1] = acc[mt][2 + c];
          }
        }
      }
    }
    __syncthreads();
    {
      float *dst = p.ws + p.slot0 + ((int64_t)u + blockIdx.x) * kSlot;
      for (int o = tid; o < gh * (kD + 3); o += kThreads) {
        const int hh = o / (kD + 3), e = o % (kD + 3);
        float mstar = -INFINITY, Mstar = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          mstar = fmaxf(mstar, s_part[(w * 8 + hh) * kPW + 0]);
          Mstar = fmaxf(Mstar, s_part[(w * 8 + hh) * kPW + 2]);
        }
        const float m0 = mstar == -INFINITY ? 0.f : mstar;
        const float M0 = Mstar == -INFINITY ? 0.f : Mstar;
        float v = 0.f;
        if (e == 0) {
          v = mstar;
        } else if (e == 2) {
          v = Mstar;
        } else if (e == 1) {
#pragma unroll
          for (int w = 0; w < kWarps; ++w) {
            const float *q = s_part + (w * 8 + hh) * kPW;
            v += q[1] * ex2(q[0] - m0);
          }
        } else {
          const int dd = e - 3;
#pragma unroll
          for (int w = 0; w < kWarps; ++w) {
            const float *q = s_part + (w * 8 + hh) * kPW;
            v += q[4 + dd] * ex2(q[2] - M0);
          }
          v *= inv_sV;
        }
        dst[hh * kPW + (e < 3 ? e : e + 1)] = v;
      }
    }
    // ---- the last CTA to finish a unit merges its slots into the output.
    // Every CTA publishes its slot, then thread 0 fences (after the barrier,
    // so the fence covers the whole CTA's stores) and bumps the unit's
    // counter once; the last arrival fences again before the merge reads.
    // No CTA ever waits on another.
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const int c0 = cta_of(s_cut, p.ctas, ustart), c1 = cta_of(s_cut, p.ctas, ustart + ulen - 1);
      // CTAs with an empty range (only when the space is shorter than the
      // grid) never arrive, so count the non-empty ones of the span
      unsigned n = 0;
      for (int c = c0; c <= c1; ++c) n += s_cut[c + 1] > s_cut[c] ? 1u : 0u;
      const unsigned prev = atomicAdd(p.cnt + u, 1u);
      s_last = (prev + 1 == n) ? 1 : 0;
      if (prev + 1 == n) __threadfence();
    }
    __syncthreads();
    if (s_last) {
      const int c0 = cta_of(s_cut, p.ctas, ustart), c1 = cta_of(s_cut, p.ctas, ustart + ulen - 1);
      merge_unit(p, s_cut, u, c0, c1, b, h0, gh, warp, kWarps, lane, s_part);
    }
  }
}

__global__ void zero_out_kernel(float *out, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = 0.f;
}

// Dynamic shared memory: enough to reach kLutAddr + kLutBytes + the warps'
// partials from any dynamic base at or above 0.
constexpr size_t split_smem_bytes(int warps) {
  return (size_t)kLutAddr + kLutBytes + (size_t)warps * 8 * kPW * sizeof(float);
}

// Static shared memory plus the per-block reserve must end at or below
// kLutAddr, where the dynamic region's pair tables start.
template <typename K>
cudaError_t check_smem_layout(K kern) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  int dev = 0, reserved = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  if (e != cudaSuccess) return e;
  if ((size_t)reserved + fa.sharedSizeBytes > kLutAddr) return cudaErrorInvalidConfiguration;
  return cudaSuccess;
}

// Raises a kernel's dynamic shared memory limit once per device (the
// setting belongs to the kernel, so later launches skip the driver call).
template <auto Kern>
cudaError_t set_smem_once(size_t smem) {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t)1 << dev : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
  return e;
}

template <int KBM, bool KPROD, int VBM, bool PACK>
cudaError_t run_split(const SplitParams &sp, cudaStream_t s) {
  auto kern = decode_split_kernel<KBM, KPROD, VBM, PACK>;
  const int warps = PACK && !KPROD ? 12 : 8;
  const size_t smem = split_smem_bytes(warps);
  static const cudaError_t layout = check_smem_layout(kern);
  if (layout != cudaSuccess) return layout;
  cudaError_t e = set_smem_once<decode_split_kernel<KBM, KPROD, VBM, PACK>>(smem);
  if (e != cudaSuccess) return e;
  // programmatic dependent launch: the grid may start while the prep kernel
  // before it in the stream is still running (the kernel waits for it with
  // griddepcontrol.wait before touching the workspace)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)sp.ctas);
  cfg.blockDim = dim3((unsigned)(warps * 32));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, sp);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <bool KPROD, int VBM, bool PACK>
cudaError_t by_kbits(int kbm, const SplitParams &sp, cudaStream_t s) {
  switch (kbm) {
    case 0: if constexpr (KPROD) return run_split<0, true, VBM, PACK>(sp, s); else return cudaErrorInvalidValue;
    case 1: return run_split<1, KPROD, VBM, PACK>(sp, s);
    case 2: return run_split<2, KPROD, VBM, PACK>(sp, s);
    case 3: return run_split<3, KPROD, VBM, PACK>(sp, s);
    case 4: return run_split<4, KPROD, VBM, PACK>(sp, s);
  }
  return cudaErrorInvalidValue;
}

template <int VBM>
cudaError_t by_kvariant(int kbm, bool kprod, bool pack, const SplitParams &sp, cudaStream_t s) {
  if (pack) return kprod ? by_kbits<true, VBM, true>(kbm, sp, s) : by_kbits<false, VBM, true>(kbm, sp, s);
  return kprod ? by_kbits<true, VBM, false>(kbm, sp, s) : by_kbits<false, VBM, false>(kbm, sp, s);
}

}  // namespace

bool decode_supported(int d, int kbm, bool kprod, int vbm, bool vprod) {
  return d == kD && !vprod && vbm >= 1 && vbm <= 4 && kbm >= (kprod ? 0 : 1) && kbm <= 4;
}

size_t decode_workspace_floats(int B, int Hq, int Hkv, bool prod, int ctas) {
  const int64_t units = (int64_t)B * Hkv * ((Hq / Hkv + 7) / 8);
  (void)prod;  // the fragment block has room for the prod words either way
  return (size_t)kHdr + (size_t)units * kFragWords + (size_t)(units + ctas) * kSlot + (size_t)units;
}

cudaError_t take_device_faults(unsigned *faults) {
  unsigned w = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&w, g_tq_faults, sizeof(w));
  if (e != cudaSuccess) return e;
  *faults = w;
  if (w) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_tq_faults, &zero, sizeof(zero));
  }
  return e;
}

cudaError_t static_scratch(void **ptr) {
  // Looked up once per device, with that device current, and cached.
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void *addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *a = nullptr;
    e = cudaGetSymbolAddress(&a, g_tq_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = a;
  }
  *ptr = addr[dev];
  return cudaSuccess;
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
  const int64_t outn = (int64_t)a.B * a.Hq * kD;
  if (a.seq_len == 0) {
    zero_out_kernel<<<(unsigned)((outn + 255) / 256), 256, 0, s>>>(a.out, outn);
    return cudaGetLastError();
  }
  SplitParams sp{};
  sp.q = a.q;
  sp.q_dtype = a.q_dtype;
  sp.B = a.B;
  sp.Hq = a.Hq;
  sp.Hkv = a.Hkv;
  sp.g = a.Hq / a.Hkv;
  sp.groups = (sp.g + 7) / 8;
  sp.seq_len = a.seq_len;
  sp.seq_lens = a.seq_lens;
  // When the units fit the grid, a CTA count that is a multiple of the unit
  // count (if it idles at most 5% of the CTAs) keeps every CTA inside one
  // unit: no CTA then works on two pieces in sequence.
  {
    const int64_t units = (int64_t)a.B * a.Hkv * sp.groups;
    int ctas = a.splits;
    if (units <= ctas) {
      const int64_t aligned = (ctas / units) * units;
      if (aligned * 20 >= (int64_t)ctas * 19) ctas = (int)aligned;
    }
    sp.ctas = ctas;
  }
  sp.kc = a.k.codes;
  sp.kj = a.k.qjl;
  sp.kn = a.k.norms;
  sp.kr = a.k.rnorms;
  sp.ksb = a.k.sb;
  sp.ksh = a.k.sh;
  sp.ksn = a.k.sn;
  sp.kcent = a.kq.centroids;
  sp.ksign = a.kq.signs;
  sp.kS = a.kq.S;
  sp.vc = a.v.codes;
  sp.vn = a.v.norms;
  sp.vsb = a.v.sb;
  sp.vsh = a.v.sh;
  sp.vsn = a.v.sn;
  sp.vcent = a.vq.centroids;
  sp.scale_log2 = a.scale * kLog2e;
  sp.scores = a.scores;
  sp.ws = a.ws;
  const int units = a.B * a.Hkv * sp.groups;
  sp.frag = reinterpret_cast<const uint4 *>(a.ws + kHdr);
  sp.slot0 = (int64_t)kHdr + (int64_t)units * kFragWords;
  sp.cnt = reinterpret_cast<unsigned *>(a.ws + sp.slot0 + (int64_t)(units + sp.ctas) * kSlot);
  sp.out = a.out;
  sp.vsign = a.vq.signs;
  PrepParams pp{a.q, a.q_dtype, a.B * a.Hq, a.kq.signs, a.kq.prod ? a.kq.S : nullptr,
                a.kq.centroids, a.kq.bm, a.vq.centroids, a.vq.bm, a.ws, sp.cnt, units,
                a.Hq, a.Hkv, sp.g, sp.groups, a.seq_len, a.seq_lens, a.out,
                reinterpret_cast<uint32_t *>(a.ws + kHdr)};
  cudaError_t pe;
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((a.B * a.Hq + 1) / 2 + 2));
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = a.prep_pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    pe = cudaLaunchKernelEx(&cfg, decode_prep_kernel, pp);
  }
  if (pe != cudaSuccess) return pe;
  pe = cudaGetLastError();
  if (pe != cudaSuccess) return pe;
  const bool pack = sp.g <= 4;
  cudaError_t e = cudaErrorInvalidValue;
  switch (a.vq.bm) {
    case 1: e = by_kvariant<1>(a.kq.bm, a.kq.prod, pack, sp, s); break;
    case 2: e = by_kvariant<2>(a.kq.bm, a.kq.prod, pack, sp, s); break;
    case 3: e = by_kvariant<3>(a.kq.bm, a.kq.prod, pack, sp, s); break;
    case 4: e = by_kvariant<4>(a.kq.bm, a.kq.prod, pack, sp, s); break;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace tq
