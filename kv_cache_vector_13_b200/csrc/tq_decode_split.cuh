// Split kernel of the decode attention on the packed TurboQuant cache,
// shared by the translation units that instantiate its two variants.
//
// What it computes (the pages, by title and section): attention for one new
// query per head over every cached token ("I Spent 31 Hours On The Math
// Behind Turboquant", "KV Cache: The problem"), keys scored by the
// asymmetric estimator -- the full-precision query against compressed keys
// ("内存厂商的噩梦来了", 4.2 and its asymmetric_attention_score):
//   s_j = n_j ( <q', c_K[idx_j]> + [prod] ||r_j|| sqrt(pi/2)/d <S q', sign_j> ),
// values summed in the value-rotated basis, o' = sum_j p_j n_j c_V[idx_j],
// and rotated back once by the merge, o = Pi_V^T o'.
//
// Persistent grid, one CTA per SM.  The work is the flattened space of
// (unit = batch x kv head x group of <= 8 query heads, token) pairs, cut into
// one equal contiguous range per CTA; a range covers one or a few "pieces"
// (CTA, unit), and each warp of the CTA takes a contiguous share of a
// piece's 32-token chunks.  Per CTA, once: the two pair tables are copied into
// shared memory at address 64 KiB, replicated per lane (entry e, lane l at
// 64 KiB + e*256 + 4l, values at +128) so that table reads never conflict on
// banks and one byte permute forms a lookup's whole address.
//
// How the packed records reach the warps (the two variants):
//   * staged (unit token stride, 16-byte aligned norm rows): every warp owns
//     a ring of 2..4 shared-memory slots, each holding one chunk's K codes,
//     QJL signs, V codes and norms.  Lane-parallel bulk copies
//     (cp.async.bulk, this GPU's own memory, no multicast) fill a slot and
//     complete on the slot's mbarrier; the warp waits on it with a bounded
//     try_wait loop, reads its fragments from shared memory, and refills the
//     slot with the chunk R ahead as soon as it is done with it.  Value code
//     rows of 16 or 64 bytes are copied one token per lane into rows padded
//     by 16 bytes (48 / 80), so that the four lanes of a quad, which read the
//     same dims of tokens two apart, hit different banks.  Nothing of the
//     stream is held in registers.
//   * register-fed (any record strides): packed words go from HBM straight
//     to registers, the next chunk's loads issued while the current one is
//     worked on, with bulk L2 prefetches a window ahead.
// Per chunk, in both:
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
//   * the QJL term runs on int8 MMAs (mma.m16n8k32.s8): a sign-replicating
//     byte permute turns four sign bits into four 0 / -1 bytes, against S q'
//     held as two int8 digits (<S q', 2 bit - 1> = -2 (digit sum) - sum S q');
//   * online softmax in base 2 against one reference M per head column,
//     taken over u = logit + max(log2 n_V, kNvlFloor) and moved only when
//     some u passes it by more than kLazy: the PV weights 2^(logit + log2 n_V
//     - M) stay below 2^kLazy (fp16 range), the normaliser's terms
//     2^(logit - M) below 2^(kLazy - kNvlFloor) (fp32 range).
// The warps' partials (m, l, M, o') of a piece are merged in shared memory
// and written to workspace slot (unit + CTA index).  Each CTA then bumps its
// unit's counter; the CTA that completes the count merges the unit's slots,
// divides by l and applies Pi_V^T = diag(sigma_V) H / sqrt(d).  No CTA waits
// for another.
#pragma once

#include "../../include/tq.h"
#include "tq_device.cuh"
#include "tq_internal.h"

#include <float.h>
#include <math.h>

#include <atomic>

namespace tq {
namespace dec {

constexpr int kD = 128;
constexpr int kMaxCtas = 1024;  // persistent CTAs supported (one per SM)
constexpr int kChunk = 32;               // tokens per warp iteration
constexpr int kLutBytes = 256 * 256;     // K and V pair tables, per-lane copies
// Shared-window address of the pair tables.  Entry e, lane l sits at
// kLutAddr + 256 e + 4 l (+128 for the value table): with the tables on a
// 64 KiB boundary, one byte permute of (code byte, lane offset) yields the
// complete shared address of a lookup.
constexpr uint32_t kLutAddr = 0x10000;
// Register-fed kernel with 2-bit key codes: one code byte (four codes) is
// one lookup of a 64-bit entry (four fp16 centroids), so the key table takes
// the whole 64 KiB window (entry e, lane l at kLutAddr + 256 e + 8 l) and the
// value table moves to the next window (kVTab4Addr + 256 e + 4 l).  The query
// digit fragments and the warps' partials then sit below kLutAddr.
constexpr uint32_t kVTab4Addr = 0x20000;
template <int KBM, bool STAGED>
__host__ __device__ constexpr bool key_quads() {
  return KBM == 2 && !STAGED;
}
constexpr int kPfWin = 4;                // chunks per L2 prefetch window (register-fed variant)
constexpr int kMaxRing = 4;              // ring slots per warp (staged variant)
// A bounded wait gives up after this long without progress (ns).
constexpr uint64_t kWaitLimitNs = 1000000000ull;
// The PV weights' reference maximum M moves only when a chunk's maximum of
// logit + log2 n_V passes it by more than kLazy (log2 units); the weights
// then stay below 2^kLazy and most rescales of the accumulators are skipped.
constexpr float kLazy = 8.0f;
// Floor of log2 n_V in the reference: the normaliser's terms 2^(logit - M)
// then stay below 2^(kLazy - kNvlFloor), tiny or zero value norms included.
constexpr float kNvlFloor = -64.0f;
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
//                      w = 16 + 2S + j : dig(Sq'[g8 & 3][32 tig + 8i + 7 - 2S - j]), i = 0..3
//                                        (byte i; dig = hi digit, lo digit for g8 >= 4)
//   8 heads          : w = 2s + j / 16 + 2s + j  : hi / lo of q'[g8][32 tig + 4s + 2j, +1]
//                      w = 32 + 2S + j / 40 + 2S + j : hi / lo digit of Sq'[g8][...] as above
//   (s < 8, S < 4, j < 2).  Sq' travels as int8 digits, round(Sq' / c_h) =
//   256 hi + lo with |round(Sq' / c_h)| <= 32000; word 60 of lane h holds
//   c_h and word 61 of lane h holds T_h = sum_k Sq'_h[k] (h < 8, the
//   unit's heads).
constexpr int kFragWords = 32 * 64;
// Bytes of a unit's QJL digit fragments in shared memory ([4][2][32] uint2).
constexpr uint32_t kQsBytes = 2 * 4 * 32 * 8;
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
  const float *vrot;  // dense value rotation Pi_V (row-major), else NULL
  unsigned *faults;   // the GPU's fault word (kFault* bits)
  int dyn_bytes;      // dynamic shared memory of the launch
  bool early;         // the cache is complete when the grid starts (no append before it)
};

struct PrepParams {
  const void *q;
  int q_dtype;
  int nheads;  // B * Hq
  const int8_t *ksign;
  const float *krot;  // dense key rotation Pi_K (row-major), else NULL
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

// The prep kernel (tq_decode.cu): query rotation and fragments of every
// unit, the pair tables, the units' counters zeroed.
cudaError_t launch_prep(const PrepParams &pp, bool pdl, cudaStream_t s);

// Split-kernel launchers of the two variants (one translation unit each).
// Each picks the instantiation for (K b_m, K prod, V b_m, <= 4 heads per kv
// head) and launches it with programmatic stream serialization.
cudaError_t launch_split_staged(int kbm, bool kprod, int vbm, bool pack, const SplitParams &sp, cudaStream_t s);
cudaError_t launch_split_regs(int kbm, bool kprod, int vbm, bool pack, const SplitParams &sp, cudaStream_t s);

// Bytes of one staged ring slot (one 32-token chunk of every array).
__host__ __device__ constexpr int ring_vpitch(int vbm) { return (vbm == 4 || vbm == 2) ? 16 * vbm + 16 : 16 * vbm; }
__host__ __device__ constexpr int ring_slot_bytes(int kbm, bool kprod, int vbm) {
  return kChunk * (16 * kbm + (kprod ? 16 : 0) + ring_vpitch(vbm)) + kChunk * 4 * (kprod ? 3 : 2);
}

}  // namespace dec

namespace {

using namespace dec;

// ------------------------------------------------------------------ PTX

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D += A B on int8 operands (mma.m16n8k32, s8 x s8 -> s32).
__device__ __forceinline__ void mma16832_s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four int8 lanes, each 0 or -1 as bit 7 of byte 0..3 of w is clear or set
// (a byte permute in sign-replicating mode).
__device__ __forceinline__ uint32_t sign_bytes(uint32_t w) {
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, 0xBA98;\n" : "=r"(r) : "r"(w));
  return r;
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

// 64-bit table entry (two half2) at shared-window address `addr`
__device__ __forceinline__ uint2 lut64(uint32_t addr) {
  uint2 v;
  asm("ld.shared.v2.b32 {%0, %1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(addr));
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
  float d0, d1;
  dev::sub_x2(d0, d1, a, b, f.x, f.y);
  lo = pack_half2(d0, d1);
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
// The word is shifted by the bit residue s % 8 only and the byte s / 8 of
// the result selected, so every field of a word at the same residue shares
// one shift.
template <int SH>
__device__ __forceinline__ uint32_t lut_addr(uint32_t w0, uint32_t w1, uint32_t laneoff) {
  constexpr int s = SH & 31, r = s % 8, by = s / 8;
  if constexpr (r == 0) {
    return __byte_perm(w0, laneoff, 0x7604 | (by << 4));
  } else if constexpr (s + 8 <= 32) {
    return __byte_perm(w0 >> r, laneoff, 0x7604 | (by << 4));
  } else {  // the byte crosses into w1 (by == 3)
    return __byte_perm(__funnelshift_r(w0, w1, r), laneoff, 0x7604 | (by << 4));
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

template <int BM>
struct VChunk {  // 16 dims of one token: 2*BM bytes
  static constexpr int NW = (2 * BM + 3) / 4;
};

// Two tokens' BM-bit streams of 16 dims (a, b) interleaved field by field:
// field j of xe holds (a's code, b's code) of dim 2j as one 2BM-bit pair
// index (a in the low bits: the pair tables' layout), xo the same for dim
// 2j + 1; field j sits at bit 2 BM j, where pair j of a token's own stream
// sits.
template <int BM>
__device__ __forceinline__ void interleave_tokens(const uint32_t (&a)[VChunk<BM>::NW],
                                                  const uint32_t (&b)[VChunk<BM>::NW],
                                                  uint32_t (&xe)[VChunk<BM>::NW], uint32_t (&xo)[VChunk<BM>::NW]) {
  if constexpr (BM == 3) {
    constexpr uint64_t Me = 0x1C71C71C71C7ull;  // bits [6j, 6j + 3), j < 8
    const uint64_t A = ((uint64_t)a[1] << 32) | a[0], B = ((uint64_t)b[1] << 32) | b[0];
    const uint64_t e = (A & Me) | ((B << 3) & (Me << 3));
    const uint64_t o = ((A >> 3) & Me) | (B & (Me << 3));
    xe[0] = (uint32_t)e;
    xe[1] = (uint32_t)(e >> 32);
    xo[0] = (uint32_t)o;
    xo[1] = (uint32_t)(o >> 32);
  } else if constexpr (BM == 2) {
    xe[0] = (a[0] & 0x33333333u) | ((b[0] << 2) & 0xCCCCCCCCu);
    xo[0] = ((a[0] >> 2) & 0x33333333u) | (b[0] & 0xCCCCCCCCu);
  } else if constexpr (BM == 1) {
    xe[0] = (a[0] & 0x5555u) | ((b[0] << 1) & 0xAAAAu);
    xo[0] = ((a[0] >> 1) & 0x5555u) | (b[0] & 0xAAAAu);
  } else {  // BM == 4: fields stay inside their bytes
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      xe[w] = (a[w] & 0x0F0F0F0Fu) | ((b[w] << 4) & 0xF0F0F0F0u);
      xo[w] = ((a[w] >> 4) & 0x0F0F0F0Fu) | (b[w] & 0xF0F0F0F0u);
    }
  }
}

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
  } else {  // BM == 3: 6 bytes at 6g of a 48-byte record, 2-byte aligned:
    // the two words at the 4-byte boundary below (still inside the record),
    // shifted down by 16 bits for odd g, with no branch
    const uint32_t *q = reinterpret_cast<const uint32_t *>(p - 2 * (g & 1));
    const uint32_t lo = __ldg(q), hi = __ldg(q + 1);
    const int sh = 16 * (g & 1);
    W[0] = __funnelshift_r(lo, hi, sh);
    W[1] = (hi >> sh) & 0xFFFFu;
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

// The lane's record indices of the fast path (unit record strides) at chunk
// 0 of a piece: the key rows' (token g8) and the value rows' (token 2 tig);
// chunk c adds c * kChunk records.  The array bases stay in the kernel
// parameters, so a piece keeps two indices live rather than six pointers.
struct FastPtrs {
  int64_t kr0, vr0;
};

__device__ __forceinline__ FastPtrs fast_ptrs(int64_t krec0, int64_t vrec0, int tig, int g8) {
  return FastPtrs{krec0 + g8, vrec0 + 2 * tig};
}

// Key side of full chunk c through the fast-path indices.
template <int KBM, bool KPROD, int VBM>
__device__ __forceinline__ void load_k_fast(KBuf<KBM, KPROD> &c, const SplitParams &p, const FastPtrs &f, int ci,
                                            int tig, int g8) {
  constexpr int KCB = kD * KBM / 8;
  const int64_t r0 = f.kr0 + (int64_t)ci * kChunk;
  const int64_t v0 = f.vr0 - 2 * tig + g8 + (int64_t)ci * kChunk;  // the key rows' value norms
#pragma unroll
  for (int ms = 0; ms < 2; ++ms) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int t = 16 * ms + 8 * r;
      if constexpr (KBM > 0) load_k32<KBM>(p.kc + (r0 + t) * KCB + tig * (4 * KBM), c.w[ms][r]);
      if constexpr (KPROD) {
        c.qj[ms][r] = __ldg(reinterpret_cast<const uint32_t *>(p.kj + (r0 + t) * (kD / 8)) + tig);
        c.kr[ms][r] = __ldg(p.kr + r0 + t);
      }
      c.kn[ms][r] = __ldg(p.kn + r0 + t);
      c.vn[ms][r] = __ldg(p.vn + v0 + t);
    }
  }
}

// Value side of full chunk c through the fast-path indices.
template <int KBM, bool KPROD, int VBM>
__device__ __forceinline__ void load_v_fast(VBuf<VBM> &c, const SplitParams &p, const FastPtrs &f, int ci, int g8) {
  constexpr int VCB = kD * VBM / 8;
  const int64_t r0 = f.vr0 + (int64_t)ci * kChunk;
#pragma unroll
  for (int ms = 0; ms < 2; ++ms) {
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4)
      load_v16<VBM>(p.vc + (r0 + 16 * ms + (q4 & 1) + 8 * (q4 >> 1)) * VCB + g8 * (2 * VBM), c.w[ms][q4], g8);
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
  const bool had = p.vrot == nullptr;
  const int8_t sg0 = had ? p.vsign[lane * 4] : 1, sg1 = had ? p.vsign[lane * 4 + 1] : 1;
  const int8_t sg2 = had ? p.vsign[lane * 4 + 2] : 1, sg3 = had ? p.vsign[lane * 4 + 3] : 1;
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
      if (p.vrot) {
        // o = Pi_V^T (o' / l): stage o' in this head's own row of s_m (read
        // only by this warp), then out_j = sum_k Pi[k][j] o'_k
        const float f = ex2(Ms - m_all) / l;
        float *st = s_m + hh * kPW + 4;
        *reinterpret_cast<float4 *>(st + lane * 4) = make_float4(a[0] * f, a[1] * f, a[2] * f, a[3] * f);
        __syncwarp();
        float o4[4] = {0.f, 0.f, 0.f, 0.f};
        const float4 *R = reinterpret_cast<const float4 *>(p.vrot) + lane;
        for (int k = 0; k < kD; ++k) {
          const float4 r = __ldg(R + k * (kD / 4));
          const float ok = st[k];
          o4[0] = fmaf(r.x, ok, o4[0]);
          o4[1] = fmaf(r.y, ok, o4[1]);
          o4[2] = fmaf(r.z, ok, o4[2]);
          o4[3] = fmaf(r.w, ok, o4[3]);
        }
        *reinterpret_cast<float4 *>(out) = make_float4(o4[0], o4[1], o4[2], o4[3]);
      } else {
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


// ------------------------------------------------------ staged ring (PTX)

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
  return t;
}

// Orders this thread's earlier shared-memory accesses (generic proxy) before
// its later bulk copies into the same memory (async proxy).
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned)
// from global memory of this GPU into shared memory; completes on `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// Waits, with the whole warp, for phase `parity` of `bar`.  After
// kWaitLimitNs without completion it records kFaultTimeout in the fault word
// and marks the warp dead: a dead warp no longer waits and carries on with
// whatever the slots hold, so that every warp still reaches every barrier
// and the kernel ends (its outputs are then invalid, and tq_check says so).
__device__ __noinline__ bool ring_wait(uint32_t bar, uint32_t parity, unsigned *faults, bool &dead) {
  if (dead) return false;
  uint64_t t0 = 0;
  for (uint32_t spin = 0;; ++spin) {
    if (__all_sync(dev::kFull, mbar_try_wait(bar, parity))) return true;
    if ((spin & 255u) == 255u) {
      const uint64_t now = globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (__any_sync(dev::kFull, now - t0 > kWaitLimitNs)) {
        if ((threadIdx.x & 31) == 0) atomicOr(faults, kFaultTimeout);
        dead = true;
        return false;
      }
    }
  }
}

// Sub-array offsets inside one ring slot (all multiples of 16 bytes).
template <int KBM, bool KPROD, int VBM>
struct SlotLayout {
  static constexpr int KCB = kD * KBM / 8, VCB = kD * VBM / 8, VP = ring_vpitch(VBM);
  static constexpr bool kVRows = VP != VCB;  // value rows copied one token per lane, padded
  static constexpr int oKC = 0;
  static constexpr int oKJ = oKC + kChunk * KCB;
  static constexpr int oVC = oKJ + (KPROD ? kChunk * 16 : 0);
  static constexpr int oKN = oVC + kChunk * VP;
  static constexpr int oVN = oKN + kChunk * 4;
  static constexpr int oKR = oVN + kChunk * 4;
  static constexpr int kBytes = oKR + (KPROD ? kChunk * 4 : 0);
  static_assert(kBytes == ring_slot_bytes(KBM, KPROD, VBM), "slot layout");
};

// Lane-parallel fill of one ring slot with the n (1..32) records starting at
// records krec / vrec (n4 = n rounded down to 4 of them carry their norms by
// bulk copy; the 0..3 left over are loaded by lanes and stored directly).
// Called by the whole warp once it is done reading the slot.
template <int KBM, bool KPROD, int VBM>
__device__ __forceinline__ void ring_fill(const SplitParams &p, uint32_t slot, uint32_t bar, int64_t krec,
                                          int64_t vrec, int n, int lane) {
  using SL = SlotLayout<KBM, KPROD, VBM>;
  const int n4 = n & ~3;
  uint32_t bytes = (uint32_t)n * (SL::KCB + SL::VCB + (KPROD ? 16 : 0)) + (uint32_t)n4 * 4u * (KPROD ? 3u : 2u);
  if (lane == 0) mbar_arrive_expect_tx(bar, bytes);
  __syncwarp();
  fence_proxy_async();
  if constexpr (KBM > 0) {
    if (lane == 0) bulk_g2s(slot + SL::oKC, p.kc + krec * SL::KCB, (uint32_t)n * SL::KCB, bar);
  }
  if constexpr (KPROD) {
    if (lane == 1) bulk_g2s(slot + SL::oKJ, p.kj + krec * 16, (uint32_t)n * 16u, bar);
    if (lane == 3 && n4) bulk_g2s(slot + SL::oKR, p.kr + krec, (uint32_t)n4 * 4u, bar);
  }
  if (n4) {
    if (lane == 2) bulk_g2s(slot + SL::oKN, p.kn + krec, (uint32_t)n4 * 4u, bar);
    if (lane == 4) bulk_g2s(slot + SL::oVN, p.vn + vrec, (uint32_t)n4 * 4u, bar);
  }
  if constexpr (SL::kVRows) {
    if (lane < n) bulk_g2s(slot + SL::oVC + lane * SL::VP, p.vc + (vrec + lane) * SL::VCB, SL::VCB, bar);
  } else {
    if (lane == 5) bulk_g2s(slot + SL::oVC, p.vc + vrec * SL::VCB, (uint32_t)n * SL::VCB, bar);
  }
  if (lane >= n4 && lane < n) {  // the ragged last rows' norms
    float *s = reinterpret_cast<float *>(__cvta_shared_to_generic(slot));
    s[SL::oKN / 4 + lane] = __ldg(p.kn + krec + lane);
    s[SL::oVN / 4 + lane] = __ldg(p.vn + vrec + lane);
    if constexpr (KPROD) s[SL::oKR / 4 + lane] = __ldg(p.kr + krec + lane);
  }
}

// Key side of a chunk from a ring slot: rows t outside [lo, hi) are masked
// (norm -1), their other values are whatever the slot holds.
template <int KBM, bool KPROD, int VBM>
__device__ __forceinline__ void load_k_ring(KBuf<KBM, KPROD> &c, const char *slot, int lo, int hi, int tig, int g8) {
  using SL = SlotLayout<KBM, KPROD, VBM>;
#pragma unroll
  for (int ms = 0; ms < 2; ++ms) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int t = 16 * ms + 8 * r + g8;
      const bool ok = t >= lo && t < hi;
      if constexpr (KBM > 0) {
        const char *src = slot + SL::oKC + t * SL::KCB + tig * (4 * KBM);
        if constexpr (KBM == 4) {
          const uint4 v = *reinterpret_cast<const uint4 *>(src);
          c.w[ms][r][0] = v.x; c.w[ms][r][1] = v.y; c.w[ms][r][2] = v.z; c.w[ms][r][3] = v.w;
        } else if constexpr (KBM == 2) {
          const uint2 v = *reinterpret_cast<const uint2 *>(src);
          c.w[ms][r][0] = v.x; c.w[ms][r][1] = v.y;
        } else {
#pragma unroll
          for (int i = 0; i < KBM; ++i) c.w[ms][r][i] = reinterpret_cast<const uint32_t *>(src)[i];
        }
      }
      if constexpr (KPROD) {
        c.qj[ms][r] = *reinterpret_cast<const uint32_t *>(slot + SL::oKJ + t * 16 + tig * 4);
        c.kr[ms][r] = reinterpret_cast<const float *>(slot + SL::oKR)[t];
      }
      const float kn = reinterpret_cast<const float *>(slot + SL::oKN)[t];
      c.kn[ms][r] = ok ? kn : -1.f;  // -1 marks a masked row
      c.vn[ms][r] = ok ? reinterpret_cast<const float *>(slot + SL::oVN)[t] : 1.f;
    }
  }
}

// Value side of a chunk from a ring slot (rows outside the valid range get
// weight 0, so their codes need no masking: every table entry is finite).
template <int KBM, bool KPROD, int VBM>
__device__ __forceinline__ void load_v_ring(VBuf<VBM> &c, const char *slot, int g8, int tig) {
  using SL = SlotLayout<KBM, KPROD, VBM>;
#pragma unroll
  for (int ms = 0; ms < 2; ++ms) {
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const int t = 16 * ms + 2 * tig + (q4 & 1) + 8 * (q4 >> 1);
      const char *src = slot + SL::oVC + t * SL::VP + g8 * (2 * VBM);
      if constexpr (VBM == 4) {
        const uint2 v = *reinterpret_cast<const uint2 *>(src);
        c.w[ms][q4][0] = v.x;
        c.w[ms][q4][1] = v.y;
      } else if constexpr (VBM == 2) {
        c.w[ms][q4][0] = *reinterpret_cast<const uint32_t *>(src);
      } else if constexpr (VBM == 1) {
        c.w[ms][q4][0] = *reinterpret_cast<const unsigned short *>(src);
      } else {  // 6 bytes at 48 t + 6 g8: 2-byte aligned
        if ((g8 & 1) == 0) {
          c.w[ms][q4][0] = *reinterpret_cast<const uint32_t *>(src);
          c.w[ms][q4][1] = *reinterpret_cast<const unsigned short *>(src + 4);
        } else {
          const uint32_t lo16 = *reinterpret_cast<const unsigned short *>(src);
          const uint32_t hi32 = *reinterpret_cast<const uint32_t *>(src + 2);
          c.w[ms][q4][0] = lo16 | (hi32 << 16);
          c.w[ms][q4][1] = hi32 >> 16;
        }
      }
    }
  }
}

// Warps per CTA: 12 with <= 4 query heads per kv head (the hi and lo query
// halves share one MMA); 8 with more, whose extra fragments need the
// registers.  The register-fed variant keeps the QJL term's query fragments
// (S q') in shared memory, which leaves room for 12 warps with prod keys.
template <bool PACK, bool KPROD, bool STAGED>
__host__ __device__ constexpr int split_warps() {
  return PACK ? 12 : 8;
}

// Whether the QJL term's query fragments are read from shared memory.
template <bool KPROD, bool STAGED>
__host__ __device__ constexpr bool qs_in_smem() {
  return KPROD && !STAGED;
}

template <int KBM, bool KPROD, int VBM, bool PACK, bool STAGED>
__global__ void __launch_bounds__(split_warps<PACK, KPROD, STAGED>() * 32, 1) decode_split_kernel(SplitParams p) {
  constexpr int kWarps = split_warps<PACK, KPROD, STAGED>();
  constexpr int kThreads = kWarps * 32;
  constexpr int KW = KBM > 0 ? KBM : 1;
  constexpr int VW = VChunk<VBM>::NW;
  constexpr int kSlotBytes = (ring_slot_bytes(KBM, KPROD, VBM) + 127) & ~127;
  extern __shared__ float4 smem4[];
  char *smem = reinterpret_cast<char *>(smem4);
  // [kLutAddr, +64 KB): the pair tables.  Register-fed: the warps' partials
  // follow them.  Staged: the ring slots fill [dynamic base, kLutAddr) and
  // [kLutAddr + 64 KB, end of the allocation); the partials reuse the start
  // of the second region once a piece's slots are drained.  The host sizes
  // the allocation so that both layouts fit from any dynamic base at or
  // below kLutAddr.
  const uint32_t dyn_base = smem_addr(smem4);
  if (dyn_base > kLutAddr) {  // excluded on the host; reported, never silent
    if (threadIdx.x == 0) atomicOr(p.faults, kFaultSmemLayout);
    return;
  }
  constexpr bool K4 = key_quads<KBM, STAGED>();
  char *s_lut = smem + (kLutAddr - dyn_base);
  // [kWarps][8][kPW]; with key quads below the tables, past the digit fragments
  float *s_part = K4 ? reinterpret_cast<float *>(smem + (((dyn_base + 15u) & ~15u) - dyn_base) + kQsBytes)
                     : reinterpret_cast<float *>(s_lut + kLutBytes);
  if (K4 && ((dyn_base + 15u) & ~15u) + kQsBytes + (uint32_t)(kWarps * 8 * kPW * 4) > kLutAddr) {
    if (threadIdx.x == 0) atomicOr(p.faults, kFaultSmemLayout);  // excluded on the host
    return;
  }
  __shared__ int s_last;
  __shared__ int64_t s_cut[kMaxCtas + 1];
  __shared__ __align__(8) uint64_t s_bar[STAGED ? kWarps * kMaxRing : 1];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g8 = lane >> 2, tig = lane & 3;
  const int UH = p.Hkv * p.groups;
  const int64_t T = flat_total(p.seq_lens, p.seq_len, p.B, UH);
  const int64_t x0 = cut(T, p.ctas, blockIdx.x), x1 = cut(T, p.ctas, blockIdx.x + 1);
  if (x0 >= x1) return;
  const bool unit = p.ksn == 1 && p.vsn == 1;

  // ---- staged: this warp's ring (R slots, their mbarriers) and the first
  // piece's first R chunks, issued before anything else when the cache is
  // already complete
  int R = 1;
  uint32_t ring0 = 0, ring1 = 0;  // shared address of slot 0, and of the first slot past the tables
  int ring_split = 0;             // slots of this warp below the tables
  uint32_t kk_issued = 0, kk_used = 0;  // chunks issued into / consumed from the ring
  uint32_t dead_at = 0;                 // kk_used when a wait first gave up
  bool dead = false;
  auto slot_addr = [&](uint32_t k) -> uint32_t {
    const int j = (int)(k % (uint32_t)R);
    return j < ring_split ? ring0 + (uint32_t)j * kSlotBytes : ring1 + (uint32_t)(j - ring_split) * kSlotBytes;
  };
  auto bar_addr = [&](uint32_t k) -> uint32_t { return smem_addr(&s_bar[warp * kMaxRing + (int)(k % (uint32_t)R)]); };
  // piece geometry of position x: unit, its start and length, the piece's
  // tokens [t0, t1), the chunk origin cs0 and this warp's chunks [cb, ce)
  struct Piece {
    int u;
    int64_t ustart, ulen, t0, t1, cs0;
    int nch, cb, ce;
  };
  auto piece_at = [&](int64_t x) {
    Piece q;
    locate(p.seq_lens, p.seq_len, p.B, UH, x, &q.u, &q.ustart, &q.ulen);
    q.t0 = x - q.ustart;
    q.t1 = min(x1, q.ustart + q.ulen) - q.ustart;
    q.cs0 = STAGED ? (q.t0 & ~(int64_t)3) : q.t0;
    // a piece is shorter than 2^31 tokens
    q.nch = (int)((q.t1 - q.cs0 + kChunk - 1) / kChunk);
    const int per_warp = (q.nch + kWarps - 1) / kWarps;
    q.cb = min(q.nch, warp * per_warp);
    q.ce = min(q.nch, q.cb + per_warp);
    return q;
  };
  // issue chunk ci of piece q into the ring (whole warp); a dead warp
  // issues nothing more
  auto issue = [&](const Piece &q, int ci) {
    if (dead) return;
    const int b = q.u / UH, kvh = (q.u % UH) / p.groups;
    const int64_t cs = q.cs0 + (int64_t)ci * kChunk;
    const int n = (int)min((int64_t)kChunk, q.t1 - cs);
    ring_fill<KBM, KPROD, VBM>(p, slot_addr(kk_issued), bar_addr(kk_issued),
                               (int64_t)b * p.ksb + (int64_t)kvh * p.ksh + cs,
                               (int64_t)b * p.vsb + (int64_t)kvh * p.vsh + cs, n, lane);
    ++kk_issued;
  };
  Piece first = piece_at(x0);
  if constexpr (STAGED) {
    const uint32_t lo0 = (dyn_base + 127u) & ~127u;
    const uint32_t hi0 = kLutAddr + kLutBytes, end = dyn_base + (uint32_t)p.dyn_bytes;
    const int n_lo = (int)((kLutAddr - lo0) / kSlotBytes);
    const int n_hi = end > hi0 ? (int)((end - hi0) / kSlotBytes) : 0;
    R = min(kMaxRing, (n_lo + n_hi) / kWarps);
    if (R < 2) {  // excluded on the host; reported, never silent
      if (tid == 0) atomicOr(p.faults, kFaultSmemLayout);
      return;
    }
    // global slot index s = warp * R + j: the first n_lo below the tables
    const int s0 = warp * R;
    ring_split = max(0, min(R, n_lo - s0));
    ring0 = lo0 + (uint32_t)s0 * kSlotBytes;
    ring1 = hi0 + (uint32_t)max(0, s0 - n_lo) * kSlotBytes;
    if (lane == 0) {
      for (int j = 0; j < R; ++j) mbar_init(smem_addr(&s_bar[warp * kMaxRing + j]), 1);
      asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncwarp();
    if (p.early) {
      for (int ci = first.cb; ci < min(first.ce, first.cb + R); ++ci) issue(first, ci);
    }
  } else {
    // warm L2 with this warp's first two chunks while the tables are set up
    if (unit && lane == 0 && first.cb < first.ce) {
      const int b = first.u / UH, kvh = (first.u % UH) / p.groups;
      const int64_t j = first.t0 + (int64_t)first.cb * kChunk;
      prefetch_chunk<KBM, KPROD, VBM>(p, (int64_t)b * p.ksb + (int64_t)kvh * p.ksh + j,
                                      (int64_t)b * p.vsb + (int64_t)kvh * p.vsh + j,
                                      min(2 * (int64_t)kChunk, first.t1 - j));
    }
  }

  for (int c = tid; c <= p.ctas; c += kThreads) s_cut[c] = cut(T, p.ctas, c);
  // Everything above reads only the arguments and the cache (and the cache
  // only when it is complete); the workspace (tables, query fragments,
  // counters) is written by the prep kernel, which may still be running
  // when this grid starts (programmatic dependent launch).
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  if constexpr (STAGED) {
    if (!p.early) {
      for (int ci = first.cb; ci < min(first.ce, first.cb + R); ++ci) issue(first, ci);
    }
  }

  // ---- once per CTA: the two pair tables, one copy per lane, read from the
  // workspace (L2) directly
  float inv_sK, inv_sV;
  {
    const uint32_t *ktab = reinterpret_cast<const uint32_t *>(p.ws + 64);
    const uint32_t *vtab = reinterpret_cast<const uint32_t *>(p.ws + 320);
    inv_sK = __ldg(p.ws + 0);
    inv_sV = __ldg(p.ws + 1);
    uint4 *tab = reinterpret_cast<uint4 *>(s_lut);
    // register-fed: the 256 + 256 distinct entries first (one load a thread,
    // all in flight) into the partials' memory, idle until the first piece
    // ends, then the per-lane copies from there; staged: the partials'
    // memory may hold ring slots already in flight, so from L2 directly
    const uint32_t *ks = ktab, *vs = vtab;
    if constexpr (!STAGED) {
      uint32_t *raw = reinterpret_cast<uint32_t *>(s_part);
      for (int i = tid; i < 512; i += kThreads) raw[i] = i < 256 ? (KBM > 0 ? __ldg(ktab + i) : 0u) : __ldg(vtab + i - 256);
      __syncthreads();
      ks = raw;
      vs = raw + 256;
    }
    if constexpr (K4) {
      // key entry e: the pair entries of its low and high nibbles
      for (int i = tid; i < 256 * 16; i += kThreads) {
        const int e = i >> 4;
        const uint32_t lo = ks[e & 15], hi = ks[e >> 4];
        tab[i] = make_uint4(lo, hi, lo, hi);
      }
      uint4 *vt = reinterpret_cast<uint4 *>(s_lut + (kVTab4Addr - kLutAddr));
      for (int i = tid; i < 256 * 8; i += kThreads) {  // the first 128 bytes of each row
        const uint32_t v = vs[i >> 3];
        vt[(i >> 3) * 16 + (i & 7)] = make_uint4(v, v, v, v);
      }
    } else {
      for (int i = tid; i < 256 * 16; i += kThreads) {  // 16 uint4 per 256-byte row
        const int e = i >> 4, part = i & 15;
        const uint32_t v = part < 8 ? (KBM > 0 ? ks[e] : 0u) : vs[e];
        tab[i] = make_uint4(v, v, v, v);
      }
    }
  }
  const float sK = 1.0f / inv_sK;
  const float kscale = inv_sK * p.scale_log2;  // logit = raw score * n_K * kscale
  const uint32_t koff = kLutAddr + lane * (K4 ? 8 : 4);
  const uint32_t voff = (K4 ? kVTab4Addr : kLutAddr + 128) + lane * 4;
  const bool want_scores = p.scores != nullptr;

  bool first_piece = true;
  for (int64_t x = x0; x < x1;) {
    const Piece pc = first_piece ? first : piece_at(x);
    first_piece = false;
    const int u = pc.u;
    const int64_t ustart = pc.ustart, ulen = pc.ulen, t0 = pc.t0, t1 = pc.t1, cs0 = pc.cs0;
    x = ustart + t1;
    const int b = u / UH;
    const int kvh = (u % UH) / p.groups;
    const int grp = (u % UH) % p.groups;
    const int h0 = kvh * p.g + grp * 8;
    const int gh = min(8, p.g - grp * 8);

    __syncthreads();  // tables ready / the previous piece's shared data consumed
    if constexpr (STAGED) {
      // the first R chunks of a later piece (the previous piece's merge, which
      // reuses ring memory, is over)
      if (kk_issued == kk_used) {
        for (int ci = pc.cb; ci < min(pc.ce, pc.cb + R); ++ci) issue(pc, ci);
      }
    }

    // ---- B fragments of the unit, written by the prep kernel in this
    // lane's register order.  PACK: column n < 4 is the hi half of head n,
    // n >= 4 the lo half of head n - 4.  Else qf = hi and qf2 = lo of head
    // g8.  Lanes whose head is absent (fewer than 4 or 8 heads) hold zeros.
    constexpr bool QS_SMEM = qs_in_smem<KPROD, STAGED>();
    uint32_t qf[8][2], qf2[PACK ? 1 : 8][2];
    uint32_t qsf[(KPROD && !QS_SMEM) ? 4 : 1][2], qsf2[(KPROD && !PACK && !QS_SMEM) ? 4 : 1][2];
    // QS_SMEM: the unit's S q' digit fragments at the start of the dynamic
    // region, [S][hi 0 / lo 1][lane] word pairs (one 8-byte load per lane and
    // step)
    const uint2 *s_qs = reinterpret_cast<const uint2 *>(smem + (((dyn_base + 15u) & ~15u) - dyn_base));
    // the QJL term of this lane's two head columns c: sum_i digit-weighted
    // MMA results, qd[c][0] * hi (+ qd[c][1] * lo) + qd[c][2] = <S q', sign>
    float qd[2][3];
    {
      const bool has = (PACK ? (g8 & 3) : g8) < gh;
      const uint4 *fr = p.frag + (int64_t)u * (kFragWords / 4) + lane;
      auto ld4 = [&](int w4) { return has ? __ldg(fr + w4 * 32) : make_uint4(0u, 0u, 0u, 0u); };
      auto put = [](auto &f, int k, uint4 v) {
        f[2 * k][0] = v.x;
        f[2 * k][1] = v.y;
        f[2 * k + 1][0] = v.z;
        f[2 * k + 1][1] = v.w;
      };
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        put(qf, k, ld4(k));
        if constexpr (!PACK) put(qf2, k, ld4(4 + k));
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        if constexpr (KPROD && !QS_SMEM) put(qsf, k, ld4((PACK ? 4 : 8) + k));
        if constexpr (KPROD && !PACK && !QS_SMEM) put(qsf2, k, ld4(10 + k));
      }
      if constexpr (KPROD) {
        const uint32_t *fw = reinterpret_cast<const uint32_t *>(p.frag + (int64_t)u * (kFragWords / 4));
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int h = PACK ? 2 * (tig & 1) + c : 2 * tig + c;  // this lane's head columns
          const float ch = h < gh ? __uint_as_float(__ldg(fw + (15 * 32 + h) * 4 + 0)) : 0.f;
          const float th = h < gh ? __uint_as_float(__ldg(fw + (15 * 32 + h) * 4 + 1)) : 0.f;
          // the MMAs sum -bit * digit: <S q', 2 bit - 1> = -2 c_h (256 hi + lo) - T_h,
          // scaled by kappa s_K (the estimator's sqrt(pi/2)/d; the table holds s_K c)
          const float ks = kKappa * sK;
          if constexpr (PACK) {  // lanes tig < 2 hold the hi digits' columns, the others the lo digits'
            qd[c][0] = -2.f * ch * (tig < 2 ? 256.f : 1.f) * ks;
            qd[c][1] = 0.f;
            qd[c][2] = tig < 2 ? -th * ks : 0.f;
          } else {
            qd[c][0] = -512.f * ch * ks;
            qd[c][1] = -2.f * ch * ks;
            qd[c][2] = -th * ks;
          }
        }
      }
      if constexpr (QS_SMEM) {
        // every thread copies its share; the barrier below (before the
        // chunk loop) publishes them
        uint2 *dst = const_cast<uint2 *>(s_qs);
        for (int i = tid; i < 2 * 4 * 32; i += kThreads) {
          const int ln = i & 31, S = (i >> 5) & 3, j2 = i >> 7;
          if (PACK && j2 == 1) continue;
          const bool h = (PACK ? ((ln >> 2) & 3) : (ln >> 2)) < gh;
          const int w4 = (PACK ? 4 : (j2 ? 10 : 8)) + (S >> 1);
          uint4 v = h ? __ldg(p.frag + (int64_t)u * (kFragWords / 4) + ln + w4 * 32) : make_uint4(0u, 0u, 0u, 0u);
          dst[(S * 2 + j2) * 32 + ln] = (S & 1) ? make_uint2(v.z, v.w) : make_uint2(v.x, v.y);
        }
        __syncthreads();
      }
    }

    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    // M_run: the column's reference (finite; -FLT_MAX until a valid token);
    // M_thr = M_run + kLazy
    float M_run[2] = {-FLT_MAX, -FLT_MAX}, M_thr[2] = {-FLT_MAX, -FLT_MAX};
    float l_run[2] = {0.f, 0.f};

    const int64_t kbase = (int64_t)b * p.ksb + (int64_t)kvh * p.ksh;
    const int64_t vbase = (int64_t)b * p.vsb + (int64_t)kvh * p.vsh;
    // the piece's chunks [0, nch) from cs0, of which [0, nfull) are full and
    // unmasked (register-fed); this warp takes [c_begin, c_end)
    const int nch = pc.nch;
    const int nfull = (int)((t1 - cs0) / kChunk);
    const int c_begin = pc.cb, c_end = pc.ce;

    KBuf<KBM, KPROD> kb;
    VBuf<VBM> vb;
    FastPtrs fp{};
    if constexpr (!STAGED) {
      fp = fast_ptrs(kbase + t0, vbase + t0, tig, g8);
      // warm L2 up to the end of the first prefetch window
      if (unit && lane == 0 && c_begin + 1 < c_end) {
        const int64_t jp = t0 + (int64_t)(c_begin + 1) * kChunk;
        const int pe = min(c_end, c_begin + kPfWin);
        prefetch_chunk<KBM, KPROD, VBM>(p, kbase + jp, vbase + jp,
                                        min((int64_t)(pe - c_begin - 1) * kChunk, t1 - jp));
      }
      if (c_begin < c_end) {
        if (unit && c_begin < nfull) {
          load_k_fast<KBM, KPROD, VBM>(kb, p, fp, c_begin, tig, g8);
          load_v_fast<KBM, KPROD, VBM>(vb, p, fp, c_begin, g8);
        } else {
          const int64_t j0 = t0 + (int64_t)c_begin * kChunk;
          const int nv = (int)min((int64_t)kChunk, t1 - j0);
          load_k_slow(kb, p, kbase + j0 * p.ksn, vbase + j0 * p.vsn, nv, tig, g8);
          load_v_slow(vb, p, vbase + j0 * p.vsn, nv, g8, tig);
        }
      }
    }
    (void)nch;
    for (int ci = c_begin; ci < c_end; ++ci) {
      const int cn = ci + 1;
      const bool more = cn < c_end;
      const bool fast_next = unit && cn < nfull;
      const int64_t cstart = cs0 + (int64_t)ci * kChunk;  // the chunk's first token
      const char *slot = nullptr;
      if constexpr (STAGED) {
        const uint32_t k = kk_used++;
        slot = smem + (slot_addr(k) - dyn_base);
        const bool was_dead = dead;
        ring_wait(bar_addr(k), (k / (uint32_t)R) & 1u, p.faults, dead);
        if (dead && !was_dead) dead_at = k;  // from here on the slots hold what they hold
        const int lo = (int)max((int64_t)0, t0 - cstart), hi = (int)min((int64_t)kChunk, t1 - cstart);
        load_k_ring<KBM, KPROD, VBM>(kb, slot, lo, hi, tig, g8);
      } else {
        // every kPfWin chunks, warm L2 with the window after the next one
        if (unit && lane == 0 && ((ci - c_begin) % kPfWin) == 0 && ci + kPfWin < c_end) {
          const int64_t jp = t0 + (int64_t)(ci + kPfWin) * kChunk;
          const int pe = min(c_end, ci + 2 * kPfWin);
          prefetch_chunk<KBM, KPROD, VBM>(p, kbase + jp, vbase + jp,
                                          min((int64_t)(pe - ci - kPfWin) * kChunk, t1 - jp));
        }
      }
      // -------- scores: rows (ms, r) -> token cstart + 16 ms + 8 r + g8
      float sc[2][4];
      float nvl[2][2];  // log2 n_V of the lane's rows (masked rows: any value, their logit is -inf)
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
          kr[r] = KPROD ? kb.kr[ms][r] : 0.f;
          // (staged masked rows hold whatever the slot holds: kept finite)
          nvl[ms][r] = (STAGED && !ok[r]) ? 0.f : __log2f(kb.vn[ms][r]);
        }
        // the lo halves (more than 4 heads) accumulate apart: two chains of
        // dependent MMAs instead of one twice as long
        float cm[4] = {0.f, 0.f, 0.f, 0.f}, cm2[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (K4) {
          // byte S of a row's 64-bit stream: pairs 2S and 2S + 1 in one read
#define TQ_KSTEP4(S)                                                              \
  {                                                                               \
    constexpr uint32_t sel = 0x7604u | (((S) & 3) << 4);                          \
    const uint2 e0 = lut64(__byte_perm(kw[0][(S) >> 2], koff, sel));              \
    const uint2 e1 = lut64(__byte_perm(kw[1][(S) >> 2], koff, sel));              \
    const uint32_t a[4] = {e0.x, e1.x, e0.y, e1.y};                               \
    mma16816(cm, a, qf[S][0], qf[S][1]);                                          \
    if constexpr (!PACK) mma16816(cm2, a, qf2[S][0], qf2[S][1]);                  \
  }
          TQ_KSTEP4(0) TQ_KSTEP4(1) TQ_KSTEP4(2) TQ_KSTEP4(3)
          TQ_KSTEP4(4) TQ_KSTEP4(5) TQ_KSTEP4(6) TQ_KSTEP4(7)
#undef TQ_KSTEP4
        } else if constexpr (KBM > 0) {
#define TQ_KSTEP(S)                                                               \
  {                                                                               \
    uint32_t a[4];                                                                \
    a[0] = lut(pair_addr<KBM, 2 * (S), KW>(kw[0], koff));                         \
    a[1] = lut(pair_addr<KBM, 2 * (S), KW>(kw[1], koff));                         \
    a[2] = lut(pair_addr<KBM, 2 * (S) + 1, KW>(kw[0], koff));                     \
    a[3] = lut(pair_addr<KBM, 2 * (S) + 1, KW>(kw[1], koff));                     \
    mma16816(cm, a, qf[S][0], qf[S][1]);                                          \
    if constexpr (!PACK) mma16816(cm2, a, qf2[S][0], qf2[S][1]);                  \
  }
          TQ_KSTEP(0) TQ_KSTEP(1) TQ_KSTEP(2) TQ_KSTEP(3)
          TQ_KSTEP(4) TQ_KSTEP(5) TQ_KSTEP(6) TQ_KSTEP(7)
#undef TQ_KSTEP
        }
        if constexpr (!PACK) {
#pragma unroll
          for (int i = 0; i < 4; ++i) cm[i] += cm2[i];
        }
        float cq[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (KPROD) {
          // the signs as int8 0 / -1 (four a register, bits 7, 15, 23, 31 of
          // the lane's word shifted left by 2S + j) against the S q' digits
          int ch[4] = {0, 0, 0, 0}, cl[4] = {0, 0, 0, 0};
#define TQ_QSTEP(S)                                                               \
  {                                                                               \
    uint32_t a[4];                                                                \
    a[0] = sign_bytes(qj[0] << (2 * (S)));                                        \
    a[1] = sign_bytes(qj[1] << (2 * (S)));                                        \
    a[2] = sign_bytes(qj[0] << (2 * (S) + 1));                                    \
    a[3] = sign_bytes(qj[1] << (2 * (S) + 1));                                    \
    if constexpr (QS_SMEM) {                                                      \
      const uint2 f = s_qs[((S) * 2) * 32 + lane];                                \
      mma16832_s8(ch, a, f.x, f.y);                                               \
      if constexpr (!PACK) {                                                      \
        const uint2 f2 = s_qs[((S) * 2 + 1) * 32 + lane];                         \
        mma16832_s8(cl, a, f2.x, f2.y);                                           \
      }                                                                           \
    } else {                                                                      \
      mma16832_s8(ch, a, qsf[S][0], qsf[S][1]);                                   \
      if constexpr (!PACK) mma16832_s8(cl, a, qsf2[S][0], qsf2[S][1]);            \
    }                                                                             \
  }
          TQ_QSTEP(0) TQ_QSTEP(1) TQ_QSTEP(2) TQ_QSTEP(3)
#undef TQ_QSTEP
          // the two head columns of a row as one pair
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            float b0 = qd[0][2], b1 = qd[1][2];
            if constexpr (!PACK)
              dev::fma_x2(b0, b1, (float)cl[2 * r], (float)cl[2 * r + 1], qd[0][1], qd[1][1], b0, b1);
            dev::fma_x2(cq[2 * r], cq[2 * r + 1], (float)ch[2 * r], (float)ch[2 * r + 1], qd[0][0], qd[1][0], b0, b1);
          }
        }
        // raw score = main + kappa gamma s_K qjl (the table holds s_K c; kappa
        // s_K is folded into qd)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          if constexpr (KPROD)
            dev::fma_x2(cm[2 * r], cm[2 * r + 1], kr[r], kr[r], cq[2 * r], cq[2 * r + 1], cm[2 * r], cm[2 * r + 1]);
          if constexpr (PACK) {  // hi + lo columns
            const float o0 = __shfl_xor_sync(dev::kFull, cm[2 * r], 2);
            const float o1 = __shfl_xor_sync(dev::kFull, cm[2 * r + 1], 2);
            dev::add_x2(cm[2 * r], cm[2 * r + 1], cm[2 * r], cm[2 * r + 1], o0, o1);
          }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          float t0, t1;
          dev::mul_x2(t0, t1, cm[2 * r], cm[2 * r + 1], fs[r], fs[r]);
          sc[ms][2 * r] = ok[r] ? t0 : -INFINITY;
          sc[ms][2 * r + 1] = ok[r] ? t1 : -INFINITY;
        }
        if (want_scores) {
#pragma unroll
          for (int r = 0; r < 2; ++r) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const int head = PACK ? 2 * (tig & 1) + c : 2 * tig + c;
              if (ok[r] && head < gh && (!PACK || tig < 2)) {
                const int64_t j = cstart + 16 * ms + 8 * r + g8;
                p.scores[((int64_t)b * p.Hq + h0 + head) * p.seq_len + j] =
                    cm[2 * r + c] * (kb.kn[ms][r] * inv_sK);
              }
            }
          }
        }
      }
      // the key registers are free: start the next chunk's key loads
      if constexpr (!STAGED) {
        if (more) {
          if (fast_next) {
            load_k_fast<KBM, KPROD, VBM>(kb, p, fp, cn, tig, g8);
          } else {
            const int64_t jn = t0 + (int64_t)cn * kChunk;
            load_k_slow(kb, p, kbase + jn * p.ksn, vbase + jn * p.vsn, (int)min((int64_t)kChunk, t1 - jn), tig,
                        g8);
          }
        }
      }

      // -------- online softmax, per head column c, against the column's
      // reference M_run, which moves only when some lane's u = logit +
      // max(log2 n_V, kNvlFloor) passes it by more than kLazy: one vote for
      // both columns, and the column maxima, the rescale of l and of the
      // accumulators only then (warp-uniform branch)
      float wgt[2][4];
      float Mx[2];
      {
        // u[row][c], the two columns of a row as one pair
        float u[4][2];
#pragma unroll
        for (int ms = 0; ms < 2; ++ms) {
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float nf = fmaxf(nvl[ms][r], kNvlFloor);
            dev::add_x2(u[2 * ms + r][0], u[2 * ms + r][1], sc[ms][2 * r], sc[ms][2 * r + 1], nf, nf);
          }
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) Mx[c] = fmaxf(fmaxf(u[0][c], u[1][c]), fmaxf(u[2][c], u[3][c]));
      }
      if (__any_sync(dev::kFull, Mx[0] > M_thr[0] || Mx[1] > M_thr[1])) {
        float aM[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float m = Mx[c];
#pragma unroll
          for (int o = 4; o <= 16; o <<= 1) m = fmaxf(m, __shfl_xor_sync(dev::kFull, m, o));
          const float Mn = m > M_thr[c] ? m : M_run[c];
          aM[c] = ex2(M_run[c] - Mn);
          l_run[c] *= aM[c];
          M_run[c] = Mn;
          M_thr[c] = Mn + kLazy;
        }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          acc[mt][0] *= aM[0];
          acc[mt][1] *= aM[1];
          acc[mt][2] *= aM[0];
          acc[mt][3] *= aM[1];
        }
      }
      {
        float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
        for (int ms = 0; ms < 2; ++ms) {
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            float e0, e1, w0, w1;
            dev::sub_x2(e0, e1, sc[ms][2 * r], sc[ms][2 * r + 1], M_run[0], M_run[1]);
            dev::add_x2(ls0, ls1, ls0, ls1, ex2(e0), ex2(e1));
            dev::add_x2(w0, w1, e0, e1, nvl[ms][r], nvl[ms][r]);
            wgt[ms][2 * r] = ex2(w0);
            wgt[ms][2 * r + 1] = ex2(w1);
          }
        }
        dev::add_x2(l_run[0], l_run[1], l_run[0], l_run[1], ls0, ls1);
      }

      // -------- PV: for each 16-token half, B = W^T via movmatrix
      if constexpr (STAGED) load_v_ring<KBM, KPROD, VBM>(vb, slot, g8, tig);
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
        // tokens (q4 = 0, 1) and (2, 3) interleaved into pair indices: the
        // table then yields A's (token, token) pairs at one dim directly
        uint32_t xe[2][VW], xo[2][VW];
        interleave_tokens<VBM>(vw[0], vw[1], xe[0], xo[0]);
        interleave_tokens<VBM>(vw[2], vw[3], xe[1], xo[1]);
#define TQ_VSTEP(MT)                                                              \
  {                                                                               \
    uint32_t a[4];                                                                \
    a[0] = lut(pair_addr<VBM, MT, VW>(xe[0], voff));                              \
    a[1] = lut(pair_addr<VBM, MT, VW>(xo[0], voff));                              \
    a[2] = lut(pair_addr<VBM, MT, VW>(xe[1], voff));                              \
    a[3] = lut(pair_addr<VBM, MT, VW>(xo[1], voff));                              \
    mma16816(acc[MT], a, b0, b1);                                                 \
    if constexpr (!PACK) mma16816(acc[MT], a, b2, b3);                            \
  }
        TQ_VSTEP(0) TQ_VSTEP(1) TQ_VSTEP(2) TQ_VSTEP(3)
        TQ_VSTEP(4) TQ_VSTEP(5) TQ_VSTEP(6) TQ_VSTEP(7)
#undef TQ_VSTEP
      }
      if constexpr (STAGED) {
        // the slot is read: refill it with the chunk R ahead
        __syncwarp();
        if (ci + R < c_end) issue(pc, ci + R);
      } else {
        // the value registers are free: start the next chunk's value loads
        if (more) {
          if (fast_next) {
            load_v_fast<KBM, KPROD, VBM>(vb, p, fp, cn, g8);
          } else {
            const int64_t jn = t0 + (int64_t)cn * kChunk;
            load_v_slow(vb, p, vbase + jn * p.vsn, (int)min((int64_t)kChunk, t1 - jn), g8, tig);
          }
        }
      }
    }

    // ---- warp totals: l over the 8 row groups (one reference per column);
    // a column that saw no valid token reports -inf; PACK: hi + lo columns
    // of acc
    float m_run[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
#pragma unroll
      for (int o = 4; o <= 16; o <<= 1) l_run[c] += __shfl_xor_sync(dev::kFull, l_run[c], o);
      if (M_run[c] == -FLT_MAX) M_run[c] = -INFINITY;
      m_run[c] = M_run[c];
    }
    if constexpr (PACK) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[mt][i] += __shfl_xor_sync(dev::kFull, acc[mt][i], 2);
      }
    }

    // ---- CTA merge of the warps' partials for this piece (staged: their
    // shared memory is ring memory, free once every warp is past its loop)
    if constexpr (STAGED) __syncthreads();
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

  // a warp that gave up a wait drains the copies it still has in flight
  // (bounded again) before the CTA's shared memory goes away
  if constexpr (STAGED) {
    if (dead) {
      bool dead2 = false;
      for (uint32_t k = dead_at; k < kk_issued && !dead2; ++k)
        ring_wait(bar_addr(k), (k / (uint32_t)R) & 1u, p.faults, dead2);
    }
  }
}

__global__ void zero_out_kernel(float *out, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = 0.f;
}

// Register-fed variant's dynamic shared memory: enough to reach the end of
// the tables (key quads: the value table's window; else the warps'
// partials past the shared window) from any dynamic base at or above 0.
// Every table keeps 256 rows: a lookup's byte may carry bits of the next
// field above a pair index.
constexpr size_t split_smem_bytes(int warps, bool k4) {
  return k4 ? (size_t)kVTab4Addr + kLutBytes
            : (size_t)kLutAddr + kLutBytes + (size_t)warps * 8 * kPW * sizeof(float);
}

// Static shared memory plus the per-block reserve must end at or below
// kLutAddr, where the dynamic region's pair tables start.  *dyn_max gets the
// largest dynamic allocation the kernel can have on this device, *base the
// highest address its dynamic region can start at.
template <typename K>
cudaError_t smem_layout(K kern, size_t *dyn_max, size_t *base) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  int dev = 0, reserved = 0, optin = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  *base = (size_t)reserved + fa.sharedSizeBytes + 128;
  if (*base > kLutAddr) return cudaErrorInvalidConfiguration;
  *dyn_max = (size_t)optin > fa.sharedSizeBytes ? (size_t)optin - fa.sharedSizeBytes : 0;
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

// Launches one instantiation.  The staged variant takes all the dynamic
// shared memory the device allows; it needs room for at least two ring
// slots per warp next to the tables, which the record sizes of d = 128
// always leave (else cudaErrorInvalidConfiguration).
template <int KBM, bool KPROD, int VBM, bool PACK, bool STAGED>
cudaError_t run_split(SplitParams sp, cudaStream_t s) {
  auto kern = decode_split_kernel<KBM, KPROD, VBM, PACK, STAGED>;
  constexpr int warps = split_warps<PACK, KPROD, STAGED>();
  size_t dyn_max = 0, base = 0;
  static const cudaError_t layout = smem_layout(kern, &dyn_max, &base);
  static const size_t dyn_keep = dyn_max, base_keep = base;
  if (layout != cudaSuccess) return layout;
  constexpr bool k4 = key_quads<KBM, STAGED>();
  size_t smem = split_smem_bytes(warps, k4);
  // key quads: digit fragments and partials below the tables
  if (k4 && ((base_keep + 15) & ~(size_t)15) + kQsBytes + (size_t)warps * 8 * kPW * 4 > kLutAddr)
    return cudaErrorInvalidConfiguration;
  if constexpr (STAGED) {
    smem = dyn_keep;
    constexpr size_t sb = (ring_slot_bytes(KBM, KPROD, VBM) + 127) & ~(size_t)127;
    const size_t lo0 = (base_keep + 127) & ~(size_t)127;
    const size_t n_lo = (kLutAddr - lo0) / sb;
    const size_t end = base_keep - 128 + dyn_keep;  // lowest possible end of the allocation
    const size_t n_hi = end > (size_t)kLutAddr + kLutBytes ? (end - kLutAddr - kLutBytes) / sb : 0;
    if ((n_lo + n_hi) / warps < 2 || end < (size_t)kLutAddr + kLutBytes + (size_t)warps * 8 * kPW * 4)
      return cudaErrorInvalidConfiguration;
  }
  sp.dyn_bytes = (int)smem;
  cudaError_t e = set_smem_once<decode_split_kernel<KBM, KPROD, VBM, PACK, STAGED>>(smem);
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

template <bool STAGED, bool KPROD, int VBM, bool PACK>
cudaError_t by_kbits(int kbm, const SplitParams &sp, cudaStream_t s) {
  switch (kbm) {
    case 0: if constexpr (KPROD) return run_split<0, true, VBM, PACK, STAGED>(sp, s); else return cudaErrorInvalidValue;
    case 1: return run_split<1, KPROD, VBM, PACK, STAGED>(sp, s);
    case 2: return run_split<2, KPROD, VBM, PACK, STAGED>(sp, s);
    case 3: return run_split<3, KPROD, VBM, PACK, STAGED>(sp, s);
    case 4: return run_split<4, KPROD, VBM, PACK, STAGED>(sp, s);
  }
  return cudaErrorInvalidValue;
}

template <bool STAGED, int VBM>
cudaError_t by_kvariant(int kbm, bool kprod, bool pack, const SplitParams &sp, cudaStream_t s) {
  if (pack) return kprod ? by_kbits<STAGED, true, VBM, true>(kbm, sp, s) : by_kbits<STAGED, false, VBM, true>(kbm, sp, s);
  return kprod ? by_kbits<STAGED, true, VBM, false>(kbm, sp, s) : by_kbits<STAGED, false, VBM, false>(kbm, sp, s);
}

template <bool STAGED>
cudaError_t launch_split_variant(int kbm, bool kprod, int vbm, bool pack, const SplitParams &sp, cudaStream_t s) {
  switch (vbm) {
    case 1: return by_kvariant<STAGED, 1>(kbm, kprod, pack, sp, s);
    case 2: return by_kvariant<STAGED, 2>(kbm, kprod, pack, sp, s);
    case 3: return by_kvariant<STAGED, 3>(kbm, kprod, pack, sp, s);
    case 4: return by_kvariant<STAGED, 4>(kbm, kprod, pack, sp, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace
}  // namespace tq
