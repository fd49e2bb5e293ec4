// Decode attention on CUDA cores (sm_100a) for the caches the tensor-core
// split kernel does not take: d = 64 or 256 with the Hadamard rotation,
// dense (Haar) rotations of any supported d other than 128, TurboQuant_prod
// values, and outlier-channel split caches.  Same definition as the main
// path ("I Spent 31 Hours On The Math Behind Turboquant", section "KV Cache:
// The problem"; "内存厂商的噩梦来了", section 4.2, the asymmetric score):
//   s_j = sum_g n_gj (<q'_g, c_g[idx_gj]> + [prod] ||r_gj|| sqrt(pi/2)/d_g <S_g q'_g, sign_gj>),
//   q'_g = Pi_g q[channels_g], softmax over s_j * scale, and each value group
//   summed in its rotated basis, o'_g = sum_j p_j n_gj (c_g[idx_gj] + [prod]
//   ||r_gj|| sqrt(pi/2)/d_g S_g^T sign_gj), rotated back once into its
//   channels, o[channels_g] = Pi_g^T o'_g.  A plain cache is one group over
//   all d channels; an outlier-channel split cache ("TurboQuant của Google",
//   the correction in the experiments section) is two.
//
// Flash-decoding split over the sequence:
//   general_partial_kernel, grid (splits, B * Hkv * head groups): up to 8
//     query heads of one kv head over one token slice, in tiles of 64
//     tokens: the tile's records and norms staged in shared memory with
//     coalesced copies, scores (4 threads a token, q' and S q' read
//     coordinate-major, all heads of a coordinate in one vector load), an
//     online softmax per head, then the values: a thread per coordinate (and
//     token class when d <= 128) accumulating every head's weighted
//     centroids (and, for prod values, weighted signs); the slice's (m, l,
//     o', signs) go to a workspace slot;
//   general_merge_kernel, a block per (batch, query head): merges the slots,
//   adds S_g^T of the sign sums, applies each group's inverse rotation and
//   1/l, and scatters the groups into their channels.

#include "../../include/tq.h"
#include "tq_device.cuh"
#include "tq_internal.h"

#include <atomic>

namespace tq {
namespace {

constexpr int kGnThreads = 256;
constexpr int kGnMaxD = 256;
constexpr int kGnHeads = 8;   // query heads a block
constexpr int kGnTile = 64;   // tokens a tile
constexpr int kGnMaxSplits = 128;  // sequence splits at most
constexpr float kGnLog2e = 1.4426950408889634f;
constexpr float kGnSqrtHalfPi = 1.2533141373155003f;

// One quantizer group: its dimension and offset among the head's
// rotated coordinates, codebook, rotation (dense Pi, or the Hadamard signs
// when rot is NULL), channel list (NULL: channels 0..d-1), and its cache.
struct GnGroup {
  int d, off, bm;
  bool prod;
  const float *cent, *rot, *S;
  const int8_t *signs;
  const int32_t *chan;
  const uint8_t *codes, *qjl;
  const float *norms, *rnorms;
  int64_t sb, sh, sn;
};

struct GnParams {
  GnGroup k[2], v[2];
  int nk, nv;        // groups per side (1 or 2)
  const void *q;
  int q_dtype;
  int B, Hq, Hkv, g, hg, d, splits;
  int64_t seq_len, per_split;
  const int32_t *seq_lens;
  float scale_log2;  // softmax scale * log2(e)
  float *out, *scores;
  float *ws;         // slots [splits][B * Hq][4 + 2 d]
};

__device__ __forceinline__ int64_t gn_len(const GnParams &p, int b) {
  if (!p.seq_lens) return p.seq_len;
  const int64_t L = p.seq_lens[b];
  return L < 0 ? 0 : (L > p.seq_len ? p.seq_len : L);
}

__device__ __forceinline__ float gn_q(const GnParams &p, int64_t i) {
  if (p.q_dtype == TQ_F32) return __ldg(static_cast<const float *>(p.q) + i);
  const unsigned short h = __ldg(static_cast<const unsigned short *>(p.q) + i);
  return p.q_dtype == TQ_BF16 ? __uint_as_float((uint32_t)h << 16) : __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ float gn_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// In-place unnormalised FWHT of nv vectors of length d (power of two) in
// shared memory, rows `stride` floats apart; the whole block takes part.
__device__ void gn_fwht(float *x, int nv, int d, int stride) {
  for (int h = d / 2; h >= 1; h >>= 1) {
    __syncthreads();
    for (int e = threadIdx.x; e < nv * (d / 2); e += blockDim.x) {
      const int v = e / (d / 2), k = e % (d / 2);
      const int i = (k / h) * 2 * h + (k % h);
      float *r = x + v * stride;
      const float a = r[i], b = r[i + h];
      r[i] = a + b;
      r[i + h] = a - b;
    }
  }
  __syncthreads();
}

// Staged records sit in shared memory token-major with a pitch of whole
// 32-bit words, so that a field is read as a word (two at a word boundary).
__device__ __forceinline__ int gn_pitch(int nbytes) { return (nbytes + 3) & ~3; }

// Index pair (fields i, i + 1; i even) of an LSB-first bm-bit stream held in
// the words rec[]: a 2 bm-bit pair-table index, field i in the low bits.
__device__ __forceinline__ uint32_t gn_pair_s(const uint32_t *rec, int i, int bm) {
  const int q = i * bm;
  const int wi = q >> 5, sh = q & 31;
  uint32_t v = rec[wi] >> sh;
  if (sh + 2 * bm > 32) v |= rec[wi + 1] << (32 - sh);
  return v & ((1u << (2 * bm)) - 1u);
}

// Bits i, i + 1 (i even) of a sign stream held in words: bit 0 / bit 1.
__device__ __forceinline__ uint32_t gn_bits2_s(const uint32_t *rec, int i) { return (rec[i >> 5] >> (i & 31)) & 3u; }

// Copies nbytes-byte records rec0, rec0 + sn, ... (nt of them) of src into
// dst, token-major at gn_pitch(nbytes) bytes a token: 32-bit words when the
// records are contiguous whole words (the cache arrays are 16-byte
// aligned), else bytes.  The whole block takes part.
__device__ __forceinline__ void gn_stage(const uint8_t *src, int64_t rec0, int64_t sn, int nbytes, int nt,
                                         uint8_t *dst) {
  if (sn == 1 && (nbytes & 3) == 0) {
    const uint32_t *s4 = reinterpret_cast<const uint32_t *>(src + rec0 * nbytes);
    uint32_t *d4 = reinterpret_cast<uint32_t *>(dst);
    const int nw = nt * (nbytes >> 2);
    for (int e = threadIdx.x; e < nw; e += kGnThreads) d4[e] = __ldg(s4 + e);
  } else {
    const int pitch = gn_pitch(nbytes);
    const int nb = nt * nbytes;
    for (int e = threadIdx.x; e < nb; e += kGnThreads) {
      const int tt = e / nbytes, by = e - tt * nbytes;
      dst[tt * pitch + by] = __ldg(src + (rec0 + tt * sn) * nbytes + by);
    }
  }
}

// Staging capacity of one side's tile (two groups at most, each padded to
// whole words): codes at most 4 bits a coordinate, and the QJL signs.
constexpr int kGnCodeBytes = kGnTile * (kGnMaxD / 2 + 8);
constexpr int kGnSignBytes = kGnTile * (kGnMaxD / 8 + 8);
constexpr int kGnStageBytes = 2 * (kGnCodeBytes + kGnSignBytes);
// Pair tables in dynamic shared memory: [K / V][group][256] centroid pairs.
constexpr int kGnPairBytes = 2 * 2 * 256 * 8;

// Loads of the query fragments by head count: NH consecutive floats.
template <int NH>
__device__ __forceinline__ void gn_ld_heads(const float *src, float (&v)[NH]) {
  if constexpr (NH % 4 == 0) {
#pragma unroll
    for (int k = 0; k < NH / 4; ++k) {
      const float4 t = reinterpret_cast<const float4 *>(src)[k];
      v[4 * k] = t.x, v[4 * k + 1] = t.y, v[4 * k + 2] = t.z, v[4 * k + 3] = t.w;
    }
  } else if constexpr (NH == 2) {
    const float2 t = *reinterpret_cast<const float2 *>(src);
    v[0] = t.x, v[1] = t.y;
  } else {
    v[0] = src[0];
  }
}

// y_h = A x_h for the block's heads h < nh: A is n x n row-major in global
// memory, x_h and y_h rows of shared memory kGnMaxD floats apart.  A warp
// takes a row, its lanes read consecutive columns (coalesced) and sum across
// the warp; the whole block takes part.
template <int NH>
__device__ __forceinline__ void gn_rows_times(const float *A, int n, const float *x, float *y, int nh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int r = warp; r < n; r += kGnThreads / 32) {
    const float *row = A + (int64_t)r * n;
    float acc[NH];
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) acc[hh] = 0.f;
    for (int c = lane; c < n; c += 32) {
      const float a = __ldg(row + c);
#pragma unroll
      for (int hh = 0; hh < NH; ++hh)
        if (hh < nh) acc[hh] = fmaf(a, x[hh * kGnMaxD + c], acc[hh]);
    }
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) {
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) acc[hh] += __shfl_xor_sync(dev::kFull, acc[hh], o);
      if (lane == 0 && hh < nh) y[hh * kGnMaxD + r] = acc[hh];
    }
  }
}

// NH: the most query heads a block handles (1, 2, 4 or 8): the per-token
// head loops are unrolled to it.
template <int NH>
__global__ void __launch_bounds__(kGnThreads) general_partial_kernel(GnParams p) {
  // setup: q'_g and S_g q'_g by head ([8][kGnMaxD] each); tiles: the staged
  // records, K codes | K signs | V codes | V signs; end: the halves' sums
  __shared__ __align__(16) unsigned char s_raw[kGnStageBytes];
  __shared__ __align__(16) float s_qT[kGnMaxD][NH];   // q'_g, coordinate-major
  __shared__ __align__(16) float s_qsT[kGnMaxD][NH];  // S_g q'_g (prod key groups)
  __shared__ float s_w[kGnHeads][kGnTile];            // logits
  __shared__ __align__(16) float s_wT[kGnTile][NH];   // weights, token-major
  __shared__ float s_kn[2][kGnTile], s_kr[2][kGnTile], s_vn[2][kGnTile], s_vr[2][kGnTile];
  extern __shared__ float2 s_pt[];   // pair tables [K / V][group][256]
  __shared__ float s_alpha[kGnHeads], s_m[kGnHeads], s_l[kGnHeads];
  float(*s_q)[kGnMaxD] = reinterpret_cast<float(*)[kGnMaxD]>(s_raw);
  float(*s_qs)[kGnMaxD] = reinterpret_cast<float(*)[kGnMaxD]>(s_raw + kGnHeads * kGnMaxD * 4);
  static_assert(2 * kGnHeads * kGnMaxD * 4 <= kGnStageBytes, "setup scratch");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = p.d;
  const int split = blockIdx.x;
  const int u = blockIdx.y;  // (b, kv head, head group)
  const int hgi = u % p.hg, bk = u / p.hg;
  const int b = bk / p.Hkv, kvh = bk % p.Hkv;
  const int h0 = kvh * p.g + kGnHeads * hgi;
  const int nh = min(NH, p.g - kGnHeads * hgi);
  const int64_t L = gn_len(p, b);
  const int64_t t0 = (int64_t)split * p.per_split;
  const int64_t t1 = min(L, t0 + p.per_split);

  for (int e = tid; e < 4 * 256; e += kGnThreads) {  // pair tables: entry e = (c[e & m], c[e >> bm])
    const int side = e >> 9, gr = (e >> 8) & 1, pe = e & 255;
    const GnGroup &G = side ? p.v[gr] : p.k[gr];
    float2 v = make_float2(0.f, 0.f);
    if (gr < (side ? p.nv : p.nk) && G.bm > 0 && pe < (1 << (2 * G.bm)))
      v = make_float2(__ldg(G.cent + (pe & ((1 << G.bm) - 1))), __ldg(G.cent + (pe >> G.bm)));
    s_pt[e] = v;
  }
  // ---- q'_g = Pi_g q[channels_g] for the block's heads (and S_g q'_g)
  for (int gr = 0; gr < p.nk; ++gr) {
    const GnGroup &G = p.k[gr];
    for (int e = tid; e < nh * G.d; e += kGnThreads) {
      const int hh = e / G.d, c = e % G.d;
      const int ch = G.chan ? min(max(__ldg(G.chan + c), 0), d - 1) : c;
      const float x = gn_q(p, ((int64_t)b * p.Hq + h0 + hh) * d + ch);
      if (G.rot) {
        s_qs[hh][G.off + c] = x;
      } else {
        s_q[hh][G.off + c] = G.signs[c] < 0 ? -x : x;
      }
    }
  }
  __syncthreads();
  for (int gr = 0; gr < p.nk; ++gr) {
    const GnGroup &G = p.k[gr];
    if (G.rot) {
      gn_rows_times<NH>(G.rot, G.d, &s_qs[0][G.off], &s_q[0][G.off], nh);
    } else {  // Hadamard: a single group at offset 0
      gn_fwht(&s_q[0][0], nh, G.d, kGnMaxD);
      const float inv = rsqrtf((float)G.d);
      for (int e = tid; e < nh * G.d; e += kGnThreads) s_q[e / G.d][e % G.d] *= inv;
    }
  }
  __syncthreads();
  for (int gr = 0; gr < p.nk; ++gr) {
    const GnGroup &G = p.k[gr];
    if (G.prod) gn_rows_times<NH>(G.S, G.d, &s_q[0][G.off], &s_qs[0][G.off], nh);
  }
  if (tid < kGnHeads) {
    s_m[tid] = -INFINITY;
    s_l[tid] = 0.f;
  }
  __syncthreads();

  if (tid < kGnHeads) s_alpha[tid] = 1.f;
  // coordinate-major copies of q' and S q' (zero for absent heads)
  for (int e = tid; e < kGnMaxD * NH; e += kGnThreads) {
    const int i = e / NH, hh = e - i * NH;
    const bool live = hh < nh && i < d;
    s_qT[i][hh] = live ? s_q[hh][i] : 0.f;
    s_qsT[i][hh] = live ? s_qs[hh][i] : 0.f;
  }
  __syncthreads();

  // staged-record offsets in s_raw: K codes | K signs | V codes | V signs,
  // each side's groups one after the other (a tile of a group is a
  // multiple of 64 bytes, so every part stays 16-byte aligned)
  int kc_off[2] = {0, 0}, kj_off[2] = {0, 0}, vc_off[2] = {0, 0}, vj_off[2] = {0, 0};
  {
    int oc = 0, oj = kGnCodeBytes;
    for (int gr = 0; gr < p.nk; ++gr) {
      kc_off[gr] = oc;
      kj_off[gr] = oj;
      oc += kGnTile * gn_pitch(p.k[gr].d * p.k[gr].bm / 8);
      oj += kGnTile * gn_pitch(p.k[gr].d / 8);
    }
    oc = kGnCodeBytes + kGnSignBytes;
    oj = 2 * kGnCodeBytes + kGnSignBytes;
    for (int gr = 0; gr < p.nv; ++gr) {
      vc_off[gr] = oc;
      vj_off[gr] = oj;
      oc += kGnTile * gn_pitch(p.v[gr].d * p.v[gr].bm / 8);
      oj += kGnTile * gn_pitch(p.v[gr].d / 8);
    }
  }

  // value threads: coordinates (2 vp, 2 vp + 1) of the tokens tt = half
  // (mod nhalf); a group's coordinates start at a multiple of 8, so a pair
  // never straddles two groups
  const int np = d / 2;
  const int nhalf = kGnThreads / np;
  const int half = tid / np, vp = tid - half * np;
  const bool vact = half < nhalf;
  const int gv = (p.nv == 2 && 2 * vp >= p.v[1].off) ? 1 : 0;
  const int li = 2 * vp - p.v[gv].off;
  float acc[NH][2], sacc[NH][2];
#pragma unroll
  for (int hh = 0; hh < NH; ++hh) acc[hh][0] = acc[hh][1] = sacc[hh][0] = sacc[hh][1] = 0.f;

  for (int64_t base = t0; base < t1; base += kGnTile) {
    const int nt = (int)min((int64_t)kGnTile, t1 - base);
    // ---- stage the tile's records and norms
    for (int gr = 0; gr < p.nk; ++gr) {
      const GnGroup &G = p.k[gr];
      const int64_t rec0 = (int64_t)b * G.sb + (int64_t)kvh * G.sh + base * G.sn;
      if (G.bm > 0) gn_stage(G.codes, rec0, G.sn, G.d * G.bm / 8, nt, s_raw + kc_off[gr]);
      if (G.prod) gn_stage(G.qjl, rec0, G.sn, G.d / 8, nt, s_raw + kj_off[gr]);
    }
    for (int gr = 0; gr < p.nv; ++gr) {
      const GnGroup &G = p.v[gr];
      const int64_t rec0 = (int64_t)b * G.sb + (int64_t)kvh * G.sh + base * G.sn;
      if (G.bm > 0) gn_stage(G.codes, rec0, G.sn, G.d * G.bm / 8, nt, s_raw + vc_off[gr]);
      if (G.prod) gn_stage(G.qjl, rec0, G.sn, G.d / 8, nt, s_raw + vj_off[gr]);
    }
    for (int e = tid; e < 4 * kGnTile; e += kGnThreads) {  // (side, group, token)
      const int side = e / (2 * kGnTile), gr = (e / kGnTile) & 1, tt = e % kGnTile;
      const GnGroup &G = side ? p.v[gr] : p.k[gr];
      if (gr < (side ? p.nv : p.nk) && tt < nt) {
        const int64_t r = (int64_t)b * G.sb + (int64_t)kvh * G.sh + (base + tt) * G.sn;
        const float n = __ldg(G.norms + r);
        const float kr = G.prod ? __ldg(G.rnorms + r) * (kGnSqrtHalfPi / (float)G.d) : 0.f;
        if (side) {
          s_vn[gr][tt] = n;
          s_vr[gr][tt] = kr;
        } else {
          s_kn[gr][tt] = n;
          s_kr[gr][tt] = kr;
        }
      }
    }
    __syncthreads();

    // ---- scores: 4 threads a token, a quarter of every group's coordinates each
    {
      const int tt = tid >> 2, qq = tid & 3;
      const bool ok = tt < nt;
      const int64_t j = base + (ok ? tt : 0);
      float tot[NH];
#pragma unroll
      for (int hh = 0; hh < NH; ++hh) tot[hh] = 0.f;
      if (ok) {
        for (int gr = 0; gr < p.nk; ++gr) {
          const GnGroup &G = p.k[gr];
          const uint32_t *kc = reinterpret_cast<const uint32_t *>(
              s_raw + kc_off[gr] + tt * gn_pitch(G.d * G.bm / 8));
          const uint32_t *kj = reinterpret_cast<const uint32_t *>(s_raw + kj_off[gr] + tt * gn_pitch(G.d / 8));
          const float2 *pt = s_pt + gr * 256;
          float part[NH], qpart[NH];
#pragma unroll
          for (int hh = 0; hh < NH; ++hh) part[hh] = qpart[hh] = 0.f;
          // a quarter of the group's coordinates, two at a time (G.d / 4 is even)
          const int i0 = qq * (G.d / 4), i1 = i0 + G.d / 4;
          for (int i = i0; i < i1; i += 2) {
            float q0[NH], q1[NH];
            gn_ld_heads<NH>(&s_qT[G.off + i][0], q0);
            gn_ld_heads<NH>(&s_qT[G.off + i + 1][0], q1);
            const float2 c = G.bm > 0 ? pt[gn_pair_s(kc, i, G.bm)] : make_float2(0.f, 0.f);
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) part[hh] = fmaf(c.y, q1[hh], fmaf(c.x, q0[hh], part[hh]));
            if (G.prod) {
              float s0[NH], s1[NH];
              gn_ld_heads<NH>(&s_qsT[G.off + i][0], s0);
              gn_ld_heads<NH>(&s_qsT[G.off + i + 1][0], s1);
              const uint32_t bb = gn_bits2_s(kj, i);
              const float g0 = (bb & 1u) ? 1.f : -1.f, g1 = (bb & 2u) ? 1.f : -1.f;
#pragma unroll
              for (int hh = 0; hh < NH; ++hh) qpart[hh] = fmaf(g1, s1[hh], fmaf(g0, s0[hh], qpart[hh]));
            }
          }
          const float n = s_kn[gr][tt], kap = s_kr[gr][tt];
#pragma unroll
          for (int hh = 0; hh < NH; ++hh) tot[hh] = fmaf(n, fmaf(kap, qpart[hh], part[hh]), tot[hh]);
        }
      }
#pragma unroll
      for (int hh = 0; hh < NH; ++hh) {
        tot[hh] += __shfl_xor_sync(dev::kFull, tot[hh], 1);
        tot[hh] += __shfl_xor_sync(dev::kFull, tot[hh], 2);
      }
      if (qq == 0) {
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
          if (hh < nh) {
            s_w[hh][tt] = ok ? tot[hh] * p.scale_log2 : -INFINITY;
            if (ok && p.scores) p.scores[((int64_t)b * p.Hq + h0 + hh) * p.seq_len + j] = tot[hh];
          }
        }
      }
    }
    __syncthreads();
    // ---- online softmax: warp hh updates head hh and writes its weights
    // token-major
    if (warp < nh) {
      const float a0 = s_w[warp][lane], a1 = s_w[warp][lane + 32];
      float mx = fmaxf(a0, a1);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(dev::kFull, mx, o));
      const float mo = s_m[warp];
      const float mn = fmaxf(mo, mx);
      const float ms = mn == -INFINITY ? 0.f : mn;
      const float w0 = gn_ex2(a0 - ms), w1 = gn_ex2(a1 - ms);
      s_wT[lane][warp] = w0;
      s_wT[lane + 32][warp] = w1;
      float sum = w0 + w1;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(dev::kFull, sum, o);
      if (lane == 0) {
        const float al = gn_ex2(mo - ms);
        s_alpha[warp] = al;
        s_l[warp] = fmaf(s_l[warp], al, sum);
        s_m[warp] = mn;
      }
    } else if (warp < NH) {  // absent heads: zero weights
      s_wT[lane][warp] = 0.f;
      s_wT[lane + 32][warp] = 0.f;
    }
    __syncthreads();
    // ---- values: this thread's coordinate pair of every head, its token class
    if (vact) {
      const GnGroup &G = p.v[gv];
#pragma unroll
      for (int hh = 0; hh < NH; ++hh) {
        const float al = s_alpha[hh];
        acc[hh][0] *= al;
        acc[hh][1] *= al;
        sacc[hh][0] *= al;
        sacc[hh][1] *= al;
      }
      const int cw = gn_pitch(G.d * G.bm / 8) >> 2, jw = gn_pitch(G.d / 8) >> 2;  // words a token
      const uint32_t *vc = reinterpret_cast<const uint32_t *>(s_raw + vc_off[gv]);
      const uint32_t *vj = reinterpret_cast<const uint32_t *>(s_raw + vj_off[gv]);
      const float2 *pt = s_pt + (2 + gv) * 256;
      for (int tt = half; tt < nt; tt += nhalf) {
        float w[NH];
        gn_ld_heads<NH>(&s_wT[tt][0], w);
        const float n = s_vn[gv][tt];
        float2 c = G.bm > 0 ? pt[gn_pair_s(vc + tt * cw, li, G.bm)] : make_float2(0.f, 0.f);
        c.x *= n;
        c.y *= n;
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
          acc[hh][0] = fmaf(w[hh], c.x, acc[hh][0]);
          acc[hh][1] = fmaf(w[hh], c.y, acc[hh][1]);
        }
        if (G.prod) {
          const float r = n * s_vr[gv][tt];
          const uint32_t bb = gn_bits2_s(vj + tt * jw, li);
          const float r0 = (bb & 1u) ? r : -r, r1 = (bb & 2u) ? r : -r;
#pragma unroll
          for (int hh = 0; hh < NH; ++hh) {
            sacc[hh][0] = fmaf(w[hh], r0, sacc[hh][0]);
            sacc[hh][1] = fmaf(w[hh], r1, sacc[hh][1]);
          }
        }
      }
    }
    __syncthreads();  // the staged records are read before the next tile's copy
  }

  // ---- the slice's partial state: the token classes' sums added per
  // (head, coordinate), the value sums first, then (prod value groups) the
  // sign sums, through the staging memory
  float *s_red = reinterpret_cast<float *>(s_raw);  // [threads][NH][2]
  static_assert(kGnThreads * kGnHeads * 2 * 4 <= kGnStageBytes, "reduction scratch");
  const int stride = 4 + 2 * d;
  const bool any_prod = p.v[0].prod || (p.nv == 2 && p.v[1].prod);
  for (int round = 0; round < (any_prod ? 2 : 1); ++round) {
    if (vact) {
#pragma unroll
      for (int hh = 0; hh < NH; ++hh) {
        s_red[(tid * NH + hh) * 2] = round ? sacc[hh][0] : acc[hh][0];
        s_red[(tid * NH + hh) * 2 + 1] = round ? sacc[hh][1] : acc[hh][1];
      }
    }
    __syncthreads();
    for (int e = tid; e < nh * d; e += kGnThreads) {
      const int hh = e / d, i = e - hh * d;
      float a = 0.f;
      for (int hf = 0; hf < nhalf; ++hf) a += s_red[((hf * np + (i >> 1)) * NH + hh) * 2 + (i & 1)];
      float *slot = p.ws + ((int64_t)split * p.B * p.Hq + (int64_t)b * p.Hq + h0 + hh) * stride;
      slot[4 + round * d + i] = a;
      if (round == 0 && i == 0) {
        slot[0] = s_m[hh];
        slot[1] = s_l[hh];
      }
      if (!any_prod) slot[4 + d + i] = 0.f;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kGnThreads) general_merge_kernel(GnParams p) {
  __shared__ float s_o[kGnMaxD], s_s[kGnMaxD];
  __shared__ float s_hdr[2];
  __shared__ float s_f[kGnMaxSplits];  // each slot's factor 2^(m_s - M), 0 for an empty slot
  __shared__ float s_part[2 * kGnThreads];  // the parts' partial sums, [thread]
  const int head = blockIdx.x;  // b * Hq + hq
  const int b = head / p.Hq;
  const int tid = threadIdx.x;
  const int d = p.d;
  const int stride = 4 + 2 * d;
  float *out = p.out + (int64_t)head * d;
  if (gn_len(p, b) == 0) {
    for (int i = tid; i < d; i += kGnThreads) out[i] = 0.f;
    return;
  }
  if (tid < 32) {  // the first warp: the slots' maximum, factors and l, lanes over slots
    const int lane = tid;
    float m[kGnMaxSplits / 32], lv[kGnMaxSplits / 32];
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < kGnMaxSplits / 32; ++k) {
      const int sl = lane + 32 * k;
      const float *slot = p.ws + ((int64_t)sl * p.B * p.Hq + head) * stride;
      m[k] = sl < p.splits ? slot[0] : -INFINITY;
      lv[k] = sl < p.splits ? slot[1] : 0.f;
      M = fmaxf(M, m[k]);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(dev::kFull, M, o));
    float l = 0.f;
#pragma unroll
    for (int k = 0; k < kGnMaxSplits / 32; ++k) {
      const float f = m[k] == -INFINITY ? 0.f : gn_ex2(m[k] - M);
      s_f[lane + 32 * k] = f;
      l = fmaf(lv[k], f, l);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) l += __shfl_xor_sync(dev::kFull, l, o);
    if (lane == 0) {
      s_hdr[0] = M;
      s_hdr[1] = l;
    }
  }
  __syncthreads();
  const float l = s_hdr[1];
  // the coordinates' loops split over P parts (P threads a coordinate when d
  // leaves threads idle), each part a stride of the batches of 8 loads, the
  // parts' sums added through shared memory (thread part * d + i)
  const int P = d >= kGnThreads ? 1 : min(8, kGnThreads / d);
  const int part = tid / d, pi = tid - part * d;
  const bool pact = part < P;
  const int pgv = (p.nv == 2 && pi >= p.v[1].off) ? 1 : 0;
  const GnGroup &PG = p.v[pgv];
  const int pc = pi - PG.off;  // the coordinate inside its group
  float *s_pa = s_part, *s_pb = s_part + kGnThreads;
  if (pact) {
    float o = 0.f, so = 0.f;
    const float *slot = p.ws + (int64_t)head * stride + 4 + pi;
    const int64_t sstride = (int64_t)p.B * p.Hq * stride;
    // batches of 8 slots, every load of a batch issued before its sums
    // (empty slots have f = 0 and finite sums)
    for (int s0 = 8 * part; s0 < p.splits; s0 += 8 * P) {
      float x[8], y[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int sl = min(s0 + k, p.splits - 1);
        x[k] = __ldcg(slot + sl * sstride);
        y[k] = __ldcg(slot + sl * sstride + d);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float f = s0 + k < p.splits ? s_f[s0 + k] : 0.f;
        o = fmaf(x[k], f, o);
        so = fmaf(y[k], f, so);
      }
    }
    s_pa[tid] = o;
    s_pb[tid] = so;
  }
  __syncthreads();
  for (int i = tid; i < d; i += kGnThreads) {
    float o = 0.f, so = 0.f;
    for (int q = 0; q < P; ++q) {
      o += s_pa[q * d + i];
      so += s_pb[q * d + i];
    }
    s_o[i] = o;
    s_s[i] = so;
  }
  __syncthreads();
  // prod value groups: o'_g += S_g^T (weighted signs); sqrt(pi/2)/d_g is in the weights
  if (p.v[0].prod || (p.nv == 2 && p.v[1].prod)) {
    if (pact) {
      float a = 0.f;
      if (PG.prod) {
        for (int k0 = 8 * part; k0 < PG.d; k0 += 8 * P) {  // PG.d is a multiple of 8: batches of 8 loads
          float x[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) x[k] = __ldg(PG.S + (int64_t)(k0 + k) * PG.d + pc);
#pragma unroll
          for (int k = 0; k < 8; ++k) a = fmaf(x[k], s_s[PG.off + k0 + k], a);
        }
      }
      s_pa[tid] = a;
    }
    __syncthreads();
    for (int i = tid; i < d; i += kGnThreads) {
      float a = 0.f;
      for (int q = 0; q < P; ++q) a += s_pa[q * d + i];
      s_o[i] += a;
    }
    __syncthreads();
  }
  const float inv_l = l > 0.f ? 1.0f / l : 0.f;
  if (p.v[0].rot) {  // o[channels_g] = Pi_g^T o'_g
    if (pact) {
      float a = 0.f;
      for (int r0 = 8 * part; r0 < PG.d; r0 += 8 * P) {  // batches of 8 loads
        float x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = __ldg(PG.rot + (int64_t)(r0 + k) * PG.d + pc);
#pragma unroll
        for (int k = 0; k < 8; ++k) a = fmaf(x[k], s_o[PG.off + r0 + k], a);
      }
      s_pa[tid] = a;
    }
    __syncthreads();
    for (int i = tid; i < d; i += kGnThreads) {
      const int gv = (p.nv == 2 && i >= p.v[1].off) ? 1 : 0;
      const GnGroup &G = p.v[gv];
      const int c = i - G.off;
      float a = 0.f;
      for (int q = 0; q < P; ++q) a += s_pa[q * d + i];
      const int ch = G.chan ? min(max(__ldg(G.chan + c), 0), d - 1) : c;
      out[ch] = a * inv_l;
    }
  } else {  // a single Hadamard group: o = sigma * H o' / sqrt(d)
    gn_fwht(s_o, 1, d, kGnMaxD);
    const float f = rsqrtf((float)d) * inv_l;
    for (int i = tid; i < d; i += kGnThreads) out[i] = (p.v[0].signs[i] < 0 ? -s_o[i] : s_o[i]) * f;
  }
}

GnGroup group_of(const QuantParams &q, const CacheView &v, int off) {
  GnGroup g{};
  g.d = q.d;
  g.off = off;
  g.bm = q.bm;
  g.prod = q.prod;
  g.cent = q.centroids;
  g.rot = q.rot;
  g.S = q.S;
  g.signs = q.signs;
  g.chan = q.channels;
  g.codes = v.codes;
  g.qjl = v.qjl;
  g.norms = v.norms;
  g.rnorms = v.rnorms;
  g.sb = v.sb;
  g.sh = v.sh;
  g.sn = v.sn;
  return g;
}

// One partial-kernel launch with the pair tables' dynamic shared memory;
// the kernel's limit is raised once per device (the setting belongs to the
// kernel, so later launches skip the driver call).
template <int NH>
cudaError_t launch_partial(const GnParams &p, dim3 grid, cudaStream_t s) {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t)1 << dev : 0;
  if (!bit || !(done.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(general_partial_kernel<NH>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGnPairBytes);
    if (e != cudaSuccess) return e;
    if (bit) done.fetch_or(bit, std::memory_order_release);
  }
  general_partial_kernel<NH><<<grid, kGnThreads, kGnPairBytes, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_general(GnParams &p, cudaStream_t s) {
  p.g = p.Hq / p.Hkv;
  p.hg = (p.g + kGnHeads - 1) / kGnHeads;
  if (p.d > kGnMaxD || p.d % 8) return cudaErrorInvalidValue;
  p.splits = general_decode_splits(p.B, p.Hq, p.Hkv, p.seq_len);
  p.per_split = (p.seq_len + p.splits - 1) / p.splits;
  if (p.seq_len > 0) {
    const dim3 grid((unsigned)p.splits, (unsigned)(p.B * p.Hkv * p.hg));
    const cudaError_t e = p.g <= 1   ? launch_partial<1>(p, grid, s)
                          : p.g <= 2 ? launch_partial<2>(p, grid, s)
                          : p.g <= 4 ? launch_partial<4>(p, grid, s)
                                     : launch_partial<8>(p, grid, s);
    if (e != cudaSuccess) return e;
  } else {
    p.splits = 0;
  }
  general_merge_kernel<<<(unsigned)(p.B * p.Hq), kGnThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

int general_decode_splits(int B, int Hq, int Hkv, int64_t seq_len) {
  const int64_t blocks = (int64_t)B * Hkv * ((Hq / Hkv + kGnHeads - 1) / kGnHeads);
  int64_t s = (4 * (int64_t)decode_ctas() + blocks - 1) / blocks;  // about 4 blocks an SM
  const int64_t by_len = (seq_len + 4 * kGnTile - 1) / (4 * kGnTile);  // at least 4 tiles a split
  if (s > by_len) s = by_len;
  if (s > kGnMaxSplits) s = kGnMaxSplits;
  return (int)(s < 1 ? 1 : s);
}

size_t general_decode_workspace_floats(int B, int Hq, int Hkv, int64_t seq_len, int d) {
  return (size_t)general_decode_splits(B, Hq, Hkv, seq_len) * B * Hq * (4 + 2 * (size_t)d);
}

cudaError_t launch_decode_general(const DecodeArgs &a, cudaStream_t s) {
  GnParams p{};
  p.k[0] = group_of(a.kq, a.k, 0);
  p.v[0] = group_of(a.vq, a.v, 0);
  p.nk = p.nv = 1;
  p.q = a.q;
  p.q_dtype = a.q_dtype;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.d = a.kq.d;
  p.seq_len = a.seq_len;
  p.seq_lens = a.seq_lens;
  p.scale_log2 = a.scale * kGnLog2e;
  p.out = a.out;
  p.scores = a.scores;
  p.ws = a.ws;
  return launch_general(p, s);
}

cudaError_t launch_decode_split(const SplitDecodeArgs &a, cudaStream_t s) {
  GnParams p{};
  for (int g = 0; g < 2; ++g) {
    p.k[g] = group_of(a.kq[g], a.k[g], g == 0 ? 0 : a.kq[0].d);
    p.v[g] = group_of(a.vq[g], a.v[g], g == 0 ? 0 : a.vq[0].d);
  }
  p.nk = p.nv = 2;
  p.q = a.q;
  p.q_dtype = a.q_dtype;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.d = a.d;
  p.seq_len = a.seq_len;
  p.seq_lens = a.seq_lens;
  p.scale_log2 = a.scale * kGnLog2e;
  p.out = a.out;
  p.scores = nullptr;
  p.ws = a.ws;
  return launch_general(p, s);
}

}  // namespace tq
