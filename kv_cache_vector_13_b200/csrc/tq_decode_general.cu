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
//     tokens: scores (4 threads a token), an online softmax per head, then
//     the values 8 tokens at a time: each (token, coordinate) decoded once
//     into shared memory, and a thread per (head, coordinate) accumulating
//     the weighted centroids (and, for prod values, the weighted signs); the
//     slice's (m, l, o', signs) go to a workspace slot;
//   general_merge_kernel, a block per (batch, query head): merges the slots,
//   adds S_g^T of the sign sums, applies each group's inverse rotation and
//   1/l, and scatters the groups into their channels.

#include "../../include/tq.h"
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kGnThreads = 256;
constexpr int kGnMaxD = 256;
constexpr int kGnHeads = 8;   // query heads a block
constexpr int kGnTile = 64;   // tokens a tile
constexpr int kGnSub = 8;     // tokens a value-decode step
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

// Index i of a record's LSB-first bm-bit stream (bm <= 4: at most two bytes).
__device__ __forceinline__ int gn_field(const uint8_t *rec, int i, int bm, int nbytes) {
  const int q = i * bm;
  const int by = q >> 3, sh = q & 7;
  uint32_t w = __ldg(rec + by);
  if (sh + bm > 8 && by + 1 < nbytes) w |= (uint32_t)__ldg(rec + by + 1) << 8;
  return (int)((w >> sh) & ((1u << bm) - 1u));
}

__device__ __forceinline__ bool gn_bit(const uint8_t *rec, int i) { return (__ldg(rec + (i >> 3)) >> (i & 7)) & 1; }

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

// NH: the most query heads a block handles (1, 2, 4 or 8): the per-token
// head loops are unrolled to it.
template <int NH>
__global__ void __launch_bounds__(kGnThreads) general_partial_kernel(GnParams p) {
  __shared__ float s_q[kGnHeads][kGnMaxD];   // q'_g at the group's offset
  __shared__ float s_qs[kGnHeads][kGnMaxD];  // S_g q'_g (prod groups); staging of q[channels] first
  __shared__ float s_w[kGnHeads][kGnTile];   // logits, then weights
  __shared__ float s_vn[2][kGnTile], s_vr[2][kGnTile];
  __shared__ float s_alpha[kGnHeads], s_m[kGnHeads], s_l[kGnHeads];
  __shared__ float s_vx[2][kGnSub][kGnMaxD];  // decoded values (and prod sign terms)
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
      for (int e = tid; e < nh * G.d; e += kGnThreads) {
        const int hh = e / G.d, r = e % G.d;
        const float *row = G.rot + (int64_t)r * G.d;
        float acc = 0.f;
        for (int c = 0; c < G.d; ++c) acc = fmaf(__ldg(row + c), s_qs[hh][G.off + c], acc);
        s_q[hh][G.off + r] = acc;
      }
    } else {  // Hadamard: a single group at offset 0
      gn_fwht(&s_q[0][0], nh, G.d, kGnMaxD);
      const float inv = rsqrtf((float)G.d);
      for (int e = tid; e < nh * G.d; e += kGnThreads) s_q[e / G.d][e % G.d] *= inv;
    }
  }
  __syncthreads();
  for (int gr = 0; gr < p.nk; ++gr) {
    const GnGroup &G = p.k[gr];
    if (!G.prod) continue;
    for (int e = tid; e < nh * G.d; e += kGnThreads) {
      const int hh = e / G.d, r = e % G.d;
      const float *row = G.S + (int64_t)r * G.d;
      float acc = 0.f;
      for (int c = 0; c < G.d; ++c) acc = fmaf(__ldg(row + c), s_q[hh][G.off + c], acc);
      s_qs[hh][G.off + r] = acc;
    }
  }
  if (tid < kGnHeads) {
    s_m[tid] = -INFINITY;
    s_l[tid] = 0.f;
  }
  __syncthreads();

  // this thread's (head, coordinate) pairs: e = tid + kGnThreads * c
  constexpr int kCoords = NH * kGnMaxD / kGnThreads > 0 ? NH * kGnMaxD / kGnThreads : 1;
  float acc[kCoords], sacc[kCoords];
  int c_h[kCoords], c_i[kCoords];
  bool c_prod[kCoords];
#pragma unroll
  for (int c = 0; c < kCoords; ++c) {
    acc[c] = sacc[c] = 0.f;
    const int e = tid + kGnThreads * c;
    c_h[c] = e < nh * d ? e / d : -1;
    c_i[c] = e % d;
    c_prod[c] = p.v[(p.nv == 2 && c_i[c] >= p.v[1].off) ? 1 : 0].prod;
  }
  // the value decode's (token, coordinate) share: coordinate dec_i of
  // tokens dec_t, dec_t + dec_step, ...
  const int dec_step = kGnThreads / d;
  const int dec_i = tid < dec_step * d ? tid % d : -1;
  const int dec_t = tid / d;

  for (int64_t base = t0; base < t1; base += kGnTile) {
    const int nt = (int)min((int64_t)kGnTile, t1 - base);
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
          const int64_t kr = (int64_t)b * G.sb + (int64_t)kvh * G.sh + j * G.sn;
          const int kcb = G.d * G.bm / 8;
          const uint8_t *kc = G.bm > 0 ? G.codes + kr * kcb : nullptr;
          const uint8_t *kj = G.prod ? G.qjl + kr * (G.d / 8) : nullptr;
          float part[NH], qpart[NH];
#pragma unroll
          for (int hh = 0; hh < NH; ++hh) part[hh] = qpart[hh] = 0.f;
          const int i0 = qq * (G.d / 4), i1 = i0 + G.d / 4;
          for (int i = i0; i < i1; ++i) {
            const float c = G.bm > 0 ? __ldg(G.cent + gn_field(kc, i, G.bm, kcb)) : 0.f;
            const float sg = G.prod ? (gn_bit(kj, i) ? 1.f : -1.f) : 0.f;
            if (G.prod) {
#pragma unroll
              for (int hh = 0; hh < NH; ++hh) {
                part[hh] = fmaf(c, s_q[hh][G.off + i], part[hh]);
                qpart[hh] = fmaf(sg, s_qs[hh][G.off + i], qpart[hh]);
              }
            } else {
#pragma unroll
              for (int hh = 0; hh < NH; ++hh) part[hh] = fmaf(c, s_q[hh][G.off + i], part[hh]);
            }
          }
          const float n = __ldg(G.norms + kr);
          const float kap = G.prod ? __ldg(G.rnorms + kr) * (kGnSqrtHalfPi / (float)G.d) : 0.f;
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
      if (qq < p.nv) {  // thread qq of the token loads value group qq's norms
        const GnGroup &G = p.v[qq];
        const int64_t vr = (int64_t)b * G.sb + (int64_t)kvh * G.sh + j * G.sn;
        s_vn[qq][tt] = ok ? __ldg(G.norms + vr) : 0.f;
        s_vr[qq][tt] = (ok && G.prod) ? __ldg(G.rnorms + vr) * (kGnSqrtHalfPi / (float)G.d) : 0.f;
      }
    }
    __syncthreads();
    // ---- online softmax: warp hh updates head hh
    if (warp < nh) {
      const float a0 = s_w[warp][lane], a1 = s_w[warp][lane + 32];
      float mx = fmaxf(a0, a1);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(dev::kFull, mx, o));
      const float mo = s_m[warp];
      const float mn = fmaxf(mo, mx);
      const float ms = mn == -INFINITY ? 0.f : mn;
      const float w0 = gn_ex2(a0 - ms), w1 = gn_ex2(a1 - ms);
      s_w[warp][lane] = w0;
      s_w[warp][lane + 32] = w1;
      float sum = w0 + w1;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(dev::kFull, sum, o);
      if (lane == 0) {
        const float al = gn_ex2(mo - ms);
        s_alpha[warp] = al;
        s_l[warp] = fmaf(s_l[warp], al, sum);
        s_m[warp] = mn;
      }
    }
    __syncthreads();
    // ---- values, kGnSub tokens at a time: every (token, coordinate) is
    // decoded once into shared memory (n_V c[idx], and for prod groups
    // n_V ||r|| sqrt(pi/2)/d sign), then each (head, coordinate) thread
    // accumulates its weights times them
#pragma unroll
    for (int c = 0; c < kCoords; ++c) {
      if (c_h[c] >= 0) {
        acc[c] *= s_alpha[c_h[c]];
        sacc[c] *= s_alpha[c_h[c]];
      }
    }
    for (int t8 = 0; t8 < nt; t8 += kGnSub) {
      const int ns = min(kGnSub, nt - t8);
      if (dec_i >= 0) {
        const int gv = (p.nv == 2 && dec_i >= p.v[1].off) ? 1 : 0;
        const GnGroup &G = p.v[gv];
        const int li = dec_i - G.off;
        const int vcb = G.d * G.bm / 8;
        const int64_t vbase = (int64_t)b * G.sb + (int64_t)kvh * G.sh;
        for (int tt = dec_t; tt < ns; tt += dec_step) {
          const int64_t vr = vbase + (base + t8 + tt) * G.sn;
          const float n = s_vn[gv][t8 + tt];
          s_vx[0][tt][dec_i] = G.bm > 0 ? n * __ldg(G.cent + gn_field(G.codes + vr * vcb, li, G.bm, vcb)) : 0.f;
          if (G.prod) {
            const float r = n * s_vr[gv][t8 + tt];
            s_vx[1][tt][dec_i] = gn_bit(G.qjl + vr * (G.d / 8), li) ? r : -r;
          }
        }
      }
      __syncthreads();
#pragma unroll
      for (int c = 0; c < kCoords; ++c) {
        if (c_h[c] >= 0) {
          const int hh = c_h[c], i = c_i[c];
          float a = acc[c], sa = sacc[c];
          for (int tt = 0; tt < ns; ++tt) {
            const float w = s_w[hh][t8 + tt];
            a = fmaf(w, s_vx[0][tt][i], a);
            if (c_prod[c]) sa = fmaf(w, s_vx[1][tt][i], sa);
          }
          acc[c] = a;
          sacc[c] = sa;
        }
      }
      __syncthreads();
    }
  }

  // ---- the slice's partial state
  const int stride = 4 + 2 * d;
#pragma unroll
  for (int c = 0; c < kCoords; ++c) {
    const int e = tid + kGnThreads * c;
    if (e < nh * d) {
      const int hh = e / d, i = e % d;
      float *slot = p.ws + ((int64_t)split * p.B * p.Hq + (int64_t)b * p.Hq + h0 + hh) * stride;
      slot[4 + i] = acc[c];
      slot[4 + d + i] = sacc[c];
      if (i == 0) {
        slot[0] = s_m[hh];
        slot[1] = s_l[hh];
      }
    }
  }
}

__global__ void __launch_bounds__(kGnThreads) general_merge_kernel(GnParams p) {
  __shared__ float s_o[kGnMaxD], s_s[kGnMaxD];
  __shared__ float s_hdr[2];
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
  if (tid == 0) {
    float M = -INFINITY;
    for (int s = 0; s < p.splits; ++s) M = fmaxf(M, p.ws[((int64_t)s * p.B * p.Hq + head) * stride]);
    float l = 0.f;
    for (int s = 0; s < p.splits; ++s) {
      const float *slot = p.ws + ((int64_t)s * p.B * p.Hq + head) * stride;
      if (slot[0] != -INFINITY) l += slot[1] * gn_ex2(slot[0] - M);
    }
    s_hdr[0] = M;
    s_hdr[1] = l;
  }
  __syncthreads();
  const float M = s_hdr[0], l = s_hdr[1];
  for (int i = tid; i < d; i += kGnThreads) {
    float o = 0.f, so = 0.f;
    for (int s = 0; s < p.splits; ++s) {
      const float *slot = p.ws + ((int64_t)s * p.B * p.Hq + head) * stride;
      if (slot[0] == -INFINITY) continue;
      const float f = gn_ex2(slot[0] - M);
      o = fmaf(slot[4 + i], f, o);
      so = fmaf(slot[4 + d + i], f, so);
    }
    s_o[i] = o;
    s_s[i] = so;
  }
  __syncthreads();
  // prod value groups: o'_g += S_g^T (weighted signs); sqrt(pi/2)/d_g is in the weights
  float add[kGnMaxD / kGnThreads];
  for (int i = tid, c = 0; i < d; i += kGnThreads, ++c) {
    const int gv = (p.nv == 2 && i >= p.v[1].off) ? 1 : 0;
    const GnGroup &G = p.v[gv];
    float a = 0.f;
    if (G.prod) {
      const int li = i - G.off;
      for (int k = 0; k < G.d; ++k) a = fmaf(__ldg(G.S + (int64_t)k * G.d + li), s_s[G.off + k], a);
    }
    add[c] = a;
  }
  __syncthreads();
  for (int i = tid, c = 0; i < d; i += kGnThreads, ++c) s_o[i] += add[c];
  __syncthreads();
  const float inv_l = l > 0.f ? 1.0f / l : 0.f;
  if (p.v[0].rot) {  // o[channels_g] = Pi_g^T o'_g
    for (int i = tid; i < d; i += kGnThreads) {
      const int gv = (p.nv == 2 && i >= p.v[1].off) ? 1 : 0;
      const GnGroup &G = p.v[gv];
      const int c = i - G.off;
      float a = 0.f;
      for (int r = 0; r < G.d; ++r) a = fmaf(__ldg(G.rot + (int64_t)r * G.d + c), s_o[G.off + r], a);
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

cudaError_t launch_general(GnParams &p, cudaStream_t s) {
  p.g = p.Hq / p.Hkv;
  p.hg = (p.g + kGnHeads - 1) / kGnHeads;
  if (p.d > kGnMaxD || p.d % 8) return cudaErrorInvalidValue;
  p.splits = general_decode_splits(p.B, p.Hq, p.Hkv, p.seq_len);
  p.per_split = (p.seq_len + p.splits - 1) / p.splits;
  if (p.seq_len > 0) {
    const dim3 grid((unsigned)p.splits, (unsigned)(p.B * p.Hkv * p.hg));
    if (p.g <= 1) {
      general_partial_kernel<1><<<grid, kGnThreads, 0, s>>>(p);
    } else if (p.g <= 2) {
      general_partial_kernel<2><<<grid, kGnThreads, 0, s>>>(p);
    } else if (p.g <= 4) {
      general_partial_kernel<4><<<grid, kGnThreads, 0, s>>>(p);
    } else {
      general_partial_kernel<8><<<grid, kGnThreads, 0, s>>>(p);
    }
    const cudaError_t e = cudaGetLastError();
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
  int64_t s = (2 * (int64_t)decode_ctas() + blocks - 1) / blocks;
  const int64_t by_len = (seq_len + 4 * kGnTile - 1) / (4 * kGnTile);  // at least 4 tiles a split
  if (s > by_len) s = by_len;
  if (s > 64) s = 64;
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
