// Decode attention on CUDA cores (sm_100a) for the quantizers the
// tensor-core split kernel does not take: d = 64 or 256 with the Hadamard
// rotation, dense (Haar) rotations of any supported d other than 128, and
// TurboQuant_prod values.  Same definition as the main path ("I Spent 31
// Hours On The Math Behind Turboquant", section "KV Cache: The problem";
// "内存厂商的噩梦来了", section 4.2, the asymmetric score):
//   s_j = n_j (<q', c_K[idx_j]> + [prod] ||r_j|| sqrt(pi/2)/d <S_K q', sign_j>),
//   q' = Pi_K q, softmax over s_j * scale, and the values summed in their
//   rotated basis, o' = sum_j p_j n_j (c_V[idx_j] + [prod] ||r_j|| sqrt(pi/2)/d
//   S_V^T sign_j), rotated back once, o = Pi_V^T o'.
//
// Flash-decoding split over the sequence:
//   general_partial_kernel, grid (splits, B * Hkv * head groups): up to 8
//     query heads of one kv head over one token slice, in tiles of 64
//     tokens: scores (4 threads a token), an online softmax per head, then a
//     thread per (head, coordinate) accumulates the weighted centroids (and,
//     for prod values, the weighted signs) of the tile; the slice's
//     (m, l, o', signs) go to a workspace slot;
//   general_merge_kernel, a block per (batch, query head): merges the slots,
//   adds S_V^T of the sign sums, applies the inverse rotation and 1/l.

#include "../../include/tq.h"
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kGnThreads = 256;
constexpr int kGnMaxD = 256;
constexpr int kGnHeads = 8;   // query heads a block
constexpr int kGnTile = 64;   // tokens a tile
constexpr int kGnCoords = kGnHeads * kGnMaxD / kGnThreads;  // (head, coordinate) pairs a thread
constexpr float kGnLog2e = 1.4426950408889634f;
constexpr float kGnSqrtHalfPi = 1.2533141373155003f;

struct GnSide {
  int bm;
  bool prod;
  const float *cent, *rot, *S;
  const int8_t *signs;
  const uint8_t *codes, *qjl;
  const float *norms, *rnorms;
  int64_t sb, sh, sn;
};

struct GnParams {
  GnSide k, v;
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

__global__ void __launch_bounds__(kGnThreads) general_partial_kernel(GnParams p) {
  __shared__ float s_q[kGnHeads][kGnMaxD];   // q' (rotated query)
  __shared__ float s_qs[kGnHeads][kGnMaxD];  // S_K q' (prod keys); staging of q otherwise
  __shared__ float s_w[kGnHeads][kGnTile];   // logits, then weights
  __shared__ float s_vn[kGnTile], s_vr[kGnTile];
  __shared__ float s_alpha[kGnHeads], s_m[kGnHeads], s_l[kGnHeads];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = p.d;
  const int split = blockIdx.x;
  const int u = blockIdx.y;  // (b, kv head, head group)
  const int hgi = u % p.hg, bk = u / p.hg;
  const int b = bk / p.Hkv, kvh = bk % p.Hkv;
  const int h0 = kvh * p.g + kGnHeads * hgi;
  const int nh = min(kGnHeads, p.g - kGnHeads * hgi);
  const int64_t L = gn_len(p, b);
  const int64_t t0 = (int64_t)split * p.per_split;
  const int64_t t1 = min(L, t0 + p.per_split);

  // ---- q' = Pi_K q for the block's heads (and S_K q' for prod keys)
  for (int e = tid; e < nh * d; e += kGnThreads) {
    const int hh = e / d, i = e % d;
    const float x = gn_q(p, ((int64_t)b * p.Hq + h0 + hh) * d + i);
    if (p.k.rot) {
      s_qs[hh][i] = x;
    } else {
      s_q[hh][i] = p.k.signs[i] < 0 ? -x : x;
    }
  }
  __syncthreads();
  if (p.k.rot) {
    for (int e = tid; e < nh * d; e += kGnThreads) {
      const int hh = e / d, r = e % d;
      const float *row = p.k.rot + (int64_t)r * d;
      float acc = 0.f;
      for (int c = 0; c < d; ++c) acc = fmaf(__ldg(row + c), s_qs[hh][c], acc);
      s_q[hh][r] = acc;
    }
  } else {
    gn_fwht(&s_q[0][0], nh, d, kGnMaxD);
    const float inv = rsqrtf((float)d);
    for (int e = tid; e < nh * d; e += kGnThreads) s_q[e / d][e % d] *= inv;
  }
  __syncthreads();
  if (p.k.prod) {
    for (int e = tid; e < nh * d; e += kGnThreads) {
      const int hh = e / d, r = e % d;
      const float *row = p.k.S + (int64_t)r * d;
      float acc = 0.f;
      for (int c = 0; c < d; ++c) acc = fmaf(__ldg(row + c), s_q[hh][c], acc);
      s_qs[hh][r] = acc;
    }
  }
  if (tid < kGnHeads) {
    s_m[tid] = -INFINITY;
    s_l[tid] = 0.f;
  }
  __syncthreads();

  // this thread's (head, coordinate) pairs: e = tid + kGnThreads * c
  float acc[kGnCoords], sacc[kGnCoords];
#pragma unroll
  for (int c = 0; c < kGnCoords; ++c) acc[c] = sacc[c] = 0.f;
  const int kcb = d * p.k.bm / 8, vcb = d * p.v.bm / 8;
  const int64_t kbase = (int64_t)b * p.k.sb + (int64_t)kvh * p.k.sh;
  const int64_t vbase = (int64_t)b * p.v.sb + (int64_t)kvh * p.v.sh;
  const float kkap = kGnSqrtHalfPi / (float)d;

  for (int64_t base = t0; base < t1; base += kGnTile) {
    const int nt = (int)min((int64_t)kGnTile, t1 - base);
    // ---- scores: 4 threads a token, d/4 coordinates each
    {
      const int tt = tid >> 2, qq = tid & 3;
      const bool ok = tt < nt;
      const int64_t j = base + (ok ? tt : 0);
      const int64_t kr = kbase + j * p.k.sn;
      float part[kGnHeads], qpart[kGnHeads];
#pragma unroll
      for (int hh = 0; hh < kGnHeads; ++hh) part[hh] = qpart[hh] = 0.f;
      if (ok) {
        const uint8_t *kc = p.k.bm > 0 ? p.k.codes + kr * kcb : nullptr;
        const uint8_t *kj = p.k.prod ? p.k.qjl + kr * (d / 8) : nullptr;
        const int i0 = qq * (d / 4), i1 = i0 + d / 4;
        for (int i = i0; i < i1; ++i) {
          const float c = p.k.bm > 0 ? __ldg(p.k.cent + gn_field(kc, i, p.k.bm, kcb)) : 0.f;
          const float sg = p.k.prod ? (gn_bit(kj, i) ? 1.f : -1.f) : 0.f;
#pragma unroll
          for (int hh = 0; hh < kGnHeads; ++hh) {
            if (hh < nh) {
              part[hh] = fmaf(c, s_q[hh][i], part[hh]);
              if (p.k.prod) qpart[hh] = fmaf(sg, s_qs[hh][i], qpart[hh]);
            }
          }
        }
      }
#pragma unroll
      for (int hh = 0; hh < kGnHeads; ++hh) {
        part[hh] += __shfl_xor_sync(dev::kFull, part[hh], 1);
        part[hh] += __shfl_xor_sync(dev::kFull, part[hh], 2);
        qpart[hh] += __shfl_xor_sync(dev::kFull, qpart[hh], 1);
        qpart[hh] += __shfl_xor_sync(dev::kFull, qpart[hh], 2);
      }
      if (qq == 0 && tt < kGnTile) {
        const float n = ok ? __ldg(p.k.norms + kr) : 0.f;
        const float kap = (ok && p.k.prod) ? __ldg(p.k.rnorms + kr) * kkap : 0.f;
#pragma unroll
        for (int hh = 0; hh < kGnHeads; ++hh) {
          if (hh < nh) {
            const float s = n * (part[hh] + kap * qpart[hh]);
            s_w[hh][tt] = ok ? s * p.scale_log2 : -INFINITY;
            if (ok && p.scores) p.scores[((int64_t)b * p.Hq + h0 + hh) * p.seq_len + j] = s;
          }
        }
        const int64_t vr = vbase + j * p.v.sn;
        s_vn[tt] = ok ? __ldg(p.v.norms + vr) : 0.f;
        s_vr[tt] = (ok && p.v.prod) ? __ldg(p.v.rnorms + vr) * kkap : 0.f;
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
    // ---- values: thread (head, coordinate) pairs over the tile
#pragma unroll
    for (int c = 0; c < kGnCoords; ++c) {
      const int e = tid + kGnThreads * c;
      if (e < nh * d) {
        const int hh = e / d, i = e % d;
        float a = acc[c] * s_alpha[hh], sa = sacc[c] * s_alpha[hh];
        for (int tt = 0; tt < nt; ++tt) {
          const float w = s_w[hh][tt] * s_vn[tt];
          const int64_t vr = vbase + (base + tt) * p.v.sn;
          if (p.v.bm > 0) a = fmaf(w, __ldg(p.v.cent + gn_field(p.v.codes + vr * vcb, i, p.v.bm, vcb)), a);
          if (p.v.prod) {
            const float wr = w * s_vr[tt];
            sa += gn_bit(p.v.qjl + vr * (d / 8), i) ? wr : -wr;
          }
        }
        acc[c] = a;
        sacc[c] = sa;
      }
    }
    __syncthreads();
  }

  // ---- the slice's partial state
  const int stride = 4 + 2 * d;
#pragma unroll
  for (int c = 0; c < kGnCoords; ++c) {
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
  if (p.v.prod) {  // o' += S_V^T (weighted signs); sqrt(pi/2)/d is in the weights
    float add[kGnMaxD / kGnThreads];
    for (int i = tid, c = 0; i < d; i += kGnThreads, ++c) {
      float a = 0.f;
      for (int k = 0; k < d; ++k) a = fmaf(__ldg(p.v.S + (int64_t)k * d + i), s_s[k], a);
      add[c] = a;
    }
    __syncthreads();
    for (int i = tid, c = 0; i < d; i += kGnThreads, ++c) s_o[i] += add[c];
    __syncthreads();
  }
  const float inv_l = l > 0.f ? 1.0f / l : 0.f;
  if (p.v.rot) {  // o = Pi^T o'
    for (int c = tid; c < d; c += kGnThreads) {
      float a = 0.f;
      for (int r = 0; r < d; ++r) a = fmaf(__ldg(p.v.rot + (int64_t)r * d + c), s_o[r], a);
      out[c] = a * inv_l;
    }
  } else {  // o = sigma * H o' / sqrt(d)
    gn_fwht(s_o, 1, d, kGnMaxD);
    const float f = rsqrtf((float)d) * inv_l;
    for (int i = tid; i < d; i += kGnThreads) out[i] = (p.v.signs[i] < 0 ? -s_o[i] : s_o[i]) * f;
  }
}

GnSide side_of(const QuantParams &q, const CacheView &v) {
  GnSide s{};
  s.bm = q.bm;
  s.prod = q.prod;
  s.cent = q.centroids;
  s.rot = q.rot;
  s.S = q.S;
  s.signs = q.signs;
  s.codes = v.codes;
  s.qjl = v.qjl;
  s.norms = v.norms;
  s.rnorms = v.rnorms;
  s.sb = v.sb;
  s.sh = v.sh;
  s.sn = v.sn;
  return s;
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
  p.k = side_of(a.kq, a.k);
  p.v = side_of(a.vq, a.v);
  p.q = a.q;
  p.q_dtype = a.q_dtype;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.g = a.Hq / a.Hkv;
  p.hg = (p.g + kGnHeads - 1) / kGnHeads;
  p.d = a.kq.d;
  p.seq_len = a.seq_len;
  p.seq_lens = a.seq_lens;
  p.scale_log2 = a.scale * kGnLog2e;
  p.out = a.out;
  p.scores = a.scores;
  p.ws = a.ws;
  if (p.d > kGnMaxD || p.d % 8) return cudaErrorInvalidValue;
  p.splits = general_decode_splits(a.B, a.Hq, a.Hkv, a.seq_len);
  p.per_split = (a.seq_len + p.splits - 1) / p.splits;
  if (a.seq_len > 0) {
    const dim3 grid((unsigned)p.splits, (unsigned)(a.B * a.Hkv * p.hg));
    general_partial_kernel<<<grid, kGnThreads, 0, s>>>(p);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  } else {
    p.splits = 0;
  }
  general_merge_kernel<<<(unsigned)(a.B * a.Hq), kGnThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace tq
