// Decode attention over an outlier-channel split cache (sm_100a), plain
// CUDA cores.
//
// A head's channels are in two groups quantized separately, the outlier
// channels at a higher bit width ("TurboQuant của Google: nén KV cache 6
// lần", the correction in the experiments section).  Each group is its own
// TurboQuant quantizer with the dense rotation, so for one query
//   s_j = sum_g n_gj ( <q'_g, c_g[idx_gj]> + [prod] ||r_gj|| sqrt(pi/2)/d_g <S_g q'_g, sign_gj> ),
// q'_g = Pi_g q[channels_g]; softmax over the tokens; each value group is
// summed in its rotated basis and rotated back into its channels.
//
// split_scores_kernel: a thread per token, all query heads of its kv head
// (the codes are unpacked once for the GQA group); writes the logits.
// split_attend_kernel: a block per query head: the logits' maximum and sum,
// then a thread per rotated coordinate accumulates the weighted centroids
// (prod values: the weighted sign vectors, projected once by S^T at the
// end), and the inverse rotation scatters the group into its channels.

#include "../../include/tq.h"
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kSpMaxD = 256;
constexpr int kSpMaxG = 8;  // query heads per kv head handled by one thread

struct SpGroup {
  int d, bm;
  bool prod;
  const float *cent, *rot, *S;
  const int32_t *chan;
  const uint8_t *codes, *qjl;
  const float *norms, *rnorms;
  int64_t sb, sh, sn;
};

struct SpParams {
  SpGroup k[2], v[2];
  const void *q;
  int q_dtype;
  int B, Hq, Hkv, g, d;
  int64_t seq_len;
  const int32_t *seq_lens;
  float scale;
  float *out;
  float *logits;  // [B * Hq][seq_len]
};

__device__ __forceinline__ float ld_q(const SpParams &p, int64_t i) {
  if (p.q_dtype == TQ_F32) return __ldg(static_cast<const float *>(p.q) + i);
  const unsigned short h = __ldg(static_cast<const unsigned short *>(p.q) + i);
  return p.q_dtype == TQ_BF16 ? __uint_as_float((uint32_t)h << 16) : __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ int64_t blen(const SpParams &p, int b) {
  if (!p.seq_lens) return p.seq_len;
  const int64_t L = p.seq_lens[b];
  return L < 0 ? 0 : (L > p.seq_len ? p.seq_len : L);
}

// index of coordinate i of a record's LSB-first bitstream
__device__ __forceinline__ int field(const uint8_t *rec, int i, int bm) {
  int v = 0;
  for (int t = 0; t < bm; ++t) {
    const int q = i * bm + t;
    v |= ((rec[q >> 3] >> (q & 7)) & 1) << t;
  }
  return v;
}

__global__ void __launch_bounds__(256) split_scores_kernel(SpParams p) {
  __shared__ float s_qr[2][kSpMaxG][kSpMaxD];  // q'_g per head of the group
  __shared__ float s_qs[2][kSpMaxG][kSpMaxD];  // S_g q'_g
  __shared__ float s_q[kSpMaxG][kSpMaxD];
  const int bk = blockIdx.y;  // (b, kv head)
  const int b = bk / p.Hkv, kvh = bk % p.Hkv;
  const int tid = threadIdx.x;
  for (int i = tid; i < p.g * p.d; i += blockDim.x) {
    const int hh = i / p.d, c = i % p.d;
    s_q[hh][c] = ld_q(p, ((int64_t)b * p.Hq + kvh * p.g + hh) * p.d + c);
  }
  __syncthreads();
  for (int gr = 0; gr < 2; ++gr) {
    const SpGroup &G = p.k[gr];
    for (int i = tid; i < p.g * G.d; i += blockDim.x) {
      const int hh = i / G.d, r = i % G.d;
      float acc = 0.f;
      for (int c = 0; c < G.d; ++c) {
        const int ch = min(max(__ldg(G.chan + c), 0), p.d - 1);  // lists partition [0, d)
        acc = fmaf(__ldg(G.rot + (int64_t)r * G.d + c), s_q[hh][ch], acc);
      }
      s_qr[gr][hh][r] = acc;
    }
  }
  __syncthreads();
  for (int gr = 0; gr < 2; ++gr) {
    const SpGroup &G = p.k[gr];
    if (!G.prod) continue;
    for (int i = tid; i < p.g * G.d; i += blockDim.x) {
      const int hh = i / G.d, r = i % G.d;
      float acc = 0.f;
      for (int c = 0; c < G.d; ++c) acc = fmaf(__ldg(G.S + (int64_t)r * G.d + c), s_qr[gr][hh][c], acc);
      s_qs[gr][hh][r] = acc;
    }
  }
  __syncthreads();
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + tid;
  const int64_t L = blen(p, b);
  if (j >= p.seq_len) return;
  float sc[kSpMaxG];
#pragma unroll
  for (int hh = 0; hh < kSpMaxG; ++hh) sc[hh] = 0.f;
  if (j < L) {
    for (int gr = 0; gr < 2; ++gr) {
      const SpGroup &G = p.k[gr];
      const int64_t rec = (int64_t)b * G.sb + (int64_t)kvh * G.sh + j * G.sn;
      const uint8_t *cr = G.codes ? G.codes + rec * (G.d * G.bm / 8) : nullptr;
      const uint8_t *qr = G.prod ? G.qjl + rec * (G.d / 8) : nullptr;
      const float n = __ldg(G.norms + rec);
      const float kap = G.prod ? __ldg(G.rnorms + rec) * (1.2533141373155003f / (float)G.d) : 0.f;
      float part[kSpMaxG];
#pragma unroll
      for (int hh = 0; hh < kSpMaxG; ++hh) part[hh] = 0.f;
      for (int i = 0; i < G.d; ++i) {
        const float c = G.bm > 0 ? __ldg(G.cent + field(cr, i, G.bm)) : 0.f;
        const float sg = G.prod ? (((qr[i >> 3] >> (i & 7)) & 1) ? kap : -kap) : 0.f;
#pragma unroll
        for (int hh = 0; hh < kSpMaxG; ++hh) {
          if (hh < p.g) part[hh] = fmaf(c, s_qr[gr][hh][i], fmaf(sg, G.prod ? s_qs[gr][hh][i] : 0.f, part[hh]));
        }
      }
#pragma unroll
      for (int hh = 0; hh < kSpMaxG; ++hh) sc[hh] = fmaf(n, part[hh], sc[hh]);
    }
  }
#pragma unroll
  for (int hh = 0; hh < kSpMaxG; ++hh) {
    if (hh < p.g)
      p.logits[((int64_t)b * p.Hq + kvh * p.g + hh) * p.seq_len + j] = j < L ? sc[hh] * p.scale : -INFINITY;
  }
}

__device__ float block_reduce(float v, bool is_max, float *s_red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const float w = __shfl_xor_sync(dev::kFull, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  __syncthreads();
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  float r = is_max ? -INFINITY : 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = is_max ? fmaxf(r, s_red[w]) : r + s_red[w];
  return r;
}

__global__ void __launch_bounds__(256) split_attend_kernel(SpParams p) {
  __shared__ float s_red[8];
  __shared__ float s_acc[2][kSpMaxD];  // weighted centroids, rotated basis
  __shared__ float s_sgn[2][kSpMaxD];  // weighted sign sums (prod values)
  const int head = blockIdx.x;  // b * Hq + hq
  const int b = head / p.Hq, hq = head % p.Hq, kvh = hq / p.g;
  const int tid = threadIdx.x;
  const int64_t L = blen(p, b);
  float *out = p.out + (int64_t)head * p.d;
  if (L == 0) {
    for (int c = tid; c < p.d; c += blockDim.x) out[c] = 0.f;
    return;
  }
  const float *lg = p.logits + (int64_t)head * p.seq_len;
  float m = -INFINITY;
  for (int64_t j = tid; j < L; j += blockDim.x) m = fmaxf(m, lg[j]);
  m = block_reduce(m, true, s_red);
  float l = 0.f;
  for (int64_t j = tid; j < L; j += blockDim.x) l += __expf(lg[j] - m);
  l = block_reduce(l, false, s_red);
  const float inv_l = 1.0f / l;
  // thread t < d_0 + d_1: coordinate t of group 0, or t - d_0 of group 1
  const int d0 = p.v[0].d;
  const int gr = tid < d0 ? 0 : 1;
  const int i = gr == 0 ? tid : tid - d0;
  const bool mine = tid < d0 + p.v[1].d;
  if (mine) {
    const SpGroup &G = p.v[gr];
    float acc = 0.f, sacc = 0.f;
    for (int64_t j = 0; j < L; ++j) {
      const int64_t rec = (int64_t)b * G.sb + (int64_t)kvh * G.sh + j * G.sn;
      const float w = __expf(lg[j] - m) * inv_l * __ldg(G.norms + rec);
      if (G.bm > 0) acc = fmaf(w, __ldg(G.cent + field(G.codes + rec * (G.d * G.bm / 8), i, G.bm)), acc);
      if (G.prod) {
        const float wr = w * __ldg(G.rnorms + rec);
        sacc += ((G.qjl[rec * (G.d / 8) + (i >> 3)] >> (i & 7)) & 1) ? wr : -wr;
      }
    }
    s_acc[gr][i] = acc;
    s_sgn[gr][i] = sacc;
  }
  __syncthreads();
  // prod values: add sqrt(pi/2)/d_g S_g^T (weighted signs) in the rotated basis
  float add = 0.f;
  if (mine && p.v[gr].prod) {
    const SpGroup &G = p.v[gr];
    for (int k = 0; k < G.d; ++k) add = fmaf(__ldg(G.S + (int64_t)k * G.d + i), s_sgn[gr][k], add);
    add *= 1.2533141373155003f / (float)G.d;
  }
  __syncthreads();
  if (mine) s_acc[gr][i] += add;
  __syncthreads();
  // back to the channels: out[chan_g[c]] = sum_r Pi_g[r][c] o'_g[r]
  if (mine) {
    const SpGroup &G = p.v[gr];
    float o = 0.f;
    for (int r = 0; r < G.d; ++r) o = fmaf(__ldg(G.rot + (int64_t)r * G.d + i), s_acc[gr][r], o);
    out[min(max(__ldg(G.chan + i), 0), p.d - 1)] = o;
  }
}

SpGroup group_of(const QuantParams &q, const CacheView &v) {
  SpGroup g{};
  g.d = q.d;
  g.bm = q.bm;
  g.prod = q.prod;
  g.cent = q.centroids;
  g.rot = q.rot;
  g.S = q.S;
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

}  // namespace

cudaError_t launch_decode_split(const SplitDecodeArgs &a, cudaStream_t s) {
  SpParams p{};
  for (int g = 0; g < 2; ++g) {
    p.k[g] = group_of(a.kq[g], a.k[g]);
    p.v[g] = group_of(a.vq[g], a.v[g]);
  }
  p.q = a.q;
  p.q_dtype = a.q_dtype;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.g = a.Hq / a.Hkv;
  p.d = a.d;
  p.seq_len = a.seq_len;
  p.seq_lens = a.seq_lens;
  p.scale = a.scale;
  p.out = a.out;
  p.logits = a.ws;
  if (p.g > kSpMaxG || p.d > kSpMaxD) return cudaErrorInvalidValue;
  const dim3 g1((unsigned)((a.seq_len + 255) / 256), (unsigned)(a.B * a.Hkv));
  split_scores_kernel<<<g1, 256, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  split_attend_kernel<<<(unsigned)(a.B * a.Hq), 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace tq
