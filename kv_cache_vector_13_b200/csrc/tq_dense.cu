// TurboQuant with the dense (Haar) rotation, any d that is a multiple of 8
// up to 256 (sm_100a): encode and dequant, one warp per vector.
//
// The rotation is the pages' own definition ("TurboQuant của Google: nén KV
// cache 6 lần", section "Trick đầu tiên": Pi is the Q of a Gaussian
// matrix's QR), y = Pi x, a d x d product per vector -- the cost the critique
// of the runtime names ("Steel-man: ReturningTarzan của ExLlama đã đúng ở
// đâu", point 1).  Per vector, in the pages' order: keep the norm (canonical
// fp32 fold-halves sum of squares over the zero-padded power-of-two length,
// sqrt_rn), u = fl(Pi x) * fl(1/n) in fp32, idx = #{j : u > t_j}, bit-pack;
// prod adds r = u - c[idx], ||r|| and sign(S r).  The products are fp32 FMAs
// in ascending input order, so u differs from the exact value by a few
// units in the last place of sum |Pi_jk x_k| / n: codes can differ from
// the exact ones only for coordinates that close to a threshold.
//
// Lane l of a warp holds coordinates l + 32 m; the warp's x and u (or r) are
// staged in shared memory so that every lane can read all of them.  The
// matrices (Pi, S) are read from global memory (L1/L2-resident).

#include "../../include/tq.h"
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kDnWarps = 8;
constexpr int kDnMax = 256;  // largest d
constexpr int kDnJ = kDnMax / 32;

struct DenseParams {
  const void *x;
  int dtype;
  int64_t xsb, xsh, xsn;
  int64_t B, H, N, nvec;
  uint8_t *codes;
  uint8_t *qjl;
  float *norms;
  float *rnorms;
  int64_t osb, osh, osn;
  const float *cent;
  const float *thr;
  const float *rot;
  const float *S;
  int d, bm, kcb;
  bool prod;
  float *out;  // dequant
};

__device__ __forceinline__ float load_elem(const void *base, int dtype, int64_t i) {
  if (dtype == TQ_F32) return __ldg(static_cast<const float *>(base) + i);
  const unsigned short h = __ldg(static_cast<const unsigned short *>(base) + i);
  return dtype == TQ_BF16 ? __uint_as_float((uint32_t)h << 16) : __half2float(__ushort_as_half(h));
}

// sum over k < d of M[row * d + k] * v[k] (v in shared memory), fp32 FMAs in
// ascending k; d is a multiple of 8, rows 16-byte aligned
__device__ __forceinline__ float row_dot(const float *M, int row, int d, const float *v) {
  const float4 *r = reinterpret_cast<const float4 *>(M + (int64_t)row * d);
  float acc = 0.0f;
  for (int k = 0; k < d; k += 4) {
    const float4 m = __ldg(r + k / 4);
    acc = fmaf(m.x, v[k], acc);
    acc = fmaf(m.y, v[k + 1], acc);
    acc = fmaf(m.z, v[k + 2], acc);
    acc = fmaf(m.w, v[k + 3], acc);
  }
  return acc;
}

__device__ __forceinline__ void bhn(const DenseParams &p, int64_t v, int64_t &b, int64_t &h, int64_t &n) {
  n = v % p.N;
  const int64_t bh = v / p.N;
  h = bh % p.H;
  b = bh / p.H;
}

__global__ void __launch_bounds__(kDnWarps * 32) encode_dense_kernel(DenseParams p) {
  __shared__ float s_x[kDnWarps][kDnMax];
  __shared__ float s_r[kDnWarps][kDnMax];
  __shared__ unsigned char s_idx[kDnWarps][kDnMax];
  __shared__ float s_thr[16], s_cent[16];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = 1 << p.bm;
  if (threadIdx.x < K && p.bm > 0) s_cent[threadIdx.x] = p.cent[threadIdx.x];
  if (threadIdx.x + 1 < K && p.bm > 0) s_thr[threadIdx.x] = p.thr[threadIdx.x];
  __syncthreads();
  const int64_t v = (int64_t)blockIdx.x * kDnWarps + warp;
  if (v >= p.nvec) return;
  int64_t b, h, n;
  bhn(p, v, b, h, n);
  const int64_t xoff = b * p.xsb + h * p.xsh + n * p.xsn;
  const int64_t rec = b * p.osb + h * p.osh + n * p.osn;
  const int d = p.d;
  float *xs = s_x[warp], *rs = s_r[warp];

  // load; norm = sqrt_rn of the fold-halves sum of squares over the
  // zero-padded power-of-two length P2
  float sq[kDnJ];
#pragma unroll
  for (int j = 0; j < kDnJ; ++j) {
    const int k = lane + 32 * j;
    const float a = k < d ? load_elem(p.x, p.dtype, xoff + k) : 0.0f;
    if (k < d) xs[k] = a;
    sq[j] = __fmul_rn(a, a);
  }
  int P2 = 8;
  while (P2 < d) P2 <<= 1;
  // stages h = P2/2 .. 32 pair registers j and j + h/32 of the same lane
#pragma unroll
  for (int st = kDnJ / 2; st >= 1; st >>= 1) {
    if (P2 / 2 >= 32 * st) {
#pragma unroll
      for (int j = 0; j < st; ++j) sq[j] = __fadd_rn(sq[j], sq[j + st]);
    }
  }
  float s = sq[0];
  for (int hh = min(16, P2 / 2); hh >= 1; hh >>= 1) s = __fadd_rn(s, __shfl_down_sync(dev::kFull, s, hh));
  const float nrm = __fsqrt_rn(__shfl_sync(dev::kFull, s, 0));
  const float inv = nrm > 0.0f ? __frcp_rn(nrm) : 0.0f;
  __syncwarp();

  // rotate, scale, quantize; prod keeps the residual
  for (int j = lane; j < d; j += 32) {
    const float u = __fmul_rn(row_dot(p.rot, j, d, xs), inv);
    int idx = 0;
    for (int t = 0; t + 1 < K; ++t) idx += u > s_thr[t] ? 1 : 0;
    s_idx[warp][j] = (unsigned char)idx;
    rs[j] = p.bm > 0 ? __fsub_rn(u, s_cent[idx]) : u;
  }
  __syncwarp();

  // pack: byte B of the record holds stream bits 8B .. 8B+7, bit q of the
  // stream being bit q % b_m of index q / b_m
  if (p.bm > 0) {
    for (int B = lane; B < p.kcb; B += 32) {
      uint32_t val = 0;
#pragma unroll
      for (int bit = 0; bit < 8; ++bit) {
        const int q = 8 * B + bit;
        val |= (uint32_t)((s_idx[warp][q / p.bm] >> (q % p.bm)) & 1) << bit;
      }
      p.codes[rec * p.kcb + B] = (uint8_t)val;
    }
  }
  if (lane == 0) p.norms[rec] = nrm;
  if (p.prod) {
    float g = 0.0f;
    for (int j = lane; j < d; j += 32) g = fmaf(rs[j], rs[j], g);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) g += __shfl_xor_sync(dev::kFull, g, o);
    if (lane == 0) p.rnorms[rec] = sqrtf(g);
    // bit k = [(S r)_k >= 0], k = 32 m + lane, one ballot per 32 bits
    for (int m = 0; m < (d + 31) / 32; ++m) {
      const int k = 32 * m + lane;
      const bool pos = k < d ? row_dot(p.S, k, d, rs) >= 0.0f : false;
      const unsigned w = __ballot_sync(dev::kFull, pos);
      const int nb = min(4, d / 8 - 4 * m);
      if (lane < nb) p.qjl[rec * (d / 8) + 4 * m + lane] = (uint8_t)(w >> (8 * lane));
    }
  }
}

__global__ void __launch_bounds__(kDnWarps * 32) dequant_dense_kernel(DenseParams p) {
  __shared__ float s_u[kDnWarps][kDnMax];
  __shared__ float s_sg[kDnWarps][kDnMax];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t v = (int64_t)blockIdx.x * kDnWarps + warp;
  if (v >= p.nvec) return;
  int64_t b, h, n;
  bhn(p, v, b, h, n);
  const int64_t rec = b * p.osb + h * p.osh + n * p.osn;
  const int d = p.d;
  float *us = s_u[warp], *sg = s_sg[warp];
  // u_hat in the rotated basis: c[idx] (+ prod: ||r|| sqrt(pi/2)/d S^T sign)
  for (int j = lane; j < d; j += 32) {
    float u = 0.0f;
    if (p.bm > 0) {
      int idx = 0;
      for (int t = 0; t < p.bm; ++t) {
        const int q = j * p.bm + t;
        idx |= ((p.codes[rec * p.kcb + q / 8] >> (q % 8)) & 1) << t;
      }
      u = __ldg(p.cent + idx);
    }
    us[j] = u;
    if (p.prod) sg[j] = ((p.qjl[rec * (d / 8) + j / 8] >> (j % 8)) & 1) ? 1.0f : -1.0f;
  }
  __syncwarp();
  if (p.prod) {
    const float scale = __ldg(p.rnorms + rec) * (1.2533141373155003f / (float)d);
    for (int j = lane; j < d; j += 32) {
      float acc = 0.0f;
      for (int k = 0; k < d; ++k) acc = fmaf(__ldg(p.S + (int64_t)k * d + j), sg[k], acc);
      us[j] = fmaf(scale, acc, us[j]);
    }
    __syncwarp();
  }
  // x_hat = ||x|| Pi^T u_hat
  const float nrm = __ldg(p.norms + rec);
  for (int i = lane; i < d; i += 32) {
    float acc = 0.0f;
    for (int j = 0; j < d; ++j) acc = fmaf(__ldg(p.rot + (int64_t)j * d + i), us[j], acc);
    p.out[v * d + i] = nrm * acc;
  }
}

}  // namespace

cudaError_t launch_encode_dense(const EncodeArgs &a, cudaStream_t s) {
  DenseParams p{};
  p.x = a.x;
  p.dtype = a.dtype;
  p.xsb = a.xsb;
  p.xsh = a.xsh;
  p.xsn = a.xsn;
  p.B = a.B;
  p.H = a.H;
  p.N = a.N;
  p.nvec = a.B * a.H * a.N;
  p.codes = a.out.codes;
  p.qjl = a.out.qjl;
  p.norms = a.out.norms;
  p.rnorms = a.out.rnorms;
  p.osb = a.out.sb;
  p.osh = a.out.sh;
  p.osn = a.out.sn;
  p.cent = a.q.centroids;
  p.thr = a.q.thresholds;
  p.rot = a.q.rot;
  p.S = a.q.S;
  p.d = a.q.d;
  p.bm = a.q.bm;
  p.kcb = a.q.d * a.q.bm / 8;
  p.prod = a.q.prod;
  const int64_t blocks = (p.nvec + kDnWarps - 1) / kDnWarps;
  encode_dense_kernel<<<(unsigned)blocks, kDnWarps * 32, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_dequant_dense(const DequantArgs &a, cudaStream_t s) {
  DenseParams p{};
  p.B = a.B;
  p.H = a.H;
  p.N = a.N;
  p.nvec = a.B * a.H * a.N;
  p.codes = a.in.codes;
  p.qjl = a.in.qjl;
  p.norms = a.in.norms;
  p.rnorms = a.in.rnorms;
  p.osb = a.in.sb;
  p.osh = a.in.sh;
  p.osn = a.in.sn;
  p.cent = a.q.centroids;
  p.rot = a.q.rot;
  p.S = a.q.S;
  p.d = a.q.d;
  p.bm = a.q.bm;
  p.kcb = a.q.d * a.q.bm / 8;
  p.prod = a.q.prod;
  p.out = a.out;
  const int64_t blocks = (p.nvec + kDnWarps - 1) / kDnWarps;
  dequant_dense_kernel<<<(unsigned)blocks, kDnWarps * 32, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace tq
