// TurboQuant dequant for sm_100a: x_hat = ||x|| Pi^T u_hat with
// u_hat = c[idx] (+ ||r|| sqrt(pi/2)/d S^T sign for TurboQuant_prod), i.e. the
// pseudocode's dequant step ("内存厂商的噩梦来了", section 4) and the QJL
// reconstruction of the residual ("TurboQuant của Google", section "Vấn đề
// của inner product").  A reference path for users and tests, not the decode
// hot loop (decode never materialises x_hat).

#include "../../include/tq.h"
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kDqThreads = 256;

struct DqParams {
  const uint8_t *codes;
  const uint8_t *qjl;
  const float *norms;
  const float *rnorms;
  int64_t sb, sh, sn;
  int64_t H, N, nvec;
  const float *cent;
  const int8_t *signs;
  const float *S;
  float sqrt_d;
  float *out;
};

template <int D, int BM, bool PROD>
__global__ void __launch_bounds__(kDqThreads) dequant_kernel(DqParams p) {
  constexpr int T = D <= 64 ? 1 : D / 64;
  constexpr int E = D / T;
  constexpr int VPB = kDqThreads / T;
  constexpr int NWC = BM > 0 ? E * BM / 32 : 1;
  __shared__ float s_cent[16];
  __shared__ int8_t s_sgn[D];
  const int tid = threadIdx.x;
  if (BM > 0 && tid < (1 << BM)) s_cent[tid] = p.cent[tid];
  for (int i = tid; i < D; i += blockDim.x) s_sgn[i] = p.signs[i];
  __syncthreads();

  const int t = tid % T;
  int64_t v = (int64_t)blockIdx.x * VPB + tid / T;
  const bool active = v < p.nvec;
  if (!active) v = p.nvec - 1;
  const int64_t n = v % p.N, bh = v / p.N, h = bh % p.H, b = bh / p.H;
  const int64_t rec = b * p.sb + h * p.sh + n * p.sn;

  float a[E];
  if constexpr (BM > 0) {
    uint32_t W[NWC];
    dev::load_words<NWC>(p.codes + rec * (D * BM / 8) + t * (E * BM / 8), W);
#pragma unroll
    for (int i = 0; i < E; ++i) a[i] = s_cent[dev::get_field<BM>(W, i)];
  } else {
#pragma unroll
    for (int i = 0; i < E; ++i) a[i] = 0.f;
  }
  if constexpr (PROD) {
    // + gamma sqrt(pi/2)/d * sum_k sign_k S[k][i]
    const uint32_t *qw = reinterpret_cast<const uint32_t *>(p.qjl + rec * (D / 8));
    const float coef = __ldg(p.rnorms + rec) * (1.2533141373155003f / (float)D);
    float corr[E];
#pragma unroll
    for (int i = 0; i < E; ++i) corr[i] = 0.f;
    for (int kw = 0; kw < D / 32; ++kw) {
      const uint32_t w = __ldg(qw + kw);
      for (int kb = 0; kb < 32; ++kb) {
        const float sg = ((w >> kb) & 1u) ? 1.f : -1.f;
        const float *Sk = p.S + (size_t)(32 * kw + kb) * D + t * E;
#pragma unroll
        for (int i = 0; i < E; ++i) corr[i] = fmaf(sg, __ldg(Sk + i), corr[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < E; ++i) a[i] = fmaf(coef, corr[i], a[i]);
  }
  dev::fwht<T, E>(a, t);
  const float sc = __fdiv_rn(__ldg(p.norms + rec), p.sqrt_d);
  if (active) {
    float *o = p.out + v * D + t * E;
#pragma unroll
    for (int i = 0; i < E; i += 4) {
      float4 q;
      q.x = a[i] * sc * s_sgn[t * E + i];
      q.y = a[i + 1] * sc * s_sgn[t * E + i + 1];
      q.z = a[i + 2] * sc * s_sgn[t * E + i + 2];
      q.w = a[i + 3] * sc * s_sgn[t * E + i + 3];
      *reinterpret_cast<float4 *>(o + i) = q;
    }
  }
}

template <int D, int BM, bool PROD>
cudaError_t run(const DequantArgs &a, cudaStream_t s) {
  constexpr int T = D <= 64 ? 1 : D / 64;
  constexpr int VPB = kDqThreads / T;
  DqParams p{a.in.codes, a.in.qjl, a.in.norms, a.in.rnorms, a.in.sb, a.in.sh, a.in.sn,
             a.H, a.N, a.B * a.H * a.N, a.q.centroids, a.q.signs, a.q.S, a.q.sqrt_d, a.out};
  const int64_t blocks = (p.nvec + VPB - 1) / VPB;
  dequant_kernel<D, BM, PROD><<<(unsigned)blocks, kDqThreads, 0, s>>>(p);
  return cudaGetLastError();
}

template <int D, bool PROD>
cudaError_t by_bits(const DequantArgs &a, cudaStream_t s) {
  switch (a.q.bm) {
    case 0: if constexpr (PROD) return run<D, 0, true>(a, s); else return cudaErrorInvalidValue;
    case 1: return run<D, 1, PROD>(a, s);
    case 2: return run<D, 2, PROD>(a, s);
    case 3: return run<D, 3, PROD>(a, s);
    case 4: return run<D, 4, PROD>(a, s);
  }
  return cudaErrorInvalidValue;
}

template <int D>
cudaError_t by_variant(const DequantArgs &a, cudaStream_t s) {
  return a.q.prod ? by_bits<D, true>(a, s) : by_bits<D, false>(a, s);
}

}  // namespace

bool dequant_supported(int d, int bm, bool prod, bool dense) {
  if (dense) return d >= 8 && d <= 256 && d % 8 == 0 && bm >= (prod ? 0 : 1) && bm <= 4;
  return (d == 64 || d == 128 || d == 256) && bm >= (prod ? 0 : 1) && bm <= 4;
}

cudaError_t launch_dequant(const DequantArgs &a, cudaStream_t s) {
  if (a.q.rot) return launch_dequant_dense(a, s);
  switch (a.q.d) {
    case 64: return by_variant<64>(a, s);
    case 128: return by_variant<128>(a, s);
    case 256: return by_variant<256>(a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tq
