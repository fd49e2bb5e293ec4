// TurboQuant encode (TurboQuant_mse and TurboQuant_prod) for sm_100a.
//
// Per vector, in the order the pages give ("TurboQuant của Google: nén KV
// cache 6 lần", sections "Trick đầu tiên", "Lloyd-Max quantizer" and "Vấn đề
// của inner product"; "内存厂商的噩梦来了", sections 4.1-4.3): keep the norm,
// rotate with sign flips + FWHT, scale to the unit sphere, map each
// coordinate to its Lloyd-Max index, bit-pack; for prod, take the residual,
// its norm, and the signs of S r.
//
// Work layout: T = d/E lanes per vector, each lane owning E contiguous
// coordinates in registers (E = 64 for large batches; E = 16 for small ones,
// such as appending one token, where short per-lane chains matter more than
// shuffle count); the butterfly stages with stride >= E and the first folds
// of the norm go through warp shuffles.
// Memory traffic per vector is the input read once and the packed record
// written once; nothing else touches HBM.

#include "../../include/tq.h"
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kEncThreads = 256;

struct EncParams {
  const void *x;
  int64_t xsb, xsh, xsn;
  int64_t H, N, nvec;
  uint8_t *codes;
  uint8_t *qjl;
  float *norms;
  float *rnorms;
  int64_t osb, osh, osn;
  const float *cent;
  const float *thr;
  const int8_t *signs;
  const float *S;
  float sqrt_d;
};

template <int D, int EE = 64>
struct Shape {
  static constexpr int T = D <= EE ? 1 : D / EE;  // lanes per vector
  static constexpr int E = D / T;                 // coordinates per lane
  static constexpr int VPB = kEncThreads / T;     // vectors per block
  static constexpr int RS = D + 4;                // padded smem row (floats)
  // S lives in shared memory when it fits next to the residual buffer
  static constexpr bool kSmemS = (size_t)D * RS * 4 + (size_t)VPB * RS * 4 <= 200 * 1024;
};

template <int D, bool PROD, int EE>
constexpr size_t enc_smem_bytes() {
  using Sh = Shape<D, EE>;
  if constexpr (!PROD) return 0;
  return (size_t)Sh::VPB * Sh::RS * 4 + (Sh::kSmemS ? (size_t)D * Sh::RS * 4 : 0);
}

// Stores the low NB bytes of W (little-endian) to dst, which is aligned to
// the largest power of two dividing NB (at most 16).
template <int NB, int NW>
__device__ __forceinline__ void store_bytes(uint8_t *dst, const uint32_t (&W)[NW]) {
  if constexpr (NB % 16 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 16; ++i)
      reinterpret_cast<uint4 *>(dst)[i] = make_uint4(W[4 * i], W[4 * i + 1], W[4 * i + 2], W[4 * i + 3]);
  } else if constexpr (NB % 8 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 8; ++i) reinterpret_cast<uint2 *>(dst)[i] = make_uint2(W[2 * i], W[2 * i + 1]);
  } else if constexpr (NB % 4 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 4; ++i) reinterpret_cast<uint32_t *>(dst)[i] = W[i];
  } else {
    static_assert(NB % 2 == 0, "odd byte count");
#pragma unroll
    for (int i = 0; i < NB / 2; ++i)
      reinterpret_cast<unsigned short *>(dst)[i] = (unsigned short)(W[i >> 1] >> (16 * (i & 1)));
  }
}

template <int D, int BM, bool PROD, int DT, int EE>
__global__ void __launch_bounds__(kEncThreads) encode_kernel(EncParams p) {
  using Sh = Shape<D, EE>;
  constexpr int T = Sh::T, E = Sh::E, VPB = Sh::VPB, RS = Sh::RS;
  constexpr int K = 1 << BM;
  constexpr int NWC = BM > 0 ? (E * BM + 31) / 32 : 1;  // code words per lane
  constexpr int NWQ = (E + 31) / 32;                    // qjl words per lane

  __shared__ uint32_t s_sign[D / 32];
  __shared__ float s_cent[16];
  extern __shared__ float4 s_dyn4[];
  float *s_dyn = reinterpret_cast<float *>(s_dyn4);
  float *s_r = s_dyn;                   // [VPB][RS] residuals (prod)
  float *s_S = s_dyn + (size_t)VPB * RS;  // [D][RS] projection (prod, if it fits)

  const int tid = threadIdx.x;
  if (tid < 32) {  // sign bit masks, one ballot per 32 coordinates
#pragma unroll
    for (int w = 0; w < D / 32; ++w) {
      const unsigned m = __ballot_sync(dev::kFull, p.signs[32 * w + tid] < 0);
      if (tid == 0) s_sign[w] = m;
    }
  }
  if constexpr (PROD && BM > 0) {
    if (tid < K) s_cent[tid] = p.cent[tid];
  }
  if constexpr (PROD && Sh::kSmemS) {
    for (int i = tid; i < D * D; i += blockDim.x) s_S[(i / D) * RS + (i % D)] = p.S[i];
  }
  uint32_t P[K / 2 > 0 ? K / 2 : 1];
#pragma unroll
  for (int m = 0; m + 1 < K / 2; ++m) P[m] = __float_as_uint(__ldg(p.thr + K / 2 + m));
  __syncthreads();

  const int t = tid % T;
  const int vl = tid / T;
  int64_t v = (int64_t)blockIdx.x * VPB + vl;
  const bool active = v < p.nvec;
  if (!active) v = p.nvec - 1;  // idle lanes still take part in the shuffles
  const int64_t n = v % p.N;
  const int64_t bh = v / p.N;
  const int64_t h = bh % p.H;
  const int64_t b = bh / p.H;
  const int64_t xoff = b * p.xsb + h * p.xsh + n * p.xsn + (int64_t)t * E;
  const int64_t rec = b * p.osb + h * p.osh + n * p.osn;
  constexpr int ES = DT == 0 ? 4 : 2;

  float a[E];
  dev::load_block<DT, E>(static_cast<const char *>(p.x) + xoff * ES, a);

  // norm: fold-halves sum of squares, then sqrt_rn
  float sq[E];
#pragma unroll
  for (int i = 0; i < E; ++i) sq[i] = __fmul_rn(a[i], a[i]);
  const float nrm = __fsqrt_rn(dev::fold_halves_sum<T, E>(sq));

  // rotate: sign flips, then the unnormalised FWHT
  uint32_t sw[(E + 31) / 32];
#pragma unroll
  for (int w = 0; w < (E + 31) / 32; ++w) sw[w] = s_sign[(t * E) / 32 + w] >> ((t * E) & 31);
#pragma unroll
  for (int i = 0; i < E; ++i)
    a[i] = __uint_as_float(__float_as_uint(a[i]) ^ (((sw[i >> 5] >> (i & 31)) & 1u) << 31));
  dev::fwht<T, E>(a, t);

  // scale to the unit sphere: u = y * fl(1 / fl(n * fl(sqrt d)))
  const float wsc = __fmul_rn(nrm, p.sqrt_d);
  const float inv = wsc > 0.0f ? __frcp_rn(wsc) : 0.0f;
#pragma unroll
  for (int i = 0; i < E; ++i) a[i] = __fmul_rn(a[i], inv);

  // quantize and pack; prod keeps the residual in a[]
  uint32_t W[NWC];
#pragma unroll
  for (int w = 0; w < NWC; ++w) W[w] = 0u;
  if constexpr (BM > 0) {
#pragma unroll
    for (int i = 0; i < E; ++i) {
      int idx;
      if constexpr (BM == 1) {
        idx = a[i] > 0.0f ? 1 : 0;
      } else {
        idx = dev::quantize_sym<BM>(a[i], P);
      }
      dev::put_field<BM>(W, i, (uint32_t)idx);
      if constexpr (PROD) a[i] = __fsub_rn(a[i], s_cent[idx]);
    }
    if (active) store_bytes<E * BM / 8>(p.codes + rec * (D * BM / 8) + t * (E * BM / 8), W);
  }
  if (active && t == 0) p.norms[rec] = nrm;

  if constexpr (PROD) {
    float rr[E];
#pragma unroll
    for (int i = 0; i < E; ++i) rr[i] = __fmul_rn(a[i], a[i]);
    const float gam = __fsqrt_rn(dev::fold_halves_sum<T, E>(rr));
    // z_k = sum_i S[k][i] r_i for this lane's k-block, fp32
    float *rv = s_r + (size_t)vl * RS;
#pragma unroll
    for (int i = 0; i < E; ++i) rv[t * E + i] = a[i];
    __syncwarp();
    uint32_t Q[NWQ];
    const int rot = (t * 32 / T) & 31;  // rotates the column order per lane: no bank clash
#pragma unroll
    for (int w = 0; w < NWQ; ++w) {
      uint32_t qw = 0u;
      for (int kb = 0; kb < (E < 32 ? E : 32); ++kb) {
        const int k = t * E + w * 32 + kb;
        float acc = 0.0f;
        if constexpr (Sh::kSmemS) {
          const float *Sk = s_S + (size_t)k * RS;
#pragma unroll 8
          for (int ii = 0; ii < D; ++ii) {
            const int i = (ii + rot) & (D - 1);
            acc = fmaf(Sk[i], rv[i], acc);
          }
        } else {
          const float *Sk = p.S + (size_t)k * D;
#pragma unroll 8
          for (int ii = 0; ii < D; ++ii) {
            const int i = (ii + rot) & (D - 1);
            acc = fmaf(__ldg(Sk + i), rv[i], acc);
          }
        }
        qw |= (acc >= 0.0f ? 1u : 0u) << kb;
      }
      Q[w] = qw;
    }
    if (active) {
      store_bytes<E / 8>(p.qjl + rec * (D / 8) + t * (E / 8), Q);
      if (t == 0) p.rnorms[rec] = gam;
    }
  }
}

template <int D, int BM, bool PROD, int DT, int EE>
cudaError_t run_e(const EncodeArgs &a, cudaStream_t s) {
  using Sh = Shape<D, EE>;
  EncParams p;
  p.x = a.x;
  p.xsb = a.xsb;
  p.xsh = a.xsh;
  p.xsn = a.xsn;
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
  p.signs = a.q.signs;
  p.S = a.q.S;
  p.sqrt_d = a.q.sqrt_d;
  const size_t smem = enc_smem_bytes<D, PROD, EE>();
  auto kern = encode_kernel<D, BM, PROD, DT, EE>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t blocks = (p.nvec + Sh::VPB - 1) / Sh::VPB;
  kern<<<(unsigned)blocks, kEncThreads, smem, s>>>(p);
  return cudaGetLastError();
}

// Small batches (up to one vector per lane of a full wave at E = 64) take
// the E = 16 layout: four times more lanes per vector, shorter chains.
template <int D, int BM, bool PROD, int DT>
cudaError_t run(const EncodeArgs &a, cudaStream_t s) {
  const int64_t nvec = a.B * a.H * a.N;
  if (nvec <= 148 * (kEncThreads / Shape<D, 64>::T)) return run_e<D, BM, PROD, DT, 16>(a, s);
  return run_e<D, BM, PROD, DT, 64>(a, s);
}

template <int D, int BM, bool PROD>
cudaError_t by_dtype(const EncodeArgs &a, cudaStream_t s) {
  switch (a.dtype) {
    case TQ_F32: return run<D, BM, PROD, 0>(a, s);
    case TQ_BF16: return run<D, BM, PROD, 1>(a, s);
    case TQ_F16: return run<D, BM, PROD, 2>(a, s);
  }
  return cudaErrorInvalidValue;
}

template <int D, bool PROD>
cudaError_t by_bits(const EncodeArgs &a, cudaStream_t s) {
  switch (a.q.bm) {
    case 0: if constexpr (PROD) return by_dtype<D, 0, true>(a, s); else return cudaErrorInvalidValue;
    case 1: return by_dtype<D, 1, PROD>(a, s);
    case 2: return by_dtype<D, 2, PROD>(a, s);
    case 3: return by_dtype<D, 3, PROD>(a, s);
    case 4: return by_dtype<D, 4, PROD>(a, s);
  }
  return cudaErrorInvalidValue;
}

template <int D>
cudaError_t by_variant(const EncodeArgs &a, cudaStream_t s) {
  return a.q.prod ? by_bits<D, true>(a, s) : by_bits<D, false>(a, s);
}

}  // namespace

bool encode_supported(int d, int bm, bool prod, int dtype) {
  return (d == 64 || d == 128 || d == 256) && bm >= (prod ? 0 : 1) && bm <= 4 && dtype >= 0 && dtype <= 2;
}

cudaError_t launch_encode(const EncodeArgs &a, cudaStream_t s) {
  if (a.B * a.H * a.N >= (int64_t)1 << 40) return cudaErrorInvalidValue;
  switch (a.q.d) {
    case 64: return by_variant<64>(a, s);
    case 128: return by_variant<128>(a, s);
    case 256: return by_variant<256>(a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tq
