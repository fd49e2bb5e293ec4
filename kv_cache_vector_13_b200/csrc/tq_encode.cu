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

#include <cuda_fp16.h>

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
  // v -> (n, bh) and bh -> (h, b) by multiply-shift when every index fits
  // in 31 bits (div32): q = (x * m) >> (31 + l) with l = ceil(log2 divisor),
  // m = floor(2^(31+l) / divisor) + 1, exact for x < 2^31 (Granlund and
  // Montgomery, "Division by invariant integers using multiplication").
  bool div32;
  uint32_t mN, mH;
  int sN, sH;
  bool pdl;  // launched programmatically after the kernel before it
};

// Programmatic dependent launch.  Every encode grid lets the next kernel in
// the stream start early; a grid that was itself launched early (pdl) keeps
// one thread waiting for the grid before it, so it cannot complete first and
// a chain of such grids completes in stream order.
__device__ __forceinline__ void pdl_open() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_close(bool pdl) {
  if (pdl && blockIdx.x == 0 && threadIdx.x == 0) asm volatile("griddepcontrol.wait;\n" ::: "memory");
}

// Vector index v -> (b, h, n) of a [B][H][N] batch.
__device__ __forceinline__ void split_index(const EncParams &p, int64_t v, int64_t &b, int64_t &h, int64_t &n) {
  if (p.div32) {
    const uint32_t x = (uint32_t)v;
    const uint32_t bh = (uint32_t)(((uint64_t)x * p.mN) >> p.sN);
    const uint32_t hb = (uint32_t)(((uint64_t)bh * p.mH) >> p.sH);
    n = x - bh * (uint32_t)p.N;
    h = bh - hb * (uint32_t)p.H;
    b = hb;
  } else {
    n = v % p.N;
    const int64_t bh = v / p.N;
    h = bh % p.H;
    b = bh / p.H;
  }
}

// Magic multiplier and shift for 31-bit dividends (see EncParams).
inline void magic31(int64_t d, uint32_t &m, int &s) {
  int l = 0;
  while (((int64_t)1 << l) < d) ++l;
  m = (uint32_t)((((uint64_t)1 << (31 + l)) / (uint64_t)d) + 1);
  s = 31 + l;
}

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

// Sign-flip masks (one ballot per 32 coordinates) into s_sign; the calling
// block's first warp does it.
template <int D>
__device__ __forceinline__ void load_sign_masks(const int8_t *signs, uint32_t *s_sign, int tid) {
  if (tid < 32) {
#pragma unroll
    for (int w = 0; w < D / 32; ++w) {
      const unsigned m = __ballot_sync(dev::kFull, signs[32 * w + tid] < 0);
      if (tid == 0) s_sign[w] = m;
    }
  }
}

// Per-vector front half, in the canonical fp32 order: load, norm (fold-halves
// sum of squares, sqrt_rn), sign flips + unnormalised FWHT, scale by
// fl(1 / fl(n * fl(sqrt d))), quantize and pack into W.  Returns the norm;
// a[] ends as the residual (prod) or the scaled rotation (mse).
template <int D, int BM, bool PROD, int DT, int T, int E, int NWC, int NP>
__device__ __forceinline__ float encode_front(const EncParams &p, int64_t xoff, int t, const uint32_t *s_sign,
                                              const float *s_cent, const uint32_t (&P)[NP], float (&a)[E],
                                              uint32_t (&W)[NWC]) {
  constexpr int ES = DT == 0 ? 4 : 2;
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
  }
  return nrm;
}

// The 64-coordinate layout is held to 3 resident blocks per SM (at most 85
// registers a thread): more blocks in flight hide the load latency better
// than the extra registers would help.
template <int D, int BM, bool PROD, int DT, int EE>
__global__ void __launch_bounds__(kEncThreads, EE == 64 ? 3 : 1) encode_kernel(EncParams p) {
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
  pdl_open();
  load_sign_masks<D>(p.signs, s_sign, tid);
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
  int64_t b, h, n;
  split_index(p, v, b, h, n);
  const int64_t xoff = b * p.xsb + h * p.xsh + n * p.xsn + (int64_t)t * E;
  const int64_t rec = b * p.osb + h * p.osh + n * p.osn;

  float a[E];
  uint32_t W[NWC];
  const float nrm = encode_front<D, BM, PROD, DT, T, E>(p, xoff, t, s_sign, s_cent, P, a, W);
  if constexpr (BM > 0) {
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
  pdl_close(p.pdl);
}

// ------------------------------------------------ prod, d = 128: tensor cores
//
// The QJL projection z = S r is a dense 128 x 128 contraction per vector; for
// a batch it is Z = R S^T, which runs here on mma.m16n8k16 (f16 x f16 ->
// f32).  One warp owns 16 vectors (two lanes per vector in the front half),
// exactly the M = 16 rows of an MMA tile.  Operands are split into fp16
// halves, x = hi + lo with hi = fp16(x), lo = fp16(x - hi), and
// z ~ Sh.rh + Sh.rl + Sl.rh (the dropped Sl.rl is below 2^-22 of
// sum |S_ki r_i|).  Each residual row is first scaled by a power of two,
// 2^(4 - floor(log2 ||r||)), which keeps both halves in fp16's normal range
// and leaves every sign unchanged.  The representation (about 3 * 2^-22
// per product), the dropped term and the fp32 accumulation over 24 MMA
// steps (at most 24 * 2^-23 of sum |S_ki r_i|) stay below 2^-17.4
// sum |S_ki r_i| <= 2^-17.4 ||S_k|| ||r||, a fifth of
// theta_k = 2^-15 ||S_k|| ||r||; a projection with |z| <= theta_k (about
// three in ten thousand) is recomputed by an fp32 dot product, so a stored
// sign can differ from the exact one only where an fp32 summation's sign
// could.  The block is persistent: it converts S to fp16 halves in
// shared memory once and then walks tiles of 256 vectors.
constexpr int kMmaThreads = 512;
constexpr int kMmaVPB = kMmaThreads / 2;  // vectors per tile (two lanes each)
constexpr int kSRow = 128 + 8;            // fp16 row of S halves (conflict-free B loads)
constexpr int kRRow = 128 + 4;            // fp32 residual row (conflict-free A loads)

constexpr size_t enc_mma_smem_bytes() {
  return (size_t)2 * 128 * kSRow * 2 + (size_t)kMmaVPB * kRRow * 4;
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<const uint32_t *>(&h); }

// fp16 (hi, lo) halves of the pair (x, y)
__device__ __forceinline__ void split2(float x, float y, uint32_t &hi, uint32_t &lo) {
  const __half2 h = __floats2half2_rn(x, y);
  const float2 f = __half22float2(h);
  hi = h2_bits(h);
  lo = h2_bits(__floats2half2_rn(x - f.x, y - f.y));
}

__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bits 0..3 of x to bits 0, 2, 4, 6
__device__ __forceinline__ uint32_t spread4(uint32_t x) {
  x = (x | (x << 2)) & 0x33u;
  return (x | (x << 1)) & 0x55u;
}

// sign of the fp32 dot product of one row of S (global, 16-byte aligned)
// with a residual row (shared, 16-byte aligned)
__device__ __noinline__ bool qjl_recheck(const float *S_row, const float *r) {
  const float4 *s4 = reinterpret_cast<const float4 *>(S_row);
  const float4 *r4 = reinterpret_cast<const float4 *>(r);
  float acc = 0.0f;
#pragma unroll 8
  for (int i = 0; i < 32; ++i) {
    const float4 a = __ldg(s4 + i), b = r4[i];
    acc = fmaf(a.x, b.x, acc);
    acc = fmaf(a.y, b.y, acc);
    acc = fmaf(a.z, b.z, acc);
    acc = fmaf(a.w, b.w, acc);
  }
  return acc >= 0.0f;
}

template <int BM, int DT>
__global__ void __launch_bounds__(kMmaThreads, 1) encode_prod_mma_kernel(EncParams p, int64_t ntiles) {
  constexpr int D = 128, T = 2, E = 64;
  constexpr int K = 1 << BM;
  constexpr int NWC = BM > 0 ? (E * BM + 31) / 32 : 1;

  __shared__ uint32_t s_sign[D / 32];
  __shared__ float s_cent[16];
  __shared__ float s_snorm[D];
  __shared__ float s_rs[kMmaVPB];  // per vector: scale of its residual row, theta factor
  __shared__ float s_th[kMmaVPB];
  extern __shared__ float4 s_dyn4[];
  __half *s_sh = reinterpret_cast<__half *>(s_dyn4);          // [128][kSRow] hi(S)
  __half *s_sl = s_sh + 128 * kSRow;                          // [128][kSRow] lo(S)
  float *s_r = reinterpret_cast<float *>(s_sl + 128 * kSRow);  // [256][kRRow] residuals

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_open();
  load_sign_masks<D>(p.signs, s_sign, tid);
  if constexpr (BM > 0) {
    if (tid < K) s_cent[tid] = p.cent[tid];
  }
  {  // S to fp16 halves, and its row norms: thread = (row, quarter of 32)
    const int row = tid >> 2, q = tid & 3;
    const float4 *src = reinterpret_cast<const float4 *>(p.S + row * D + 32 * q);
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 v = __ldg(src + i);
      uint32_t h0, l0, h1, l1;
      split2(v.x, v.y, h0, l0);
      split2(v.z, v.w, h1, l1);
      const int k = 32 * q + 4 * i;
      *reinterpret_cast<uint2 *>(s_sh + row * kSRow + k) = make_uint2(h0, h1);
      *reinterpret_cast<uint2 *>(s_sl + row * kSRow + k) = make_uint2(l0, l1);
      ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
    }
    ss += __shfl_xor_sync(dev::kFull, ss, 1);
    ss += __shfl_xor_sync(dev::kFull, ss, 2);
    if (q == 0) s_snorm[row] = sqrtf(ss);
  }
  uint32_t P[K / 2 > 0 ? K / 2 : 1];
#pragma unroll
  for (int m = 0; m + 1 < K / 2; ++m) P[m] = __float_as_uint(__ldg(p.thr + K / 2 + m));
  __syncthreads();

  const int t = tid & 1, vl = tid >> 1;
  const int g8 = lane >> 2, tig = lane & 3;
  const float *rw = s_r + (size_t)(warp * 16) * kRRow;  // this warp's 16 residual rows
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    int64_t v = tile * kMmaVPB + vl;
    const bool active = v < p.nvec;
    if (!active) v = p.nvec - 1;  // idle lanes still take part in the shuffles
    int64_t b, h, n;
    split_index(p, v, b, h, n);
    const int64_t xoff = b * p.xsb + h * p.xsh + n * p.xsn + (int64_t)t * E;
    const int64_t rec = b * p.osb + h * p.osh + n * p.osn;

    float a[E];
    uint32_t W[NWC];
    const float nrm = encode_front<D, BM, true, DT, T, E>(p, xoff, t, s_sign, s_cent, P, a, W);
    if constexpr (BM > 0) {
      if (active) store_bytes<E * BM / 8>(p.codes + rec * (D * BM / 8) + t * (E * BM / 8), W);
    }
    if (active && t == 0) p.norms[rec] = nrm;
    float rr[E];
#pragma unroll
    for (int i = 0; i < E; ++i) rr[i] = __fmul_rn(a[i], a[i]);
    const float gam = __fsqrt_rn(dev::fold_halves_sum<T, E>(rr));
    float *rv = s_r + (size_t)vl * kRRow + t * E;
#pragma unroll
    for (int i = 0; i < E; i += 4) *reinterpret_cast<float4 *>(rv + i) = make_float4(a[i], a[i + 1], a[i + 2], a[i + 3]);
    if (t == 0) {
      // 2^(4 - floor(log2 gam)): |scaled r_i| <= 32; gam = 0 -> 1
      const int ex = gam > 0.0f ? ((__float_as_int(gam) >> 23) & 0xff) - 127 : 0;
      const float sc = __int_as_float((127 + min(4 - ex, 100)) << 23);
      s_rs[vl] = sc;
      s_th[vl] = gam * sc * 0x1p-15f;
    }
    __syncwarp();

    // A fragments (16 vectors x 128 dims) as fp16 halves of the scaled rows
    uint32_t ah[8][4], al[8][4];
    const float sc0 = s_rs[warp * 16 + g8], sc1 = s_rs[warp * 16 + g8 + 8];
    const float th0 = s_th[warp * 16 + g8], th1 = s_th[warp * 16 + g8 + 8];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int c = ks * 16 + 2 * tig;
      const float2 r00 = *reinterpret_cast<const float2 *>(rw + g8 * kRRow + c);
      const float2 r10 = *reinterpret_cast<const float2 *>(rw + (g8 + 8) * kRRow + c);
      const float2 r01 = *reinterpret_cast<const float2 *>(rw + g8 * kRRow + c + 8);
      const float2 r11 = *reinterpret_cast<const float2 *>(rw + (g8 + 8) * kRRow + c + 8);
      split2(r00.x * sc0, r00.y * sc0, ah[ks][0], al[ks][0]);
      split2(r10.x * sc1, r10.y * sc1, ah[ks][1], al[ks][1]);
      split2(r01.x * sc0, r01.y * sc0, ah[ks][2], al[ks][2]);
      split2(r11.x * sc1, r11.y * sc1, ah[ks][3], al[ks][3]);
    }
    uint32_t Q[2] = {0u, 0u};
    const int v16 = lane >> 1;  // this lane's vector within the warp (front-half layout)
#pragma unroll 1
    for (int ng = 0; ng < 4; ++ng) {  // outputs [32 ng, 32 ng + 32)
      float c[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) c[j][0] = c[j][1] = c[j][2] = c[j][3] = 0.0f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int row = (4 * ng + j) * 8 + g8;
          const __half *ph = s_sh + row * kSRow + ks * 16 + 2 * tig;
          const __half *pl = s_sl + row * kSRow + ks * 16 + 2 * tig;
          const uint32_t bh0 = *reinterpret_cast<const uint32_t *>(ph);
          const uint32_t bh1 = *reinterpret_cast<const uint32_t *>(ph + 8);
          const uint32_t bl0 = *reinterpret_cast<const uint32_t *>(pl);
          const uint32_t bl1 = *reinterpret_cast<const uint32_t *>(pl + 8);
          mma_f16(c[j], ah[ks], bh0, bh1);
          mma_f16(c[j], al[ks], bh0, bh1);
          mma_f16(c[j], ah[ks], bl0, bl1);
        }
      }
      // signs: C element e of tile j is (row g8 + 8 (e >> 1), output
      // 8 (4 ng + j) + 2 tig + (e & 1))
      uint32_t bal[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int out = 8 * (4 * ng + j) + 2 * tig + (e & 1);
          const int rl = g8 + 8 * (e >> 1);
          const float z = c[j][e];
          bool pos = z >= 0.0f;
          if (!(fabsf(z) > (e >> 1 ? th1 : th0) * s_snorm[out])) pos = qjl_recheck(p.S + out * D, rw + rl * kRRow);
          bal[j][e] = __ballot_sync(dev::kFull, pos);
        }
      }
      // lane (v16, t) keeps outputs [64 t, 64 t + 64): groups 2t and 2t + 1
      if ((ng >> 1) == t) {
        const int e0 = v16 < 8 ? 0 : 2, sh = 4 * (v16 & 7);
        uint32_t word = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t ev = (bal[j][e0] >> sh) & 0xfu, od = (bal[j][e0 + 1] >> sh) & 0xfu;
          word |= (spread4(ev) | (spread4(od) << 1)) << (8 * j);
        }
        Q[ng & 1] = word;
      }
    }
    if (active) {
      store_bytes<8>(p.qjl + rec * (D / 8) + t * 8, Q);
      if (t == 0) p.rnorms[rec] = gam;
    }
    // keep the block's warps in step (they run the same long straight-line
    // code, which then stays in the instruction cache); also orders this
    // warp's residual-row reads before the next tile's writes
    __syncthreads();
  }
  pdl_close(p.pdl);
}

// A launch, with programmatic stream serialization when pdl is set.
template <typename K, typename... Args>
cudaError_t launch_maybe_pdl(K kern, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <int BM, int DT>
cudaError_t run_prod_mma(const EncParams &p, cudaStream_t s) {
  auto kern = encode_prod_mma_kernel<BM, DT>;
  const size_t smem = enc_mma_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t ntiles = (p.nvec + kMmaVPB - 1) / kMmaVPB;
  const int64_t grid = ntiles < decode_ctas() ? ntiles : decode_ctas();
  e = launch_maybe_pdl(kern, dim3((unsigned)grid), dim3(kMmaThreads), smem, s, p.pdl, p, ntiles);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
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
  p.pdl = a.pdl;
  p.div32 = p.nvec < ((int64_t)1 << 31) && a.N > 0 && a.H > 0;
  p.mN = p.mH = 0u;
  p.sN = p.sH = 0;
  if (p.div32) {
    magic31(a.N, p.mN, p.sN);
    magic31(a.H, p.mH, p.sH);
  }
  if constexpr (PROD && D == 128 && EE == 64) return run_prod_mma<BM, DT>(p, s);
  const size_t smem = enc_smem_bytes<D, PROD, EE>();
  auto kern = encode_kernel<D, BM, PROD, DT, EE>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t blocks = (p.nvec + Sh::VPB - 1) / Sh::VPB;
  const cudaError_t e = launch_maybe_pdl(kern, dim3((unsigned)blocks), dim3(kEncThreads), smem, s, p.pdl, p);
  if (e != cudaSuccess) return e;
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

bool encode_supported(int d, int bm, bool prod, int dtype, bool dense) {
  if (dense) return d >= 8 && d <= 256 && d % 8 == 0 && bm >= (prod ? 0 : 1) && bm <= 4 && dtype >= 0 && dtype <= 2;
  return (d == 64 || d == 128 || d == 256) && bm >= (prod ? 0 : 1) && bm <= 4 && dtype >= 0 && dtype <= 2;
}

cudaError_t launch_encode(const EncodeArgs &a, cudaStream_t s) {
  if (a.B * a.H * a.N >= (int64_t)1 << 40) return cudaErrorInvalidValue;
  if (a.q.rot) return launch_encode_dense(a, s);
  switch (a.q.d) {
    case 64: return by_variant<64>(a, s);
    case 128: return by_variant<128>(a, s);
    case 256: return by_variant<256>(a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tq
