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
#include "tq_umma.cuh"

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
  const float nrm = __fsqrt_rn(dev::fold_halves_sumsq<T, E>(a));

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
  if constexpr (PROD) {
    // the residual subtracts from these products: scalar, so that no
    // product is fused into the subtraction
#pragma unroll
    for (int i = 0; i < E; ++i) a[i] = __fmul_rn(a[i], inv);
  } else {
    dev::scale_x2<E>(a, inv);
  }

  // quantize and pack; prod keeps the residual in a[]
#pragma unroll
  for (int w = 0; w < NWC; ++w) W[w] = 0u;
  if constexpr (BM > 0) {
#pragma unroll
    for (int i = 0; i < E; i += 2) {
      int idx[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        if constexpr (BM == 1) {
          idx[j] = a[i + j] > 0.0f ? 1 : 0;
        } else {
          idx[j] = dev::quantize_sym<BM>(a[i + j], P);
        }
        dev::put_field<BM>(W, i + j, (uint32_t)idx[j]);
      }
      if constexpr (PROD) dev::sub_x2(a[i], a[i + 1], a[i], a[i + 1], s_cent[idx[0]], s_cent[idx[1]]);
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
    const float gam = __fsqrt_rn(dev::fold_halves_sumsq<T, E>(a));
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

// ------------------------------------------------ prod, d = 128: tcgen05
//
// The QJL projection z = S r is a dense 128 x 128 contraction per vector; for
// a tile of 128 vectors it is Z = R S^T (M = N = K = 128), which runs here on
// the fifth-generation tensor cores with the accumulator in tensor memory.
// fp32 is carried by fp16 halves, x = hi + lo with hi = fp16(x),
// lo = fp16(x - hi), and Z ~ Rh Sh + Rh Sl + Rl Sh (the dropped Rl Sl is
// below 2^-22 of sum |S_ki r_i|).  Scalings that keep every half in fp16's
// normal range and leave every sign unchanged: each row of S by
// 16 / ||S_k||, each residual row by sc = 2^(4 - floor(log2 ||r||)).  The
// representation (about 3 * 2^-22 per product), the dropped term and the
// fp32 accumulation stay below 2^-17.4 sum |S_ki r_i| <= 2^-17.4 ||S_k||
// ||r||, a fifth of theta_k = 2^-15 ||S_k|| ||r||; in the scaled units the
// test is |z'_k| <= sc ||r|| 2^-11 for every k.  Such a projection (about
// three in ten thousand) is recomputed exactly: the warp re-encodes the
// vector from its input in the canonical fp32 order (four coordinates a
// lane) and forms z_k = sum_i S_ki r_i in fp32, so a stored sign can differ
// from the exact one only where an fp32 summation's sign could.
//
// Per CTA (persistent, one per SM): two groups of 8 warps, each with its own
// A operand, TMEM accumulator and mbarrier, take a tile each per round (in
// step for 16-bit inputs, out of step for fp32; see the loop).
//   * once: S's scaled halves into shared memory (the B operand, K-major, no
//     swizzle), 2 x 128 TMEM columns;
//   * front half (two lanes per vector, 64 coordinates each): norm, sign
//     flips + FWHT, scale, codes, residual, ||r||; the scaled residual's
//     halves go into the group's A operand as 16-byte core-matrix rows;
//   * one thread issues the 3 x 8 tcgen05.mma and commits to the group's
//     mbarrier; the group waits on it (bounded);
//   * epilogue: warp w of the group reads TMEM lanes 32 (w % 4) + [0, 32)
//     (one vector each) and 64 of the 128 columns; a sign bit is the fp32
//     sign of z', gathered by funnel shifts.
constexpr int kPtGroups = 2;                 // tiles in flight per CTA
constexpr int kPtGroupThreads = 256;         // 8 warps a group
constexpr int kPtThreads = kPtGroups * kPtGroupThreads;
constexpr int kPtM = 128;                    // vectors per tile
constexpr int kPtLbo = 128;                  // bytes between K-adjacent core matrices
constexpr int kPtSbo = 16 * kPtLbo;          // bytes between 8-row groups (K = 128)
constexpr int kPtOp = 16 * kPtSbo;           // one 128 x 128 fp16 operand: 32 KiB
constexpr size_t kPtSmem = (size_t)(2 + 2 * kPtGroups) * kPtOp;  // S hi, S lo, then A hi, A lo per group

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// fp16 halves of 8 consecutive values: hi into H, lo into L (as uint4 rows
// of a core matrix)
__device__ __forceinline__ void split8(const float (&x)[8], uint4 &H, uint4 &L) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    h[i] = pack_h2(x[2 * i], x[2 * i + 1]);
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h[i]));
    float d0, d1;
    dev::sub_x2(d0, d1, x[2 * i], x[2 * i + 1], f.x, f.y);
    l[i] = pack_h2(d0, d1);
  }
  H = make_uint4(h[0], h[1], h[2], h[3]);
  L = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ void group_sync(int grp) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(1 + grp), "r"(kPtGroupThreads) : "memory");
}

// The exact fp32 residual of vector v, re-encoded by the whole warp in the
// canonical order: lane l holds coordinates 4l + j.  Every step is the same
// IEEE operation on the same operands as the two-lane front half (the
// butterfly and the fold-halves sum pair the same coordinates whatever the
// layout), so r[] equals the residual the front half formed.
template <int BM, int DT>
__device__ __forceinline__ void front_warp(const EncParams &p, int64_t v, const uint32_t *s_sign, const float *s_cent,
                                           float (&r)[4], int (&idx)[4], float &nrm_out) {
  constexpr int K = 1 << BM;
  const int lane = threadIdx.x & 31;
  int64_t b, h, n;
  split_index(p, v, b, h, n);
  const int64_t xoff = b * p.xsb + h * p.xsh + n * p.xsn + 4 * lane;
  float x[4];
  if constexpr (DT == 0) {
    const float4 t = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(p.x) + xoff));
    x[0] = t.x, x[1] = t.y, x[2] = t.z, x[3] = t.w;
  } else {
    const uint2 t = __ldg(reinterpret_cast<const uint2 *>(static_cast<const unsigned short *>(p.x) + xoff));
    if constexpr (DT == 1) {
      x[0] = dev::bf16lo(t.x), x[1] = dev::bf16hi(t.x), x[2] = dev::bf16lo(t.y), x[3] = dev::bf16hi(t.y);
    } else {
      x[0] = dev::f16lo(t.x), x[1] = dev::f16hi(t.x), x[2] = dev::f16lo(t.y), x[3] = dev::f16hi(t.y);
    }
  }
  // norm: fold-halves over h = 64 .. 1 (lanes < h/4 hold the live partial sums)
  float sq[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) sq[j] = __fmul_rn(x[j], x[j]);
#pragma unroll
  for (int sh = 16; sh >= 1; sh >>= 1) {
#pragma unroll
    for (int j = 0; j < 4; ++j) sq[j] = __fadd_rn(sq[j], __shfl_down_sync(dev::kFull, sq[j], sh));
  }
  sq[0] = __fadd_rn(sq[0], sq[2]);
  sq[1] = __fadd_rn(sq[1], sq[3]);
  const float nrm = __fsqrt_rn(__shfl_sync(dev::kFull, __fadd_rn(sq[0], sq[1]), 0));
  nrm_out = nrm;
  // sign flips, then the FWHT stages h = 64 .. 1
  const uint32_t sw = s_sign[lane >> 3] >> (4 * (lane & 7));
#pragma unroll
  for (int j = 0; j < 4; ++j) x[j] = __uint_as_float(__float_as_uint(x[j]) ^ (((sw >> j) & 1u) << 31));
#pragma unroll
  for (int pl = 16; pl >= 1; pl >>= 1) {
    const bool low = (lane & pl) == 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float o = __shfl_xor_sync(dev::kFull, x[j], pl);
      x[j] = low ? __fadd_rn(x[j], o) : __fsub_rn(o, x[j]);
    }
  }
  {
    const float a0 = x[0], a1 = x[1], a2 = x[2], a3 = x[3];
    x[0] = __fadd_rn(a0, a2), x[2] = __fsub_rn(a0, a2);
    x[1] = __fadd_rn(a1, a3), x[3] = __fsub_rn(a1, a3);
    const float c0 = x[0], c1 = x[1], c2 = x[2], c3 = x[3];
    x[0] = __fadd_rn(c0, c1), x[1] = __fsub_rn(c0, c1);
    x[2] = __fadd_rn(c2, c3), x[3] = __fsub_rn(c2, c3);
  }
  const float wsc = __fmul_rn(nrm, p.sqrt_d);
  const float inv = wsc > 0.0f ? __frcp_rn(wsc) : 0.0f;
  uint32_t PP[K / 2 > 0 ? K / 2 : 1];
#pragma unroll
  for (int m = 0; m + 1 < K / 2; ++m) PP[m] = __float_as_uint(__ldg(p.thr + K / 2 + m));
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float u = __fmul_rn(x[j], inv);
    if constexpr (BM == 0) {
      r[j] = u;
      idx[j] = 0;
    } else {
      idx[j] = BM == 1 ? (u > 0.0f ? 1 : 0) : dev::quantize_sym<BM>(u, PP);
      r[j] = __fsub_rn(u, s_cent[idx[j]]);
    }
  }
}

template <int BM, int DT>
__device__ __forceinline__ void residual_exact(const EncParams &p, int64_t v, const uint32_t *s_sign, const float *s_cent,
                                               float (&r)[4]) {
  int idx[4];
  float nrm;
  front_warp<BM, DT>(p, v, s_sign, s_cent, r, idx, nrm);
}

// Small d = 128 prod batches (the one-token append of a decode step, whose
// latency sits on the step's critical path): one 128-thread CTA per vector.
// Warp 0 runs the canonical front half, four coordinates a lane (the same
// operations as every other encode path, so codes and norms are identical);
// the residual's norm is the same fold-halves sum; then thread k forms
// z_k = sum_i S_ki r_i in fp32 from the residual in shared memory, and each
// warp's ballot is one 32-bit word of the sketch.
template <int BM, int DT>
__global__ void __launch_bounds__(128) encode_prod_small_kernel(EncParams p) {
  constexpr int D = 128;
  constexpr int K = 1 << BM;
  __shared__ uint32_t s_sign[D / 32];
  __shared__ float s_cent[16];
  __shared__ __align__(16) float s_r[D];
  __shared__ int s_idx[D];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_open();
  load_sign_masks<D>(p.signs, s_sign, tid);
  if constexpr (BM > 0) {
    if (tid < K) s_cent[tid] = p.cent[tid];
  }
  __syncthreads();
  const int64_t v = blockIdx.x;
  int64_t b, h, n;
  split_index(p, v, b, h, n);
  const int64_t rec = b * p.osb + h * p.osh + n * p.osn;
  if (warp == 0) {
    float r[4];
    int idx[4];
    float nrm;
    front_warp<BM, DT>(p, v, s_sign, s_cent, r, idx, nrm);
    float sq[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) sq[j] = __fmul_rn(r[j], r[j]);
#pragma unroll
    for (int sh = 16; sh >= 1; sh >>= 1) {
#pragma unroll
      for (int j = 0; j < 4; ++j) sq[j] = __fadd_rn(sq[j], __shfl_down_sync(dev::kFull, sq[j], sh));
    }
    sq[0] = __fadd_rn(sq[0], sq[2]);
    sq[1] = __fadd_rn(sq[1], sq[3]);
    const float gam = __fsqrt_rn(__fadd_rn(sq[0], sq[1]));  // lane 0's is the canonical sum
    *reinterpret_cast<float4 *>(s_r + 4 * lane) = make_float4(r[0], r[1], r[2], r[3]);
#pragma unroll
    for (int j = 0; j < 4; ++j) s_idx[4 * lane + j] = idx[j];
    if (lane == 0) {
      p.norms[rec] = nrm;
      p.rnorms[rec] = gam;
    }
  }
  __syncthreads();
  // codes: thread w < 4 BM builds word w of the record's 128 BM-bit stream
  if constexpr (BM > 0) {
    if (tid < 4 * BM) {
      const int lo = 32 * tid;
      uint32_t word = 0u;
      for (int i = lo / BM; i * BM < lo + 32; ++i) {
        const int pos = i * BM - lo;
        const uint32_t f = (uint32_t)s_idx[i];
        word |= pos >= 0 ? f << pos : f >> -pos;
      }
      reinterpret_cast<uint32_t *>(p.codes + rec * (D * BM / 8))[tid] = word;
    }
  }
  // the sketch: z_k = sum_i S_ki r_i, bit k = (z_k >= 0)
  {
    const float4 *Sk = reinterpret_cast<const float4 *>(p.S + (size_t)tid * D);
    const float4 *r4 = reinterpret_cast<const float4 *>(s_r);
    float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
#pragma unroll 8
    for (int i = 0; i < D / 4; ++i) {
      const float4 a = __ldg(Sk + i), c = r4[i];
      z0 = fmaf(a.x, c.x, z0);
      z1 = fmaf(a.y, c.y, z1);
      z2 = fmaf(a.z, c.z, z2);
      z3 = fmaf(a.w, c.w, z3);
    }
    const float z = (z0 + z1) + (z2 + z3);
    const unsigned bits = __ballot_sync(dev::kFull, z >= 0.0f);
    if (lane == 0) reinterpret_cast<uint32_t *>(p.qjl + rec * (D / 8))[warp] = bits;
  }
  pdl_close(p.pdl);
}

// The warp's exact recheck of one 32-column chunk: lanes in `need` hold a
// vector (v0 + lane) with near-zero projections k0 + i for the bits i of
// their `mine`; each such sign is recomputed from the exact residual.
// Returns the calling lane's corrected sign word.
template <int BM, int DT>
__device__ __noinline__ uint32_t recheck(const EncParams &p, int64_t v0, int k0, uint32_t need, uint32_t mine,
                                         uint32_t q, const uint32_t *s_sign, const float *s_cent) {
  const int lane = threadIdx.x & 31;
  while (need) {
    const int src = __ffs(need) - 1;
    need &= need - 1;
    uint32_t mask = __shfl_sync(dev::kFull, mine, src);
    float r[4];
    residual_exact<BM, DT>(p, v0 + src, s_sign, s_cent, r);
    while (mask) {
      const int i = __ffs(mask) - 1;
      mask &= mask - 1;
      const float4 sk = __ldg(reinterpret_cast<const float4 *>(p.S + (k0 + i) * 128) + lane);
      float z = fmaf(sk.x, r[0], fmaf(sk.y, r[1], fmaf(sk.z, r[2], sk.w * r[3])));
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) z += __shfl_xor_sync(dev::kFull, z, o);
      if (lane == src) q = (q & ~(1u << i)) | ((z >= 0.0f ? 1u : 0u) << i);
    }
  }
  return q;
}

template <int BM, int DT>
__global__ void __launch_bounds__(kPtThreads, 1) encode_prod_tc_kernel(EncParams p, unsigned *faults, int64_t ntiles) {
  constexpr int D = 128, T = 2, E = 64;
  constexpr int K = 1 << BM;
  constexpr int NWC = BM > 0 ? (E * BM + 31) / 32 : 1;
  constexpr uint32_t kIdesc = umma::idesc_f16(kPtM, D);
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ uint32_t s_sign[D / 32];
  __shared__ float s_cent[16];
  __shared__ float s_th[kPtGroups][2][kPtM];  // per tile parity: sc ||r|| 2^-11
  __shared__ __align__(8) uint64_t s_bar[kPtGroups];
  __shared__ uint32_t s_tmem;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = warp / 8, gt = tid % kPtGroupThreads, gw = warp % 8;
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
  const uint32_t bar = (uint32_t)__cvta_generic_to_shared(&s_bar[grp]);
  pdl_open();

  // ---- once: TMEM, mbarriers, S's scaled halves, codebook, sign masks
  if (warp == 0) umma::alloc(&s_tmem, kPtGroups * D);
  if (tid == 0) {
#pragma unroll
    for (int g = 0; g < kPtGroups; ++g) umma::mbar_init((uint32_t)__cvta_generic_to_shared(&s_bar[g]), 1);
  }
  load_sign_masks<D>(p.signs, s_sign, tid);
  if constexpr (BM > 0) {
    if (tid < K) s_cent[tid] = p.cent[tid];
  }
  {  // thread = (row of S, quarter of 32 columns)
    const int row = tid >> 2, q = tid & 3;
    const float4 *src = reinterpret_cast<const float4 *>(p.S + row * D + 32 * q);
    float v[32];
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 t = __ldg(src + i);
      v[4 * i] = t.x, v[4 * i + 1] = t.y, v[4 * i + 2] = t.z, v[4 * i + 3] = t.w;
      ss = fmaf(t.x, t.x, fmaf(t.y, t.y, fmaf(t.z, t.z, fmaf(t.w, t.w, ss))));
    }
    ss += __shfl_xor_sync(dev::kFull, ss, 1);
    ss += __shfl_xor_sync(dev::kFull, ss, 2);
    const float f = ss > 0.0f ? 16.0f / sqrtf(ss) : 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = v[8 * c + i] * f;
      uint4 H, L;
      split8(x, H, L);
      const uint32_t o = umma::off(row, 32 * q + 8 * c, kPtSbo, kPtLbo);
      *reinterpret_cast<uint4 *>(smem + o) = H;
      *reinterpret_cast<uint4 *>(smem + kPtOp + o) = L;
    }
  }
  uint32_t P[K / 2 > 0 ? K / 2 : 1];
#pragma unroll
  for (int m = 0; m + 1 < K / 2; ++m) P[m] = __float_as_uint(__ldg(p.thr + K / 2 + m));
  umma::fence_async_smem();
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = s_tmem + (uint32_t)(grp * D);
  const uint32_t oAh = (uint32_t)((2 + 2 * grp) * kPtOp), oAl = oAh + kPtOp;
  const int t = gt & 1, vl = gt >> 1;
  bool dead = false;

  // one tile per group a round.  With 16-bit inputs the two groups take
  // their tiles in step (one CTA barrier a round), so that the warps run the
  // same part of the long straight-line code together; with fp32 inputs
  // (twice the load latency per tile) they run out of step, one group's
  // loads overlapping the other's MMAs and epilogue.  Each measured faster
  // than the other choice on 2^20 vectors (bf16 513 vs 543 us, fp32 579 vs
  // 650 us).
  const int64_t stride = (int64_t)gridDim.x * kPtGroups;
  const int64_t rounds = (ntiles - (int64_t)blockIdx.x * kPtGroups + stride - 1) / stride;
  for (int64_t it = 0; it < rounds; ++it) {
    const int64_t tile = (int64_t)blockIdx.x * kPtGroups + grp + it * stride;
    const int par = (int)(it & 1);
    if constexpr (DT != 0) __syncthreads();
    if (tile >= ntiles) continue;
    // ---- front half: vector vl of the tile, coordinates [64 t, 64 t + 64)
    {
      int64_t v = tile * kPtM + vl;
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
      const float gam = __fsqrt_rn(dev::fold_halves_sumsq<T, E>(a));
      // 2^(4 - floor(log2 gam)): |scaled r_i| <= 32; gam = 0 -> 1
      const int ex = gam > 0.0f ? ((__float_as_int(gam) >> 23) & 0xff) - 127 : 0;
      const float sc = __int_as_float((127 + min(4 - ex, 100)) << 23);
      if (t == 0) {
        s_th[grp][par][vl] = gam * sc * 0x1p-11f;
        if (active) {
          p.norms[rec] = nrm;
          p.rnorms[rec] = gam;
        }
      }
#pragma unroll
      for (int c = 0; c < E / 8; ++c) {
        float x[8];
#pragma unroll
        for (int i = 0; i < 8; i += 2)  // sc is a power of two: exact products
          dev::mul_x2(x[i], x[i + 1], a[8 * c + i], a[8 * c + i + 1], sc, sc);
        uint4 H, L;
        split8(x, H, L);
        const uint32_t o = umma::off(vl, t * E + 8 * c, kPtSbo, kPtLbo);
        *reinterpret_cast<uint4 *>(smem + oAh + o) = H;
        *reinterpret_cast<uint4 *>(smem + oAl + o) = L;
      }
    }
    umma::fence_async_smem();
    umma::fence_before();
    group_sync(grp);

    // ---- Z' = Rh Sh + Rh Sl + Rl Sh into the group's TMEM columns
    if (gt == 0) {
      umma::fence_after();
#pragma unroll 1
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t k0 = (uint32_t)(ks * 2 * kPtLbo);
        const uint64_t ah = umma::desc(sbase + oAh + k0, kPtLbo, kPtSbo);
        const uint64_t al = umma::desc(sbase + oAl + k0, kPtLbo, kPtSbo);
        const uint64_t bh = umma::desc(sbase + k0, kPtLbo, kPtSbo);
        const uint64_t bl = umma::desc(sbase + kPtOp + k0, kPtLbo, kPtSbo);
        umma::mma_f16(tmem, ah, bh, kIdesc, ks > 0 ? 1u : 0u);
        umma::mma_f16(tmem, ah, bl, kIdesc, 1u);
        umma::mma_f16(tmem, al, bh, kIdesc, 1u);
      }
      umma::commit(bar);
    }
    if (!dead) dead = !umma::mbar_wait_bounded(bar, (uint32_t)par, faults, kFaultTimeout);
    umma::fence_after();

    // ---- epilogue: vector m, projections [64 hf, 64 hf + 64)
    {
      const int q4 = gw & 3, hf = gw >> 2;
      const int m = 32 * q4 + lane;
      const int64_t v = tile * kPtM + m;
      const float th = s_th[grp][par][m];
      uint32_t Q[2];
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t y[32];
        umma::ld32(tmem + ((uint32_t)(32 * q4) << 16) + (uint32_t)(hf * 64 + 32 * c), y);
        umma::wait_ld();
        uint32_t neg = 0u;  // bit i: the sign bit of z'_i
        bool near = false;
#pragma unroll
        for (int i = 31; i >= 0; --i) {
          neg = __funnelshift_l(y[i], neg, 1);
          near |= !(fabsf(__uint_as_float(y[i])) > th);
        }
        uint32_t q = ~neg;
        // exact recheck of the projections too close to zero to trust
        uint32_t need = __ballot_sync(dev::kFull, near && v < p.nvec);
        if (need) {
          uint32_t mine = 0u;
#pragma unroll
          for (int i = 0; i < 32; ++i) mine |= (!(fabsf(__uint_as_float(y[i])) > th) ? 1u : 0u) << i;
          q = recheck<BM, DT>(p, tile * kPtM + 32 * q4, hf * 64 + 32 * c, need, mine, q, s_sign, s_cent);
        }
        Q[c] = q;
      }
      if (v < p.nvec) {
        int64_t b, h, n;
        split_index(p, v, b, h, n);
        const int64_t rec = b * p.osb + h * p.osh + n * p.osn;
        store_bytes<8>(p.qjl + rec * (D / 8) + hf * 8, Q);
      }
    }
    umma::fence_before();
  }
  __syncthreads();
  if (warp == 0) {
    umma::fence_after();
    umma::dealloc(s_tmem, kPtGroups * D);
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
cudaError_t run_prod_tc(const EncParams &p, cudaStream_t s) {
  auto kern = encode_prod_tc_kernel<BM, DT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPtSmem);
  if (e != cudaSuccess) return e;
  unsigned *faults = nullptr;
  e = fault_word(&faults);
  if (e != cudaSuccess) return e;
  const int64_t ntiles = (p.nvec + kPtM - 1) / kPtM;
  const int64_t pairs = (ntiles + kPtGroups - 1) / kPtGroups;
  const int64_t grid = pairs < decode_ctas() ? pairs : decode_ctas();
  e = launch_maybe_pdl(kern, dim3((unsigned)grid), dim3(kPtThreads), kPtSmem, s, p.pdl, p, faults, ntiles);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

EncParams make_params(const EncodeArgs &a) {
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
  return p;
}

template <int BM, int DT>
cudaError_t run_prod_small(const EncodeArgs &a, cudaStream_t s) {
  const EncParams p = make_params(a);
  const cudaError_t e = launch_maybe_pdl(encode_prod_small_kernel<BM, DT>, dim3((unsigned)p.nvec), dim3(128), 0, s,
                                         p.pdl, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D, int BM, bool PROD, int DT, int EE>
cudaError_t run_e(const EncodeArgs &a, cudaStream_t s) {
  using Sh = Shape<D, EE>;
  const EncParams p = make_params(a);
  if constexpr (PROD && D == 128 && EE == 64) return run_prod_tc<BM, DT>(p, s);
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
// the E = 16 layout: four times more lanes per vector, shorter chains; d =
// 128 prod batches take one CTA per vector.
template <int D, int BM, bool PROD, int DT>
cudaError_t run(const EncodeArgs &a, cudaStream_t s) {
  const int64_t nvec = a.B * a.H * a.N;
  if (nvec <= 148 * (kEncThreads / Shape<D, 64>::T)) {
    if constexpr (PROD && D == 128) {
      return run_prod_small<BM, DT>(a, s);
    } else {
      return run_e<D, BM, PROD, DT, 16>(a, s);
    }
  }
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
