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
#include "tq_umma.cuh"

#include <cuda_fp16.h>

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
  const int32_t *chan;  // input element of each coordinate, or NULL
  int d, bm, kcb;
  bool prod;
  float *out;  // dequant
  dev::IndexSplit ix;
};

// Elements i, i + 1 (i even, the pair 8- or 4-byte aligned), widened to fp32.
__device__ __forceinline__ float2 load_pair(const void *base, int dtype, int64_t i) {
  if (dtype == TQ_F32) return __ldg(reinterpret_cast<const float2 *>(static_cast<const float *>(base) + i));
  const uint32_t w = __ldg(reinterpret_cast<const unsigned int *>(static_cast<const unsigned short *>(base) + i));
  if (dtype == TQ_BF16) return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  return make_float2(__half2float(__ushort_as_half((unsigned short)(w & 0xffffu))),
                     __half2float(__ushort_as_half((unsigned short)(w >> 16))));
}

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
  dev::split_bhn(p.ix, v, b, h, n);
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
    const float a = k < d ? load_elem(p.x, p.dtype, xoff + (p.chan ? __ldg(p.chan + k) : k)) : 0.0f;
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


// ------------------------------------------------ tensor cores (tcgen05)
//
// d = 64 or 128, TurboQuant_mse, large batches: the rotation of a tile of
// 128 vectors is the GEMM Y = X Pi^T (M = 128 vectors, N = K = d) on the
// fifth-generation tensor cores.  fp32 is carried by fp16 halves: each row
// of X is first scaled by 2^(13 - floor(log2 ||x||)) (exact; the row then
// lies within [-2^14, 2^14]) and Pi by 16 (exact), and x = hi + lo with
// hi = fp16(x), lo = fp16(x - hi), likewise Pi; the product is
// Xh Ph + Xh Pl + Xl Ph (the dropped Xl Pl is below 2^-22 of the terms),
// accumulated in fp32 in tensor memory.  u = y_scaled * fl(1 / fl(16 s n)).
// Per CTA (persistent, one per SM, 512 threads in two groups of 8 warps
// that walk alternate tiles, so one group's loads overlap the other's MMAs
// and epilogue):
//   * once: Pi's halves into shared memory in the K-major, no-swizzle
//     canonical layout (8 x 16-byte core matrices), and d TMEM columns per
//     group;
//   * per tile: the group's warps load 16 rows each (8 at a time, all loads
//     in flight first), take each row's canonical norm (fold-halves:
//     in-register stages, then shuffles), scale, split and store the halves
//     into the group's A operand -- its core matrices are 144 bytes apart
//     along K so that a warp's 2-byte stores of one row hit 32 different
//     banks;
//   * one thread issues the 3 d/16 tcgen05.mma and a tcgen05.commit to the
//     group's mbarrier; the group waits on it (bounded);
//   * the epilogue: warp w of the group reads TMEM lanes 32 (w % 4) + [0, 32)
//     (its rows) and half the d columns (w / 4), 32 at a time, scales,
//     quantizes and packs half a record per thread.

constexpr int kTcGroups = 2;        // tiles in flight per CTA
constexpr int kTcGroupWarps = 8;
constexpr int kTcThreads = kTcGroups * kTcGroupWarps * 32;
constexpr int kTcM = 128;          // vectors per tile
constexpr int kTcLboA = 144;       // bytes between K-adjacent core matrices of A
constexpr int kTcLboB = 128;

template <int D>
struct TcLayout {
  static constexpr int SBO_A = (D / 8) * kTcLboA;  // bytes between 8-row groups of A
  static constexpr int SBO_B = (D / 8) * kTcLboB;
  static constexpr int A_BYTES = (kTcM / 8) * SBO_A;
  static constexpr int B_BYTES = (D / 8) * SBO_B;
  static constexpr int oBh = 0, oBl = B_BYTES;
  // group g: A halves at oA(g), oA(g) + A_BYTES
  static constexpr int oA0 = 2 * B_BYTES;
  static constexpr int oInv = oA0 + kTcGroups * 2 * A_BYTES;  // [kTcGroups][kTcM] floats
  static constexpr int kBytes = oInv + kTcGroups * kTcM * 4;
};

template <int D, int BM, int DT>
__global__ void __launch_bounds__(kTcThreads, 1) encode_dense_tc_kernel(DenseParams p, unsigned *faults,
                                                                        int64_t ntiles) {
  using L = TcLayout<D>;
  constexpr int J = D / 32;          // elements per lane per row in the loads
  constexpr int K = 1 << BM;
  constexpr int kRows = kTcM / kTcGroupWarps;  // rows a warp loads per tile
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t s_bar[kTcGroups];
  __shared__ uint32_t s_tmem;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = warp / kTcGroupWarps, gw = warp % kTcGroupWarps;
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
  const uint32_t bar = (uint32_t)__cvta_generic_to_shared(&s_bar[grp]);
  const uint32_t oAh = (uint32_t)(L::oA0 + grp * 2 * L::A_BYTES), oAl = oAh + L::A_BYTES;
  float *s_inv = reinterpret_cast<float *>(smem + L::oInv) + grp * kTcM;

  // ---- once: TMEM columns, the mbarriers, Pi's halves (scaled by 16)
  if (warp == 0) umma::alloc(&s_tmem, (uint32_t)(kTcGroups * D));
  if (tid == 0) {
#pragma unroll
    for (int g = 0; g < kTcGroups; ++g) umma::mbar_init((uint32_t)__cvta_generic_to_shared(&s_bar[g]), 1);
  }
  for (int i = tid; i < D * D; i += kTcThreads) {
    const int n = i / D, k = i % D;
    const float v = 16.0f * __ldg(p.rot + i);
    const __half h = __float2half_rn(v);
    const __half l = __float2half_rn(v - __half2float(h));
    const uint32_t o = umma::off(n, k, L::SBO_B, kTcLboB);
    *reinterpret_cast<__half *>(smem + L::oBh + o) = h;
    *reinterpret_cast<__half *>(smem + L::oBl + o) = l;
  }
  uint32_t P[K / 2 > 0 ? K / 2 : 1];
#pragma unroll
  for (int m = 0; m + 1 < K / 2; ++m) P[m] = __float_as_uint(__ldg(p.thr + K / 2 + m));
  umma::fence_async_smem();
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = s_tmem + (uint32_t)(grp * D);
  constexpr uint32_t idesc = umma::idesc_f16(kTcM, D);
  bool dead = false;

  int64_t it = 0;
  for (int64_t tile = (int64_t)blockIdx.x * kTcGroups + grp; tile < ntiles;
       tile += (int64_t)gridDim.x * kTcGroups, ++it) {
    // ---- phase 1: rows gw * kRows + [0, kRows), in batches of 8 whose
    // loads are all in flight before the first row is used
#pragma unroll 1
    for (int rb = 0; rb < kRows; rb += 8) {
      // lane holds the element pairs (2 lane + 64 jj, + 1), jj < J / 2
      float2 xr[8][J / 2];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int64_t v = tile * kTcM + gw * kRows + rb + r;
        int64_t b, h, n;
        bhn(p, v < p.nvec ? v : 0, b, h, n);
        const int64_t xoff = b * p.xsb + h * p.xsh + n * p.xsn;  // even: the rows are 16-byte aligned
#pragma unroll
        for (int jj = 0; jj < J / 2; ++jj)
          xr[r][jj] = v < p.nvec ? load_pair(p.x, DT, xoff + 2 * lane + 64 * jj) : make_float2(0.0f, 0.0f);
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int m = gw * kRows + rb + r;
        const int64_t v = tile * kTcM + m;
        // norm: fold-halves in the canonical stage order, h = 64 in the
        // lane, h = 32 .. 2 across lanes 16 .. 1 apart, h = 1 in the lane
        float2 sq = make_float2(__fmul_rn(xr[r][0].x, xr[r][0].x), __fmul_rn(xr[r][0].y, xr[r][0].y));
        if constexpr (J / 2 == 2) {
          const float2 t = make_float2(__fmul_rn(xr[r][1].x, xr[r][1].x), __fmul_rn(xr[r][1].y, xr[r][1].y));
          dev::add_x2(sq.x, sq.y, sq.x, sq.y, t.x, t.y);
        }
#pragma unroll
        for (int hh = 16; hh >= 1; hh >>= 1) {
          const float o0 = __shfl_down_sync(dev::kFull, sq.x, hh), o1 = __shfl_down_sync(dev::kFull, sq.y, hh);
          dev::add_x2(sq.x, sq.y, sq.x, sq.y, o0, o1);
        }
        const float nrm = __fsqrt_rn(__shfl_sync(dev::kFull, __fadd_rn(sq.x, sq.y), 0));
        // 2^(13 - floor(log2 n)) for a normal n > 0, else 1
        const int ex = ((__float_as_int(nrm) >> 23) & 0xff) - 127;
        const bool normal = nrm > 0.0f && ex > -127;
        const float sc = normal ? __int_as_float((127 + 13 - ex) << 23) : 1.0f;
#pragma unroll
        for (int jj = 0; jj < J / 2; ++jj) {
          const int k = 2 * lane + 64 * jj;
          float xs0, xs1, lo0, lo1;
          dev::mul_x2(xs0, xs1, xr[r][jj].x, xr[r][jj].y, sc, sc);  // sc is a power of two: exact
          const __half2 hi = __floats2half2_rn(xs0, xs1);
          const float2 hf = __half22float2(hi);
          dev::sub_x2(lo0, lo1, xs0, xs1, hf.x, hf.y);
          const __half2 lo = __floats2half2_rn(lo0, lo1);
          const uint32_t o = umma::off(m, k, L::SBO_A, kTcLboA);  // k even: a 4-byte aligned pair
          *reinterpret_cast<__half2 *>(smem + oAh + o) = hi;
          *reinterpret_cast<__half2 *>(smem + oAl + o) = lo;
        }
        if (lane == 0) {
          s_inv[m] = normal ? __frcp_rn(__fmul_rn(16.0f * sc, nrm)) : 0.0f;
          if (v < p.nvec) {
            int64_t b, h, n;
            bhn(p, v, b, h, n);
            p.norms[b * p.osb + h * p.osh + n * p.osn] = nrm;
          }
        }
      }
    }
    umma::fence_async_smem();
    umma::fence_before();
    asm volatile("bar.sync %0, %1;\n" ::"r"(1 + grp), "r"(kTcGroupWarps * 32) : "memory");

    // ---- phase 2: Y = Xh Ph + Xh Pl + Xl Ph into the group's TMEM columns
    if (gw == 0 && lane == 0) {
      umma::fence_after();
#pragma unroll 1
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint64_t ah = umma::desc(sbase + oAh + ks * 2 * kTcLboA, kTcLboA, L::SBO_A);
        const uint64_t al = umma::desc(sbase + oAl + ks * 2 * kTcLboA, kTcLboA, L::SBO_A);
        const uint64_t bh = umma::desc(sbase + L::oBh + ks * 2 * kTcLboB, kTcLboB, L::SBO_B);
        const uint64_t bl = umma::desc(sbase + L::oBl + ks * 2 * kTcLboB, kTcLboB, L::SBO_B);
        umma::mma_f16(tmem, ah, bh, idesc, ks > 0 ? 1u : 0u);
        umma::mma_f16(tmem, ah, bl, idesc, 1u);
        umma::mma_f16(tmem, al, bh, idesc, 1u);
      }
      umma::commit(bar);
    }
    // bounded wait for the MMAs (phase parity = the group's tile count & 1)
    if (!dead) dead = !umma::mbar_wait_bounded(bar, (uint32_t)(it & 1), faults, kFaultTimeout);
    umma::fence_after();

    // ---- phase 3: warp gw reads TMEM lanes 32 (gw % 4) + [0, 32) (its
    // rows) and its share of the columns, 32 (BM words of codes) at a time
    {
      constexpr int kParts = kTcGroupWarps / 4, kCols = D / kParts;
      const int q4 = gw & 3, part = gw >> 2;
      const int m = 32 * q4 + lane;
      const int64_t v = tile * kTcM + m;
      const float inv = s_inv[m];
      uint8_t *dst = nullptr;
      if (v < p.nvec) {
        int64_t b, h, n;
        bhn(p, v, b, h, n);
        dst = p.codes + (b * p.osb + h * p.osh + n * p.osn) * (D * BM / 8) + part * (kCols * BM / 8);
      }
#pragma unroll 1
      for (int c = 0; c < kCols / 32; ++c) {
        uint32_t y[32];
        umma::ld32(tmem + ((uint32_t)(32 * q4) << 16) + (uint32_t)(part * kCols + 32 * c), y);
        umma::wait_ld();
        uint32_t W[BM];
#pragma unroll
        for (int w = 0; w < BM; ++w) W[w] = 0u;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float u = __fmul_rn(__uint_as_float(y[i]), inv);
          int idx;
          if constexpr (BM == 1) {
            idx = u > 0.0f ? 1 : 0;
          } else {
            idx = dev::quantize_sym<BM>(u, P);
          }
          dev::put_field<BM>(W, i, (uint32_t)idx);
        }
        if (dst) dev::store_words<BM>(dst + c * 4 * BM, W);
      }
    }
    umma::fence_before();
    // the group's next tile rewrites s_inv and A only after every thread of
    // the group has read them
    asm volatile("bar.sync %0, %1;\n" ::"r"(1 + grp), "r"(kTcGroupWarps * 32) : "memory");
  }
  __syncthreads();
  if (warp == 0) {
    umma::fence_after();
    umma::dealloc(s_tmem, (uint32_t)(kTcGroups * D));
  }
}

template <int D, int BM, int DT>
cudaError_t run_dense_tc(const DenseParams &p, unsigned *faults, cudaStream_t s) {
  auto kern = encode_dense_tc_kernel<D, BM, DT>;
  constexpr int smem = TcLayout<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t ntiles = (p.nvec + kTcM - 1) / kTcM;
  const int64_t pairs = (ntiles + kTcGroups - 1) / kTcGroups;
  const int64_t grid = pairs < decode_ctas() ? pairs : decode_ctas();
  kern<<<(unsigned)grid, kTcThreads, smem, s>>>(p, faults, ntiles);
  return cudaGetLastError();
}

template <int D, int DT>
cudaError_t dense_tc_bits(const DenseParams &p, unsigned *faults, cudaStream_t s) {
  switch (p.bm) {
    case 1: return run_dense_tc<D, 1, DT>(p, faults, s);
    case 2: return run_dense_tc<D, 2, DT>(p, faults, s);
    case 3: return run_dense_tc<D, 3, DT>(p, faults, s);
    case 4: return run_dense_tc<D, 4, DT>(p, faults, s);
  }
  return cudaErrorInvalidValue;
}

template <int D>
cudaError_t dense_tc_dtype(const DenseParams &p, unsigned *faults, cudaStream_t s) {
  switch (p.dtype) {
    case TQ_F32: return dense_tc_bits<D, TQ_F32>(p, faults, s);
    case TQ_BF16: return dense_tc_bits<D, TQ_BF16>(p, faults, s);
    case TQ_F16: return dense_tc_bits<D, TQ_F16>(p, faults, s);
  }
  return cudaErrorInvalidValue;
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
  p.chan = a.q.channels;
  p.d = a.q.d;
  p.bm = a.q.bm;
  p.kcb = a.q.d * a.q.bm / 8;
  p.prod = a.q.prod;
  p.ix = dev::make_index_split(p.H, p.N, p.nvec);
  // large TurboQuant_mse batches at d = 64 / 128: the rotation on tcgen05
  if (!p.prod && !p.chan && (p.d == 64 || p.d == 128) && p.nvec >= 8 * kTcM) {
    unsigned *faults = nullptr;
    cudaError_t e = fault_word(&faults);
    if (e != cudaSuccess) return e;
    return p.d == 64 ? dense_tc_dtype<64>(p, faults, s) : dense_tc_dtype<128>(p, faults, s);
  }
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
  p.ix = dev::make_index_split(p.H, p.N, p.nvec);
  const int64_t blocks = (p.nvec + kDnWarps - 1) / kDnWarps;
  dequant_dense_kernel<<<(unsigned)blocks, kDnWarps * 32, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace tq
