// Device helpers shared by the TurboQuant kernels (sm_100a).
//
// Vector layout inside a kernel: a d-vector is held by T consecutive lanes,
// lane t of the group owning the contiguous block of E = d/T elements
// [t*E, t*E + E) in registers.  Butterfly stages whose stride h is >= E pair
// lanes t and t ^ (h/E); the rest stay in registers.  Every add, subtract,
// multiply and square root below is IEEE round-to-nearest with no
// contraction, so the encode reproduces the canonical fp32 procedure bit for
// bit whatever T is.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tq {
namespace dev {

constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------- loading

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float f16lo(uint32_t w) {
  return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu)));
}
__device__ __forceinline__ float f16hi(uint32_t w) {
  return __half2float(__ushort_as_half((unsigned short)(w >> 16)));
}

// E contiguous elements of dtype DT (0 f32, 1 bf16, 2 f16) from a 16-byte
// aligned address, widened exactly to fp32.
template <int DT, int E>
__device__ __forceinline__ void load_block(const void *p, float (&v)[E]) {
  if constexpr (DT == 0) {
    const float4 *q = reinterpret_cast<const float4 *>(p);
#pragma unroll
    for (int i = 0; i < E / 4; ++i) {
      const float4 t = __ldg(q + i);
      v[4 * i + 0] = t.x;
      v[4 * i + 1] = t.y;
      v[4 * i + 2] = t.z;
      v[4 * i + 3] = t.w;
    }
  } else {
    const uint4 *q = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int i = 0; i < E / 8; ++i) {
      const uint4 t = __ldg(q + i);
      const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if constexpr (DT == 1) {
          v[8 * i + 2 * k] = bf16lo(w[k]);
          v[8 * i + 2 * k + 1] = bf16hi(w[k]);
        } else {
          v[8 * i + 2 * k] = f16lo(w[k]);
          v[8 * i + 2 * k + 1] = f16hi(w[k]);
        }
      }
    }
  }
}

// ------------------------------------------------- paired fp32 arithmetic

// Two independent fp32 operations in one packed f32x2 instruction (sm_100).
// Each half rounds to nearest exactly as the scalar add.rn / sub.rn / mul.rn
// does (no flush to zero), so a paired step gives the same bits as the two
// scalar ones -- with one exception the compiler makes: a packed product
// whose result feeds a packed sum can be fused into a packed multiply-add,
// which skips the product's rounding (measured on sm_100a).  So a product
// that an addition or subtraction consumes is formed with scalar mul.rn;
// packed products feed only comparisons, conversions and stores, or are
// exact (scaling by a power of two).
__device__ __forceinline__ void add_x2(float &d0, float &d1, float a0, float a1, float b0, float b1) {
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " add.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void sub_x2(float &d0, float &d1, float a0, float a1, float b0, float b1) {
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " sub.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void mul_x2(float &d0, float &d1, float a0, float a1, float b0, float b1) {
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " mul.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// d = a * b + c, each half one fused multiply-add (rounded once).
__device__ __forceinline__ void fma_x2(float &d0, float &d1, float a0, float a1, float b0, float b1, float c0,
                                       float c1) {
  asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " mov.b64 rc, {%6, %7};\n fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// a_i <- fl(a_i * s) over an even-length array, in pairs (for products that
// no addition consumes).
template <int E>
__device__ __forceinline__ void scale_x2(float (&a)[E], float s) {
  static_assert(E % 2 == 0, "pairs");
#pragma unroll
  for (int i = 0; i < E; i += 2) mul_x2(a[i], a[i + 1], a[i], a[i + 1], s, s);
}

// ------------------------------------------------------------ butterflies

// One cross-lane FWHT stage: the lane whose group index has bit P clear holds
// a (gets a+b), its partner holds b (gets a-b).  Both are one addition,
// fl(o + a) on the low lane and fl(o + (-b)) = fl(o - b) on the high one.
template <int E>
__device__ __forceinline__ void fwht_cross(float (&a)[E], int P, bool low) {
  const uint32_t neg = low ? 0u : 0x80000000u;
  if constexpr (E % 2 == 0) {
#pragma unroll
    for (int i = 0; i < E; i += 2) {
      const float o0 = __shfl_xor_sync(kFull, a[i], P), o1 = __shfl_xor_sync(kFull, a[i + 1], P);
      add_x2(a[i], a[i + 1], o0, o1, __uint_as_float(__float_as_uint(a[i]) ^ neg),
             __uint_as_float(__float_as_uint(a[i + 1]) ^ neg));
    }
  } else {
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float o = __shfl_xor_sync(kFull, a[i], P);
      a[i] = __fadd_rn(o, __uint_as_float(__float_as_uint(a[i]) ^ neg));
    }
  }
}

// In-register FWHT stages h = E/2, ..., 1.  Stages h >= 2 take the
// butterflies of elements i and i + 1 together (paired instructions); the
// last stage pairs the two halves of a pair and stays scalar.
template <int E>
__device__ __forceinline__ void fwht_local(float (&a)[E]) {
#pragma unroll
  for (int h = E / 2; h >= 2; h >>= 1) {
#pragma unroll
    for (int i = 0; i < E; i += 2) {
      if ((i & h) == 0) {
        const float x0 = a[i], x1 = a[i + 1], y0 = a[i + h], y1 = a[i + h + 1];
        add_x2(a[i], a[i + 1], x0, x1, y0, y1);
        sub_x2(a[i + h], a[i + h + 1], x0, x1, y0, y1);
      }
    }
  }
  if constexpr (E >= 2) {
#pragma unroll
    for (int i = 0; i < E; i += 2) {
      const float x = a[i], y = a[i + 1];
      a[i] = __fadd_rn(x, y);
      a[i + 1] = __fsub_rn(x, y);
    }
  }
}

// Full unnormalised FWHT of a d = T*E vector, stages h = d/2 .. 1.
template <int T, int E>
__device__ __forceinline__ void fwht(float (&a)[E], int t) {
#pragma unroll
  for (int P = T / 2; P >= 1; P >>= 1) fwht_cross<E>(a, P, (t & P) == 0);
  fwht_local<E>(a);
}

// Fold-halves sum of a[] over the d = T*E vector: for h = d/2, .., 1,
// a_i <- fl(a_i + a_{i+h}) for i < h.  Destroys a[]; every lane of the group
// returns the same value (fl(x+y) = fl(y+x)).
template <int T, int E>
__device__ __forceinline__ float fold_halves_sum(float (&a)[E]) {
  if constexpr (E % 2 == 0) {
#pragma unroll
    for (int P = T / 2; P >= 1; P >>= 1) {
#pragma unroll
      for (int i = 0; i < E; i += 2) {
        const float o0 = __shfl_xor_sync(kFull, a[i], P), o1 = __shfl_xor_sync(kFull, a[i + 1], P);
        add_x2(a[i], a[i + 1], a[i], a[i + 1], o0, o1);
      }
    }
#pragma unroll
    for (int h = E / 2; h >= 2; h >>= 1) {
#pragma unroll
      for (int i = 0; i < h; i += 2) add_x2(a[i], a[i + 1], a[i], a[i + 1], a[i + h], a[i + h + 1]);
    }
    return __fadd_rn(a[0], a[1]);
  } else {
#pragma unroll
    for (int P = T / 2; P >= 1; P >>= 1) {
#pragma unroll
      for (int i = 0; i < E; ++i) a[i] = __fadd_rn(a[i], __shfl_xor_sync(kFull, a[i], P));
    }
#pragma unroll
    for (int h = E / 2; h >= 1; h >>= 1) {
#pragma unroll
      for (int i = 0; i < h; ++i) a[i] = __fadd_rn(a[i], a[i + h]);
    }
    return a[0];
  }
}

// The same fold-halves sum of the squares fl(a_i * a_i), without a second
// array: after the cross-lane stages, element i after in-register stage h is
// W(i, h) = W(i, 2h) + W(i + h, 2h), with W(i, E) the squared element; the
// recursion visits the leaves depth first, so only log2(E) partial sums are
// live at a time.  Bit-identical to fold_halves_sum of the squares.
template <int T, int E, int I, int H>
__device__ __forceinline__ float fold_sumsq_node(const float (&a)[E]) {
  if constexpr (H == E) {
    float s = __fmul_rn(a[I], a[I]);
#pragma unroll
    for (int P = T / 2; P >= 1; P >>= 1) s = __fadd_rn(s, __shfl_xor_sync(kFull, s, P));
    return s;
  } else {
    const float lo = fold_sumsq_node<T, E, I, 2 * H>(a);
    return __fadd_rn(lo, fold_sumsq_node<T, E, I + H, 2 * H>(a));
  }
}

// The same recursion on the pairs (W(I, H), W(I + 1, H)) for even I and
// H >= 2, one paired instruction per step.
template <int T, int E, int I, int H>
__device__ __forceinline__ void fold_sumsq_node2(const float (&a)[E], float &w0, float &w1) {
  if constexpr (H == E) {
    // scalar squares: a packed product whose one use is a packed sum may be
    // fused into it, which would skip the product's rounding
    w0 = __fmul_rn(a[I], a[I]);
    w1 = __fmul_rn(a[I + 1], a[I + 1]);
#pragma unroll
    for (int P = T / 2; P >= 1; P >>= 1) {
      const float o0 = __shfl_xor_sync(kFull, w0, P), o1 = __shfl_xor_sync(kFull, w1, P);
      add_x2(w0, w1, w0, w1, o0, o1);
    }
  } else {
    float l0, l1, h0, h1;
    fold_sumsq_node2<T, E, I, 2 * H>(a, l0, l1);
    fold_sumsq_node2<T, E, I + H, 2 * H>(a, h0, h1);
    add_x2(w0, w1, l0, l1, h0, h1);
  }
}

template <int T, int E>
__device__ __forceinline__ float fold_halves_sumsq(const float (&a)[E]) {
  if constexpr (E % 2 == 0) {
    float w0, w1;
    fold_sumsq_node2<T, E, 0, 2>(a, w0, w1);
    return __fadd_rn(w0, w1);
  } else {
    return fold_sumsq_node<T, E, 0, 1>(a);
  }
}

// ------------------------------------------------------- index splitting

// Vector index v -> (b, h, n) of a [B][H][N] batch.  When every index fits
// in 31 bits the divisions are multiply-shifts, q = (x * m) >> (31 + l) with
// l = ceil(log2 divisor), m = floor(2^(31+l) / divisor) + 1, exact for
// x < 2^31 (Granlund and Montgomery, "Division by invariant integers using
// multiplication"); else 64-bit division.
struct IndexSplit {
  int64_t H, N;
  bool div32;
  uint32_t mN, mH;
  int sN, sH;
};

inline void magic31_div(int64_t d, uint32_t &m, int &s) {
  int l = 0;
  while (((int64_t)1 << l) < d) ++l;
  m = (uint32_t)((((uint64_t)1 << (31 + l)) / (uint64_t)d) + 1);
  s = 31 + l;
}

inline IndexSplit make_index_split(int64_t H, int64_t N, int64_t nvec) {
  IndexSplit x{};
  x.H = H;
  x.N = N;
  x.div32 = nvec < ((int64_t)1 << 31) && N > 0 && H > 0;
  if (x.div32) {
    magic31_div(N, x.mN, x.sN);
    magic31_div(H, x.mH, x.sH);
  }
  return x;
}

__device__ __forceinline__ void split_bhn(const IndexSplit &x, int64_t v, int64_t &b, int64_t &h, int64_t &n) {
  if (x.div32) {
    const uint32_t u = (uint32_t)v;
    const uint32_t bh = (uint32_t)(((uint64_t)u * x.mN) >> x.sN);
    const uint32_t hb = (uint32_t)(((uint64_t)bh * x.mH) >> x.sH);
    n = u - bh * (uint32_t)x.N;
    h = bh - hb * (uint32_t)x.H;
    b = hb;
  } else {
    n = v % x.N;
    const int64_t bh = v / x.N;
    h = bh % x.H;
    b = bh / x.H;
  }
}

// -------------------------------------------------------------- quantize

// idx = #{j : u > t_j} for an antisymmetric codebook with K = 2^BM levels,
// given the bit patterns P[0..K/2-2] of the positive thresholds
// t_{K/2}..t_{K-2} (the middle threshold is 0).  For u > 0,
// idx = K/2 + #{m : P_m < |u|}; for u <= 0 (and NaN), idx = K/2 - 1 -
// #{m : P_m <= |u|}.  Non-negative floats order like their bit patterns, so
// both counts are #{m : P_m < A} with A = bits(|u|) + [u <= 0], found by an
// unrolled binary search over the sorted P.
template <int BM>
__device__ __forceinline__ int quantize_sym(float u, const uint32_t (&P)[(1 << BM) / 2]) {
  constexpr int K = 1 << BM;
  const bool pos = u > 0.0f;
  const uint32_t A = (__float_as_uint(u) & 0x7fffffffu) + (pos ? 0u : 1u);
  int k = 0;
  if constexpr (BM == 2) {
    k = A > P[0] ? 1 : 0;
  } else if constexpr (BM == 3) {
    k = A > P[1] ? 2 : 0;
    const uint32_t t = k ? P[2] : P[0];
    k += A > t ? 1 : 0;
  } else if constexpr (BM == 4) {
    k = A > P[3] ? 4 : 0;
    const uint32_t t1 = k ? P[5] : P[1];
    k += A > t1 ? 2 : 0;
    const uint32_t lo = (k & 2) ? P[2] : P[0];
    const uint32_t hi = (k & 2) ? P[6] : P[4];
    const uint32_t t2 = (k & 4) ? hi : lo;
    k += A > t2 ? 1 : 0;
  }
  // K/2 + k for u > 0, K/2 - 1 - k otherwise (k < K/2)
  return k ^ (pos ? K / 2 : K / 2 - 1);
}

// ----------------------------------------------------------- bit packing

// Places the BM-bit field of element j (of E) into the LSB-first bitstream
// held in W[] (E*BM/32 words).
template <int BM, int NW>
__device__ __forceinline__ void put_field(uint32_t (&W)[NW], int j, uint32_t v) {
  const int p = j * BM;
  const int w = p >> 5, s = p & 31;
  W[w] |= v << s;
  if (s + BM > 32) W[w + 1] |= v >> (32 - s);
}

template <int BM, int NW>
__device__ __forceinline__ uint32_t get_field(const uint32_t (&W)[NW], int j) {
  const int p = j * BM;
  const int w = p >> 5, s = p & 31;
  uint32_t v = W[w] >> s;
  if (s + BM > 32) v |= W[w + 1] << (32 - s);
  return v & ((1u << BM) - 1u);
}

// Stores NW words to a 4*NW-byte aligned destination with the widest
// vector access the size allows.
template <int NW>
__device__ __forceinline__ void store_words(void *dst, const uint32_t (&W)[NW]) {
  if constexpr (NW % 4 == 0) {
    uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int i = 0; i < NW / 4; ++i) d[i] = make_uint4(W[4 * i], W[4 * i + 1], W[4 * i + 2], W[4 * i + 3]);
  } else if constexpr (NW % 2 == 0) {
    uint2 *d = reinterpret_cast<uint2 *>(dst);
#pragma unroll
    for (int i = 0; i < NW / 2; ++i) d[i] = make_uint2(W[2 * i], W[2 * i + 1]);
  } else {
    uint32_t *d = reinterpret_cast<uint32_t *>(dst);
#pragma unroll
    for (int i = 0; i < NW; ++i) d[i] = W[i];
  }
}

template <int NW>
__device__ __forceinline__ void load_words(const void *src, uint32_t (&W)[NW]) {
  if constexpr (NW % 4 == 0) {
    const uint4 *s = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int i = 0; i < NW / 4; ++i) {
      const uint4 t = __ldg(s + i);
      W[4 * i] = t.x;
      W[4 * i + 1] = t.y;
      W[4 * i + 2] = t.z;
      W[4 * i + 3] = t.w;
    }
  } else if constexpr (NW % 2 == 0) {
    const uint2 *s = reinterpret_cast<const uint2 *>(src);
#pragma unroll
    for (int i = 0; i < NW / 2; ++i) {
      const uint2 t = __ldg(s + i);
      W[2 * i] = t.x;
      W[2 * i + 1] = t.y;
    }
  } else {
    const uint32_t *s = reinterpret_cast<const uint32_t *>(src);
#pragma unroll
    for (int i = 0; i < NW; ++i) W[i] = __ldg(s + i);
  }
}

}  // namespace dev
}  // namespace tq
