// Host half of the TurboQuant C ABI: codebook fitting, seeded parameters,
// argument validation and dispatch to the CUDA launchers.
//
// Codebook: Lloyd-Max scalar quantizer for the coordinate law after a random
// rotation, N(0, 1/d) by default or the exact C (1-x^2)^((d-3)/2)
// ("TurboQuant của Google: nén KV cache 6 lần", sections "Trick đầu tiên"
// and "Lloyd-Max quantizer: chia bucket đúng chỗ"; "The Distortion
// Guarantee", section "The Gap").  Procedure (the pages give none): Lloyd's
// alternation in double -- thresholds at midpoints, centroids at conditional
// means -- from levels equally spaced on [-2, 2] (N(0,1) units) until no
// centroid moves by 1e-15; the exact law starts from the Gaussian levels
// / sqrt(d), integrates every cell with 128-node Gauss-Legendre and stops at
// 1e-16.  The levels are made exactly antisymmetric, the Gaussian ones are
// divided by sqrt(d), thresholds are double midpoints, and everything is
// rounded once to fp32.
//
// Seeded parameters: SplitMix64 (Steele, Lea, Flood 2014), output k of seed s
// = mix(s + (k+1) * 0x9E3779B97F4A7C15); sign i is -1 when bit 63 of output i
// is set; S entry e comes from Box-Muller on outputs 2(e/2), 2(e/2)+1 mapped
// to (o >> 11) 2^-53, the first replaced by 1-u, cos for even e and sin for
// odd e, in double, rounded to fp32.

#include "../../include/tq.h"
#include "tq_internal.h"

#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

namespace {

thread_local std::string g_last_error;

tq_status fail(tq_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
tq_status fail(tq_status s, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

tq_status cuda_fail(cudaError_t e, const char *what) {
  return fail(TQ_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---------------------------------------------------------------- codebook

const double kSqrt2 = 1.4142135623730951;
const double kInvSqrt2Pi = 0.3989422804014327;

double phi(double x) {
  if (std::isinf(x)) return 0.0;
  return kInvSqrt2Pi * std::exp(-0.5 * x * x);
}

double upper_tail(double x) {
  if (x == INFINITY) return 0.0;
  if (x == -INFINITY) return 1.0;
  return 0.5 * std::erfc(x / kSqrt2);
}

double mass(double a, double b) {
  if (a >= 0.0) return upper_tail(a) - upper_tail(b);
  if (b <= 0.0) return upper_tail(-b) - upper_tail(-a);
  return 1.0 - upper_tail(b) - upper_tail(-a);
}

void antisymmetrize(std::vector<double> &c) {
  const int K = (int)c.size();
  std::vector<double> o(c);
  for (int i = 0; i < K; ++i) c[i] = 0.5 * (o[i] - o[K - 1 - i]);
}

std::vector<double> lloyd_max_gauss(int K) {
  std::vector<double> c(K), t(K + 1), nc(K);
  for (int i = 0; i < K; ++i) c[i] = -2.0 + 4.0 * i / (K - 1);
  for (int sweep = 0; sweep < 200000; ++sweep) {
    t[0] = -INFINITY;
    t[K] = INFINITY;
    for (int i = 0; i + 1 < K; ++i) t[i + 1] = 0.5 * (c[i] + c[i + 1]);
    double delta = 0.0;
    for (int i = 0; i < K; ++i) {
      nc[i] = (phi(t[i]) - phi(t[i + 1])) / mass(t[i], t[i + 1]);
      delta = std::fmax(delta, std::fabs(nc[i] - c[i]));
    }
    c = nc;
    if (delta < 1e-15) break;
  }
  antisymmetrize(c);
  return c;
}

// Gauss-Legendre nodes/weights on [-1, 1] by Newton on the Legendre
// recurrence (Golub-Welsch would do as well; any accurate rule works).
void gauss_legendre(int n, std::vector<double> &x, std::vector<double> &w) {
  x.assign(n, 0.0);
  w.assign(n, 0.0);
  for (int i = 0; i < n; ++i) {
    double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));
    double dp = 1.0;
    for (int it = 0; it < 100; ++it) {
      double p0 = 1.0, p1 = z;
      for (int k = 2; k <= n; ++k) {
        double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
        p0 = p1;
        p1 = p2;
      }
      dp = n * (z * p1 - p0) / (z * z - 1.0);
      double dz = p1 / dp;
      z -= dz;
      if (std::fabs(dz) < 1e-16) break;
    }
    x[n - 1 - i] = z;
    w[n - 1 - i] = 2.0 / ((1.0 - z * z) * dp * dp);
  }
}

std::vector<double> lloyd_max_beta(int K, int d) {
  std::vector<double> gx, gw;
  gauss_legendre(128, gx, gw);
  std::vector<double> c = lloyd_max_gauss(K), t(K + 1), nc(K);
  const double sd = std::sqrt((double)d);
  for (int i = 0; i < K; ++i) c[i] /= sd;
  const double ex = 0.5 * (d - 3);
  for (int sweep = 0; sweep < 200000; ++sweep) {
    t[0] = -1.0;
    t[K] = 1.0;
    for (int i = 0; i + 1 < K; ++i) t[i + 1] = 0.5 * (c[i] + c[i + 1]);
    double delta = 0.0;
    for (int i = 0; i < K; ++i) {
      const double half = 0.5 * (t[i + 1] - t[i]);
      const double mid = 0.5 * (t[i + 1] + t[i]);
      double m0 = 0.0, m1 = 0.0;
      for (size_t g = 0; g < gx.size(); ++g) {
        const double xx = mid + half * gx[g];
        const double f = std::exp(ex * std::log1p(-xx * xx));
        m0 += gw[g] * f;
        m1 += gw[g] * xx * f;
      }
      nc[i] = (half * m1) / (half * m0);
      delta = std::fmax(delta, std::fabs(nc[i] - c[i]));
    }
    c = nc;
    if (delta < 1e-16) break;
  }
  antisymmetrize(c);
  return c;
}

// ------------------------------------------------------------- SplitMix64

uint64_t splitmix64(uint64_t seed, uint64_t k) {
  uint64_t z = seed + (k + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

double unit53(uint64_t v) { return (double)(v >> 11) * (1.0 / 9007199254740992.0); }

// Entry e of the seeded d x d Gaussian matrix (row-major), float64: the
// Box-Muller pair of outputs 2(e/2), 2(e/2)+1, cos for even e, sin for odd.
void gaussian_f64(uint64_t seed, int d, std::vector<double> &g) {
  const int64_t n = (int64_t)d * d;
  g.assign((size_t)n, 0.0);
  for (int64_t p = 0; p < (n + 1) / 2; ++p) {
    const double u1 = 1.0 - unit53(splitmix64(seed, 2 * p));
    const double u2 = unit53(splitmix64(seed, 2 * p + 1));
    const double r = std::sqrt(-2.0 * std::log(u1));
    const double ang = 2.0 * M_PI * u2;
    g[2 * p] = r * std::cos(ang);
    if (2 * p + 1 < n) g[2 * p + 1] = r * std::sin(ang);
  }
}

// Q of G = Q R (Householder, in double) with the columns' signs chosen so
// that diag(R) > 0; Q written row-major into q.
void haar_q(std::vector<double> a, int d, std::vector<double> &q) {
  // a: row-major d x d, overwritten by R; reflectors kept in v[k]
  std::vector<std::vector<double>> v((size_t)d);
  for (int k = 0; k < d; ++k) {
    double nx = 0.0;
    for (int i = k; i < d; ++i) nx += a[(size_t)i * d + k] * a[(size_t)i * d + k];
    nx = std::sqrt(nx);
    std::vector<double> w((size_t)(d - k), 0.0);
    const double x0 = a[(size_t)k * d + k];
    const double alpha = x0 >= 0.0 ? -nx : nx;
    for (int i = k; i < d; ++i) w[(size_t)(i - k)] = a[(size_t)i * d + k];
    w[0] -= alpha;
    double nw = 0.0;
    for (double t : w) nw += t * t;
    nw = std::sqrt(nw);
    if (nw > 0.0) {
      for (double &t : w) t /= nw;
      for (int j = k; j < d; ++j) {  // A[k:, j] -= 2 w (w . A[k:, j])
        double dot = 0.0;
        for (int i = k; i < d; ++i) dot += w[(size_t)(i - k)] * a[(size_t)i * d + j];
        for (int i = k; i < d; ++i) a[(size_t)i * d + j] -= 2.0 * w[(size_t)(i - k)] * dot;
      }
    }
    v[(size_t)k] = w;
  }
  // Q = H_0 H_1 ... H_{d-1} I, applied right to left
  q.assign((size_t)d * d, 0.0);
  for (int i = 0; i < d; ++i) q[(size_t)i * d + i] = 1.0;
  for (int k = d - 1; k >= 0; --k) {
    const std::vector<double> &w = v[(size_t)k];
    for (int j = 0; j < d; ++j) {
      double dot = 0.0;
      for (int i = k; i < d; ++i) dot += w[(size_t)(i - k)] * q[(size_t)i * d + j];
      for (int i = k; i < d; ++i) q[(size_t)i * d + j] -= 2.0 * w[(size_t)(i - k)] * dot;
    }
  }
  // sign fix: column j times sign(R_jj)
  for (int j = 0; j < d; ++j) {
    if (a[(size_t)j * d + j] < 0.0)
      for (int i = 0; i < d; ++i) q[(size_t)i * d + j] = -q[(size_t)i * d + j];
  }
}

// ------------------------------------------------------------- validation

bool valid_d(int d) { return d == 64 || d == 128 || d == 256; }
// the dense rotation takes any multiple of 8 up to 256
bool valid_dense_d(int d) { return d >= 8 && d <= 256 && d % 8 == 0; }

tq_status check_quantizer(const tq_quantizer *q, const char *name, tq::QuantParams *out) {
  if (!q) return fail(TQ_EINVAL, "%s: quantizer is NULL", name);
  if (q->rotation != TQ_ROT_HADAMARD && q->rotation != TQ_ROT_DENSE)
    return fail(TQ_EINVAL, "%s: rotation=%d", name, q->rotation);
  const bool dense = q->rotation == TQ_ROT_DENSE;
  if (dense ? !valid_dense_d(q->d) : !valid_d(q->d))
    return fail(TQ_EINVAL, "%s: d=%d (expected %s)", name, q->d,
                dense ? "a multiple of 8 from 8 to 256" : "64, 128 or 256");
  if (q->bits < 1 || q->bits > 4) return fail(TQ_EINVAL, "%s: bits=%d (expected 1..4)", name, q->bits);
  if (q->variant != TQ_MSE && q->variant != TQ_PROD)
    return fail(TQ_EINVAL, "%s: variant=%d", name, q->variant);
  if (dense && (!q->rot || (uintptr_t)q->rot % 16))
    return fail(TQ_EINVAL, "%s: dense rotation without a 16-byte aligned rot matrix", name);
  const bool prod = q->variant == TQ_PROD;
  const int bm = prod ? q->bits - 1 : q->bits;
  if (bm > 0 && (!q->centroids || !q->thresholds))
    return fail(TQ_EINVAL, "%s: centroids/thresholds are NULL", name);
  if (!dense && !q->signs) return fail(TQ_EINVAL, "%s: signs are NULL", name);
  if (prod && !q->qjl_S) return fail(TQ_EINVAL, "%s: prod quantizer without qjl_S", name);
  if (prod && (uintptr_t)q->qjl_S % 16) return fail(TQ_EINVAL, "%s: qjl_S not 16-byte aligned", name);
  out->d = q->d;
  out->bm = bm;
  out->prod = prod;
  out->centroids = q->centroids;
  out->thresholds = q->thresholds;
  out->signs = q->signs;
  out->S = q->qjl_S;
  out->rot = dense ? q->rot : nullptr;
  if (q->channels && !dense)
    return fail(TQ_EUNSUPPORTED, "%s: a channel list needs the dense rotation", name);
  out->channels = q->channels;
  out->sqrt_d = (float)std::sqrt((double)q->d);
  return TQ_OK;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

size_t dtype_size(int dt) { return dt == TQ_F32 ? 4 : 2; }

tq_status check_view(const tq_cache_view *v, const tq::QuantParams &q, const char *name,
                     bool need_all, tq::CacheView *out) {
  if (!v) return fail(TQ_EINVAL, "%s: cache view is NULL", name);
  if (need_all) {
    if (q.bm > 0 && !v->codes) return fail(TQ_EINVAL, "%s: codes are NULL", name);
    if (!v->norms) return fail(TQ_EINVAL, "%s: norms are NULL", name);
    if (q.prod && (!v->qjl || !v->rnorms)) return fail(TQ_EINVAL, "%s: prod needs qjl and rnorms", name);
  }
  if (v->codes && !aligned(v->codes, 16)) return fail(TQ_EINVAL, "%s: codes not 16-byte aligned", name);
  if (v->qjl && !aligned(v->qjl, 16)) return fail(TQ_EINVAL, "%s: qjl not 16-byte aligned", name);
  if (v->norms && !aligned(v->norms, 4)) return fail(TQ_EINVAL, "%s: norms not 4-byte aligned", name);
  if (v->rnorms && !aligned(v->rnorms, 4)) return fail(TQ_EINVAL, "%s: rnorms not 4-byte aligned", name);
  if (v->stride_b < 0 || v->stride_h < 0 || v->stride_n < 0)
    return fail(TQ_EINVAL, "%s: negative stride", name);
  out->codes = v->codes;
  out->qjl = q.prod ? v->qjl : nullptr;
  out->norms = v->norms;
  out->rnorms = q.prod ? v->rnorms : nullptr;
  out->sb = v->stride_b;
  out->sh = v->stride_h;
  out->sn = v->stride_n;
  return TQ_OK;
}

int g_num_sms = 0;

int num_sms() {
  if (g_num_sms > 0) return g_num_sms;
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
    g_num_sms = n;
  else
    g_num_sms = 148;
  return g_num_sms;
}

}  // namespace

// ------------------------------------------------------------ split policy

namespace tq {

// One persistent CTA per SM of the current device.
int decode_ctas() { return std::min(num_sms(), 1024); }

}  // namespace tq

// -------------------------------------------------------------------- ABI

extern "C" {

tq_status tq_make_codebook(int32_t d, int32_t bits_mse, tq_codebook_dist dist, float *centroids,
                           float *thresholds) {
  if (!valid_dense_d(d)) return fail(TQ_EINVAL, "tq_make_codebook: d=%d", d);
  if (bits_mse < 1 || bits_mse > 4) return fail(TQ_EINVAL, "tq_make_codebook: bits_mse=%d", bits_mse);
  if (!centroids || !thresholds) return fail(TQ_EINVAL, "tq_make_codebook: NULL output");
  const int K = 1 << bits_mse;
  std::vector<double> c;
  if (dist == TQ_CB_GAUSS) {
    c = lloyd_max_gauss(K);
    const double sd = std::sqrt((double)d);
    for (double &v : c) v /= sd;
  } else if (dist == TQ_CB_BETA) {
    c = lloyd_max_beta(K, d);
  } else {
    return fail(TQ_EINVAL, "tq_make_codebook: dist=%d", (int)dist);
  }
  for (int i = 0; i < K; ++i) centroids[i] = (float)c[i];
  for (int i = 0; i + 1 < K; ++i) thresholds[i] = (float)(0.5 * (c[i] + c[i + 1]));
  return TQ_OK;
}

tq_status tq_make_signs(uint64_t seed, int32_t d, int8_t *signs) {
  if (!valid_dense_d(d)) return fail(TQ_EINVAL, "tq_make_signs: d=%d", d);
  if (!signs) return fail(TQ_EINVAL, "tq_make_signs: NULL output");
  for (int i = 0; i < d; ++i) signs[i] = (splitmix64(seed, (uint64_t)i) >> 63) ? -1 : 1;
  return TQ_OK;
}

tq_status tq_make_qjl(uint64_t seed, int32_t d, float *S) {
  if (!valid_dense_d(d)) return fail(TQ_EINVAL, "tq_make_qjl: d=%d", d);
  if (!S) return fail(TQ_EINVAL, "tq_make_qjl: NULL output");
  std::vector<double> g;
  gaussian_f64(seed, d, g);
  for (size_t i = 0; i < g.size(); ++i) S[i] = (float)g[i];
  return TQ_OK;
}

tq_status tq_make_rotation(uint64_t seed, int32_t d, float *rot) {
  if (!valid_dense_d(d)) return fail(TQ_EINVAL, "tq_make_rotation: d=%d (expected a multiple of 8 from 8 to 256)", d);
  if (!rot) return fail(TQ_EINVAL, "tq_make_rotation: NULL output");
  std::vector<double> g, q;
  gaussian_f64(seed, d, g);
  haar_q(g, d, q);
  for (size_t i = 0; i < q.size(); ++i) rot[i] = (float)q[i];
  return TQ_OK;
}

size_t tq_code_bytes(int32_t d, int32_t bits, int32_t variant) {
  const int bm = variant == TQ_PROD ? bits - 1 : bits;
  return bm > 0 ? (size_t)d * bm / 8 : 0;
}

size_t tq_qjl_bytes(int32_t d, int32_t variant) { return variant == TQ_PROD ? (size_t)d / 8 : 0; }

}  // extern "C"

namespace {

// Validates an encode call into *a.  TQ_OK with *empty set means there is
// nothing to launch.
tq_status prepare_encode(const char *name, const char *out_name, const tq_quantizer *q, const void *x,
                         tq_dtype x_dtype, int64_t B, int64_t H, int64_t N, int64_t x_stride_b, int64_t x_stride_h,
                         int64_t x_stride_n, const tq_cache_view *out, tq::EncodeArgs *a, bool *empty) {
  *a = tq::EncodeArgs{};
  *empty = false;
  tq_status st = check_quantizer(q, name, &a->q);
  if (st != TQ_OK) return st;
  if (x_dtype != TQ_F32 && x_dtype != TQ_BF16 && x_dtype != TQ_F16)
    return fail(TQ_EINVAL, "%s: x_dtype=%d", name, (int)x_dtype);
  if (B < 0 || H < 0 || N < 0) return fail(TQ_EINVAL, "%s: negative size", name);
  if (x_stride_b < 0 || x_stride_h < 0 || x_stride_n < 0) return fail(TQ_EINVAL, "%s: negative stride", name);
  if (B == 0 || H == 0 || N == 0) {
    *empty = true;
    return TQ_OK;
  }
  st = check_view(out, a->q, (std::string(name) + "(" + out_name + ")").c_str(), true, &a->out);
  if (st != TQ_OK) return st;
  if (!x) return fail(TQ_EINVAL, "%s: x is NULL", name);
  const size_t es = dtype_size(x_dtype);
  if (!aligned(x, 16) || (x_stride_b * es) % 16 || (x_stride_h * es) % 16 || (x_stride_n * es) % 16)
    return fail(TQ_EINVAL, "%s: x and its strides must be 16-byte aligned", name);
  if (!tq::encode_supported(a->q.d, a->q.bm, a->q.prod, x_dtype, a->q.rot != nullptr))
    return fail(TQ_EUNSUPPORTED, "%s: d=%d b_m=%d prod=%d dtype=%d not built", name, a->q.d, a->q.bm,
                (int)a->q.prod, (int)x_dtype);
  a->x = x;
  a->dtype = x_dtype;
  a->B = B;
  a->H = H;
  a->N = N;
  a->xsb = x_stride_b;
  a->xsh = x_stride_h;
  a->xsn = x_stride_n;
  return TQ_OK;
}

}  // namespace

extern "C" {

tq_status tq_encode(const tq_quantizer *q, const void *x, tq_dtype x_dtype, int64_t B, int64_t H,
                    int64_t N, int64_t x_stride_b, int64_t x_stride_h, int64_t x_stride_n,
                    const tq_cache_view *out, tq_stream_t stream) {
  tq::EncodeArgs a;
  bool empty;
  const tq_status st =
      prepare_encode("tq_encode", "out", q, x, x_dtype, B, H, N, x_stride_b, x_stride_h, x_stride_n, out, &a, &empty);
  if (st != TQ_OK || empty) return st;
  cudaError_t e = tq::launch_encode(a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tq_encode launch");
  return TQ_OK;
}

tq_status tq_dequant(const tq_quantizer *q, const tq_cache_view *in, int64_t B, int64_t H, int64_t N,
                     float *out, tq_stream_t stream) {
  tq::DequantArgs a{};
  tq_status st = check_quantizer(q, "tq_dequant", &a.q);
  if (st != TQ_OK) return st;
  if (B < 0 || H < 0 || N < 0) return fail(TQ_EINVAL, "tq_dequant: negative size");
  if (B == 0 || H == 0 || N == 0) return TQ_OK;
  st = check_view(in, a.q, "tq_dequant(in)", true, &a.in);
  if (st != TQ_OK) return st;
  if (!out || !aligned(out, 16)) return fail(TQ_EINVAL, "tq_dequant: out NULL or not 16-byte aligned");
  if (!tq::dequant_supported(a.q.d, a.q.bm, a.q.prod, a.q.rot != nullptr))
    return fail(TQ_EUNSUPPORTED, "tq_dequant: d=%d b_m=%d prod=%d rotation=%s not built", a.q.d, a.q.bm,
                (int)a.q.prod, a.q.rot ? "dense" : "hadamard");
  a.B = B;
  a.H = H;
  a.N = N;
  a.out = out;
  cudaError_t e = tq::launch_dequant(a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tq_dequant launch");
  return TQ_OK;
}

size_t tq_decode_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int64_t seq_len, int32_t d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || seq_len <= 0 || Hq % Hkv || !valid_dense_d(d)) return 0;
  // enough for either decode path (the quantizers are not arguments): the
  // tensor-core split kernel (d = 128, sized for TurboQuant_prod keys) and
  // the CUDA-core path (any d, prod values)
  size_t fl = tq::general_decode_workspace_floats(B, Hq, Hkv, seq_len, d);
  if (d == 128) fl = std::max(fl, tq::decode_workspace_floats(B, Hq, Hkv, true, tq::decode_ctas()));
  return fl * sizeof(float);
}

}  // extern "C"

namespace {

// Validates a decode call into *a.  TQ_OK with *empty set means there is
// nothing to launch (B == 0 or Hq == 0).
tq_status prepare_decode(const char *name, const tq_quantizer *kq, const tq_quantizer *vq, const void *q,
                         tq_dtype q_dtype, int32_t B, int32_t Hq, int32_t Hkv, int64_t seq_len,
                         const int32_t *seq_lens, const tq_cache_view *k, const tq_cache_view *v,
                         float softmax_scale, float *out, float *scores_out, void *workspace,
                         size_t workspace_bytes, tq::DecodeArgs *a, bool *empty) {
  *a = tq::DecodeArgs{};
  *empty = false;
  const std::string nm(name);
  tq_status st = check_quantizer(kq, (nm + "(kq)").c_str(), &a->kq);
  if (st != TQ_OK) return st;
  st = check_quantizer(vq, (nm + "(vq)").c_str(), &a->vq);
  if (st != TQ_OK) return st;
  if (a->kq.d != a->vq.d) return fail(TQ_EINVAL, "%s: K d=%d but V d=%d", name, a->kq.d, a->vq.d);
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16 && q_dtype != TQ_F16)
    return fail(TQ_EINVAL, "%s: q_dtype=%d", name, (int)q_dtype);
  if (B < 0 || Hq < 0 || Hkv < 0 || seq_len < 0) return fail(TQ_EINVAL, "%s: negative size", name);
  if (seq_len > INT32_MAX) return fail(TQ_EINVAL, "%s: seq_len=%lld is 2^31 or more", name, (long long)seq_len);
  if (Hkv == 0 || Hq % Hkv) return fail(TQ_EINVAL, "%s: Hq=%d not a multiple of Hkv=%d", name, Hq, Hkv);
  if (!std::isfinite(softmax_scale)) return fail(TQ_EINVAL, "%s: softmax_scale not finite", name);
  if (B == 0 || Hq == 0) {
    *empty = true;
    return TQ_OK;
  }
  st = check_view(k, a->kq, (nm + "(k)").c_str(), seq_len > 0, &a->k);
  if (st != TQ_OK) return st;
  st = check_view(v, a->vq, (nm + "(v)").c_str(), seq_len > 0, &a->v);
  if (st != TQ_OK) return st;
  if (!q || !aligned(q, 16)) return fail(TQ_EINVAL, "%s: q NULL or not 16-byte aligned", name);
  if (!out || !aligned(out, 16)) return fail(TQ_EINVAL, "%s: out NULL or not 16-byte aligned", name);
  if (scores_out && !aligned(scores_out, 4)) return fail(TQ_EINVAL, "%s: scores_out misaligned", name);
  if (!tq::decode_supported(a->kq.d, a->kq.bm, a->kq.prod, a->vq.bm, a->vq.prod, a->kq.rot != nullptr,
                            a->vq.rot != nullptr))
    return fail(TQ_EUNSUPPORTED, "%s: d=%d K b_m=%d prod=%d V b_m=%d not built", name, a->kq.d, a->kq.bm,
                (int)a->kq.prod, a->vq.bm);
  a->q = q;
  a->q_dtype = q_dtype;
  a->B = B;
  a->Hq = Hq;
  a->Hkv = Hkv;
  a->seq_len = seq_len;
  a->seq_lens = seq_lens;
  a->scale = softmax_scale;
  a->out = out;
  a->scores = scores_out;
  if (seq_len > 0) {
    const size_t need = tq_decode_workspace_bytes(B, Hq, Hkv, seq_len, a->kq.d);
    if (workspace_bytes < need || !workspace || !aligned(workspace, 16))
      return fail(TQ_EWORKSPACE, "%s: workspace %zu bytes, need %zu (16-byte aligned)", name, workspace_bytes,
                  need);
    a->splits = tq::decode_ctas();
    a->ws = (float *)workspace;
  }
  return TQ_OK;
}

}  // namespace

extern "C" {

tq_status tq_decode_attention(const tq_quantizer *kq, const tq_quantizer *vq, const void *q,
                              tq_dtype q_dtype, int32_t B, int32_t Hq, int32_t Hkv, int64_t seq_len,
                              const int32_t *seq_lens, const tq_cache_view *k,
                              const tq_cache_view *v, float softmax_scale, float *out,
                              float *scores_out, void *workspace, size_t workspace_bytes,
                              tq_stream_t stream) {
  tq::DecodeArgs a;
  bool empty;
  const tq_status st = prepare_decode("tq_decode_attention", kq, vq, q, q_dtype, B, Hq, Hkv, seq_len, seq_lens, k,
                                      v, softmax_scale, out, scores_out, workspace, workspace_bytes, &a, &empty);
  if (st != TQ_OK || empty) return st;
  cudaError_t e = tq::launch_decode(a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tq_decode_attention launch");
  return TQ_OK;
}

tq_status tq_append_decode_attention(const tq_quantizer *kq, const tq_quantizer *vq, const void *k_new,
                                     const void *v_new, tq_dtype kv_dtype, int64_t new_stride_b,
                                     int64_t new_stride_h, const tq_cache_view *k_tail,
                                     const tq_cache_view *v_tail, const void *q, tq_dtype q_dtype, int32_t B,
                                     int32_t Hq, int32_t Hkv, int64_t seq_len, const int32_t *seq_lens,
                                     const tq_cache_view *k, const tq_cache_view *v, float softmax_scale,
                                     float *out, float *scores_out, void *workspace, size_t workspace_bytes,
                                     tq_stream_t stream) {
  const char *name = "tq_append_decode_attention";
  tq::EncodeArgs ak, av;
  tq::DecodeArgs ad;
  bool ek, ev, ed;
  tq_status st = prepare_encode(name, "k_tail", kq, k_new, kv_dtype, B, Hkv, 1, new_stride_b, new_stride_h, 0,
                                k_tail, &ak, &ek);
  if (st != TQ_OK) return st;
  st = prepare_encode(name, "v_tail", vq, v_new, kv_dtype, B, Hkv, 1, new_stride_b, new_stride_h, 0, v_tail, &av,
                      &ev);
  if (st != TQ_OK) return st;
  st = prepare_decode(name, kq, vq, q, q_dtype, B, Hq, Hkv, seq_len, seq_lens, k, v, softmax_scale, out,
                      scores_out, workspace, workspace_bytes, &ad, &ed);
  if (st != TQ_OK) return st;
  if (ed) return TQ_OK;  // B == 0 or Hq == 0: no tokens and no heads
  // K append (an ordinary launch: everything before it in the stream has
  // finished), then the V append, the prep kernel and the split kernel, each
  // allowed to start while the one before it runs.  The V append and prep
  // only read inputs that existed before the chain began; each keeps one
  // thread waiting for its predecessor, so the chain completes in order and
  // the split kernel reads the cache only after both appends.
  const cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  if (!ek) e = tq::launch_encode(ak, s);
  if (e == cudaSuccess && !ev) {
    av.pdl = !ek;
    e = tq::launch_encode(av, s);
  }
  if (e == cudaSuccess) {
    ad.prep_pdl = !(ek && ev);
    e = tq::launch_decode(ad, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "tq_append_decode_attention launch");
  return TQ_OK;
}

tq_status tq_decode_attention_noalloc(const tq_quantizer *kq, const tq_quantizer *vq, const void *q,
                                      tq_dtype q_dtype, int32_t B, int32_t Hq, int32_t Hkv, int64_t seq_len,
                                      const int32_t *seq_lens, const tq_cache_view *k, const tq_cache_view *v,
                                      float softmax_scale, float *out, float *scores_out, tq_stream_t stream) {
  const size_t need = tq_decode_workspace_bytes(B, Hq, Hkv, seq_len, kq ? kq->d : 0);
  if (need > (size_t)TQ_NOALLOC_SCRATCH_BYTES)
    return fail(TQ_EWORKSPACE,
                "tq_decode_attention_noalloc: B=%d Hq=%d Hkv=%d seq_len=%lld needs %zu bytes of scratch, "
                "more than the %zu-byte static scratch; use tq_decode_attention with a caller workspace",
                B, Hq, Hkv, (long long)seq_len, need, (size_t)TQ_NOALLOC_SCRATCH_BYTES);
  void *ws = nullptr;
  if (need > 0) {
    const cudaError_t e = tq::static_scratch(&ws);
    if (e != cudaSuccess) return cuda_fail(e, "tq_decode_attention_noalloc: scratch lookup");
  }
  return tq_decode_attention(kq, vq, q, q_dtype, B, Hq, Hkv, seq_len, seq_lens, k, v, softmax_scale, out,
                             scores_out, ws, need, stream);
}

size_t tq_decode_split_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int64_t seq_len, int32_t d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || seq_len <= 0 || Hq % Hkv || d < 16 || d > 256 || d % 8) return 0;
  return tq::general_decode_workspace_floats(B, Hq, Hkv, seq_len, d) * sizeof(float);
}

tq_status tq_decode_attention_split(const tq_quantizer kq[2], const tq_quantizer vq[2], const void *q,
                                    tq_dtype q_dtype, int32_t B, int32_t Hq, int32_t Hkv, int64_t seq_len,
                                    const int32_t *seq_lens, const tq_cache_view k[2], const tq_cache_view v[2],
                                    float softmax_scale, float *out, void *workspace, size_t workspace_bytes,
                                    tq_stream_t stream) {
  const char *name = "tq_decode_attention_split";
  if (!kq || !vq || !k || !v) return fail(TQ_EINVAL, "%s: NULL quantizer or cache array", name);
  tq::SplitDecodeArgs a{};
  for (int g = 0; g < 2; ++g) {
    tq_status st = check_quantizer(&kq[g], name, &a.kq[g]);
    if (st != TQ_OK) return st;
    st = check_quantizer(&vq[g], name, &a.vq[g]);
    if (st != TQ_OK) return st;
    if (!a.kq[g].rot || !a.kq[g].channels || !a.vq[g].rot || !a.vq[g].channels)
      return fail(TQ_EINVAL, "%s: every group needs the dense rotation and a channel list", name);
    if (a.vq[g].prod && a.vq[g].bm == 0 && !a.vq[g].S) return fail(TQ_EINVAL, "%s: prod value group without S", name);
  }
  const int d = a.kq[0].d + a.kq[1].d;
  if (a.vq[0].d + a.vq[1].d != d) return fail(TQ_EINVAL, "%s: key groups cover %d channels, value groups %d", name, d,
                                               a.vq[0].d + a.vq[1].d);
  if (d > 256) return fail(TQ_EINVAL, "%s: d=%d (at most 256)", name, d);
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16 && q_dtype != TQ_F16)
    return fail(TQ_EINVAL, "%s: q_dtype=%d", name, (int)q_dtype);
  if (B < 0 || Hq < 0 || Hkv <= 0 || seq_len < 0 || Hq % Hkv) return fail(TQ_EINVAL, "%s: bad sizes", name);
  if (!std::isfinite(softmax_scale)) return fail(TQ_EINVAL, "%s: softmax_scale not finite", name);
  if (B == 0 || Hq == 0) return TQ_OK;
  if (!q || !out) return fail(TQ_EINVAL, "%s: q or out is NULL", name);
  for (int g = 0; g < 2; ++g) {
    tq_status st = check_view(&k[g], a.kq[g], name, seq_len > 0, &a.k[g]);
    if (st != TQ_OK) return st;
    st = check_view(&v[g], a.vq[g], name, seq_len > 0, &a.v[g]);
    if (st != TQ_OK) return st;
  }
  if (seq_len == 0) {
    const cudaError_t e = cudaMemsetAsync(out, 0, (size_t)B * Hq * d * sizeof(float), (cudaStream_t)stream);
    return e == cudaSuccess ? TQ_OK : cuda_fail(e, name);
  }
  const size_t need = tq_decode_split_workspace_bytes(B, Hq, Hkv, seq_len, d);
  if (workspace_bytes < need || !workspace || !aligned(workspace, 16))
    return fail(TQ_EWORKSPACE, "%s: workspace %zu bytes, need %zu", name, workspace_bytes, need);
  a.q = q;
  a.q_dtype = q_dtype;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.seq_len = seq_len;
  a.seq_lens = seq_lens;
  a.scale = softmax_scale;
  a.out = out;
  a.ws = (float *)workspace;
  const cudaError_t e = tq::launch_decode_split(a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tq_decode_attention_split launch");
  return TQ_OK;
}

size_t tq_search_workspace_bytes(int32_t n_q, int64_t n_db, int32_t d) {
  if (n_q <= 0 || n_db <= 0 || n_db >= ((int64_t)1 << 31) || d != 128) return 0;
  return tq::search_workspace_floats(n_q, n_db) * sizeof(float);
}

tq_status tq_search_topk(const tq_quantizer *q, const tq_cache_view *db, int64_t n_db, const void *queries,
                         tq_dtype q_dtype, int32_t n_q, int32_t k, float *top_scores, int64_t *top_index,
                         void *workspace, size_t workspace_bytes, tq_stream_t stream) {
  const char *name = "tq_search_topk";
  tq::SearchArgs a{};
  tq_status st = check_quantizer(q, "tq_search_topk(q)", &a.q);
  if (st != TQ_OK) return st;
  if (a.q.d != 128) return fail(TQ_EUNSUPPORTED, "%s: d=%d (only 128 is built)", name, a.q.d);
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16 && q_dtype != TQ_F16)
    return fail(TQ_EINVAL, "%s: q_dtype=%d", name, (int)q_dtype);
  if (n_q < 0 || n_db < 0) return fail(TQ_EINVAL, "%s: negative size", name);
  if (n_db >= ((int64_t)1 << 31)) return fail(TQ_EINVAL, "%s: n_db=%lld is 2^31 or more", name, (long long)n_db);
  if (k < 1 || k > 32) return fail(TQ_EINVAL, "%s: k=%d (expected 1..32)", name, k);
  if (n_q == 0) return TQ_OK;
  if (!top_scores || !top_index || !aligned(top_scores, 4) || !aligned(top_index, 8))
    return fail(TQ_EINVAL, "%s: outputs NULL or misaligned", name);
  if (!queries || !aligned(queries, 16)) return fail(TQ_EINVAL, "%s: queries NULL or not 16-byte aligned", name);
  if (n_db == 0) {
    // nothing to rank: every entry is empty
    std::vector<float> v((size_t)n_q * k, -INFINITY);
    std::vector<int64_t> ix((size_t)n_q * k, -1);
    cudaError_t e = cudaMemcpyAsync(top_scores, v.data(), v.size() * sizeof(float), cudaMemcpyHostToDevice,
                                    (cudaStream_t)stream);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(top_index, ix.data(), ix.size() * sizeof(int64_t), cudaMemcpyHostToDevice,
                          (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, name);
    return TQ_OK;
  }
  st = check_view(db, a.q, "tq_search_topk(db)", true, &a.db);
  if (st != TQ_OK) return st;
  const size_t need = tq_search_workspace_bytes(n_q, n_db, 128);
  if (workspace_bytes < need || !workspace || !aligned(workspace, 16))
    return fail(TQ_EWORKSPACE, "%s: workspace %zu bytes, need %zu (16-byte aligned)", name, workspace_bytes, need);
  a.n_db = n_db;
  a.queries = queries;
  a.q_dtype = q_dtype;
  a.nq = n_q;
  a.k = k;
  a.top_v = top_scores;
  a.top_i = top_index;
  a.ws = (float *)workspace;
  const cudaError_t e = tq::launch_search(a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tq_search_topk launch");
  return TQ_OK;
}

tq_status tq_check(tq_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tq_check");
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "tq_check");
  unsigned faults = 0;
  e = tq::take_device_faults(&faults);
  if (e != cudaSuccess) return cuda_fail(e, "tq_check: reading the device fault word");
  if (faults & tq::kFaultTimeout)
    return fail(TQ_ETIMEOUT, "tq_check: a kernel gave up a bounded wait on data that never arrived; "
                             "its outputs are not valid");
  if (faults & tq::kFaultSmemLayout)
    return fail(TQ_ECUDA, "tq_check: a decode kernel found its shared-memory layout invalid and wrote nothing");
  return TQ_OK;
}

const char *tq_status_string(tq_status s) {
  switch (s) {
    case TQ_OK: return "TQ_OK";
    case TQ_EINVAL: return "TQ_EINVAL";
    case TQ_EUNSUPPORTED: return "TQ_EUNSUPPORTED";
    case TQ_ECUDA: return "TQ_ECUDA";
    case TQ_EWORKSPACE: return "TQ_EWORKSPACE";
    case TQ_ETIMEOUT: return "TQ_ETIMEOUT";
  }
  return "TQ_UNKNOWN";
}

const char *tq_last_error(void) { return g_last_error.c_str(); }

const char *tq_version(void) { return "tq-b200 0.1.0 (sm_100a)"; }

}  // extern "C"
