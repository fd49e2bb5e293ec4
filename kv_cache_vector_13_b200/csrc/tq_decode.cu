// Decode attention on the packed TurboQuant cache (sm_100a): the prep
// kernel and the host launch.
//
// Attention for one new query per head, softmax(q K^T / sqrt(d)) V over all
// cached tokens ("I Spent 31 Hours On The Math Behind Turboquant", section
// "KV Cache: The problem"), with keys scored by the asymmetric estimator: the
// full-precision query against the compressed keys ("内存厂商的噩梦来了",
// section 4.2 and its asymmetric_attention_score).
//
// Kernel 0 (prep, this file), once per call: rotates every query head (sign
// flips + FWHT, and S q' for prod keys) into the query fragments the split
// kernel's lanes hold; for each codebook finds a scale s with fp16(s c_k)
// close to s c_k for every centroid (a search over 4096 candidates in [1, 2))
// and writes the 256-entry pair table entry e -> half2(fp16(s c[e & m]),
// fp16(s c[(e >> b_m) & m])); zeroes the units' arrival counters.
// Kernel 1 (split, tq_decode_split.cuh, instantiated by
// tq_decode_staged.cu and tq_decode_regs.cu): scores, online softmax, PV and
// the merge of the splits.

#include "tq_decode_split.cuh"

#include <atomic>
#include <mutex>

// Which split-kernel variant feeds unit-stride caches: the register-fed one
// (TQ_FEED_REGISTERS, the faster one measured on B200) or the bulk-copy ring
// (TQ_FEED_BULK_STAGED); set by tq_set_decode_feed.
static std::atomic<int> g_decode_feed{TQ_FEED_REGISTERS};

// Scratch for tq_decode_attention_noalloc: a fixed array in device memory,
// one copy per GPU that loads the library, held until the process exits.
// Host code must not use its name as a device address; the address comes
// from cudaGetSymbolAddress (static_scratch below).
static __device__ __align__(256) unsigned char g_tq_noalloc_scratch[TQ_NOALLOC_SCRATCH_BYTES];

// Faults a kernel detects on its own, one word per GPU (tq::kFault* bits),
// set with atomicOr through the address the launches pass and read back and
// cleared by tq_check.
static __device__ unsigned int g_tq_faults;

namespace tq {
namespace {

// ------------------------------------------------------------- prep kernel

// Index i in [0, kScaleCands) minimising the worst relative fp16 rounding
// error of (1 + i/kScaleCands) * c_k over the K/2 positive centroids (ties ->
// smallest i); then the pair table for that scale.  One 256-thread block.
__device__ void scale_and_table(const float *cent, int bm, float *inv_scale, uint32_t *table) {
  __shared__ uint64_t s_red[8];
  __shared__ float s_c[16];
  const int K = 1 << bm;
  if (threadIdx.x < K) s_c[threadIdx.x] = cent[threadIdx.x];
  __syncthreads();
  float c[8], rc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    c[k] = K / 2 + k < K ? s_c[K / 2 + k] : s_c[K - 1];
    rc[k] = 1.0f / c[k];
  }
  uint64_t best = ~0ull;
  for (int i = threadIdx.x; i < kScaleCands; i += blockDim.x) {
    const float s = 1.0f + (float)i * (1.0f / kScaleCands);
    float worst = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float v = s * c[k];
      worst = fmaxf(worst, fabsf(__half2float(__float2half_rn(v)) - v) * rc[k]);
    }
    const uint64_t key = ((uint64_t)__float_as_uint(worst) << 32) | (uint32_t)i;
    best = key < best ? key : best;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const uint64_t other = __shfl_xor_sync(dev::kFull, best, o);
    best = other < best ? other : best;
  }
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = best;
  __syncthreads();
  uint64_t b = ~0ull;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) b = s_red[w] < b ? s_red[w] : b;
  const float sc = 1.0f + (float)(uint32_t)(b & 0xffffffffu) * (1.0f / kScaleCands);
  const uint32_t m = (uint32_t)K - 1u;
  for (int e = threadIdx.x; e < 256; e += blockDim.x)
    table[e] = pack_half2(sc * s_c[e & m], sc * s_c[(e >> bm) & m]);
  if (threadIdx.x == 0) *inv_scale = 1.0f / sc;
}

// Blocks [0, nheads/2): two query heads each (128 threads per head):
// q' = H(sigma q)/sqrt(d) and q_s = S q'.  The last two blocks: the K and
// V scale and pair table.
__global__ void __launch_bounds__(256) decode_prep_kernel(PrepParams p) {
  // the split kernel may be scheduled now: it waits for this grid to finish
  // (griddepcontrol.wait) before it reads anything written here
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  const int nqb = (p.nheads + 1) / 2;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.units; i += gridDim.x * blockDim.x) p.cnt[i] = 0u;
  if ((int)blockIdx.x >= nqb) {
    if (blockIdx.x == (unsigned)nqb) {
      if (p.kbm > 0) scale_and_table(p.kcent, p.kbm, p.ws + 0, reinterpret_cast<uint32_t *>(p.ws + 64));
      else if (threadIdx.x == 0) p.ws[0] = 1.0f;
    } else if (p.vbm > 0) {
      scale_and_table(p.vcent, p.vbm, p.ws + 1, reinterpret_cast<uint32_t *>(p.ws + 320));
    } else if (threadIdx.x == 0) {
      p.ws[1] = 1.0f;
    }
    return;
  }
  __shared__ float s_q[2][kD], s_qs[2][kD];
  const int half = threadIdx.x >> 7, t = threadIdx.x & 127;
  const int head = blockIdx.x * 2 + half;
  const bool valid = head < p.nheads;
  // a batch with no cached tokens has no work piece: its output is zero
  if (valid && p.seq_lens && batch_len(p.seq_lens, p.seq_len, head / p.Hq) == 0)
    p.out[(int64_t)head * kD + t] = 0.f;
  const int lane = threadIdx.x & 31;
  if ((t >> 5) == 0) {  // one warp per head: 4 dims per lane
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    if (valid) {
      const int64_t qoff = (int64_t)head * kD + lane * 4;
      if (p.q_dtype == TQ_F32) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(p.q) + qoff / 4);
        a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
      } else {
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(static_cast<const char *>(p.q) + qoff * 2));
        if (p.q_dtype == TQ_BF16) {
          a[0] = dev::bf16lo(v.x); a[1] = dev::bf16hi(v.x); a[2] = dev::bf16lo(v.y); a[3] = dev::bf16hi(v.y);
        } else {
          a[0] = dev::f16lo(v.x); a[1] = dev::f16hi(v.x); a[2] = dev::f16lo(v.y); a[3] = dev::f16hi(v.y);
        }
      }
      if (!p.krot) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (p.ksign[lane * 4 + i] < 0) a[i] = -a[i];
      }
    }
    if (p.krot) {  // dense rotation: stage q, the product follows below
#pragma unroll
      for (int i = 0; i < 4; ++i) s_qs[half][lane * 4 + i] = a[i];
    } else {
      dev::fwht<32, 4>(a, lane);
#pragma unroll
      for (int i = 0; i < 4; ++i) s_q[half][lane * 4 + i] = a[i] * 0.08838834764831845f;
    }
  }
  __syncthreads();
  if (p.krot) {  // q' = Pi q, one output per thread
    float acc = 0.f;
    if (valid) {
      const float4 *R = reinterpret_cast<const float4 *>(p.krot + (size_t)t * kD);
#pragma unroll 8
      for (int i = 0; i < kD / 4; ++i) {
        const float4 r = __ldg(R + i);
        acc = fmaf(r.x, s_qs[half][4 * i], acc);
        acc = fmaf(r.y, s_qs[half][4 * i + 1], acc);
        acc = fmaf(r.z, s_qs[half][4 * i + 2], acc);
        acc = fmaf(r.w, s_qs[half][4 * i + 3], acc);
      }
    }
    __syncthreads();
    s_q[half][t] = acc;
    __syncthreads();
  }
  // S q' as two int8 digits per coordinate: x = round(Sq' / c) = 256 hi + lo
  // with |x| <= 32000 (c = max |Sq'| / 32000), hi in [-125, 125], lo in
  // [-128, 127]; and T = sum_k Sq'[k]
  __shared__ int s_dig[2][2][kD];  // [half][hi / lo][k]
  __shared__ float s_red[2][4][2];
  float sq_c = 0.f, sq_t = 0.f;
  if (p.kS) {
    float acc = 0.f;
    if (valid) {
      const float4 *Sk = reinterpret_cast<const float4 *>(p.kS + (size_t)t * kD);
#pragma unroll 8
      for (int i = 0; i < kD / 4; ++i) {
        const float4 sv = __ldg(Sk + i);
        acc = fmaf(sv.x, s_q[half][4 * i], acc);
        acc = fmaf(sv.y, s_q[half][4 * i + 1], acc);
        acc = fmaf(sv.z, s_q[half][4 * i + 2], acc);
        acc = fmaf(sv.w, s_q[half][4 * i + 3], acc);
      }
    }
    float mx = fabsf(acc), sm = acc;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(dev::kFull, mx, o));
      sm += __shfl_xor_sync(dev::kFull, sm, o);
    }
    if (lane == 0) {
      s_red[half][t >> 5][0] = mx;
      s_red[half][t >> 5][1] = sm;
    }
    __syncthreads();
    mx = fmaxf(fmaxf(s_red[half][0][0], s_red[half][1][0]), fmaxf(s_red[half][2][0], s_red[half][3][0]));
    sq_t = (s_red[half][0][1] + s_red[half][1][1]) + (s_red[half][2][1] + s_red[half][3][1]);
    sq_c = mx > 0.f ? mx * (1.0f / 32000.0f) : 1.0f;
    const int x = __float2int_rn(acc / sq_c);
    const int hi = (x + 128) >> 8;
    s_dig[half][0][t] = hi;
    s_dig[half][1][t] = x - 256 * hi;
  }
  __syncthreads();
  if (!valid) return;
  // this head's fragment words (the layout of kFragWords above)
  const int b = head / p.Hq, hq = head % p.Hq;
  const int kvh = hq / p.g, grp = (hq % p.g) / 8, hh = (hq % p.g) % 8;
  const int64_t u = ((int64_t)b * p.Hkv + kvh) * p.groups + grp;
  uint32_t *fu = p.frag + u * kFragWords;
  auto put = [&](int ln, int w, uint32_t v) { fu[((w >> 2) * 32 + ln) * 4 + (w & 3)] = v; };
  const float *qv = s_q[half];
  // the digit word of lane tig, step S, register j: bytes i = 0..3 hold the
  // digit of Sq'[32 tig + 8 i + 7 - 2 S - j]
  auto dig_word = [&](int which, int tig, int S, int j) {
    uint32_t wv = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      wv |= ((uint32_t)s_dig[half][which][32 * tig + 8 * i + 7 - 2 * S - j] & 0xFFu) << (8 * i);
    return wv;
  };
  if (p.g <= 4) {
    const int ls = t >> 4, w = t & 15, sidx = w >> 1, j = w & 1;
    const int g8 = hh + 4 * (ls >> 2), tig = ls & 3, ln = g8 * 4 + tig;
    const bool lo = g8 >= 4;
    const int d0 = 32 * tig + 4 * sidx + 2 * j;
    put(ln, w, lo ? pack_lo(qv[d0], qv[d0 + 1]) : pack_hi(qv[d0], qv[d0 + 1]));
    if (p.kS && w < 8) put(ln, 16 + w, dig_word(lo ? 1 : 0, tig, w >> 1, w & 1));
  } else {
    const int tig = t >> 5, w = t & 31, sidx = (w & 15) >> 1, j = w & 1;
    const int ln = hh * 4 + tig;
    const bool lo = w >= 16;
    const int d0 = 32 * tig + 4 * sidx + 2 * j;
    put(ln, w, lo ? pack_lo(qv[d0], qv[d0 + 1]) : pack_hi(qv[d0], qv[d0 + 1]));
    if (p.kS && w < 16) put(ln, 32 + w, dig_word(w >> 3, tig, (w & 7) >> 1, w & 1));
  }
  if (p.kS && t == 0) {  // the head's digit scale and coordinate sum
    put(hh, 60, __float_as_uint(sq_c));
    put(hh, 61, __float_as_uint(sq_t));
  }
  // When this grid was launched early after the new tokens' encode (the
  // fused append + decode chain), one thread waits for that grid, so this
  // grid completes after it and the split kernel's wait covers both.  Head 0
  // (block 0, thread 0) always reaches this point.  Without such a launch
  // the wait returns at once.
  if (blockIdx.x == 0 && threadIdx.x == 0) asm volatile("griddepcontrol.wait;\n" ::: "memory");
}


}  // namespace


// The tensor-core split kernel takes d = 128 with TurboQuant_mse values
// (either rotation: only the query's and the output's rotation differ); the
// CUDA-core path takes every other valid pair of quantizers.
bool decode_fast_path(int d, bool vprod) { return d == kD && !vprod; }

bool decode_supported(int d, int kbm, bool kprod, int vbm, bool vprod, bool kdense, bool vdense) {
  (void)kdense;
  (void)vdense;
  return d >= 8 && d <= 256 && d % 8 == 0 && vbm >= (vprod ? 0 : 1) && vbm <= 4 && kbm >= (kprod ? 0 : 1) &&
         kbm <= 4;
}

size_t decode_workspace_floats(int B, int Hq, int Hkv, bool prod, int ctas) {
  const int64_t units = (int64_t)B * Hkv * ((Hq / Hkv + 7) / 8);
  (void)prod;  // the fragment block has room for the prod words either way
  return (size_t)kHdr + (size_t)units * kFragWords + (size_t)(units + ctas) * kSlot + (size_t)units;
}

cudaError_t take_device_faults(unsigned *faults) {
  unsigned w = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&w, g_tq_faults, sizeof(w));
  if (e != cudaSuccess) return e;
  *faults = w;
  if (w) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_tq_faults, &zero, sizeof(zero));
  }
  return e;
}

namespace {

// The driver's current-context query, reached through the runtime (no
// link against the driver library); NULL when the runtime cannot provide it.
using CtxCurrentFn = int (*)(void **);
CtxCurrentFn ctx_current_fn() {
  static const CtxCurrentFn fn = [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<CtxCurrentFn>(f);
  }();
  return fn;
}

// Device address of a __device__ symbol in the current context.  Cached per
// device together with the context it was looked up in, and looked up again
// when the device's context has changed (a reset destroys the primary
// context, and the symbol's address with it); without the context query it
// is looked up on every call.
template <typename Sym>
cudaError_t symbol_address(const Sym &sym, void **ptr) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void *addr[kMaxDevices] = {};
  static void *ctx_of[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void *ctx = nullptr;  // no context yet: looked up (which creates it) and not cached
  const CtxCurrentFn fn = ctx_current_fn();
  const bool keyed = fn && fn(&ctx) == 0 && ctx;
  std::lock_guard<std::mutex> lock(mu);
  if (!keyed || !addr[dev] || ctx_of[dev] != ctx) {
    void *a = nullptr;
    e = cudaGetSymbolAddress(&a, sym);
    if (e != cudaSuccess) return e;
    addr[dev] = a;
    ctx_of[dev] = keyed ? ctx : nullptr;
  }
  *ptr = addr[dev];
  return cudaSuccess;
}

}  // namespace

cudaError_t fault_word(unsigned **ptr) {
  void *a = nullptr;
  const cudaError_t e = symbol_address(g_tq_faults, &a);
  *ptr = static_cast<unsigned *>(a);
  return e;
}

cudaError_t static_scratch(void **ptr) {
  // cached per device and context
  return symbol_address(g_tq_noalloc_scratch, ptr);
}

namespace dec {

// The prep kernel: (nheads + 1) / 2 blocks of two query heads, then the key
// and value table blocks.
cudaError_t launch_prep(const PrepParams &pp, bool pdl, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((pp.nheads + 1) / 2 + 2));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_prep_kernel, pp);
}

}  // namespace dec

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
  if (!decode_fast_path(a.kq.d, a.vq.prod)) return launch_decode_general(a, s);
  const int64_t outn = (int64_t)a.B * a.Hq * kD;
  if (a.seq_len == 0) {
    zero_out_kernel<<<(unsigned)((outn + 255) / 256), 256, 0, s>>>(a.out, outn);
    return cudaGetLastError();
  }
  SplitParams sp{};
  sp.q = a.q;
  sp.q_dtype = a.q_dtype;
  sp.B = a.B;
  sp.Hq = a.Hq;
  sp.Hkv = a.Hkv;
  sp.g = a.Hq / a.Hkv;
  sp.groups = (sp.g + 7) / 8;
  sp.seq_len = a.seq_len;
  sp.seq_lens = a.seq_lens;
  // When the units fit the grid, a CTA count that is a multiple of the unit
  // count (if it idles at most 5% of the CTAs) keeps every CTA inside one
  // unit: no CTA then works on two pieces in sequence.
  {
    const int64_t units = (int64_t)a.B * a.Hkv * sp.groups;
    int ctas = a.splits;
    if (units <= ctas) {
      const int64_t aligned = (ctas / units) * units;
      if (aligned * 20 >= (int64_t)ctas * 19) ctas = (int)aligned;
    }
    sp.ctas = ctas;
  }
  sp.kc = a.k.codes;
  sp.kj = a.k.qjl;
  sp.kn = a.k.norms;
  sp.kr = a.k.rnorms;
  sp.ksb = a.k.sb;
  sp.ksh = a.k.sh;
  sp.ksn = a.k.sn;
  sp.kcent = a.kq.centroids;
  sp.ksign = a.kq.signs;
  sp.kS = a.kq.S;
  sp.vc = a.v.codes;
  sp.vn = a.v.norms;
  sp.vsb = a.v.sb;
  sp.vsh = a.v.sh;
  sp.vsn = a.v.sn;
  sp.vcent = a.vq.centroids;
  sp.scale_log2 = a.scale * kLog2e;
  sp.scores = a.scores;
  sp.ws = a.ws;
  const int units = a.B * a.Hkv * sp.groups;
  sp.frag = reinterpret_cast<const uint4 *>(a.ws + kHdr);
  sp.slot0 = (int64_t)kHdr + (int64_t)units * kFragWords;
  sp.cnt = reinterpret_cast<unsigned *>(a.ws + sp.slot0 + (int64_t)(units + sp.ctas) * kSlot);
  sp.out = a.out;
  sp.vsign = a.vq.signs;
  sp.vrot = a.vq.rot;
  {
    void *fw = nullptr;
    const cudaError_t fe = symbol_address(g_tq_faults, &fw);
    if (fe != cudaSuccess) return fe;
    sp.faults = static_cast<unsigned *>(fw);
  }
  // without an append before it in the chain, the cache is complete when the
  // split grid starts, so its first bulk copies may precede the prep kernel
  sp.early = !a.prep_pdl;
  PrepParams pp{a.q, a.q_dtype, a.B * a.Hq, a.kq.signs, a.kq.rot, a.kq.prod ? a.kq.S : nullptr,
                a.kq.centroids, a.kq.bm, a.vq.centroids, a.vq.bm, a.ws, sp.cnt, units,
                a.Hq, a.Hkv, sp.g, sp.groups, a.seq_len, a.seq_lens, a.out,
                reinterpret_cast<uint32_t *>(a.ws + kHdr)};
  cudaError_t pe = dec::launch_prep(pp, a.prep_pdl, s);
  if (pe != cudaSuccess) return pe;
  pe = cudaGetLastError();
  if (pe != cudaSuccess) return pe;
  const bool pack = sp.g <= 4;
  // the staged variant needs unit token strides and 16-byte aligned norm
  // rows in every (batch, kv head) slice (its bulk copies move whole rows)
  auto rows16 = [&](const void *ptr, int64_t sb, int64_t sh) {
    return ptr == nullptr || (((uintptr_t)ptr % 16) == 0 && (a.B == 1 || sb % 4 == 0) && (a.Hkv == 1 || sh % 4 == 0));
  };
  const bool staged = g_decode_feed.load(std::memory_order_relaxed) == TQ_FEED_BULK_STAGED && a.k.sn == 1 &&
                      a.v.sn == 1 && rows16(a.k.norms, a.k.sb, a.k.sh) && rows16(a.k.rnorms, a.k.sb, a.k.sh) &&
                      rows16(a.v.norms, a.v.sb, a.v.sh);
  cudaError_t e = cudaErrorInvalidValue;
  if (staged) e = dec::launch_split_staged(a.kq.bm, a.kq.prod, a.vq.bm, pack, sp, s);
  if (!staged || e == cudaErrorInvalidConfiguration) {
    (void)cudaGetLastError();  // a staged launch that did not fit leaves nothing behind
    e = dec::launch_split_regs(a.kq.bm, a.kq.prod, a.vq.bm, pack, sp, s);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace tq

extern "C" int32_t tq_set_decode_feed(int32_t feed) {
  if (feed != TQ_FEED_REGISTERS && feed != TQ_FEED_BULK_STAGED) return -1;
  return g_decode_feed.exchange(feed);
}
