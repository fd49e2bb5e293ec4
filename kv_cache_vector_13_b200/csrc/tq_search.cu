// Top-k vector search on a TurboQuant-packed database (sm_100a).
//
// The pages evaluate TurboQuant as a nearest-neighbour index: the database
// is quantized online and full-precision queries are ranked against it by
// the estimated inner product ("内存厂商的噩梦来了", section 6.4), the
// asymmetric estimator of the attention scores,
//   est_j = n_j ( <q', c[idx_j]> + [prod] ||r_j|| sqrt(pi/2)/d <S q', sign_j> ).
// This is the decode kernel's score stage without softmax and PV:
//   * the decode prep kernel rotates the queries (a "unit" is a group of up
//     to 8 of them) and builds the fp16 pair tables;
//   * search_score_kernel: a CTA takes one unit and a contiguous slice of the
//     database; each warp streams 32-record chunks, scores them with the
//     pair-table lookups and mma.m16n8k16 of the decode kernel, and keeps,
//     per query, its best 32 (estimate, index) pairs sorted in registers, one
//     per lane.  Each lane tests its own two query columns against their
//     lists' k-th entries and against the CTA's k-th estimate per query (the
//     best of its warps' k-th entries, kept with an atomic maximum in shared
//     memory: a candidate below it is beaten by k others); two votes say
//     which queries have a candidate that passes, and most chunks stop
//     there.  For those, a few candidates are inserted one at a time at
//     their rank (a vote counts the entries ahead, the rest shift down one
//     lane); many (a list's first chunks) are sorted by a warp bitonic sort
//     and merged (the better of pair l and the reversed pair 31 - l is a
//     bitonic sequence holding the best 32, which five exchange stages
//     sort).  The CTA's warps merge their lists the same way and write one
//     list per (query, slice);
//   * search_merge_kernel: a block per query, eight warps merging every
//     eighth slice list, then one merge of the eight; writes the first k.
// Order: estimate descending, ties by record index ascending (a total
// order, so the result is unique).

#include "tq_decode_split.cuh"

namespace tq {
namespace {

constexpr int kSrWarps = 8;
constexpr int kTop = 32;  // list length per query (k <= 32)

struct SearchParams {
  const uint8_t *kc;
  const uint8_t *kj;
  const float *kn;
  const float *kr;
  int64_t sn;  // record stride
  int64_t N;
  int nq, units, splits, k;
  const uint4 *frag;
  const float *ws;
  float *cand_v;  // [nq][splits][kTop]
  int *cand_i;
  float *top_v;  // [nq][k]
  int64_t *top_i;
};

// Order-preserving int key of a float (signed int order = float order), so
// that atomicMax keeps a running float maximum.
__device__ __forceinline__ int fkey(float f) {
  const int b = __float_as_int(f);
  return b ^ ((b >> 31) & 0x7fffffff);
}
__device__ __forceinline__ float funkey(int k) { return __int_as_float(k ^ ((k >> 31) & 0x7fffffff)); }

__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// One compare-exchange stage of a warp bitonic network: lanes l and l ^ j
// exchange so that the lower lane holds the better pair when `first`.
__device__ __forceinline__ void cmpx(float &v, int &i, int j, bool first, int lane) {
  const float ov = __shfl_xor_sync(dev::kFull, v, j);
  const int oi = __shfl_xor_sync(dev::kFull, i, j);
  const bool lower = (lane & j) == 0;
  const bool ob = better(ov, oi, v, i);
  if ((lower == first) ? ob : better(v, i, ov, oi)) {
    v = ov;
    i = oi;
  }
}

// Sorts the warp's 32 pairs, best first.
__device__ __forceinline__ void warp_sort(float &v, int &i, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int j = size / 2; j > 0; j >>= 1) cmpx(v, i, j, (lane & size) == 0, lane);
  }
}

// (v, i): a list sorted best first; (cv, ci): another.  Leaves the best 32
// of both in (v, i), sorted best first.
__device__ __forceinline__ void warp_merge(float &v, int &i, float cv, int ci, int lane) {
  const float rv = __shfl_sync(dev::kFull, cv, 31 - lane);
  const int ri = __shfl_sync(dev::kFull, ci, 31 - lane);
  if (better(rv, ri, v, i)) {
    v = rv;
    i = ri;
  }
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) cmpx(v, i, j, true, lane);
}

// The key side of 32 records from record r0 (rows at or past `end`
// masked: norm -1).
template <int KBM, bool KPROD>
__device__ __forceinline__ void load_rows(KBuf<KBM, KPROD> &c, const SearchParams &p, int64_t r0, int64_t end,
                                          int tig, int g8) {
  constexpr int KCB = kD * KBM / 8;
#pragma unroll
  for (int ms = 0; ms < 2; ++ms) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int64_t n = r0 + 16 * ms + 8 * r + g8;
      const bool ok = n < end;
      const int64_t rec = (ok ? n : 0) * p.sn;
      if constexpr (KBM > 0) {
        if (ok) {
          load_k32<KBM>(p.kc + rec * KCB + tig * (4 * KBM), c.w[ms][r]);
        } else {
#pragma unroll
          for (int w = 0; w < KBM; ++w) c.w[ms][r][w] = 0u;
        }
      }
      if constexpr (KPROD) {
        c.qj[ms][r] = ok ? __ldg(reinterpret_cast<const uint32_t *>(p.kj + rec * (kD / 8)) + tig) : 0u;
        c.kr[ms][r] = ok ? __ldg(p.kr + rec) : 0.f;
      }
      c.kn[ms][r] = ok ? __ldg(p.kn + rec) : -1.f;
    }
  }
}

template <int KBM, bool KPROD, bool PACK>
__global__ void __launch_bounds__(kSrWarps * 32) search_score_kernel(SearchParams p) {
  constexpr int KW = KBM > 0 ? KBM : 1;
  // the key pair table, one copy per lane (entry e of lane l at 128 e + 4 l:
  // lookups never conflict on banks); reused for the CTA merge at the end
  __shared__ __align__(16) uint32_t s_tab[256 * 32];
  static_assert(sizeof(s_tab) >= (size_t)kSrWarps * 8 * kTop * 8, "merge lists fit in the table");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g8 = lane >> 2, tig = lane & 3;
  // the units of one slice are adjacent in launch order, so that they read
  // the slice at about the same time and share it through L2
  const int u = blockIdx.x, split = blockIdx.y;
  const int gh = min(8, p.nq - u * 8);
  for (int i = tid; i < 256 * 32; i += blockDim.x)
    s_tab[i] = KBM > 0 ? __ldg(reinterpret_cast<const uint32_t *>(p.ws + 64) + (i >> 5)) : 0u;
  // the CTA's k-th best estimate per query so far (the best over the warps'
  // k-th entries, only ever raised): a candidate below it is beaten by k
  // others in this CTA and cannot reach the result
  __shared__ int s_kkey[8];
  if (tid < 8) s_kkey[tid] = fkey(-INFINITY);
  const float inv_sK = __ldg(p.ws + 0);
  const float sK = 1.0f / inv_sK;
  __syncthreads();
  // pair_addr with a zero lane offset yields 256 e; the lane's copy of entry
  // e sits at tab + 128 e + 4 lane
  const uint32_t tab = smem_addr(s_tab) + 4u * lane;

  // the unit's query fragments (layout of the decode prep kernel)
  uint32_t qf[8][2], qf2[PACK ? 1 : 8][2];
  uint32_t qsf[KPROD ? 4 : 1][2], qsf2[(KPROD && !PACK) ? 4 : 1][2];
  float qd[2][3];  // digit weights and constant of this lane's two query columns
  {
    const bool has = (PACK ? (g8 & 3) : g8) < gh;
    const uint4 *fr = p.frag + (int64_t)u * (kFragWords / 4) + lane;
    auto ld4 = [&](int w4) { return has ? __ldg(fr + w4 * 32) : make_uint4(0u, 0u, 0u, 0u); };
    auto put = [](auto &f, int k, uint4 v) {
      f[2 * k][0] = v.x;
      f[2 * k][1] = v.y;
      f[2 * k + 1][0] = v.z;
      f[2 * k + 1][1] = v.w;
    };
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      put(qf, k, ld4(k));
      if constexpr (!PACK) put(qf2, k, ld4(4 + k));
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if constexpr (KPROD) put(qsf, k, ld4((PACK ? 4 : 8) + k));
      if constexpr (KPROD && !PACK) put(qsf2, k, ld4(10 + k));
    }
    const uint32_t *fw = reinterpret_cast<const uint32_t *>(p.frag + (int64_t)u * (kFragWords / 4));
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int h = PACK ? 2 * (tig & 1) + c : 2 * tig + c;
      const float ch = (KPROD && h < gh) ? __uint_as_float(__ldg(fw + (15 * 32 + h) * 4 + 0)) : 0.f;
      const float th = (KPROD && h < gh) ? __uint_as_float(__ldg(fw + (15 * 32 + h) * 4 + 1)) : 0.f;
      qd[c][0] = PACK ? -2.f * ch * (tig < 2 ? 256.f : 1.f) : -512.f * ch;
      qd[c][1] = PACK ? 0.f : -2.f * ch;
      qd[c][2] = (PACK && tig >= 2) ? 0.f : -th;
    }
  }

  float lv[8], kth_v[8];  // the lists (one entry a lane) and their k-th entries
  int li[8], kth_i[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    lv[h] = kth_v[h] = -INFINITY;
    li[h] = kth_i[h] = INT_MAX;
  }
  // the k-th entries of this lane's own two query columns h = 2 tig + c
  // (PACK: lanes tig >= 2 repeat the columns of tig - 2 and own none)
  const bool own = PACK ? tig < 2 : true;
  float kthm_v[2] = {-INFINITY, -INFINITY};
  int kthm_i[2] = {INT_MAX, INT_MAX};
  // this CTA's slice of the database, this warp's chunks of it
  const int64_t s0 = p.N * split / p.splits, s1 = p.N * (split + 1) / p.splits;
  const int64_t nch = (s1 - s0 + kChunk - 1) / kChunk;
  const int64_t per = (nch + kSrWarps - 1) / kSrWarps;
  const int64_t c0 = min(nch, warp * per), c1 = min(nch, c0 + per);
  for (int64_t ci = c0; ci < c1; ++ci) {
    const int64_t r0 = s0 + ci * kChunk;
    KBuf<KBM, KPROD> kb;
    load_rows<KBM, KPROD>(kb, p, r0, s1, tig, g8);
    float est[2][4];
#pragma unroll
    for (int ms = 0; ms < 2; ++ms) {
      const auto &kw = kb.w[ms];
      const auto &qj = kb.qj[ms];
      float cm[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (KBM > 0) {
#define TQ_SKSTEP(S)                                                  \
  {                                                                   \
    uint32_t a[4];                                                    \
    a[0] = lut(tab + (pair_addr<KBM, 2 * (S), KW>(kw[0], 0u) >> 1));     \
    a[1] = lut(tab + (pair_addr<KBM, 2 * (S), KW>(kw[1], 0u) >> 1));     \
    a[2] = lut(tab + (pair_addr<KBM, 2 * (S) + 1, KW>(kw[0], 0u) >> 1)); \
    a[3] = lut(tab + (pair_addr<KBM, 2 * (S) + 1, KW>(kw[1], 0u) >> 1)); \
    mma16816(cm, a, qf[S][0], qf[S][1]);                              \
    if constexpr (!PACK) mma16816(cm, a, qf2[S][0], qf2[S][1]);       \
  }
        TQ_SKSTEP(0) TQ_SKSTEP(1) TQ_SKSTEP(2) TQ_SKSTEP(3)
        TQ_SKSTEP(4) TQ_SKSTEP(5) TQ_SKSTEP(6) TQ_SKSTEP(7)
#undef TQ_SKSTEP
      }
      float cq[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (KPROD) {
        int ch[4] = {0, 0, 0, 0}, cl[4] = {0, 0, 0, 0};
#define TQ_SQSTEP(S)                                                  \
  {                                                                   \
    uint32_t a[4];                                                    \
    a[0] = sign_bytes(qj[0] << (2 * (S)));                            \
    a[1] = sign_bytes(qj[1] << (2 * (S)));                            \
    a[2] = sign_bytes(qj[0] << (2 * (S) + 1));                        \
    a[3] = sign_bytes(qj[1] << (2 * (S) + 1));                        \
    mma16832_s8(ch, a, qsf[S][0], qsf[S][1]);                         \
    if constexpr (!PACK) mma16832_s8(cl, a, qsf2[S][0], qsf2[S][1]);  \
  }
        TQ_SQSTEP(0) TQ_SQSTEP(1) TQ_SQSTEP(2) TQ_SQSTEP(3)
#undef TQ_SQSTEP
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = i & 1;
          cq[i] = fmaf((float)ch[i], qd[c][0], PACK ? qd[c][2] : fmaf((float)cl[i], qd[c][1], qd[c][2]));
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float s = cm[i];
        if constexpr (KPROD) s = fmaf(kb.kr[ms][i >> 1] * (kKappa * sK), cq[i], s);
        if constexpr (PACK) s += __shfl_xor_sync(dev::kFull, s, 2);  // hi + lo columns
        const float kn = kb.kn[ms][i >> 1];
        est[ms][i] = kn >= 0.f ? s * (kn * inv_sK) : -INFINITY;
      }
    }
    // per query: does any of the chunk's 32 candidates beat the list's
    // k-th entry?  Each lane tests its own two columns (rows g8 + 8 r +
    // 16 ms of the score tile) against their k-th entries; two votes answer
    // for every query, and most chunks end here.
    bool hc[2] = {false, false};
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const float cta = funkey(*reinterpret_cast<volatile int *>(&s_kkey[2 * tig + c]));
#pragma unroll
      for (int ms = 0; ms < 2; ++ms) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int idx = (int)(r0 + 16 * ms + 8 * r + g8);
          const float e = est[ms][2 * r + c];
          hc[c] |= e >= cta && better(e, idx, kthm_v[c], kthm_i[c]);
        }
      }
      hc[c] = hc[c] && own && 2 * tig + c < gh;
    }
    const unsigned hit0 = __ballot_sync(dev::kFull, hc[0]), hit1 = __ballot_sync(dev::kFull, hc[1]);
    if ((hit0 | hit1) == 0u) continue;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      if (h < gh) {
        const int c = h & 1;
        // lanes l with l % 4 == h / 2 hold column h
        if ((((c ? hit1 : hit0) >> (h >> 1)) & 0x11111111u) == 0u) continue;
        // the chunk's candidates for query h, one per lane (lane L holds
        // record r0 + L)
        const int src = (lane & 7) * 4 + (h >> 1);
        float cv = -INFINITY;
#pragma unroll
        for (int ms = 0; ms < 2; ++ms) {
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float t = __shfl_sync(dev::kFull, est[ms][2 * r + c], src);
            if ((lane >> 4) == ms && ((lane >> 3) & 1) == r) cv = t;
          }
        }
        const int cidx = (int)(r0 + lane);
        const float cta = funkey(*reinterpret_cast<volatile int *>(&s_kkey[h]));
        const unsigned up = __ballot_sync(dev::kFull, cv >= cta && better(cv, cidx, kth_v[h], kth_i[h]));
        if (__popc(up) > 4) {  // many (the lists' first chunks): sort and merge
          int ci2 = cidx;
          warp_sort(cv, ci2, lane);
          warp_merge(lv[h], li[h], cv, ci2, lane);
        } else {  // a few: insert each at its rank, the entries below move down one
          for (unsigned m = up; m; m &= m - 1) {
            const int l = __ffs(m) - 1;
            const float nv = __shfl_sync(dev::kFull, cv, l);
            const int ni = __shfl_sync(dev::kFull, cidx, l);
            const int pos = __popc(__ballot_sync(dev::kFull, better(lv[h], li[h], nv, ni)));
            const float dv = __shfl_up_sync(dev::kFull, lv[h], 1);
            const int di = __shfl_up_sync(dev::kFull, li[h], 1);
            if (lane == pos) {
              lv[h] = nv;
              li[h] = ni;
            } else if (lane > pos) {
              lv[h] = dv;
              li[h] = di;
            }
          }
        }
        kth_v[h] = __shfl_sync(dev::kFull, lv[h], p.k - 1);
        kth_i[h] = __shfl_sync(dev::kFull, li[h], p.k - 1);
        if (tig == (h >> 1)) {
          kthm_v[c] = kth_v[h];
          kthm_i[c] = kth_i[h];
        }
        if (lane == 0 && kth_v[h] > -INFINITY) atomicMax(&s_kkey[h], fkey(kth_v[h]));
      }
    }
  }
  // CTA merge: warp h merges the warps' lists of query h (in the table's
  // memory, free once every warp is done scoring)
  __syncthreads();
  float *s_lv = reinterpret_cast<float *>(s_tab);          // [kSrWarps][8][kTop]
  int *s_li = reinterpret_cast<int *>(s_tab) + kSrWarps * 8 * kTop;
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    s_lv[(warp * 8 + h) * kTop + lane] = lv[h];
    s_li[(warp * 8 + h) * kTop + lane] = li[h];
  }
  __syncthreads();
  if (warp < gh) {
    const int h = warp;
    float v = s_lv[h * kTop + lane];
    int i = s_li[h * kTop + lane];
    for (int w = 1; w < kSrWarps; ++w)
      warp_merge(v, i, s_lv[(w * 8 + h) * kTop + lane], s_li[(w * 8 + h) * kTop + lane], lane);
    const int64_t o = ((int64_t)(u * 8 + h) * p.splits + split) * kTop + lane;
    p.cand_v[o] = v;
    p.cand_i[o] = i;
  }
}

// One block per query: warp w merges the slices' lists w, w + 8, ... (the
// next list's loads issued before the current merge), then warp 0 merges
// the eight results and writes the first k.
__global__ void __launch_bounds__(256) search_merge_kernel(SearchParams p) {
  __shared__ float s_v[8][kTop];
  __shared__ int s_i[8][kTop];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int qg = blockIdx.x;
  const int64_t base = (int64_t)qg * p.splits * kTop + lane;
  float v = -INFINITY;
  int i = INT_MAX;
  float nv = warp < p.splits ? p.cand_v[base + (int64_t)warp * kTop] : -INFINITY;
  int ni = warp < p.splits ? p.cand_i[base + (int64_t)warp * kTop] : INT_MAX;
  for (int sl = warp; sl < p.splits; sl += 8) {
    const float cv = nv;
    const int ci = ni;
    if (sl + 8 < p.splits) {
      nv = p.cand_v[base + (int64_t)(sl + 8) * kTop];
      ni = p.cand_i[base + (int64_t)(sl + 8) * kTop];
    }
    warp_merge(v, i, cv, ci, lane);
  }
  s_v[warp][lane] = v;
  s_i[warp][lane] = i;
  __syncthreads();
  if (warp == 0) {
    for (int w = 1; w < 8; ++w) warp_merge(v, i, s_v[w][lane], s_i[w][lane], lane);
    if (lane < p.k) {
      const bool real = v > -INFINITY;
      p.top_v[(int64_t)qg * p.k + lane] = v;
      p.top_i[(int64_t)qg * p.k + lane] = real ? (int64_t)i : -1;
    }
  }
}

template <int KBM, bool KPROD, bool PACK>
cudaError_t run_search(const SearchParams &sp, cudaStream_t s) {
  search_score_kernel<KBM, KPROD, PACK><<<dim3((unsigned)sp.units, (unsigned)sp.splits), kSrWarps * 32, 0, s>>>(sp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  search_merge_kernel<<<(unsigned)sp.nq, 256, 0, s>>>(sp);
  return cudaGetLastError();
}

template <bool KPROD, bool PACK>
cudaError_t search_by_bits(int kbm, const SearchParams &sp, cudaStream_t s) {
  switch (kbm) {
    case 0: if constexpr (KPROD) return run_search<0, true, PACK>(sp, s); else return cudaErrorInvalidValue;
    case 1: return run_search<1, KPROD, PACK>(sp, s);
    case 2: return run_search<2, KPROD, PACK>(sp, s);
    case 3: return run_search<3, KPROD, PACK>(sp, s);
    case 4: return run_search<4, KPROD, PACK>(sp, s);
  }
  return cudaErrorInvalidValue;
}

// database slices: enough CTAs to fill the GPU twice over, each slice at
// least 2048 records
int search_splits(int64_t N, int units) {
  const int64_t want = (2 * 148 + units - 1) / units;
  const int64_t most = (N + 2047) / 2048;
  return (int)std::max<int64_t>(1, std::min(want, most));
}

}  // namespace

size_t search_workspace_floats(int nq, int64_t N) {
  const int units = (nq + 7) / 8;
  const int splits = search_splits(N, units);
  return (size_t)dec::kHdr + (size_t)units * dec::kFragWords + (size_t)units + 4 +
         (size_t)nq * splits * kTop * 2;
}

cudaError_t launch_search(const SearchArgs &a, cudaStream_t s) {
  using namespace dec;
  SearchParams sp{};
  sp.kc = a.db.codes;
  sp.kj = a.db.qjl;
  sp.kn = a.db.norms;
  sp.kr = a.db.rnorms;
  sp.sn = a.db.sn;
  sp.N = a.n_db;
  sp.nq = a.nq;
  sp.units = (a.nq + 7) / 8;
  sp.splits = search_splits(a.n_db, sp.units);
  sp.k = a.k;
  float *ws = a.ws;
  sp.ws = ws;
  sp.frag = reinterpret_cast<const uint4 *>(ws + kHdr);
  unsigned *cnt = reinterpret_cast<unsigned *>(ws + kHdr + (size_t)sp.units * kFragWords);
  float *cand = ws + kHdr + (size_t)sp.units * kFragWords + sp.units + 4;
  sp.cand_v = cand;
  sp.cand_i = reinterpret_cast<int *>(cand + (size_t)a.nq * sp.splits * kTop);
  sp.top_v = a.top_v;
  sp.top_i = a.top_i;
  // the queries are the heads of one batch entry with one kv head
  PrepParams pp{a.queries, a.q_dtype, a.nq, a.q.signs, a.q.rot, a.q.prod ? a.q.S : nullptr,
                a.q.centroids, a.q.bm, nullptr, 0, ws, cnt, sp.units,
                a.nq, 1, a.nq, sp.units, a.n_db, nullptr, nullptr,
                reinterpret_cast<uint32_t *>(ws + kHdr)};
  cudaError_t e = launch_prep(pp, false, s);
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const bool pack = a.nq <= 4;
  if (pack) return a.q.prod ? search_by_bits<true, true>(a.q.bm, sp, s) : search_by_bits<false, true>(a.q.bm, sp, s);
  return a.q.prod ? search_by_bits<true, false>(a.q.bm, sp, s) : search_by_bits<false, false>(a.q.bm, sp, s);
}

}  // namespace tq
