// Internal interface between the host library (tq_host.cpp) and the CUDA
// launchers (tq_encode.cu, tq_dequant.cu, tq_decode.cu).  Not installed.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace tq {

// Everything a kernel needs about one quantizer, resolved on the host.
struct QuantParams {
  int d;
  int bm;          // MSE bits b_m (0..4)
  bool prod;
  const float *centroids;   // 2^bm
  const float *thresholds;  // 2^bm - 1
  const int8_t *signs;      // d
  const float *S;           // d*d (prod)
  const float *rot;         // d*d row-major Pi (dense rotation), else NULL
  const int32_t *channels;  // d input-element indices (channel group), else NULL
  float sqrt_d;             // fl32(sqrt(d)) (double sqrt rounded once)
};

struct CacheView {
  uint8_t *codes;
  uint8_t *qjl;
  float *norms;
  float *rnorms;
  int64_t sb, sh, sn;  // record strides
};

struct EncodeArgs {
  QuantParams q;
  const void *x;
  int dtype;           // tq_dtype
  int64_t B, H, N;
  int64_t xsb, xsh, xsn;  // element strides
  CacheView out;
  // launched with programmatic stream serialization after the kernel before
  // it (the fused append + decode chain); the grid then waits for that
  // kernel before it completes
  bool pdl = false;
};

struct DequantArgs {
  QuantParams q;
  CacheView in;
  int64_t B, H, N;
  float *out;
};

struct DecodeArgs {
  QuantParams kq, vq;
  const void *q;
  int q_dtype;
  int B, Hq, Hkv;
  int64_t seq_len;
  const int32_t *seq_lens;
  CacheView k, v;
  float scale;
  float *out;
  float *scores;
  float *ws;           // partial slots
  int splits;          // persistent CTAs of the split kernel
  // the prep kernel is launched with programmatic stream serialization after
  // the kernel before it (the fused append + decode chain)
  bool prep_pdl = false;
};

struct SearchArgs {
  QuantParams q;
  CacheView db;   // records n * db.sn, n < n_db
  int64_t n_db;
  const void *queries;
  int q_dtype;
  int nq, k;
  float *top_v;
  int64_t *top_i;
  float *ws;
};

struct SplitDecodeArgs {
  QuantParams kq[2], vq[2];
  const void *q;
  int q_dtype;
  int B, Hq, Hkv, d;
  int64_t seq_len;
  const int32_t *seq_lens;
  CacheView k[2], v[2];
  float scale;
  float *out;
  float *ws;  // partial slots of the split over the sequence
};
cudaError_t launch_decode_split(const SplitDecodeArgs &a, cudaStream_t s);

// Workspace of a search, in floats.
size_t search_workspace_floats(int nq, int64_t n_db);
cudaError_t launch_search(const SearchArgs &a, cudaStream_t s);

// Decode work split shared by the workspace query and the launch: the number
// of persistent CTAs, and the workspace size in floats (a header with the
// centroid tables, the rotated queries, and (units + CTAs) partial slots,
// units = B * Hkv * ceil((Hq/Hkv) / 8)).
int decode_ctas();
size_t decode_workspace_floats(int B, int Hq, int Hkv, bool prod, int ctas);

// The CUDA-core decode for what the tensor-core split kernel does not take
// (d other than 128, prod values): its sequence splits and workspace in
// floats (both depend only on the arguments), and the launch.
bool decode_fast_path(int d, bool vprod);
int general_decode_splits(int B, int Hq, int Hkv, int64_t seq_len);
size_t general_decode_workspace_floats(int B, int Hq, int Hkv, int64_t seq_len, int d);
cudaError_t launch_decode_general(const DecodeArgs &a, cudaStream_t s);

// Faults the kernels detect themselves (bits of a per-GPU word): a bounded
// wait that expired, and a launch whose shared-memory layout check failed
// (the kernel then writes nothing).
constexpr unsigned kFaultTimeout = 1u;
constexpr unsigned kFaultSmemLayout = 2u;

// Device address of the current device's fault word (for kernels that set
// bits in it).
cudaError_t fault_word(unsigned **ptr);

// Reads the current device's fault word and clears it (synchronous).
cudaError_t take_device_faults(unsigned *faults);

// Device address of the allocation-free decode's fixed scratch array on
// the current device (looked up once per device with cudaGetSymbolAddress).
cudaError_t static_scratch(void **ptr);

cudaError_t launch_encode(const EncodeArgs &a, cudaStream_t s);
// the dense (Haar) rotation, any d that is a multiple of 8 up to 256
cudaError_t launch_encode_dense(const EncodeArgs &a, cudaStream_t s);
cudaError_t launch_dequant_dense(const DequantArgs &a, cudaStream_t s);
cudaError_t launch_dequant(const DequantArgs &a, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s);

// Whether a (d, bm, prod, dtype, rotation) instantiation exists.
bool encode_supported(int d, int bm, bool prod, int dtype, bool dense);
bool dequant_supported(int d, int bm, bool prod, bool dense);
bool decode_supported(int d, int kbm, bool kprod, int vbm, bool vprod, bool kdense, bool vdense);

}  // namespace tq
