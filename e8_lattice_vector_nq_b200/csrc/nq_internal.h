// nq_internal.h -- launch descriptors shared by the C ABI layer (nq_abi.cu)
// and the kernel files.  Arguments are validated by the ABI layer before any
// launcher below is called.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nq.h"
#include "nq_device.cuh"

namespace nq {

// Heads per CTA of the tiled kernels (one warp per head): the largest divisor
// of the head count up to 8.
inline int pick_head_group(int heads) {
  for (int g = 8; g >= 1; --g)
    if (heads % g == 0) return g;
  return 1;
}

struct EncodeLaunch {
  const void* K;
  nq_kv_strides ks;
  const void* V;
  nq_kv_strides vs;
  int units, heads;
  int64_t T_in, n;
  const int32_t* kept;
  int64_t kept_stride;
  int64_t pos_base;
  const float* rope_tab;
  int64_t rope_max_pos;
  nq_packed k_out, v_out;  // exact layout: meta points to the uint16 scales
  int64_t slot0;
  bool exact;
};

struct DecodeLaunch {
  nq_packed k_in, v_in;  // exact layout: meta points to the uint16 scales
  bool exact;
  int units, heads;
  int64_t n, slot0;
  const int32_t* positions;
  int64_t pos_stride;
  int64_t pos_base;
  const float* rope_tab;
  int64_t rope_max_pos;
  void* K_out;
  nq_kv_strides kos;
  void* V_out;
  nq_kv_strides vos;
};

struct AttendLaunch {
  const float* q;
  int units, heads, G;
  nq_packed k_in, v_in;
  int64_t n, slot0;
  const int32_t* positions;
  int64_t pos_stride, pos_base;
  const float* rope_tab;
  int64_t rope_max_pos;
  float scale;
  float* out;
  float* lse;
  void* ws;
};

cudaError_t launch_encode(const EncodeLaunch& L, cudaStream_t stream);
cudaError_t launch_decode(const DecodeLaunch& L, cudaStream_t stream);

cudaError_t codec_read_clear_error(uint32_t* flags);
// Decode engine (nq_decode_engine values), read at each decode launch.
void set_decode_engine(int engine);
int decode_engine();
size_t attend_workspace_floats(int units, int heads, int G, int64_t n);
int64_t attend_ctas(int units, int heads, int64_t n);  // CTAs of the partial kernel
cudaError_t launch_attend(const AttendLaunch& L, cudaStream_t stream);
cudaError_t launch_e8_quantise(const float* y, int64_t groups, int bits, uint32_t* codes,
                               uint8_t* coset, cudaStream_t stream);
cudaError_t launch_e8_box_quantise(const float* y, int64_t groups, int bits, uint32_t* codes,
                                   uint8_t* coset, cudaStream_t stream);

int64_t entropy_streams(int units, int heads, int64_t n);
int64_t entropy_max_words(int units, int heads, int64_t n);
size_t entropy_workspace_bytes(int units, int heads, int64_t n);
cudaError_t launch_entropy_encode(const nq_packed& in, int units, int heads, int64_t n,
                                  int64_t slot0, int delta, uint16_t* freq, uint32_t* offsets,
                                  uint16_t* words, void* ws, cudaStream_t stream);
cudaError_t launch_entropy_decode(const uint16_t* words, const uint32_t* offsets,
                                  const uint16_t* freq, int units, int heads, int64_t n,
                                  int delta, const nq_packed& out, int64_t slot0,
                                  cudaStream_t stream);

cudaError_t launch_score(const void* K, nq_kv_strides ks, int units, int heads, int64_t T, int W,
                         double* scores, float* mean_ws, cudaStream_t stream);
cudaError_t launch_score_static(const void* K, nq_kv_strides ks, int units, int heads, int64_t T,
                                int W, double* scores, cudaStream_t stream);
cudaError_t launch_select(const double* scores, int units, int64_t T, int W, int evict_pct,
                          int64_t n_kept, int32_t* kept, int64_t kept_stride,
                          cudaStream_t stream);

}  // namespace nq
