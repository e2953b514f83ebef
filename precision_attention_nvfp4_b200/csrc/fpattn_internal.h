// Internal host-side interfaces between the C ABI layer and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace fpattn {

cudaError_t launch_quantize_fp8_tile(const void* x, int BH, int N, int d, uint8_t* codes, float* scales,
                                     int* nonfinite, cudaStream_t st);
cudaError_t launch_quantize_fp8_channel(const void* x, int BH, int N, int d, uint8_t* codes, float* scales,
                                        int* nonfinite, cudaStream_t st);
cudaError_t launch_quantize_nvfp4(const void* x, int BH, int N, int d, const float* static_amax,
                                  uint8_t* codes, uint8_t* block_sf, float* tensor_scale, int* nonfinite,
                                  cudaStream_t st);

struct AttnArgs {
  const void* q;  // codes
  const void* k;
  const void* v;
  const uint8_t* q_sf;  // NVFP4 block scales (tensor-core layout) or null
  const uint8_t* k_sf;
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  void* out;   // bf16
  float* lse;  // or null
  const int32_t* row_ptr;  // tile mask CSR or null
  const int32_t* col_idx;
  const int32_t* row_order;
  int B, H, N, d;
  bool qk_fp4;
  bool causal;
  float softmax_scale;
};

// Returns cudaErrorNotSupported when the driver's tensor-map encoder is
// unavailable, other errors as produced by the CUDA runtime.
cudaError_t launch_attn_fwd(const AttnArgs& a, cudaStream_t st);

// Device error word access (defined next to the kernels).
cudaError_t read_device_error(cudaStream_t st, int clear, int* code);

}  // namespace fpattn
