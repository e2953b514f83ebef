// Internal host-side interfaces between the C ABI layer and the kernels.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "token_map.cuh"

#ifndef FPATTN_MAX_DEVICES
#define FPATTN_MAX_DEVICES 64
#endif
constexpr int kMaxDevices = FPATTN_MAX_DEVICES;

namespace fpattn {

// SM count of the current device, cached per device (a process may drive
// several GPUs, one after another or from several threads).
inline int device_sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= kMaxDevices) {
    int n = 148;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
  }
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    n = 148;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// tmap: NULL when x is already in the order the codes take; otherwise x is
// read in raster order and the codes are written in tile-major order.
cudaError_t launch_quantize_fp8_tile(const void* x, int BH, int N, int d, uint8_t* codes, float* scales,
                                     int* nonfinite, const TokenMap* tmap, cudaStream_t st);
// NVFP4 V with 16-token blocks along the sequence, transposed: codes
// [BH][d][ceil(N/128)*64] bytes, scales [BH][ceil(N/128)][2][512].
cudaError_t launch_quantize_nvfp4_tokens(const void* x, int BH, int N, int d, const float* static_amax,
                                         uint8_t* codes, uint8_t* block_sf, float* tensor_scale, int* nonfinite,
                                         const TokenMap* tmap, cudaStream_t st);
// One scale per group of `group` consecutive 128-token tiles (group 1: per tile).
cudaError_t launch_quantize_fp8_group(const void* x, int BH, int N, int d, int group, uint8_t* codes,
                                      float* scales, int* nonfinite, const TokenMap* tmap, cudaStream_t st);
cudaError_t launch_quantize_fp8_channel(const void* x, int BH, int N, int d, uint8_t* codes, float* scales,
                                        int* nonfinite, const TokenMap* tmap, cudaStream_t st);
cudaError_t launch_quantize_nvfp4(const void* x, int BH, int N, int d, const float* static_amax,
                                  uint8_t* codes, uint8_t* block_sf, float* tensor_scale, int* nonfinite,
                                  const TokenMap* tmap, cudaStream_t st);

// max|x| folded into *amax (zeroed first unless accumulate).
cudaError_t launch_tensor_amax_accum(const void* x, int BH, int N, int d, bool accumulate, float* amax, int* nonfinite,
                               cudaStream_t st);
// Q, K (NVFP4 when qk_fp4, else FP8 per 128-token tile) and V (FP8 per
// channel) in four launches; results equal the separate launchers'.
cudaError_t launch_quantize_qkv(const void* q, const void* k, const void* v, int BH, int N, int d, bool qk_fp4,
                                uint8_t* q_codes, uint8_t* q_sf, float* q_scale, uint8_t* k_codes, uint8_t* k_sf,
                                float* k_scale, uint8_t* v_codes, float* v_scales, int* nonfinite,
                                const TokenMap* tmap, cudaStream_t st);

// Video grid and tile of a tile-major token order.
struct VideoLayout {
  int T, Hs, W;
  int tt, th, tw;
};

// Box (w, h, t extents) that one 32-row chunk of a 128-token block covers in
// the raster grid. False when the layout does not cut every such chunk into a
// box, or the tile volume is not a multiple of 128.
inline bool video_chunk_box(const VideoLayout& v, int& bw, int& bh, int& bt) {
  const int plane = v.th * v.tw;
  if ((v.tt * plane) % 128 != 0) return false;
  if (v.tw >= 32) {
    if (v.tw % 32 != 0) return false;
    bw = 32, bh = 1, bt = 1;
  } else if (plane >= 32) {
    if (32 % v.tw != 0 || v.th % (32 / v.tw) != 0) return false;
    bw = v.tw, bh = 32 / v.tw, bt = 1;
  } else {
    if (32 % plane != 0 || v.tt % (32 / plane) != 0) return false;
    bw = v.tw, bh = v.th, bt = 32 / plane;
  }
  return true;
}

struct AttnArgs {
  const void* q;  // codes
  const void* k;
  const void* v;
  const uint8_t* q_sf;  // NVFP4 block scales (tensor-core layout) or null
  const uint8_t* k_sf;
  const uint8_t* v_sf;  // NVFP4 V block scales [BH][nkb][2][512] (pv_fp4)
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  void* out;   // bf16
  float* lse;  // or null
  const int32_t* row_ptr;  // tile mask CSR or null
  const int32_t* col_idx;
  const int32_t* row_order;
  int nnz;  // entries of col_idx
  int B, H, N, d;
  bool qk_fp4;
  bool pv_fp4;  // P and V in NVFP4: v is transposed NVFP4 codes, v_scale its tensor scale
  bool causal;
  float softmax_scale;
  float rescale_threshold;  // tau in [0, 8], log2 units
  // Non-null: Q, K, V are in tile-major order and out / lse are written back
  // in raster order of this video layout (validated by video_chunk_box).
  const VideoLayout* video;
};

// Returns cudaErrorNotSupported when the driver's tensor-map encoder is
// unavailable, other errors as produced by the CUDA runtime.
cudaError_t launch_attn_fwd(const AttnArgs& a, cudaStream_t st);

// Causal schedule of an attention launch over BH (batch, head) problems of N
// tokens on `grid` CTAs. Either heads in groups (hgroup heads a group, gspan
// positions a full group, items plus padding; hpairs = 0), or pairs of query
// blocks head by head (hpairs pairs a head). num_items: all positions of the
// launch. Host only.
struct CausalPlan {
  int hgroup, gspan, hpairs, num_items;
};
void causal_plan(int BH, int N, int D, bool qk_fp4, bool pv_fp4, int grid, CausalPlan* plan);

// Device error word access (defined next to the kernels).
cudaError_t read_device_error(cudaStream_t st, int clear, int* code);

}  // namespace fpattn
