// Quantize kernels: bf16 [B,H,N,d] -> NVFP4 (packed E2M1 + E4M3 block scales
// + FP32 tensor scale) or FP8 E4M3 (per-128-token-tile or per-channel
// scales).
//
// NVFP4 follows the micro-scaling scheme of the Blackwell FP4 practice page
// (section 1: values divided by a block scale and rounded to FP4, the scale
// itself stored in FP8). FP8 follows the FPSAttention conversion formula
// (section 2.1) and staged granularities (section 3.1).
//
// With a video token map the kernels read raster-order (time-major) input
// and write codes and scales in tile-major order, so the permutation costs no
// pass of its own (FPSAttention page, section 3.3, item 1).
//
// Also here: NVFP4 V with its blocks along the sequence (for the all-NVFP4
// P V product), and FP8 Q/K with one scale per group of tiles (the coarser
// granularities of the denoising-step schedule, FPSAttention page, section
// 3.2). Every kernel takes part in the programmatic launch chain (see
// griddep_wait).
//
// All kernels are bandwidth-bound streams: 16-byte loads per thread,
// consecutive threads on consecutive 16-byte chunks, warp-shuffle reductions.
// Every scale step is one correctly rounded fp32 operation (__fdiv_rn,
// __fmul_rn: never contracted into an FMA) so the codes are bit-exact against
// the CPU oracle, and the element conversions use the hardware's
// round-to-nearest-even, saturating cvt instructions.
#include <cfloat>
#include <cstdint>
#include <cuda_fp16.h>

#include "fpattn_internal.h"
#include "sm100.cuh"
#include "token_map.cuh"

namespace fpattn {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
  f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
  f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// max |x| over 8 bf16 values; *bad |= non-finite seen.
__device__ __forceinline__ float amax8(const uint4& v, bool* bad) {
  float f[8];
  unpack8(v, f);
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float a = fabsf(f[i]);
    *bad |= !(a <= FLT_MAX);
    m = fmaxf(m, a);
  }
  return m;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide max over kThreads threads; result valid in all threads.
__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < kThreads / 32; ++i) r = fmaxf(r, red[i]);
  __syncthreads();
  return r;
}

// s = 448 / A (fp32, correctly rounded); 1 when A == 0.
__device__ __forceinline__ float fp8_scale_from_amax(float a) { return a == 0.f ? 1.f : __fdiv_rn(448.f, a); }

// 8 bf16 * s -> 8 E4M3 codes packed in a uint2 (element 0 in the low byte).
__device__ __forceinline__ uint2 quant8_e4m3(const uint4& v, float s) {
  float f[8];
  unpack8(v, f);
  uint2 r;
  r.x = static_cast<uint32_t>(cvt_e4m3x2(__fmul_rn(f[0], s), __fmul_rn(f[1], s))) |
        (static_cast<uint32_t>(cvt_e4m3x2(__fmul_rn(f[2], s), __fmul_rn(f[3], s))) << 16);
  r.y = static_cast<uint32_t>(cvt_e4m3x2(__fmul_rn(f[4], s), __fmul_rn(f[5], s))) |
        (static_cast<uint32_t>(cvt_e4m3x2(__fmul_rn(f[6], s), __fmul_rn(f[7], s))) << 16);
  return r;
}

// ---------------------------------------------------------------------------
// FP8, one scale per (b, h, 128-token tile). grid = (ceil(N/128), B*H).
// The tile (<= 128 x 128 bf16 = 32 KiB) stays in registers between the amax
// reduction and the conversion, so x is read from HBM exactly once. With a
// token map (kMap) the tile's 128 source rows are looked up once into shared
// memory.
//
// Grouped scales (one scale for several consecutive tiles) run the same
// kernel twice around fp8_group_finalize_kernel: kAmaxOnly writes each tile's
// amax into its scale slot, kConvert converts with the scale found there.
// ---------------------------------------------------------------------------
enum TileMode { kFused = 0, kAmaxOnly = 1, kConvert = 2 };

// Body of one CTA: tile `tile` of (b, h) = bh, ntiles tiles per (b, h).
template <int D, bool kMap, int kMode>
__device__ __forceinline__ void fp8_tile_body(const uint4* __restrict__ x, int N, uint2* __restrict__ codes,
                                              float* __restrict__ scales, int* nonfinite, const TokenMap& tmap,
                                              int tile, size_t bh, int ntiles) {
  constexpr int kChunksPerRow = D / 8;
  constexpr int kChunks = 128 * kChunksPerRow;  // 16-byte chunks per full tile
  constexpr int kPer = kChunks / kThreads;
  __shared__ float red[kThreads / 32];
  __shared__ int src_row[kMap ? 128 : 1];
  const int rows = min(128, N - tile * 128);
  const size_t base = (bh * N + static_cast<size_t>(tile) * 128) * kChunksPerRow;
  if (kMap) {
    if (threadIdx.x < rows) src_row[threadIdx.x] = to_raster(tmap, tile * 128 + threadIdx.x);
    __syncthreads();
  }
  uint4 v[kPer];
  float m = 0.f;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int c = threadIdx.x + i * kThreads;
    if (c / kChunksPerRow < rows) {
      v[i] = kMap ? x[(bh * N + src_row[c / kChunksPerRow]) * kChunksPerRow + c % kChunksPerRow] : x[base + c];
      if (kMode != kConvert) m = fmaxf(m, amax8(v[i], &bad));
    }
  }
  float s;
  if (kMode == kConvert) {
    s = scales[bh * ntiles + tile];
  } else {
    if (bad && nonfinite) atomicExch(nonfinite, 1);
    const float a = block_max(m, red);
    if (kMode == kAmaxOnly) {
      if (threadIdx.x == 0) scales[bh * ntiles + tile] = a;
      return;
    }
    s = fp8_scale_from_amax(a);
    if (threadIdx.x == 0) scales[bh * ntiles + tile] = s;
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int c = threadIdx.x + i * kThreads;
    if (c / kChunksPerRow < rows) codes[base + c] = quant8_e4m3(v[i], s);
  }
}

template <int D, bool kMap, int kMode = kFused>
__global__ void __launch_bounds__(kThreads) fp8_tile_kernel(const uint4* __restrict__ x, int N,
                                                            uint2* __restrict__ codes, float* __restrict__ scales,
                                                            int* nonfinite, TokenMap tmap) {
  griddep_wait();
  fp8_tile_body<D, kMap, kMode>(x, N, codes, scales, nonfinite, tmap, blockIdx.x, blockIdx.y, gridDim.x);
  griddep_launch_dependents();
}

// One thread per (b*h, group of `group` tiles): the group's amax is the max of
// its tiles' amaxes (left in the scale slots by the kAmaxOnly pass); every
// tile of the group gets s = 448 / amax.
__global__ void fp8_group_finalize_kernel(float* __restrict__ scales, int nblk, int group, int ngroups,
                                          int total) {
  griddep_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  float* sc = scales + static_cast<size_t>(i / ngroups) * nblk;
  const int b0 = (i % ngroups) * group;
  const int b1 = min(nblk, b0 + group);
  float a = 0.f;
  for (int b = b0; b < b1; ++b) a = fmaxf(a, sc[b]);
  const float s = fp8_scale_from_amax(a);
  for (int b = b0; b < b1; ++b) sc[b] = s;
  griddep_launch_dependents();
}

// ---------------------------------------------------------------------------
// FP8, one scale per (b, h, channel), amax over all N tokens.
// Pass 1 reduces per-channel amax of a token chunk and folds it into
// amax[bh, c] with an integer atomicMax (valid for non-negative floats).
// Pass 2 converts with s_c = 448 / amax_c. Pass 3 turns amax into s in place.
// grid = (ceil(N / kRowsPerCta), B*H).
// ---------------------------------------------------------------------------
constexpr int kRowsPerCta = 256;

// Body of one CTA: rows [256 bx, 256 bx + 256) of (b, h) = bh.
template <int D>
__device__ __forceinline__ void fp8_channel_amax_body(const uint4* __restrict__ x, int N, float* __restrict__ amax,
                                                      int* nonfinite, int bx, size_t bh) {
  constexpr int kCpr = D / 8;                 // chunks per row
  constexpr int kRowsPerIter = kThreads / kCpr;
  __shared__ float part[kRowsPerIter][D];
  const int r0 = bx * kRowsPerCta;
  const int cg = threadIdx.x % kCpr;          // channel group of 8
  const int rr = threadIdx.x / kCpr;
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = 0.f;
  bool bad = false;
  const int rend = min(N, r0 + kRowsPerCta);
#pragma unroll 4
  for (int r = r0 + rr; r < rend; r += kRowsPerIter) {
    const uint4 v = x[(bh * N + r) * kCpr + cg];
    float f[8];
    unpack8(v, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float a = fabsf(f[i]);
      bad |= !(a <= FLT_MAX);
      m[i] = fmaxf(m[i], a);
    }
  }
  if (bad && nonfinite) atomicExch(nonfinite, 1);
#pragma unroll
  for (int i = 0; i < 8; ++i) part[rr][cg * 8 + i] = m[i];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += kThreads) {
    float a = 0.f;
#pragma unroll 4
    for (int j = 0; j < kRowsPerIter; ++j) a = fmaxf(a, part[j][c]);
    atomicMax(reinterpret_cast<int*>(amax) + bh * D + c, __float_as_int(a));
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads) fp8_channel_amax_kernel(const uint4* __restrict__ x, int N,
                                                                    float* __restrict__ amax, int* nonfinite) {
  griddep_wait();
  fp8_channel_amax_body<D>(x, N, amax, nonfinite, blockIdx.x, blockIdx.y);
  griddep_launch_dependents();
}

// The amax pass is order-free, so only the conversion pass reads through the
// token map (output row r, tile-major, from source row to_raster(r)).
template <int D, bool kMap>
__device__ __forceinline__ void fp8_channel_quant_body(const uint4* __restrict__ x, int N,
                                                       const float* __restrict__ amax, uint2* __restrict__ codes,
                                                       const TokenMap& tmap, int bx, size_t bh) {
  constexpr int kCpr = D / 8;
  constexpr int kRowsPerIter = kThreads / kCpr;
  static_assert(kRowsPerCta == kThreads, "one source-row lookup per thread");
  __shared__ int src_row[kMap ? kRowsPerCta : 1];
  const int r0 = bx * kRowsPerCta;
  const int cg = threadIdx.x % kCpr;
  const int rr = threadIdx.x / kCpr;
  const int rend = min(N, r0 + kRowsPerCta);
  if (kMap) {
    if (r0 + static_cast<int>(threadIdx.x) < rend) src_row[threadIdx.x] = to_raster(tmap, r0 + threadIdx.x);
    __syncthreads();
  }
  // four rows' loads are issued before any of them is converted, so that a
  // thread keeps 64 bytes in flight
  constexpr int kBatch = 4;
  uint4 v[kBatch];
#pragma unroll
  for (int u = 0; u < kBatch; ++u) {
    const int ru = r0 + rr + u * kRowsPerIter;
    v[u] = ru < rend ? x[(bh * N + (kMap ? src_row[ru - r0] : ru)) * kCpr + cg] : make_uint4(0u, 0u, 0u, 0u);
  }
  float s[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) s[i] = fp8_scale_from_amax(amax[bh * D + cg * 8 + i]);
  for (int r = r0 + rr; r < rend; r += kBatch * kRowsPerIter) {
    uint4 nxt[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int ru = r + (kBatch + u) * kRowsPerIter;
      nxt[u] = ru < rend ? x[(bh * N + (kMap ? src_row[ru - r0] : ru)) * kCpr + cg] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int ru = r + u * kRowsPerIter;
      if (ru < rend) {
        float f[8];
        unpack8(v[u], f);
        uint2 o;
        o.x = static_cast<uint32_t>(cvt_e4m3x2(__fmul_rn(f[0], s[0]), __fmul_rn(f[1], s[1]))) |
              (static_cast<uint32_t>(cvt_e4m3x2(__fmul_rn(f[2], s[2]), __fmul_rn(f[3], s[3]))) << 16);
        o.y = static_cast<uint32_t>(cvt_e4m3x2(__fmul_rn(f[4], s[4]), __fmul_rn(f[5], s[5]))) |
              (static_cast<uint32_t>(cvt_e4m3x2(__fmul_rn(f[6], s[6]), __fmul_rn(f[7], s[7]))) << 16);
        codes[(bh * N + ru) * kCpr + cg] = o;
      }
      v[u] = nxt[u];
    }
  }
}

template <int D, bool kMap>
__global__ void __launch_bounds__(kThreads) fp8_channel_quant_kernel(const uint4* __restrict__ x, int N,
                                                                     const float* __restrict__ amax,
                                                                     uint2* __restrict__ codes, TokenMap tmap) {
  griddep_wait();
  fp8_channel_quant_body<D, kMap>(x, N, amax, codes, tmap, blockIdx.x, blockIdx.y);
  griddep_launch_dependents();
}

__global__ void fp8_channel_finalize_kernel(float* __restrict__ s, int n) {
  griddep_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) s[i] = fp8_scale_from_amax(s[i]);
  griddep_launch_dependents();
}

// ---------------------------------------------------------------------------
// NVFP4.
// Pass 1 (dynamic only): tensor amax -> *amax_out via integer atomicMax.
// Pass 2 (nvfp4_quant_kernel), per 16-element block along d:
//   s_t = A_t / 2688 (1 if A_t == 0)
//   sb  = E4M3(A_b / (6 * s_t)), den = dec(sb) * s_t, inv = 1 / den,
//   code = E2M1(x * inv)   (all zero when den == 0 or inv is not finite)
//   codes in place of x's elements, scales in the tensor-core scale layout
//   (zero for the rows that pad N up to 128).
// Pass 3: *tensor_scale = s_t.
// ---------------------------------------------------------------------------
// Body of CTA `block` of `nblocks` reducing |x| over nchunks 16-byte chunks
// (grid-stride) into *amax_out.
__device__ __forceinline__ void tensor_amax_body(const uint4* __restrict__ x, size_t nchunks,
                                                 float* __restrict__ amax_out, int* nonfinite, int block,
                                                 int nblocks) {
  __shared__ float red[kThreads / 32];
  float m = 0.f;
  bool bad = false;
  const size_t stride = static_cast<size_t>(nblocks) * kThreads;
  size_t c = block * static_cast<size_t>(kThreads) + threadIdx.x;
  // four loads in flight per thread
  for (; c + 3 * stride < nchunks; c += 4 * stride) {
    const uint4 v0 = x[c], v1 = x[c + stride], v2 = x[c + 2 * stride], v3 = x[c + 3 * stride];
    m = fmaxf(fmaxf(m, amax8(v0, &bad)), fmaxf(amax8(v1, &bad), fmaxf(amax8(v2, &bad), amax8(v3, &bad))));
  }
  for (; c < nchunks; c += stride) m = fmaxf(m, amax8(x[c], &bad));
  if (bad && nonfinite) atomicExch(nonfinite, 1);
  m = block_max(m, red);
  if (threadIdx.x == 0) atomicMax(reinterpret_cast<int*>(amax_out), __float_as_int(m));
}

__global__ void __launch_bounds__(kThreads) tensor_amax_kernel(const uint4* __restrict__ x, size_t nchunks,
                                                               float* __restrict__ amax_out, int* nonfinite) {
  griddep_wait();
  tensor_amax_body(x, nchunks, amax_out, nonfinite, blockIdx.x, gridDim.x);
  griddep_launch_dependents();
}

__device__ __forceinline__ float nvfp4_tensor_scale(float amax) {
  return amax == 0.f ? 1.f : __fdiv_rn(amax, 2688.f);
}

// One warp per 128 consecutive 16-byte chunks (8 rows at D = 128, 16 at
// D = 64), that is 64 16-element scale blocks: lane i takes blocks i and
// i + 32, each whole (two adjacent chunks), so the scale of a block is worked
// out once, by the lane that converts it. Each load instruction covers 1 KB
// of contiguous rows; each lane writes the 8 code bytes of a block (a warp
// store covers 256 contiguous bytes) and its scale byte.
// grid = (nblk * 128 / kRowsPerCta, B*H): rows are padded to 128 per (b, h),
// and the padding rows only write zero scales.
template <int D, bool kMap>
__device__ __forceinline__ void nvfp4_quant_body(const uint4* __restrict__ x, int N, int nblk,
                                                 const float* __restrict__ amax_ptr, uint32_t* __restrict__ codes,
                                                 uint8_t* __restrict__ sf, const TokenMap& tmap, int bx, int bh) {
  constexpr int kCpr = D / 8;                // 16-byte chunks per row
  constexpr int kBpr = D / 16;               // 16-element scale blocks per row
  constexpr int kRowsPerWarp = 128 / kCpr;   // 8 or 16
  constexpr int kGroups = D / 64;            // 512-byte scale groups per 128-row block
  const int lane = threadIdx.x & 31;
  const int r0 = (bx * (kThreads / 32) + (threadIdx.x >> 5)) * kRowsPerWarp;
  int src = 0;
  if (kMap && lane < kRowsPerWarp && r0 + lane < N) src = to_raster(tmap, r0 + lane);
  // lane takes blocks lane and lane + 32 of the warp's rows: each a whole
  // 16-element scale block (two 16-byte chunks), all four loads issued first
  uint4 v[2][2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int blk = 32 * k + lane;
    const int rl = blk / kBpr;
    const int srow = kMap ? __shfl_sync(0xffffffffu, src, rl) : r0 + rl;
    const size_t base = (static_cast<size_t>(bh) * N + srow) * kCpr + 2 * (blk % kBpr);
#pragma unroll
    for (int h = 0; h < 2; ++h) v[k][h] = r0 + rl < N ? x[base + h] : make_uint4(0u, 0u, 0u, 0u);
  }
  const float s_t = nvfp4_tensor_scale(*amax_ptr);
  const float six_st = __fmul_rn(6.f, s_t);
  uint2* codes2 = reinterpret_cast<uint2*>(codes);
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int blk = 32 * k + lane;
    const int r = r0 + blk / kBpr;
    const int col = blk % kBpr;
    float f[16];
    unpack8(v[k][0], f);
    unpack8(v[k][1], f + 8);
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(f[i]));
    const uint32_t sb = cvt_e4m3x2(__fdiv_rn(a, six_st), 0.f) & 0xFFu;
    const float den = __fmul_rn(e4m3_to_float(sb), s_t);
    const float inv = __fdiv_rn(1.f, den);
    const bool usable = (den != 0.f) && (fabsf(inv) <= FLT_MAX);
    // an unusable scale (zero block, or 1/den not finite) gives zero codes,
    // so the products need no select of their own
    float y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(f[i], inv);
    if (r < N)
      codes2[(static_cast<size_t>(bh) * N + r) * kBpr + col] =
          usable ? make_uint2(cvt_e2m1x8(y), cvt_e2m1x8(y + 8)) : make_uint2(0u, 0u);
    // row r = 128 nb + 32 j + i, scale column col = 4 grp + s: byte
    // 16 i + 4 j + s of the 512-byte group (bh, nb, grp)
    const int rr = r & 127;
    const size_t byte = ((static_cast<size_t>(bh) * nblk + (r >> 7)) * kGroups + (col >> 2)) * 512 +
                        16 * (rr & 31) + 4 * (rr >> 5) + (col & 3);
    sf[byte] = r < N ? static_cast<uint8_t>(sb) : 0u;
  }
}

template <int D, bool kMap>
__global__ void __launch_bounds__(kThreads) nvfp4_quant_kernel(const uint4* __restrict__ x, int N, int nblk,
                                                               const float* __restrict__ amax_ptr,
                                                               uint32_t* __restrict__ codes,
                                                               uint8_t* __restrict__ sf, TokenMap tmap) {
  griddep_wait();
  nvfp4_quant_body<D, kMap>(x, N, nblk, amax_ptr, codes, sf, tmap, blockIdx.x, blockIdx.y);
  griddep_launch_dependents();
}

// NVFP4 V for a block-scaled P V product: 16-token blocks along the sequence.
// grid = (ceil(N/128), B*H), D threads. Thread t takes channels 2*(t % (D/2))
// and +1 over tokens 64*(t / (D/2)) .. +63 of the key block: per channel four
// 16-token blocks -> 32 code bytes of the transposed row and one 32-bit word
// of block scales. Output, per (b, h): codes [D][nkb*64] (channel-major, two
// tokens per byte, zero past N) and scales [nkb][2][512] in the tensor-core
// scale layout with channels as rows. Same fp32 operation sequence as
// nvfp4_quant_kernel, so the codes are bit-exact against the oracle.
template <int D, bool kMap>
__global__ void __launch_bounds__(D) nvfp4_tokens_quant_kernel(const uint32_t* __restrict__ x, int N, int nkb,
                                                              const float* __restrict__ amax_ptr,
                                                              uint8_t* __restrict__ codes,
                                                              uint32_t* __restrict__ sf, TokenMap tmap) {
  griddep_wait();
  constexpr int kPairs = D / 2;
  __shared__ int src_row[kMap ? 128 : 1];
  const int kb = blockIdx.x;
  const size_t bh = blockIdx.y;
  const int pair = threadIdx.x % kPairs;
  const int half = threadIdx.x / kPairs;
  if (kMap) {
    for (int i = threadIdx.x; i < 128; i += D) src_row[i] = kb * 128 + i < N ? to_raster(tmap, kb * 128 + i) : 0;
    __syncthreads();
  }
  const float s_t = nvfp4_tensor_scale(*amax_ptr);
  const float six_st = __fmul_rn(6.f, s_t);
  uint32_t cw[2][8];  // [channel of the pair][word]: 4 blocks x 8 codes each = 32 bytes per channel
  uint32_t sfw[2] = {0u, 0u};
#pragma unroll
  for (int blk = 0; blk < 4; ++blk) {
    float f[2][16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int tl = half * 64 + blk * 16 + k;  // token within the key block
      const int n = kb * 128 + tl;
      uint32_t w = 0u;
      if (n < N) {
        const size_t row = bh * N + (kMap ? src_row[tl] : n);
        w = x[row * kPairs + pair];
      }
      f[0][k] = bf16_lo(w);
      f[1][k] = bf16_hi(w);
    }
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      float a = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) a = fmaxf(a, fabsf(f[ch][k]));
      const uint32_t sb = cvt_e4m3x2(__fdiv_rn(a, six_st), 0.f) & 0xFFu;
      const float den = __fmul_rn(e4m3_to_float(sb), s_t);
      const float inv = __fdiv_rn(1.f, den);
      const bool usable = (den != 0.f) && (fabsf(inv) <= FLT_MAX);
      float y[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) y[k] = usable ? __fmul_rn(f[ch][k], inv) : 0.f;
      cw[ch][2 * blk] = usable ? cvt_e2m1x8(y) : 0u;
      cw[ch][2 * blk + 1] = usable ? cvt_e2m1x8(y + 8) : 0u;
      sfw[ch] |= sb << (8 * blk);
    }
  }
  const size_t pitch = static_cast<size_t>(nkb) * 64;
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    const int c = 2 * pair + ch;
    uint4* dst = reinterpret_cast<uint4*>(codes + (bh * D + c) * pitch + kb * 64 + half * 32);
    dst[0] = make_uint4(cw[ch][0], cw[ch][1], cw[ch][2], cw[ch][3]);
    dst[1] = make_uint4(cw[ch][4], cw[ch][5], cw[ch][6], cw[ch][7]);
    // channel c = 32 j + i, scale columns 4*half .. +3 of the key block:
    // bytes 16 i + 4 j .. +3 of the block's 512-byte group `half`
    uint32_t* group = sf + ((bh * nkb + kb) * 2 + half) * 128;
    group[(c & 31) * 4 + (c >> 5)] = sfw[ch];
    if (D == 64) group[(c & 31) * 4 + (c >> 5) + 2] = 0u;  // rows 64..127 of the layout are zero
  }
  griddep_launch_dependents();
}

// ---------------------------------------------------------------------------
// Q, K and V of one attention call in four launches: zero the accumulators,
// one amax pass over all three tensors, one conversion pass, one finalize.
// Each CTA runs the body of the stand-alone kernel for its share (the block
// index picks the tensor), so the codes and scales are those of the separate
// calls, bit for bit. With FP8 Q/K the per-tile quantization is one pass and
// runs in the amax launch.
// ---------------------------------------------------------------------------
struct QkvParams {
  const uint4* q;
  const uint4* k;
  const uint4* v;
  int N, BH, nblk;
  void* q_codes;       // NVFP4: packed E2M1 words; FP8: E4M3 bytes
  void* k_codes;
  uint8_t* q_sf;       // NVFP4 block scales (tensor-core layout)
  uint8_t* k_sf;
  float* q_scale;      // NVFP4: amax accumulator, then s_t; FP8: per-tile scales
  float* k_scale;
  uint2* v_codes;
  float* v_scales;     // amax accumulators, then per-channel scales
  int* nonfinite;
  TokenMap tmap;
  int amax_ctas;       // NVFP4: CTAs per tensor in the tensor-amax share
  int vgx;             // channel passes: CTAs per (b, h) (256 rows each)
  int qgx;             // NVFP4 conversion: CTAs per (b, h)
};

template <int D, bool kMap, bool kFp4>
__global__ void __launch_bounds__(kThreads) qkv_amax_kernel(const __grid_constant__ QkvParams p) {
  griddep_wait();
  int b = blockIdx.x;
  const int nqk = kFp4 ? p.amax_ctas : p.nblk * p.BH;  // CTAs of the Q share (and of the K share)
  if (b < 2 * nqk) {
    const bool isq = b < nqk;
    const int bb = isq ? b : b - nqk;
    if (kFp4) {
      tensor_amax_body(isq ? p.q : p.k, static_cast<size_t>(p.BH) * p.N * (D / 8), isq ? p.q_scale : p.k_scale,
                       p.nonfinite, bb, nqk);
    } else {
      fp8_tile_body<D, kMap, kFused>(isq ? p.q : p.k, p.N, static_cast<uint2*>(isq ? p.q_codes : p.k_codes),
                                     isq ? p.q_scale : p.k_scale, p.nonfinite, p.tmap, bb % p.nblk, bb / p.nblk,
                                     p.nblk);
    }
  } else {
    b -= 2 * nqk;
    fp8_channel_amax_body<D>(p.v, p.N, p.v_scales, p.nonfinite, b % p.vgx, b / p.vgx);
  }
  griddep_launch_dependents();
}

// Resident CTAs a SM the conversion kernel is compiled for: its loads are
// issued before the arithmetic, so more warps keep more of them in flight.
#ifndef FPATTN_CONVERT_CTAS
#define FPATTN_CONVERT_CTAS 5
#endif
constexpr int kConvertCtasPerSm = FPATTN_CONVERT_CTAS;

// V first, then K, then Q: the reverse of the amax pass, whose last reads are
// the likeliest to be still in L2.
template <int D, bool kMap, bool kFp4>
__global__ void __launch_bounds__(kThreads, kConvertCtasPerSm) qkv_convert_kernel(const __grid_constant__ QkvParams p) {
  griddep_wait();
  int b = blockIdx.x;
  const int nv = p.vgx * p.BH;
  if (b < nv) {
    fp8_channel_quant_body<D, kMap>(p.v, p.N, p.v_scales, p.v_codes, p.tmap, b % p.vgx, b / p.vgx);
  } else if (kFp4) {
    b -= nv;
    const int nq = p.qgx * p.BH;
    const bool isk = b < nq;
    const int bb = isk ? b : b - nq;
    nvfp4_quant_body<D, kMap>(isk ? p.k : p.q, p.N, p.nblk, isk ? p.k_scale : p.q_scale,
                              static_cast<uint32_t*>(isk ? p.k_codes : p.q_codes), isk ? p.k_sf : p.q_sf, p.tmap,
                              bb % p.qgx, bb / p.qgx);
  }
  griddep_launch_dependents();
}

// amax -> scale in place: s_t = A/2688 for NVFP4 Q and K (thread 0), 448/A
// per V channel.
template <bool kFp4>
__global__ void qkv_finalize_kernel(float* __restrict__ q_scale, float* __restrict__ k_scale,
                                    float* __restrict__ v_scales, int nv) {
  griddep_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (kFp4 && i == 0) {
    *q_scale = nvfp4_tensor_scale(*q_scale);
    *k_scale = nvfp4_tensor_scale(*k_scale);
  }
  if (i < nv) v_scales[i] = fp8_scale_from_amax(v_scales[i]);
  griddep_launch_dependents();
}

// Zeroes the accumulators of qkv_amax_kernel: a[0..na), b[0..nb), c[0..nc).
__global__ void zero3_kernel(float* __restrict__ a, int na, float* __restrict__ b, int nb, float* __restrict__ c,
                             int nc) {
  griddep_wait();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < na + nb + nc; i += gridDim.x * blockDim.x) {
    if (i < na) a[i] = 0.f;
    else if (i < na + nb) b[i - na] = 0.f;
    else c[i - na - nb] = 0.f;
  }
  griddep_launch_dependents();
}

// Zeroes n floats (the amax accumulators), as a kernel so that it takes
// part in the programmatic launch chain like every other step.
__global__ void zero_kernel(float* __restrict__ p, int n) {
  griddep_wait();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p[i] = 0.f;
  griddep_launch_dependents();
}

__global__ void nvfp4_finalize_kernel(const float* __restrict__ amax_ptr, float* __restrict__ tensor_scale) {
  griddep_wait();
  if (threadIdx.x == 0 && blockIdx.x == 0) *tensor_scale = nvfp4_tensor_scale(*amax_ptr);
  griddep_launch_dependents();
}

inline int num_sms() { return device_sm_count(); }

}  // namespace

// ---------------------------------------------------------------------------
// Host launchers (arguments already validated by the C ABI layer). Every
// launch goes through launch_pdl; the instantiation is picked first.
// ---------------------------------------------------------------------------
namespace {

// Zeroes the tensor-amax accumulator, then reduces |x| into it.
void launch_tensor_amax(const void* x, int BH, int N, int d, float* acc, int* nonfinite, cudaStream_t st) {
  launch_pdl(zero_kernel, dim3(1), dim3(32), 0, st, acc, 1);
  const size_t nchunks = static_cast<size_t>(BH) * N * d / 8;
  launch_pdl(tensor_amax_kernel, dim3(num_sms() * 8), dim3(kThreads), 0, st, static_cast<const uint4*>(x), nchunks,
             acc, nonfinite);
}

}  // namespace

cudaError_t launch_tensor_amax_accum(const void* x, int BH, int N, int d, bool accumulate, float* amax, int* nonfinite,
                               cudaStream_t st) {
  if (!accumulate) launch_pdl(zero_kernel, dim3(1), dim3(32), 0, st, amax, 1);
  const size_t nchunks = static_cast<size_t>(BH) * N * d / 8;
  launch_pdl(tensor_amax_kernel, dim3(num_sms() * 8), dim3(kThreads), 0, st, static_cast<const uint4*>(x), nchunks,
             amax, nonfinite);
  return cudaGetLastError();
}

cudaError_t launch_quantize_nvfp4_tokens(const void* x, int BH, int N, int d, const float* static_amax,
                                         uint8_t* codes, uint8_t* block_sf, float* tensor_scale, int* nonfinite,
                                         const TokenMap* tmap, cudaStream_t st) {
  const float* amax_ptr = static_amax;
  if (!static_amax) {
    // tensor_scale doubles as the amax accumulator until the finalize overwrites it
    launch_tensor_amax(x, BH, N, d, tensor_scale, nonfinite, st);
    amax_ptr = tensor_scale;
  }
  const int nkb = (N + 127) / 128;
  auto kern = d == 128 ? (tmap ? nvfp4_tokens_quant_kernel<128, true> : nvfp4_tokens_quant_kernel<128, false>)
                       : (tmap ? nvfp4_tokens_quant_kernel<64, true> : nvfp4_tokens_quant_kernel<64, false>);
  launch_pdl(kern, dim3(nkb, BH), dim3(d), 0, st, static_cast<const uint32_t*>(x), N, nkb, amax_ptr, codes,
             reinterpret_cast<uint32_t*>(block_sf), tmap ? *tmap : TokenMap{});
  launch_pdl(nvfp4_finalize_kernel, dim3(1), dim3(32), 0, st, amax_ptr, tensor_scale);
  return cudaGetLastError();
}

cudaError_t launch_quantize_fp8_tile(const void* x, int BH, int N, int d, uint8_t* codes, float* scales,
                                     int* nonfinite, const TokenMap* tmap, cudaStream_t st) {
  auto kern = d == 128 ? (tmap ? fp8_tile_kernel<128, true> : fp8_tile_kernel<128, false>)
                       : (tmap ? fp8_tile_kernel<64, true> : fp8_tile_kernel<64, false>);
  launch_pdl(kern, dim3((N + 127) / 128, BH), dim3(kThreads), 0, st, static_cast<const uint4*>(x), N,
             reinterpret_cast<uint2*>(codes), scales, nonfinite, tmap ? *tmap : TokenMap{});
  return cudaGetLastError();
}

namespace {

template <int D, bool kMap>
void launch_fp8_grouped(const uint4* xv, int BH, int N, int group, uint2* cv, float* scales, int* nonfinite,
                        const TokenMap& tm, cudaStream_t st) {
  const int nblk = (N + 127) / 128;
  const dim3 grid(nblk, BH);
  launch_pdl(fp8_tile_kernel<D, kMap, kAmaxOnly>, grid, dim3(kThreads), 0, st, xv, N, cv, scales, nonfinite, tm);
  const int ngroups = (nblk + group - 1) / group;
  const int total = BH * ngroups;
  launch_pdl(fp8_group_finalize_kernel, dim3((total + 255) / 256), dim3(256), 0, st, scales, nblk, group, ngroups,
             total);
  launch_pdl(fp8_tile_kernel<D, kMap, kConvert>, grid, dim3(kThreads), 0, st, xv, N, cv, scales, nonfinite, tm);
}

}  // namespace

cudaError_t launch_quantize_fp8_group(const void* x, int BH, int N, int d, int group, uint8_t* codes,
                                      float* scales, int* nonfinite, const TokenMap* tmap, cudaStream_t st) {
  if (group <= 1) return launch_quantize_fp8_tile(x, BH, N, d, codes, scales, nonfinite, tmap, st);
  const uint4* xv = static_cast<const uint4*>(x);
  uint2* cv = reinterpret_cast<uint2*>(codes);
  const TokenMap tm = tmap ? *tmap : TokenMap{};
  if (d == 128) {
    if (tmap) launch_fp8_grouped<128, true>(xv, BH, N, group, cv, scales, nonfinite, tm, st);
    else launch_fp8_grouped<128, false>(xv, BH, N, group, cv, scales, nonfinite, tm, st);
  } else {
    if (tmap) launch_fp8_grouped<64, true>(xv, BH, N, group, cv, scales, nonfinite, tm, st);
    else launch_fp8_grouped<64, false>(xv, BH, N, group, cv, scales, nonfinite, tm, st);
  }
  return cudaGetLastError();
}

cudaError_t launch_quantize_fp8_channel(const void* x, int BH, int N, int d, uint8_t* codes, float* scales,
                                        int* nonfinite, const TokenMap* tmap, cudaStream_t st) {
  const int n = BH * d;
  launch_pdl(zero_kernel, dim3((n + 255) / 256), dim3(256), 0, st, scales, n);
  const dim3 grid((N + kRowsPerCta - 1) / kRowsPerCta, BH);
  const uint4* xv = static_cast<const uint4*>(x);
  auto amax = d == 128 ? fp8_channel_amax_kernel<128> : fp8_channel_amax_kernel<64>;
  auto quant = d == 128 ? (tmap ? fp8_channel_quant_kernel<128, true> : fp8_channel_quant_kernel<128, false>)
                        : (tmap ? fp8_channel_quant_kernel<64, true> : fp8_channel_quant_kernel<64, false>);
  launch_pdl(amax, grid, dim3(kThreads), 0, st, xv, N, scales, nonfinite);
  launch_pdl(quant, grid, dim3(kThreads), 0, st, xv, N, static_cast<const float*>(scales),
             reinterpret_cast<uint2*>(codes), tmap ? *tmap : TokenMap{});
  launch_pdl(fp8_channel_finalize_kernel, dim3((n + 255) / 256), dim3(256), 0, st, scales, n);
  return cudaGetLastError();
}

cudaError_t launch_quantize_nvfp4(const void* x, int BH, int N, int d, const float* static_amax,
                                  uint8_t* codes, uint8_t* block_sf, float* tensor_scale, int* nonfinite,
                                  const TokenMap* tmap, cudaStream_t st) {
  const float* amax_ptr = static_amax;
  if (!static_amax) {
    // tensor_scale doubles as the amax accumulator until the finalize overwrites it
    launch_tensor_amax(x, BH, N, d, tensor_scale, nonfinite, st);
    amax_ptr = tensor_scale;
  }
  const int nblk = (N + 127) / 128;
  // rows per CTA: 8 warps x 128 chunks; 128 divides by it, so CTAs tile the padded rows
  const int rows_per_cta = (kThreads / 32) * (128 / (d / 8));
  auto kern = d == 128 ? (tmap ? nvfp4_quant_kernel<128, true> : nvfp4_quant_kernel<128, false>)
                       : (tmap ? nvfp4_quant_kernel<64, true> : nvfp4_quant_kernel<64, false>);
  launch_pdl(kern, dim3(nblk * 128 / rows_per_cta, BH), dim3(kThreads), 0, st, static_cast<const uint4*>(x), N,
             nblk, amax_ptr, reinterpret_cast<uint32_t*>(codes), block_sf, tmap ? *tmap : TokenMap{});
  launch_pdl(nvfp4_finalize_kernel, dim3(1), dim3(32), 0, st, amax_ptr, tensor_scale);
  return cudaGetLastError();
}

namespace {

template <int D, bool kMap, bool kFp4>
void launch_qkv(const QkvParams& p, cudaStream_t st) {
  const int nv = p.BH * D;
  launch_pdl(zero3_kernel, dim3((2 + nv + 255) / 256), dim3(256), 0, st, kFp4 ? p.q_scale : nullptr,
             kFp4 ? 1 : 0, kFp4 ? p.k_scale : nullptr, kFp4 ? 1 : 0, p.v_scales, nv);
  const int nqk = kFp4 ? p.amax_ctas : p.nblk * p.BH;
  launch_pdl(qkv_amax_kernel<D, kMap, kFp4>, dim3(2 * nqk + p.vgx * p.BH), dim3(kThreads), 0, st, p);
  launch_pdl(qkv_convert_kernel<D, kMap, kFp4>, dim3(p.vgx * p.BH + (kFp4 ? 2 * p.qgx * p.BH : 0)),
             dim3(kThreads), 0, st, p);
  launch_pdl(qkv_finalize_kernel<kFp4>, dim3((nv + 255) / 256), dim3(256), 0, st, p.q_scale, p.k_scale,
             p.v_scales, nv);
}

}  // namespace

cudaError_t launch_quantize_qkv(const void* q, const void* k, const void* v, int BH, int N, int d, bool qk_fp4,
                                uint8_t* q_codes, uint8_t* q_sf, float* q_scale, uint8_t* k_codes, uint8_t* k_sf,
                                float* k_scale, uint8_t* v_codes, float* v_scales, int* nonfinite,
                                const TokenMap* tmap, cudaStream_t st) {
  QkvParams p{};
  p.q = static_cast<const uint4*>(q);
  p.k = static_cast<const uint4*>(k);
  p.v = static_cast<const uint4*>(v);
  p.N = N;
  p.BH = BH;
  p.nblk = (N + 127) / 128;
  p.q_codes = q_codes;
  p.k_codes = k_codes;
  p.q_sf = q_sf;
  p.k_sf = k_sf;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.v_codes = reinterpret_cast<uint2*>(v_codes);
  p.v_scales = v_scales;
  p.nonfinite = nonfinite;
  p.tmap = tmap ? *tmap : TokenMap{};
  p.amax_ctas = num_sms() * 4;
  p.vgx = (N + kRowsPerCta - 1) / kRowsPerCta;
  p.qgx = p.nblk * 128 / ((kThreads / 32) * (128 / (d / 8)));
  const bool map = tmap != nullptr;
  if (d == 128) {
    if (qk_fp4) map ? launch_qkv<128, true, true>(p, st) : launch_qkv<128, false, true>(p, st);
    else map ? launch_qkv<128, true, false>(p, st) : launch_qkv<128, false, false>(p, st);
  } else {
    if (qk_fp4) map ? launch_qkv<64, true, true>(p, st) : launch_qkv<64, false, true>(p, st);
    else map ? launch_qkv<64, true, false>(p, st) : launch_qkv<64, false, false>(p, st);
  }
  return cudaGetLastError();
}

}  // namespace fpattn
