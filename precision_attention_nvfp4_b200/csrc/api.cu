// C ABI of the library: argument validation, dispatch to the kernels, the
// host-side sliding-tile planner, status strings. See include/fpattn.h.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/fpattn.h"
#include "fpattn_internal.h"

namespace {

using fpattn::AttnArgs;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fpattn_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return FPATTN_OK;
  if (e == cudaErrorNotSupported) return FPATTN_ERR_UNSUPPORTED;
  return FPATTN_ERR_CUDA;
}

// Common shape checks for a [B,H,N,d] tensor with the given dtype.
fpattn_status check_tensor(const fpattn_tensor* t, int dtype) {
  if (!t || !t->data) return FPATTN_ERR_INVALID_ARG;
  if (t->dtype != dtype) return FPATTN_ERR_INVALID_ARG;
  if (t->B <= 0 || t->H <= 0 || t->N <= 0 || t->d <= 0) return FPATTN_ERR_INVALID_ARG;
  if (t->d != 64 && t->d != 128) return FPATTN_ERR_UNSUPPORTED;
  // keep every index of the kernels inside 32-bit block / item counters
  const long long bh = static_cast<long long>(t->B) * t->H;
  const long long nblk = (t->N + 127) / 128;
  // (b, h) is the grid's y index in the quantize kernels: at most 65535
  if (bh > 65535 || bh * nblk > (1ll << 30) || t->N > (1 << 28)) return FPATTN_ERR_UNSUPPORTED;
  if (!aligned16(t->data)) return FPATTN_ERR_ALIGNMENT;
  return FPATTN_OK;
}

// Validates a video layout for N tokens and converts it; on success *tm
// receives the tile-major -> raster map.
fpattn_status check_layout(const fpattn_video_layout* l, int N, fpattn::VideoLayout* v, fpattn::TokenMap* tm) {
  if (!l) return FPATTN_ERR_INVALID_ARG;
  if (l->T <= 0 || l->Hs <= 0 || l->W <= 0 || l->tt <= 0 || l->th <= 0 || l->tw <= 0) return FPATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(l->T) * l->Hs * l->W != N) return FPATTN_ERR_INVALID_ARG;
  if (l->T % l->tt != 0 || l->Hs % l->th != 0 || l->W % l->tw != 0) return FPATTN_ERR_UNSUPPORTED;
  *v = fpattn::VideoLayout{l->T, l->Hs, l->W, l->tt, l->th, l->tw};
  int bw, bh, bt;
  if (!fpattn::video_chunk_box(*v, bw, bh, bt)) return FPATTN_ERR_UNSUPPORTED;
  *tm = fpattn::make_token_map(l->T, l->Hs, l->W, l->tt, l->th, l->tw);
  return FPATTN_OK;
}

fpattn_status quantize_nvfp4(const fpattn_tensor* x, const fpattn_video_layout* layout, const float* static_amax,
                             uint8_t* codes, uint8_t* block_sf, float* tensor_scale, int32_t* nonfinite_flag,
                             fpattn_stream_t stream) {
  fpattn_status s = check_tensor(x, FPATTN_BF16);
  if (s != FPATTN_OK) return s;
  fpattn::VideoLayout vl;
  fpattn::TokenMap tm;
  if (layout && (s = check_layout(layout, x->N, &vl, &tm)) != FPATTN_OK) return s;
  if (!codes || !block_sf || !tensor_scale) return FPATTN_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(block_sf) || (reinterpret_cast<uintptr_t>(tensor_scale) & 3u))
    return FPATTN_ERR_ALIGNMENT;
  return from_cuda(fpattn::launch_quantize_nvfp4(x->data, x->B * x->H, x->N, x->d, static_amax, codes, block_sf,
                                                 tensor_scale, nonfinite_flag, layout ? &tm : nullptr,
                                                 reinterpret_cast<cudaStream_t>(stream)));
}

fpattn_status quantize_fp8(const fpattn_tensor* x, const fpattn_video_layout* layout, int32_t granularity,
                           uint8_t* codes, float* scales, int32_t* nonfinite_flag, fpattn_stream_t stream) {
  fpattn_status s = check_tensor(x, FPATTN_BF16);
  if (s != FPATTN_OK) return s;
  fpattn::VideoLayout vl;
  fpattn::TokenMap tm;
  if (layout && (s = check_layout(layout, x->N, &vl, &tm)) != FPATTN_OK) return s;
  if (!codes || !scales) return FPATTN_ERR_INVALID_ARG;
  if (!aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u)) return FPATTN_ERR_ALIGNMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int BH = x->B * x->H;
  const fpattn::TokenMap* tmp = layout ? &tm : nullptr;
  if (granularity == FPATTN_FP8_TILE128)
    return from_cuda(
        fpattn::launch_quantize_fp8_tile(x->data, BH, x->N, x->d, codes, scales, nonfinite_flag, tmp, st));
  if (granularity == FPATTN_FP8_CHANNEL)
    return from_cuda(
        fpattn::launch_quantize_fp8_channel(x->data, BH, x->N, x->d, codes, scales, nonfinite_flag, tmp, st));
  return FPATTN_ERR_INVALID_ARG;
}

fpattn_status quantize_qkv(const fpattn_tensor* q, const fpattn_tensor* k, const fpattn_tensor* v, int32_t qk_dtype,
                          const fpattn_video_layout* layout, uint8_t* q_codes, uint8_t* q_block_sf, float* q_scale,
                          uint8_t* k_codes, uint8_t* k_block_sf, float* k_scale, uint8_t* v_codes,
                          float* v_scales, int32_t* nonfinite_flag, fpattn_stream_t stream) {
  fpattn_status s;
  if ((s = check_tensor(q, FPATTN_BF16)) != FPATTN_OK) return s;
  if ((s = check_tensor(k, FPATTN_BF16)) != FPATTN_OK) return s;
  if ((s = check_tensor(v, FPATTN_BF16)) != FPATTN_OK) return s;
  if (k->B != q->B || k->H != q->H || k->N != q->N || k->d != q->d || v->B != q->B || v->H != q->H ||
      v->N != q->N || v->d != q->d)
    return FPATTN_ERR_INVALID_ARG;
  if (qk_dtype != FPATTN_NVFP4 && qk_dtype != FPATTN_E4M3) return FPATTN_ERR_UNSUPPORTED;
  const bool fp4 = qk_dtype == FPATTN_NVFP4;
  fpattn::VideoLayout vl;
  fpattn::TokenMap tm;
  if (layout && (s = check_layout(layout, q->N, &vl, &tm)) != FPATTN_OK) return s;
  if (!q_codes || !k_codes || !v_codes || !q_scale || !k_scale || !v_scales) return FPATTN_ERR_INVALID_ARG;
  if (fp4 ? (!q_block_sf || !k_block_sf) : (q_block_sf || k_block_sf)) return FPATTN_ERR_INVALID_ARG;
  if (!aligned16(q_codes) || !aligned16(k_codes) || !aligned16(v_codes)) return FPATTN_ERR_ALIGNMENT;
  if (fp4 && (!aligned16(q_block_sf) || !aligned16(k_block_sf))) return FPATTN_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(q_scale) | reinterpret_cast<uintptr_t>(k_scale) |
       reinterpret_cast<uintptr_t>(v_scales)) & 3u)
    return FPATTN_ERR_ALIGNMENT;
  return from_cuda(fpattn::launch_quantize_qkv(q->data, k->data, v->data, q->B * q->H, q->N, q->d, fp4, q_codes,
                                               q_block_sf, q_scale, k_codes, k_block_sf, k_scale, v_codes,
                                               v_scales, nonfinite_flag, layout ? &tm : nullptr,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

fpattn_status quantize_nvfp4_v(const fpattn_tensor* x, const fpattn_video_layout* layout, const float* static_amax,
                              uint8_t* codes, uint8_t* block_sf, float* tensor_scale, int32_t* nonfinite_flag,
                              fpattn_stream_t stream) {
  fpattn_status s = check_tensor(x, FPATTN_BF16);
  if (s != FPATTN_OK) return s;
  fpattn::VideoLayout vl;
  fpattn::TokenMap tm;
  if (layout && (s = check_layout(layout, x->N, &vl, &tm)) != FPATTN_OK) return s;
  if (!codes || !block_sf || !tensor_scale) return FPATTN_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(block_sf) || (reinterpret_cast<uintptr_t>(tensor_scale) & 3u))
    return FPATTN_ERR_ALIGNMENT;
  return from_cuda(fpattn::launch_quantize_nvfp4_tokens(x->data, x->B * x->H, x->N, x->d, static_amax, codes,
                                                        block_sf, tensor_scale, nonfinite_flag,
                                                        layout ? &tm : nullptr,
                                                        reinterpret_cast<cudaStream_t>(stream)));
}

fpattn_status quantize_fp8_group(const fpattn_tensor* x, const fpattn_video_layout* layout, int32_t group,
                                 uint8_t* codes, float* scales, int32_t* nonfinite_flag, fpattn_stream_t stream) {
  fpattn_status s = check_tensor(x, FPATTN_BF16);
  if (s != FPATTN_OK) return s;
  fpattn::VideoLayout vl;
  fpattn::TokenMap tm;
  if (layout && (s = check_layout(layout, x->N, &vl, &tm)) != FPATTN_OK) return s;
  if (group < 1 || !codes || !scales) return FPATTN_ERR_INVALID_ARG;
  if (!aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u)) return FPATTN_ERR_ALIGNMENT;
  const int nblk = (x->N + 127) / 128;
  return from_cuda(fpattn::launch_quantize_fp8_group(x->data, x->B * x->H, x->N, x->d, std::min<int>(group, nblk),
                                                     codes, scales, nonfinite_flag, layout ? &tm : nullptr,
                                                     reinterpret_cast<cudaStream_t>(stream)));
}

fpattn_status fwd(const fpattn_tensor* q, const fpattn_tensor* k, const fpattn_tensor* v,
                  const fpattn_scales* scales, const fpattn_tile_mask_desc* tile_mask, int32_t causal,
                  const fpattn_video_layout* layout, void* out, float* lse, fpattn_stream_t stream) {
  if (!q || !k || !v || !scales || !out) return FPATTN_ERR_INVALID_ARG;
  const int qk_dtype = q->dtype;
  if (qk_dtype != FPATTN_NVFP4 && qk_dtype != FPATTN_E4M3) return FPATTN_ERR_UNSUPPORTED;
  fpattn_status s;
  if ((s = check_tensor(q, qk_dtype)) != FPATTN_OK) return s;
  if ((s = check_tensor(k, qk_dtype)) != FPATTN_OK) return s;
  const bool pv4 = v->dtype == FPATTN_NVFP4;
  if ((s = check_tensor(v, pv4 ? FPATTN_NVFP4 : FPATTN_E4M3)) != FPATTN_OK) return s;
  if (k->B != q->B || k->H != q->H || k->N != q->N || k->d != q->d || v->B != q->B || v->H != q->H ||
      v->N != q->N || v->d != q->d)
    return FPATTN_ERR_INVALID_ARG;
  fpattn::VideoLayout vl;
  fpattn::TokenMap tm;
  if (layout && (s = check_layout(layout, q->N, &vl, &tm)) != FPATTN_OK) return s;
  if (!aligned16(out) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))) return FPATTN_ERR_ALIGNMENT;
  if (!scales->q_scale || !scales->k_scale || !scales->v_scale) return FPATTN_ERR_INVALID_ARG;
  const bool fp4 = qk_dtype == FPATTN_NVFP4;
  if (fp4 && (!scales->q_block_sf || !scales->k_block_sf)) return FPATTN_ERR_INVALID_ARG;
  if (fp4 && (!aligned16(scales->q_block_sf) || !aligned16(scales->k_block_sf))) return FPATTN_ERR_ALIGNMENT;
  if (pv4 && !scales->v_block_sf) return FPATTN_ERR_INVALID_ARG;
  if (pv4 && !aligned16(scales->v_block_sf)) return FPATTN_ERR_ALIGNMENT;
  // P is stored in E4M3 at the fixed scale 1/448.
  if (!(scales->p_scale > 0.f) || std::abs(scales->p_scale * 448.f - 1.f) > 1e-6f) return FPATTN_ERR_INVALID_ARG;
  if (!(scales->softmax_scale >= 0.f) || scales->softmax_scale > 1e30f) return FPATTN_ERR_INVALID_ARG;
  if (!(scales->rescale_threshold >= 0.f && scales->rescale_threshold <= 8.f)) return FPATTN_ERR_INVALID_ARG;
  const int nblk = (q->N + 127) / 128;
  if (tile_mask) {
    if (tile_mask->nblk_q != nblk || !tile_mask->row_ptr || !tile_mask->col_idx || tile_mask->nnz < 0)
      return FPATTN_ERR_INVALID_ARG;
  }
  AttnArgs a{};
  a.q = q->data;
  a.k = k->data;
  a.v = v->data;
  a.q_sf = fp4 ? scales->q_block_sf : nullptr;
  a.k_sf = fp4 ? scales->k_block_sf : nullptr;
  a.v_sf = pv4 ? scales->v_block_sf : nullptr;
  a.pv_fp4 = pv4;
  a.q_scale = scales->q_scale;
  a.k_scale = scales->k_scale;
  a.v_scale = scales->v_scale;
  a.out = out;
  a.lse = lse;
  a.row_ptr = tile_mask ? tile_mask->row_ptr : nullptr;
  a.col_idx = tile_mask ? tile_mask->col_idx : nullptr;
  a.row_order = tile_mask ? tile_mask->row_order : nullptr;
  a.nnz = tile_mask ? tile_mask->nnz : 0;
  a.B = q->B;
  a.H = q->H;
  a.N = q->N;
  a.d = q->d;
  a.qk_fp4 = fp4;
  a.causal = causal != 0;
  a.softmax_scale = scales->softmax_scale > 0.f ? scales->softmax_scale : 1.0f / std::sqrt(static_cast<float>(q->d));
  a.rescale_threshold = scales->rescale_threshold;
  a.video = layout ? &vl : nullptr;
  return from_cuda(fpattn::launch_attn_fwd(a, reinterpret_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

size_t fpattn_nvfp4_sf_bytes(int32_t B, int32_t H, int32_t N, int32_t d) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || d % 64 != 0) return 0;
  return static_cast<size_t>(B) * H * ((N + 127) / 128) * (d / 64) * 512;
}

fpattn_status fpattn_quantize_nvfp4(const fpattn_tensor* x, const float* static_amax, uint8_t* codes,
                                    uint8_t* block_sf, float* tensor_scale, int32_t* nonfinite_flag,
                                    fpattn_stream_t stream) {
  return quantize_nvfp4(x, nullptr, static_amax, codes, block_sf, tensor_scale, nonfinite_flag, stream);
}

fpattn_status fpattn_quantize_fp8(const fpattn_tensor* x, int32_t granularity, uint8_t* codes, float* scales,
                                  int32_t* nonfinite_flag, fpattn_stream_t stream) {
  return quantize_fp8(x, nullptr, granularity, codes, scales, nonfinite_flag, stream);
}

fpattn_status fpattn_quantize_qkv(const fpattn_tensor* q, const fpattn_tensor* k, const fpattn_tensor* v,
                                  int32_t qk_dtype, const fpattn_video_layout* layout, uint8_t* q_codes,
                                  uint8_t* q_block_sf, float* q_scale, uint8_t* k_codes, uint8_t* k_block_sf,
                                  float* k_scale, uint8_t* v_codes, float* v_scales, int32_t* nonfinite_flag,
                                  fpattn_stream_t stream) {
  return quantize_qkv(q, k, v, qk_dtype, layout, q_codes, q_block_sf, q_scale, k_codes, k_block_sf, k_scale,
                      v_codes, v_scales, nonfinite_flag, stream);
}

fpattn_status fpattn_tensor_amax(const fpattn_tensor* x, int32_t accumulate, float* amax, int32_t* nonfinite_flag,
                                 fpattn_stream_t stream) {
  fpattn_status s = check_tensor(x, FPATTN_BF16);
  if (s != FPATTN_OK) return s;
  if (!amax) return FPATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(amax) & 3u) return FPATTN_ERR_ALIGNMENT;
  return from_cuda(fpattn::launch_tensor_amax_accum(x->data, x->B * x->H, x->N, x->d, accumulate != 0, amax,
                                              nonfinite_flag, reinterpret_cast<cudaStream_t>(stream)));
}

fpattn_status fpattn_video_layout_check(const fpattn_video_layout* layout, int32_t N) {
  fpattn::VideoLayout vl;
  fpattn::TokenMap tm;
  return check_layout(layout, N, &vl, &tm);
}

fpattn_status fpattn_quantize_nvfp4_video(const fpattn_tensor* x, const fpattn_video_layout* layout,
                                          const float* static_amax, uint8_t* codes, uint8_t* block_sf,
                                          float* tensor_scale, int32_t* nonfinite_flag, fpattn_stream_t stream) {
  if (!layout) return FPATTN_ERR_INVALID_ARG;
  return quantize_nvfp4(x, layout, static_amax, codes, block_sf, tensor_scale, nonfinite_flag, stream);
}

fpattn_status fpattn_quantize_fp8_video(const fpattn_tensor* x, const fpattn_video_layout* layout,
                                        int32_t granularity, uint8_t* codes, float* scales, int32_t* nonfinite_flag,
                                        fpattn_stream_t stream) {
  if (!layout) return FPATTN_ERR_INVALID_ARG;
  return quantize_fp8(x, layout, granularity, codes, scales, nonfinite_flag, stream);
}

size_t fpattn_nvfp4_v_bytes(int32_t B, int32_t H, int32_t N, int32_t d, size_t* block_sf_bytes) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || d % 64 != 0) {
    if (block_sf_bytes) *block_sf_bytes = 0;
    return 0;
  }
  const size_t nkb = static_cast<size_t>((N + 127) / 128);
  if (block_sf_bytes) *block_sf_bytes = static_cast<size_t>(B) * H * nkb * 1024;
  return static_cast<size_t>(B) * H * d * nkb * 64;
}

fpattn_status fpattn_quantize_nvfp4_v(const fpattn_tensor* x, const fpattn_video_layout* layout,
                                      const float* static_amax, uint8_t* codes, uint8_t* block_sf,
                                      float* tensor_scale, int32_t* nonfinite_flag, fpattn_stream_t stream) {
  return quantize_nvfp4_v(x, layout, static_amax, codes, block_sf, tensor_scale, nonfinite_flag, stream);
}

fpattn_status fpattn_quantize_fp8_group(const fpattn_tensor* x, const fpattn_video_layout* layout,
                                        int32_t group_tiles, uint8_t* codes, float* scales,
                                        int32_t* nonfinite_flag, fpattn_stream_t stream) {
  return quantize_fp8_group(x, layout, group_tiles, codes, scales, nonfinite_flag, stream);
}

fpattn_status fpattn_step_phase(int32_t t, int32_t num_steps, double alpha1, double alpha2, int32_t* phase) {
  if (!phase || num_steps < 1 || t < 1 || t > num_steps) return FPATTN_ERR_INVALID_ARG;
  if (!(alpha1 >= 0.0 && alpha1 <= alpha2 && alpha2 <= 1.0)) return FPATTN_ERR_INVALID_ARG;
  const double td = static_cast<double>(t);
  *phase = td <= alpha1 * num_steps ? FPATTN_PHASE_EARLY
                                    : (td <= alpha2 * num_steps ? FPATTN_PHASE_MIDDLE : FPATTN_PHASE_LATE);
  return FPATTN_OK;
}

fpattn_status fpattn_causal_plan(int64_t bh, int64_t n, int32_t d, int32_t qk_dtype, int32_t pv_dtype,
                                 int32_t sm_count, int32_t* heads_per_group, int32_t* group_positions,
                                 int32_t* pairs_per_head, int32_t* positions, int32_t* ctas) {
  if (!heads_per_group || !group_positions || !pairs_per_head || !positions || !ctas) return FPATTN_ERR_INVALID_ARG;
  if (bh <= 0 || n <= 0 || sm_count <= 0) return FPATTN_ERR_INVALID_ARG;
  if ((qk_dtype != FPATTN_NVFP4 && qk_dtype != FPATTN_E4M3) || (pv_dtype != FPATTN_NVFP4 && pv_dtype != FPATTN_E4M3))
    return FPATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FPATTN_ERR_UNSUPPORTED;
  const long long nblk = (n + 127) / 128;
  if (bh > 65535 || bh * nblk > (1ll << 30) || n > (1 << 28)) return FPATTN_ERR_UNSUPPORTED;
  const int items = static_cast<int>(bh * nblk);
  const int grid = items < sm_count ? items : sm_count;
  fpattn::CausalPlan cp;
  fpattn::causal_plan(static_cast<int>(bh), static_cast<int>(n), d, qk_dtype == FPATTN_NVFP4,
                      pv_dtype == FPATTN_NVFP4, grid, &cp);
  *heads_per_group = cp.hgroup;
  *group_positions = cp.gspan;
  *pairs_per_head = cp.hpairs;
  *positions = cp.num_items;
  *ctas = grid;
  return FPATTN_OK;
}

fpattn_status fpattn_sta_plan(int32_t nt, int32_t nh, int32_t nw, int32_t tt, int32_t th, int32_t tw, int32_t wt,
                              int32_t wh, int32_t ww, int32_t* row_ptr, int32_t* col_idx, int32_t* row_order,
                              size_t col_cap, int32_t* nblk_q_out, int32_t* nnz_out) {
  if (nt <= 0 || nh <= 0 || nw <= 0 || tt <= 0 || th <= 0 || tw <= 0 || wt <= 0 || wh <= 0 || ww <= 0)
    return FPATTN_ERR_INVALID_ARG;
  if (!nblk_q_out || !nnz_out) return FPATTN_ERR_INVALID_ARG;
  const long long vol = static_cast<long long>(tt) * th * tw;
  const long long ntiles = static_cast<long long>(nt) * nh * nw;
  if (vol % 128 != 0) return FPATTN_ERR_UNSUPPORTED;
  const long long per = vol / 128;  // 128-token blocks per tile
  if (ntiles * per > (1ll << 28)) return FPATTN_ERR_UNSUPPORTED;
  const int ht = wt / 2, hh = wh / 2, hw = ww / 2;
  // tiles in W(u) for tile u = (a, b, c): clipped ranges per axis
  auto range = [](int u, int half, int n, int* lo, int* hi) {
    *lo = std::max(0, u - half);
    *hi = std::min(n - 1, u + half);
  };
  long long nnz = 0;
  for (int a = 0; a < nt; ++a)
    for (int b = 0; b < nh; ++b)
      for (int c = 0; c < nw; ++c) {
        int a0, a1, b0, b1, c0, c1;
        range(a, ht, nt, &a0, &a1);
        range(b, hh, nh, &b0, &b1);
        range(c, hw, nw, &c0, &c1);
        nnz += static_cast<long long>(a1 - a0 + 1) * (b1 - b0 + 1) * (c1 - c0 + 1) * per * per;
      }
  if (nnz > (1ll << 31) - 1) return FPATTN_ERR_UNSUPPORTED;
  const int nblk = static_cast<int>(ntiles * per);
  *nblk_q_out = nblk;
  *nnz_out = static_cast<int32_t>(nnz);
  if (!row_ptr || !col_idx || !row_order || col_cap < static_cast<size_t>(nnz)) return FPATTN_OK;
  int32_t pos = 0;
  int qb = 0;
  row_ptr[0] = 0;
  std::vector<int32_t> blocks;
  for (int a = 0; a < nt; ++a)
    for (int b = 0; b < nh; ++b)
      for (int c = 0; c < nw; ++c) {
        int a0, a1, b0, b1, c0, c1;
        range(a, ht, nt, &a0, &a1);
        range(b, hh, nh, &b0, &b1);
        range(c, hw, nw, &c0, &c1);
        // key blocks of W(u): tile indices in raster order are ascending, so
        // the list comes out sorted
        blocks.clear();
        for (int x = a0; x <= a1; ++x)
          for (int y = b0; y <= b1; ++y)
            for (int z = c0; z <= c1; ++z) {
              const long long v = (static_cast<long long>(x) * nh + y) * nw + z;
              for (long long i = 0; i < per; ++i) blocks.push_back(static_cast<int32_t>(v * per + i));
            }
        // every 128-token query block of tile u gets the same list
        for (long long i = 0; i < per; ++i) {
          std::memcpy(col_idx + pos, blocks.data(), sizeof(int32_t) * blocks.size());
          pos += static_cast<int32_t>(blocks.size());
          row_ptr[qb + 1] = pos;
          ++qb;
        }
      }
  std::vector<int32_t> order(nblk);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int32_t x, int32_t y) {
    return (row_ptr[x + 1] - row_ptr[x]) > (row_ptr[y + 1] - row_ptr[y]);
  });
  std::memcpy(row_order, order.data(), sizeof(int32_t) * nblk);
  return FPATTN_OK;
}

fpattn_status fpattn_tile_mask_check(int32_t nblk, int32_t nnz, const int32_t* row_ptr, const int32_t* col_idx,
                                     const int32_t* row_order) {
  if (nblk <= 0 || nnz < 0 || !row_ptr || (nnz > 0 && !col_idx)) return FPATTN_ERR_INVALID_ARG;
  if (row_ptr[0] != 0 || row_ptr[nblk] != nnz) return FPATTN_ERR_INVALID_ARG;
  for (int32_t r = 0; r < nblk; ++r) {
    const int32_t b = row_ptr[r], e = row_ptr[r + 1];
    if (e < b || e > nnz) return FPATTN_ERR_INVALID_ARG;
    for (int32_t i = b; i < e; ++i) {
      if (col_idx[i] < 0 || col_idx[i] >= nblk) return FPATTN_ERR_INVALID_ARG;
      if (i > b && col_idx[i] <= col_idx[i - 1]) return FPATTN_ERR_INVALID_ARG;
    }
  }
  if (row_order) {
    std::vector<char> seen(static_cast<size_t>(nblk), 0);
    for (int32_t r = 0; r < nblk; ++r) {
      const int32_t x = row_order[r];
      if (x < 0 || x >= nblk || seen[x]) return FPATTN_ERR_INVALID_ARG;
      seen[x] = 1;
    }
  }
  return FPATTN_OK;
}

fpattn_status fpattn_fwd(const fpattn_tensor* q, const fpattn_tensor* k, const fpattn_tensor* v,
                         const fpattn_scales* scales, const fpattn_tile_mask_desc* tile_mask, int32_t causal,
                         void* out, float* lse, fpattn_stream_t stream) {
  return fwd(q, k, v, scales, tile_mask, causal, nullptr, out, lse, stream);
}

fpattn_status fpattn_fwd_video(const fpattn_tensor* q, const fpattn_tensor* k, const fpattn_tensor* v,
                               const fpattn_scales* scales, const fpattn_tile_mask_desc* tile_mask, int32_t causal,
                               const fpattn_video_layout* layout, void* out, float* lse, fpattn_stream_t stream) {
  if (!layout) return FPATTN_ERR_INVALID_ARG;
  return fwd(q, k, v, scales, tile_mask, causal, layout, out, lse, stream);
}

fpattn_status fpattn_device_error(fpattn_stream_t stream, int32_t clear, int32_t* code) {
  int v = 0;
  cudaError_t e = fpattn::read_device_error(reinterpret_cast<cudaStream_t>(stream), clear, &v);
  if (code) *code = v;
  if (e != cudaSuccess) return FPATTN_ERR_CUDA;
  return v == 0 ? FPATTN_OK : FPATTN_ERR_TIMEOUT;
}

const char* fpattn_status_string(fpattn_status status) {
  switch (status) {
    case FPATTN_OK: return "ok";
    case FPATTN_ERR_INVALID_ARG: return "invalid argument";
    case FPATTN_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case FPATTN_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case FPATTN_ERR_CUDA: return "CUDA error";
    case FPATTN_ERR_TIMEOUT: return "bounded device wait expired";
  }
  return "unknown status";
}

const char* fpattn_version(void) { return "fpattn 0.1 sm_100a"; }

}  // extern "C"
