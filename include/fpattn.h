/*
 * fpattn: quantized attention forward for NVIDIA B200 (sm_100a).
 *
 * C ABI of the library. Every entry point takes plain pointers and sizes; no
 * C++ or framework types cross this boundary.
 *
 * What the library computes
 *   softmax(Q K^T / sqrt(d)) V  (FP4-attention tutorial page, section 2.1),
 *   with Q, K, V first quantized either
 *     - to NVFP4: E2M1 values in 16-element blocks along d, an E4M3 block
 *       scale per block and an FP32 tensor scale (Blackwell FP4 practice page,
 *       section 1, "micro-scaling": the scale is stored in FP8), or
 *     - to FP8 E4M3 in the FPSAttention staged scheme (FPSAttention page,
 *       section 2.1 conversion formula, section 3.1 "staged quantization":
 *       Q/K per block, V per channel, P per tensor at a fixed scale 1/448),
 *   and attention then run as one fused kernel with FP32 accumulation and an
 *   online softmax over 128-key tiles (FlashAttention-4 article: tiling,
 *   online softmax, kernel fusion), optionally restricted to a 3D
 *   sliding-tile pattern over video tokens (FPSAttention page, section 2.2)
 *   and/or a causal mask.
 *
 * Conventions shared by all entry points
 *   - The caller owns all memory. Tensor data pointers are DEVICE pointers on
 *     the current CUDA device unless stated otherwise. The library allocates
 *     no memory and never synchronizes the device; work is enqueued on the
 *     given stream in stream order.
 *   - Tensors are contiguous [B, H, N, d] row-major (d fastest). Data pointers
 *     must be 16-byte aligned (FPATTN_ERR_ALIGNMENT otherwise).
 *   - Argument and shape errors are returned before any work is enqueued.
 *     A failed launch returns FPATTN_ERR_CUDA. A bounded device-side wait
 *     that expired is recorded in a device error word that
 *     fpattn_device_error() reads.
 *   - Inputs are expected to be finite; non-finite inputs give unspecified
 *     codes and set the optional device flag *nonfinite_flag to 1.
 *   - Self-attention only: Q, K and V share B, H, N and d.
 */
#ifndef FPATTN_H_
#define FPATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fpattn_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  FPATTN_OK = 0,
  FPATTN_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, inconsistent tensors */
  FPATTN_ERR_UNSUPPORTED = 2,  /* d not in {64, 128}, dtype pair not supported, tile mask shape */
  FPATTN_ERR_ALIGNMENT = 3,    /* a data pointer is not 16-byte aligned */
  FPATTN_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
  FPATTN_ERR_TIMEOUT = 5       /* a bounded device wait expired (see fpattn_device_error) */
} fpattn_status;

typedef enum {
  FPATTN_BF16 = 0,  /* 2 bytes per element */
  FPATTN_E4M3 = 1,  /* 1 byte per element (OCP FP8 E4M3, max 448) */
  FPATTN_NVFP4 = 2  /* packed E2M1 codes, 2 per byte: element 2i in the low nibble of byte i */
} fpattn_dtype;

/* A contiguous [B, H, N, d] tensor. For NVFP4 the data holds B*H*N*d/2 bytes. */
typedef struct {
  void* data;
  int32_t dtype; /* fpattn_dtype */
  int32_t B, H, N, d;
} fpattn_tensor;

/* Quantization granularity for fpattn_quantize_fp8. */
typedef enum {
  FPATTN_FP8_TILE128 = 0, /* one scale per (b, h, 128-token tile): Q and K */
  FPATTN_FP8_CHANNEL = 1  /* one scale per (b, h, channel) over all N tokens: V */
} fpattn_fp8_granularity;

/*
 * Size in bytes of the NVFP4 block-scale buffer for a [B, H, N, d] tensor:
 * B*H*ceil(N/128)*(d/64)*512.
 *
 * Layout ("tensor-core scale layout"): for each (b, h), each 128-row block nb
 * and each group a of four 16-element scale columns, 512 bytes in which the
 * E4M3 scale of row r = nb*128 + 32*j + i (i < 32, j < 4) and column
 * 4*a + c (c < 4) is byte 16*i + 4*j + c. Rows at or past N are zero. This is
 * the arrangement the block-scaled tensor-core MMA reads its scale vectors
 * in, so the attention kernel copies it to tensor memory unchanged.
 */
size_t fpattn_nvfp4_sf_bytes(int32_t B, int32_t H, int32_t N, int32_t d);

/*
 * NVFP4 quantization of a bf16 tensor (Blackwell FP4 practice page,
 * section 1, micro-scaling with an FP8 scale; two-level arithmetic as below).
 *
 *   A_t = static_amax ? *static_amax : max|x| over the whole tensor
 *   s_t = A_t / 2688            (2688 = 6 * 448; 1 when A_t == 0)
 *   per 16-element block along d:
 *     sb   = E4M3(A_b / (6 * s_t)),   den = dec(sb) * s_t,
 *     code = E2M1(x * (1/den))  (round to nearest even, saturating at 6;
 *                                all codes 0 when den == 0)
 * Every step is one correctly rounded fp32 operation, so results are bit-exact
 * against the CPU oracle. Dequantized value: E2M1val * dec(sb) * s_t.
 *
 * x             bf16 input tensor (dtype FPATTN_BF16), d in {64, 128}
 * static_amax   device pointer to one float, or NULL for dynamic (per call)
 * codes         device, B*H*N*d/2 bytes, packed E2M1
 * block_sf      device, fpattn_nvfp4_sf_bytes() bytes, tensor-core scale layout
 * tensor_scale  device pointer to one float: receives s_t
 * nonfinite_flag  optional device int, set to 1 if x holds a non-finite value
 *                 (only written in dynamic mode; the caller zeroes it)
 */
fpattn_status fpattn_quantize_nvfp4(const fpattn_tensor* x, const float* static_amax,
                                    uint8_t* codes, uint8_t* block_sf, float* tensor_scale,
                                    int32_t* nonfinite_flag, fpattn_stream_t stream);

/*
 * The amax pass of fpattn_quantize_nvfp4 on its own (Blackwell FP4 practice
 * page, section 1: the tensor scale comes from the largest magnitude): folds
 * max|x| over the bf16 tensor x into the device float *amax, which is zeroed
 * first unless accumulate != 0. Several calls on consecutive pieces of one
 * tensor, the first with accumulate = 0 and the rest in stream order with
 * accumulate = 1, leave the amax of the whole tensor; passed as static_amax
 * to fpattn_quantize_nvfp4 on each piece it gives the codes and scales of
 * the whole-tensor call (the tensor is quantized as its pieces arrive).
 * nonfinite_flag as in fpattn_quantize_nvfp4. Errors as there.
 */
fpattn_status fpattn_tensor_amax(const fpattn_tensor* x, int32_t accumulate, float* amax, int32_t* nonfinite_flag,
                                 fpattn_stream_t stream);

/*
 * FP8 E4M3 quantization of a bf16 tensor (FPSAttention page, section 2.1:
 * X_hat = dequantize(FP8_convert(X * s_g)) / s_g; section 3.1: Q/K per block,
 * V per channel).
 *
 *   s    = 448 / A   (A = amax of the tile or channel; 1 when A == 0)
 *   code = E4M3(x * s), round to nearest even, saturating at 448.
 *
 * x            bf16 input tensor, d in {64, 128}
 * granularity  FPATTN_FP8_TILE128: A over one (b, h, 128-token tile) x d
 *              (a last partial tile uses its valid tokens); scales has
 *              B*H*ceil(N/128) floats.
 *              FPATTN_FP8_CHANNEL: A over all N tokens of one (b, h, channel);
 *              scales has B*H*d floats.
 * codes        device, B*H*N*d bytes, same [B, H, N, d] layout as x
 * scales       device floats: receives s (a multiplier: x ~ dec(code) / s)
 * nonfinite_flag  optional device int (see above)
 */
fpattn_status fpattn_quantize_fp8(const fpattn_tensor* x, int32_t granularity, uint8_t* codes,
                                  float* scales, int32_t* nonfinite_flag, fpattn_stream_t stream);

/*
 * FP8 E4M3 quantization of Q or K with one scale per group of `group_tiles`
 * consecutive 128-token tiles of each (b, h): the coarser Q/K granularities
 * of the FPSAttention page's denoising-step-aware schedule (section 3.2).
 * group_tiles = 1 is FPATTN_FP8_TILE128; ceil(N/128) (or more) is one scale
 * per (b, h); the tiles of one 3D video tile (tt*th*tw/128) is one scale per
 * video tile.
 *
 *   A = amax over the group's tokens (a last partial group: its valid
 *       tokens); s = 448 / A (1 when A == 0); code = E4M3(x * s).
 *
 * scales receives B*H*ceil(N/128) floats, the scale of every tile (its
 * group's scale, repeated), so fpattn_fwd takes them as per-tile scales
 * unchanged. layout: NULL for x in kernel order, else x is in raster order
 * and codes / scales come out tile-major, as in fpattn_quantize_fp8_video.
 * group_tiles < 1: FPATTN_ERR_INVALID_ARG; other arguments as
 * fpattn_quantize_fp8. x is read twice when group_tiles > 1 (amax pass,
 * then conversion).
 */
fpattn_status fpattn_quantize_fp8_group(const fpattn_tensor* x, const struct fpattn_video_layout_s* layout,
                                        int32_t group_tiles, uint8_t* codes, float* scales,
                                        int32_t* nonfinite_flag, fpattn_stream_t stream);

/*
 * Q, K and V of one attention call quantized together, in four launches
 * (zero the accumulators, one amax pass over the three tensors, one
 * conversion pass, one finalize) instead of four per tensor. The results are
 * bit for bit those of the separate calls:
 *   qk_dtype FPATTN_NVFP4: q, k as fpattn_quantize_nvfp4 (dynamic amax),
 *     q_block_sf / k_block_sf fpattn_nvfp4_sf_bytes() each, q_scale /
 *     k_scale one float each (s_t);
 *   qk_dtype FPATTN_E4M3: q, k as fpattn_quantize_fp8(FPATTN_FP8_TILE128),
 *     q_scale / k_scale B*H*ceil(N/128) floats, q_block_sf = k_block_sf =
 *     NULL;
 *   v as fpattn_quantize_fp8(FPATTN_FP8_CHANNEL): v_codes B*H*N*d bytes,
 *     v_scales B*H*d floats.
 * q, k, v: bf16 tensors of one shape. layout: NULL, or all three in raster
 * order of a video (codes and per-tile scales come out tile-major, as from
 * the _video calls). Errors as the separate calls; q, k, v of different
 * shapes or a qk_dtype other than the two: FPATTN_ERR_INVALID_ARG /
 * FPATTN_ERR_UNSUPPORTED. The Q/K scale outputs hold amax partial results
 * until the last launch has run (stream order makes that invisible).
 */
fpattn_status fpattn_quantize_qkv(const fpattn_tensor* q, const fpattn_tensor* k, const fpattn_tensor* v,
                                  int32_t qk_dtype, const struct fpattn_video_layout_s* layout, uint8_t* q_codes,
                                  uint8_t* q_block_sf, float* q_scale, uint8_t* k_codes, uint8_t* k_block_sf,
                                  float* k_scale, uint8_t* v_codes, float* v_scales, int32_t* nonfinite_flag,
                                  fpattn_stream_t stream);

/*
 * Phase of denoising step t of num_steps (FPSAttention page, section 3.2):
 * with t1 = alpha1 * num_steps and t2 = alpha2 * num_steps (the page deploys
 * alpha1 = 0.2, alpha2 = 0.7), t <= t1 is early (coarse granularity, sparse
 * window), t1 < t <= t2 middle (fine, dense), later steps late
 * (intermediate, medium). t counts steps in run order, 1 .. num_steps;
 * comparisons in double. HOST-only. Errors: t outside 1..num_steps, or not
 * 0 <= alpha1 <= alpha2 <= 1: FPATTN_ERR_INVALID_ARG.
 */
typedef enum { FPATTN_PHASE_EARLY = 0, FPATTN_PHASE_MIDDLE = 1, FPATTN_PHASE_LATE = 2 } fpattn_phase;
fpattn_status fpattn_step_phase(int32_t t, int32_t num_steps, double alpha1, double alpha2, int32_t* phase);

/*
 * NVFP4 quantization of V for the all-NVFP4 attention (P and V in NVFP4, P V
 * on block-scaled FP4 tensor cores). Same two-level recipe as
 * fpattn_quantize_nvfp4 (Blackwell FP4 practice page, section 1; tensor amax
 * over all of V, or *static_amax), but the 16-element blocks run along the
 * sequence, the contraction axis of P V, and the result is channel-major:
 *
 *   codes     device, fpattn_nvfp4_v_bytes() bytes: [B, H, d, Np/2] with
 *             Np = 128 * ceil(N/128); byte t/2 of row (b, h, c) holds
 *             tokens t (low nibble) and t+1; tokens >= N are 0
 *   block_sf  device, *block_sf_bytes bytes: per (b, h) and 128-token block
 *             kb, two 512-byte groups g (tokens 64g .. 64g+63): the E4M3
 *             scale of channel c = 32j + i and token block 4g + s at byte
 *             16i + 4j + s (the tensor-core scale layout with channels as
 *             rows; rows >= d are 0)
 *   tensor_scale  device float: s_t = A_t / 2688
 *
 * layout: NULL, or x in raster order of a video (tokens permuted to
 * tile-major order on the way, as in fpattn_quantize_fp8_video). Pass the
 * codes as an FPATTN_NVFP4 tensor [B, H, N, d] to fpattn_fwd with
 * scales.v_scale = tensor_scale and scales.v_block_sf = block_sf.
 */
size_t fpattn_nvfp4_v_bytes(int32_t B, int32_t H, int32_t N, int32_t d, size_t* block_sf_bytes);
fpattn_status fpattn_quantize_nvfp4_v(const fpattn_tensor* x, const struct fpattn_video_layout_s* layout,
                                      const float* static_amax, uint8_t* codes, uint8_t* block_sf,
                                      float* tensor_scale, int32_t* nonfinite_flag, fpattn_stream_t stream);

/* Scales consumed by fpattn_fwd. */
typedef struct {
  /* NVFP4 Q/K: device pointer to the one-float tensor scale s_t.
     E4M3 Q/K: device pointer to B*H*ceil(N/128) per-tile multipliers. */
  const float* q_scale;
  const float* k_scale;
  /* E4M3 V: device pointer to B*H*d per-channel multipliers.
     NVFP4 V: device pointer to its one-float tensor scale s_t. */
  const float* v_scale;
  /* NVFP4 Q/K: device block scales in the tensor-core scale layout; else NULL. */
  const uint8_t* q_block_sf;
  const uint8_t* k_block_sf;
  /* Scale of the E4M3 softmax probabilities; must be 1/448 (FPSAttention
     page, section 3.1: P per tensor at a fixed 1/448). */
  float p_scale;
  /* Multiplier of Q K^T before the softmax; 0 selects 1/sqrt(d). */
  float softmax_scale;
  /* Conditional softmax rescale (FlashAttention-4 article, co-design list,
     online-softmax item: rescale only once the running max has moved past a
     threshold). tau in [0, 8], log2 units; 0 (the default of a zeroed struct)
     is the exact running max. With tau > 0 a row's reference max m moves to
     the running max only when that exceeds m by more than tau; otherwise O
     and l are not rescaled, P = 2^(s - m) may reach 2^tau, and P is stored
     in E4M3 at the scale 448 * 2^-tau (p_scale above stays 1/448: the
     2^-tau is applied inside the kernel and cancels in O / l). Outside
     [0, 8]: FPATTN_ERR_INVALID_ARG. */
  float rescale_threshold;
  /* NVFP4 V (fpattn_quantize_nvfp4_v): device block scales; else NULL. */
  const uint8_t* v_block_sf;
} fpattn_scales;

/*
 * Block-sparse tile mask over 128-token blocks, shared by all (b, h):
 * query block qb attends exactly key blocks col_idx[row_ptr[qb] ..
 * row_ptr[qb+1]), which must be ascending and < ceil(N/128). All arrays are
 * DEVICE int32. row_order (optional, may be NULL) lists the query blocks in
 * the order the kernel should schedule them (a permutation of 0..nblk_q-1,
 * e.g. longest row first).
 */
typedef struct {
  int32_t nblk_q;          /* must equal ceil(N/128) */
  int32_t nnz;             /* row_ptr[nblk_q] */
  const int32_t* row_ptr;  /* nblk_q + 1 entries */
  const int32_t* col_idx;  /* nnz entries */
  const int32_t* row_order;
} fpattn_tile_mask_desc;

/*
 * HOST-only check of a tile mask held in HOST arrays (for instance before
 * copying it to the device for fpattn_fwd), with no CUDA call. FPATTN_OK when
 * row_ptr[0] = 0, row_ptr is non-decreasing with row_ptr[nblk] = nnz, every
 * row's col_idx entries are strictly ascending and in [0, nblk), and
 * row_order (may be NULL) is a permutation of 0 .. nblk-1; else
 * FPATTN_ERR_INVALID_ARG. fpattn_fwd cannot read device arrays before its
 * launch: given a mask that fails this check, it reads no memory outside the
 * arrays and tensors, but its results are unspecified.
 */
fpattn_status fpattn_tile_mask_check(int32_t nblk, int32_t nnz, const int32_t* row_ptr, const int32_t* col_idx,
                                     const int32_t* row_order);

/*
 * 3D sliding-tile planner (FPSAttention page, section 2.2: query tile u
 * attends key tiles v with ||c_u - c_v||_inf within the window). HOST-only,
 * integer work.
 *
 * Tokens of an nt*tt x nh*th x nw*tw video are taken in tile-major order
 * (tiles in raster order, tokens raster order within a tile). The tile volume
 * tt*th*tw must be a multiple of 128 so that every 128-token block lies in one
 * tile (FPATTN_ERR_UNSUPPORTED otherwise). The window (wt, wh, ww) is in
 * tiles; the half-width per axis is floor(w/2), clipped at the grid edges.
 *
 * Writes the CSR of fpattn_tile_mask_desc into HOST arrays:
 *   row_ptr[nblk_q + 1], col_idx[nnz], row_order[nblk_q] (rows sorted by
 *   descending length, ties by index). *nblk_q_out and *nnz_out receive the
 *   sizes. If col_cap < nnz (or any array is NULL), nothing but the sizes is
 *   written and FPATTN_OK is returned, so a first call with col_cap = 0 sizes
 *   the buffers.
 */
fpattn_status fpattn_sta_plan(int32_t nt, int32_t nh, int32_t nw, int32_t tt, int32_t th,
                              int32_t tw, int32_t wt, int32_t wh, int32_t ww,
                              int32_t* row_ptr, int32_t* col_idx, int32_t* row_order,
                              size_t col_cap, int32_t* nblk_q_out, int32_t* nnz_out);

/*
 * HOST-only, no CUDA call: the schedule fpattn_fwd uses for a causal launch
 * without a tile mask over bh = B*H (batch, head) problems of n tokens with
 * head dimension d (64 or 128), Q/K in qk_dtype and V in pv_dtype
 * (FPATTN_NVFP4 or FPATTN_E4M3), on a device with sm_count SMs. This is the
 * library's own scheduling, not a step of the pages' method: the results are
 * the same under any schedule.
 *
 * The kernel's work items are (head, 128-query block) pairs; a causal row of
 * query block qb attends qb + 1 key blocks. *ctas persistent CTAs take them
 * in one of two orders:
 *
 * Longest first (*pairs_per_head = 0). Items are taken longest row first and
 * dealt in a snake order (CTA 0..C-1 on even rounds, C-1..0 on odd ones:
 * position r*C + c or r*C + C-1-c). Over all heads at once, the same query
 * block of every head would be in flight together and the K/V of all heads
 * would pass through the L2 at once, so the heads are grouped so that one
 * group's K and V bytes fit in a 32 MiB share of the L2, the groups following
 * one another, and each group's positions are padded to whole pairs of snake
 * rounds so that every group is dealt evenly. Groups are used for NVFP4 Q/K
 * with at most 32 query blocks (measured faster there; with FP8 Q/K slower),
 * and a group size only when the padded schedule is modelled within 0.5% of
 * the ungrouped one's balance.
 * Position p of group p / group_positions holds an item when its offset in
 * the group is below group_heads*nblk (group_heads = heads of that group);
 * that item is head group*heads_per_group + offset % group_heads, query block
 * nblk - 1 - offset / group_heads. Ungrouped: heads_per_group = bh and
 * group_positions = bh*nblk.
 *
 * Pairs (*pairs_per_head = P = ceil(nblk/2) > 0), at d = 128 with at least
 * 32 query blocks, no head groups, and the heads' K/V beyond four shares (the
 * whole L2): pair j = h*P + i of
 * head h holds query blocks nblk-1-i and i, which together always cover nblk
 * + 1 key blocks, so pairs dealt round-robin (CTA c takes pairs c, c + C, ...)
 * balance the CTAs, and the CTAs in flight work on a few consecutive heads.
 * CTA c's round r is position 2*((r/2)*C + c) + r%2; position 2j is query
 * block nblk-1-i of pair j and 2j+1 is block i, absent when both are the
 * same block (the middle one of an odd nblk). Used only when modelled within
 * 1.5% of the snake's balance.
 *
 * *positions receives the positions of the whole launch. Sizes out of
 * fpattn_fwd's range give FPATTN_ERR_UNSUPPORTED; non-positive sizes, other
 * dtypes or NULL outputs FPATTN_ERR_INVALID_ARG.
 */
fpattn_status fpattn_causal_plan(int64_t bh, int64_t n, int32_t d, int32_t qk_dtype, int32_t pv_dtype,
                                 int32_t sm_count, int32_t* heads_per_group, int32_t* group_positions,
                                 int32_t* pairs_per_head, int32_t* positions, int32_t* ctas);

/*
 * Fused quantized attention forward.
 *
 * q, k        both FPATTN_NVFP4 (QK^T on block-scaled FP4 tensor cores) or
 *             both FPATTN_E4M3 (FP8 tensor cores)
 * v           FPATTN_E4M3 with per-channel scales (PV on FP8 tensor cores,
 *             P in E4M3 at scale 1/448), or FPATTN_NVFP4 from
 *             fpattn_quantize_nvfp4_v: all-NVFP4 attention, P quantized to
 *             NVFP4 in 16-key blocks with its tensor amax fixed at 2^tau (the
 *             bound of P under the reference max; the pages give no P rule
 *             for FP4, this is the library's reading) and P V on block-scaled
 *             FP4 tensor cores
 * scales      as described in fpattn_scales
 * tile_mask   NULL for dense, else a block mask (may be combined with causal)
 * causal      nonzero: key j attends query i only when j <= i
 * out         device bf16 [B, H, N, d]
 * lse         device float [B, H, N], natural-log log-sum-exp of the scaled
 *             scores of each row, or NULL
 * Per row, keys are walked in ascending 128-key tiles with a running max m,
 * a running sum l of the unquantized P, and O += E4M3(448 P) V; the output is
 * O / (448 l) with the V and P scales folded in. A row with no allowed key
 * gets out = 0 and lse = -inf.
 */
fpattn_status fpattn_fwd(const fpattn_tensor* q, const fpattn_tensor* k, const fpattn_tensor* v,
                         const fpattn_scales* scales, const fpattn_tile_mask_desc* tile_mask,
                         int32_t causal, void* out, float* lse, fpattn_stream_t stream);

/*
 * Video token order (FPSAttention page, section 2.2: attention over 3D tiles
 * of the video token grid; section 3.3, item 1: contiguous memory access
 * through a tile transpose).
 *
 * A video of T x Hs x W tokens in raster (time-major) order holds token
 * (t, h, w) in row (t*Hs + h)*W + w of its N = T*Hs*W rows. The attention
 * kernel works in tile-major order: tiles of tt x th x tw tokens in raster
 * order over the tile grid, and inside each tile its tokens in raster order
 * (the order fpattn_sta_plan numbers blocks in). The _video entry points
 * fuse that permutation into passes that touch the data anyway: the
 * quantizers read raster-order bf16 and write tile-major codes and scales,
 * and fpattn_fwd_video reads tile-major codes and writes out and lse in
 * raster order. No pass or buffer of its own is needed.
 *
 * Supported when T, Hs and W are multiples of tt, th and tw, the tile volume
 * tt*th*tw is a multiple of 128, and every 32 consecutive tile-major tokens
 * of a tile form one box of the grid, that is: tw is a multiple of 32; or 32
 * is a multiple of tw and th a multiple of 32/tw; or 32 is a multiple of
 * th*tw and tt a multiple of 32/(th*tw). Tiles (6,8,8), (4,8,8) and
 * (6,16,16) qualify. Other tiles give FPATTN_ERR_UNSUPPORTED; a layout with
 * T*Hs*W != N gives FPATTN_ERR_INVALID_ARG.
 */
typedef struct fpattn_video_layout_s {
  int32_t T, Hs, W;    /* grid, in tokens */
  int32_t tt, th, tw;  /* tile, in tokens */
} fpattn_video_layout;

/*
 * HOST-only check of a video layout for N tokens, with no CUDA call:
 * FPATTN_OK when the _video entry points accept it, FPATTN_ERR_UNSUPPORTED
 * or FPATTN_ERR_INVALID_ARG (NULL, non-positive sizes, T*Hs*W != N) as they
 * would return.
 */
fpattn_status fpattn_video_layout_check(const fpattn_video_layout* layout, int32_t N);

/*
 * fpattn_quantize_nvfp4 / fpattn_quantize_fp8 for raster-order input: x is
 * bf16 [B, H, N, d] in raster order of `layout` (HOST pointer to the layout
 * struct, read during the call); codes, block scales and per-tile scales are
 * written in tile-major order, exactly as the non-video call would write them
 * for x permuted to tile-major order. Per-tensor and per-channel scales are
 * order-free and equal to the non-video call's. Arguments and errors
 * otherwise as the non-video calls; layout NULL is FPATTN_ERR_INVALID_ARG.
 */
fpattn_status fpattn_quantize_nvfp4_video(const fpattn_tensor* x, const fpattn_video_layout* layout,
                                          const float* static_amax, uint8_t* codes, uint8_t* block_sf,
                                          float* tensor_scale, int32_t* nonfinite_flag,
                                          fpattn_stream_t stream);
fpattn_status fpattn_quantize_fp8_video(const fpattn_tensor* x, const fpattn_video_layout* layout,
                                        int32_t granularity, uint8_t* codes, float* scales,
                                        int32_t* nonfinite_flag, fpattn_stream_t stream);

/*
 * fpattn_fwd with q, k, v (and their block or tile scales) in tile-major
 * order of `layout` (HOST pointer), and out [B, H, N, d] and lse [B, H, N]
 * written in raster order: row r of the tile-major computation lands in the
 * raster row of the same token. tile_mask, if given, is over tile-major
 * blocks (as fpattn_sta_plan writes it). Results equal fpattn_fwd's,
 * permuted. Arguments and errors otherwise as fpattn_fwd; layout NULL is
 * FPATTN_ERR_INVALID_ARG.
 */
fpattn_status fpattn_fwd_video(const fpattn_tensor* q, const fpattn_tensor* k, const fpattn_tensor* v,
                               const fpattn_scales* scales, const fpattn_tile_mask_desc* tile_mask,
                               int32_t causal, const fpattn_video_layout* layout, void* out, float* lse,
                               fpattn_stream_t stream);

/*
 * Reads (and, if clear != 0, resets) the library's device error word on the
 * current device. Synchronizes `stream`. Returns FPATTN_OK when no bounded
 * wait has expired, FPATTN_ERR_TIMEOUT otherwise; *code (if non-NULL)
 * receives the raw word (which wait gave up).
 */
fpattn_status fpattn_device_error(fpattn_stream_t stream, int32_t clear, int32_t* code);

/* Human-readable name of a status code (static storage). */
const char* fpattn_status_string(fpattn_status status);

/* Library version string, e.g. "fpattn 0.1 sm_100a". */
const char* fpattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FPATTN_H_ */
