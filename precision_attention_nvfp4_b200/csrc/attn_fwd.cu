// Fused quantized attention forward for sm_100a.
//
// Computes softmax(Q K^T * softmax_scale) V for quantized operands:
//   Q, K: NVFP4 (E2M1 + E4M3 per-16 block scale + FP32 tensor scale), QK^T on
//         the block-scaled FP4 tensor-core MMA (kind::mxf4nvf4), or
//         FP8 E4M3 with one scale per 128-token tile, QK^T on kind::f8f6f4;
//   P:    E4M3 at the fixed scale 1/448 (FPSAttention page, section 3.1);
//   V:    E4M3 with per-channel scales; PV on kind::f8f6f4 with P read
//         straight from tensor memory.
// The online softmax follows the FlashAttention tiling the pages describe
// (FlashAttention-4 article: S and P kept on chip, O accumulated in tensor
// memory, asynchronous pipeline between loads, MMA and softmax). The running
// row max is always the exact max; the O/l rescale is skipped for rows whose
// max did not change (a warp skips the tensor-memory round trip when none of
// its rows changed), which is exact.
//
// CTA organisation (persistent, one CTA per SM, 384 threads):
//   warp 0       TMA producer: Q once per work item, K/V tiles into a
//                4-stage shared-memory ring (plus NVFP4 block scales)
//   warp 1       tensor-memory allocator and single-thread MMA issuer
//   warps 2-3    idle
//   warps 4-11   two softmax warpgroups; warpgroup h owns keys 64h..64h+63 of
//                every 128-key S tile and output columns h*d/2..(h+1)*d/2-1;
//                thread (warp w, lane t) owns query row 32*(w%4)+t. They
//                exchange row maxima through shared memory once per tile.
// Tensor memory (512 columns): S double buffer at columns 0 and 128 (fp32
// 128x128), P (E4M3) written over the first 16 columns of each 64-column half
// of its S buffer, O at column 256 (d fp32 columns), NVFP4 scale vectors of Q
// and of two K tiles after O.
// Work items are (batch*head, 128-query block); causal runs schedule the
// longest query blocks first, tile-mask runs follow the mask's row order.
#include <cfloat>
#include <cstdint>
#include <cstdio>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "fpattn_internal.h"
#include "sm100.cuh"

namespace fpattn {

__device__ int g_error_word = 0;

namespace {

constexpr int kThreads = 384;
constexpr int kStages = 4;
constexpr float kLog2_448 = 8.807354922057604f;  // log2(448)
constexpr float kLn2 = 0.6931471805599453f;

// error codes recorded on a wait timeout (which wait gave up)
enum : int {
  kErrQEmpty = 0x101, kErrKvEmpty = 0x102, kErrQFull = 0x201, kErrKFull = 0x202, kErrVFull = 0x203,
  kErrPFull = 0x204, kErrSFull = 0x301, kErrODone = 0x302, kErrDrain = 0x401
};

template <int D, bool FP4>
struct Cfg {
  static constexpr int kQKRow = FP4 ? D / 2 : D;          // bytes per Q/K row
  static constexpr int kQKTile = 128 * kQKRow;            // bytes per 128-row Q/K tile
  static constexpr int kVTile = 128 * D;                  // bytes per 128-row V tile
  static constexpr int kSF = FP4 ? 512 * (D / 64) : 0;    // block-scale bytes per 128 rows
  static constexpr uint32_t kQKSwz = kQKRow == 128 ? 2u : (kQKRow == 64 ? 4u : 6u);
  static constexpr uint32_t kQKSbo = 8 * kQKRow;
  static constexpr uint32_t kVSwz = D == 128 ? 2u : 4u;
  static constexpr uint32_t kVSbo = 8 * D;
  static constexpr int kKSteps = FP4 ? D / 64 : D / 32;   // MMAs per S tile
#ifndef FPATTN_POLY_PAIRS
  static constexpr int kPolyPairs = 12;                   // of 32 exp2 pairs per thread and tile
#else
  static constexpr int kPolyPairs = FPATTN_POLY_PAIRS;
#endif
  static constexpr uint32_t kColO = 256;
  static constexpr uint32_t kColSFQ = 256 + D;
  static constexpr uint32_t kSFCols = 4 * (D / 64);
  static constexpr uint32_t kColSFK = kColSFQ + kSFCols;  // + buf * kSFCols
  // shared memory layout (offsets from a 1024-byte aligned base)
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQKTile;
  static constexpr int kOffV = kOffK + kStages * kQKTile;
  static constexpr int kOffSFQ = kOffV + kStages * kVTile;
  static constexpr int kOffSFK = kOffSFQ + kSF;
  static constexpr int kOffBar = kOffSFK + kStages * kSF;
  static constexpr int kNumBars = 2 + 3 * kStages + 2 + 2 + 2;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffXMax = (kOffMisc + 64 + 15) & ~15;   // float[2][2][128]
  static constexpr int kOffXL = kOffXMax + 2 * 2 * 128 * 4;     // float[2][2][128]
  static constexpr int kBytes = kOffXL + 2 * 2 * 128 * 4;
  // Request at least this much so that a single CTA fits per SM (it takes
  // all 512 tensor-memory columns).
  static constexpr int kSmemRequest = (kBytes + 1024 > 120 * 1024 ? kBytes + 1024 : 120 * 1024);
};

struct __align__(64) Params {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  __nv_bfloat16* out;
  float* lse;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const int32_t* row_order;
  int N, nblk, BH, num_items;
  int causal, sparse;
  float sm_scale_log2;
};

struct KList {
  int begin, count;
};

__device__ __forceinline__ void decode_item(const Params& p, int item, int& bh, int& qb) {
  if (p.sparse) {
    const int r = item / p.BH;
    bh = item % p.BH;
    qb = p.row_order ? p.row_order[r] : r;
  } else if (p.causal) {
    qb = p.nblk - 1 - item / p.BH;  // longest rows first
    bh = item % p.BH;
  } else {
    bh = item / p.nblk;             // one head's blocks together: K/V shared in L2
    qb = item % p.nblk;
  }
}

__device__ __forceinline__ KList key_list(const Params& p, int qb) {
  if (p.sparse) {
    const int b = p.row_ptr[qb];
    int e = p.row_ptr[qb + 1];
    if (p.causal) {
      int n = b;
      while (n < e && p.col_idx[n] <= qb) ++n;
      e = n;
    }
    return {b, e - b};
  }
  return {0, p.causal ? qb + 1 : p.nblk};
}

__device__ __forceinline__ int key_block(const Params& p, const KList& L, int j) {
  return p.sparse ? p.col_idx[L.begin + j] : j;
}

// Row max of 64 scores: a tree of three-input max instructions (depth 5).
__device__ __forceinline__ float row_max64(const float (&s)[64]) {
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = fmax3(s[8 * k], s[8 * k + 1], s[8 * k + 2]);
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = fmax3(a[k], s[8 * k + 3], s[8 * k + 4]);
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = fmax3(a[k], s[8 * k + 5], s[8 * k + 6]);
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = fmaxf(a[k], s[8 * k + 7]);
  return fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
}

// P = 2^(c*s + nbias) for 64 scores (nbias folds -m and log2 448), packed to
// E4M3 four per word (key 4j+b in byte b of pk[j]); returns the sum of the
// unquantized P. kPoly of the 32 pairs take the FMA-pipe polynomial exp2, the
// rest the MUFU ex2, spread evenly so both pipes stay busy.
template <int kPoly>
__device__ __forceinline__ float exp_pack64(const float (&s)[64], float c, float nbias, uint32_t (&pk)[16]) {
  const uint64_t c2 = f2_pack(c, c), nb2 = f2_pack(nbias, nbias);
  uint64_t acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = 0ull;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint64_t x = f2_fma(f2_pack(s[2 * i], s[2 * i + 1]), c2, nb2);
    uint64_t p;
    if (((i * kPoly) % 32) < kPoly) {
      p = exp2_poly2(x);
    } else {
      float x0, x1;
      f2_unpack(x, x0, x1);
      p = f2_pack(ex2_approx(x0), ex2_approx(x1));
    }
    acc[i & 3] = f2_add(acc[i & 3], p);
    float p0, p1;
    f2_unpack(p, p0, p1);
    const uint32_t h = cvt_e4m3x2(p0, p1);
    if (i & 1) pk[i >> 1] |= h << 16;
    else pk[i >> 1] = h;
  }
  const uint64_t t = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
  float lo, hi;
  f2_unpack(t, lo, hi);
  return lo + hi;
}

// AND of `v` over the 256 softmax threads; doubles as their shared barrier.
__device__ __forceinline__ bool softmax_sync_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, 256, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

// Lane 0 waits, the result is broadcast to the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* err, int code) {
  uint32_t ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, err, code) ? 1u : 0u;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  return ok != 0;
}

template <int D, bool FP4>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ Params p) {
  using C = Cfg<D, FP4>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* v_full = bars + 2 + kStages;
  uint64_t* kv_empty = bars + 2 + 2 * kStages;
  uint64_t* s_full = bars + 2 + 3 * kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* drain = o_done + 1;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  volatile int* issued_cnt = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);
  volatile int* consumed_cnt = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 12);
  float* xmax = reinterpret_cast<float*>(smem + C::kOffXMax);
  float* xl = reinterpret_cast<float*>(smem + C::kOffXL);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(v_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(p_full + b, 8);  // one arrival per softmax warp
    }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    *issued_cnt = 0;
    *consumed_cnt = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_k);
    prefetch_tensormap(&p.tm_v);
  }
  if (warp == 1) {
    tmem_alloc(const_cast<uint32_t*>(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      int g = 0, it = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < p.num_items && ok; item += gridDim.x, ++it) {
        int bh, qb;
        decode_item(p, item, bh, qb);
        const KList L = key_list(p, qb);
        if (it > 0) ok = mbar_wait(q_empty, (it - 1) & 1, abort_flag, &g_error_word, kErrQEmpty);
        if (!ok) break;
        mbar_arrive_expect_tx(q_full, C::kQKTile + C::kSF);
        tma_load_3d(smem + C::kOffQ, &p.tm_q, q_full, 0, qb * 128, bh);
        if (FP4)
          bulk_load(smem + C::kOffSFQ, p.q_sf + (static_cast<size_t>(bh) * p.nblk + qb) * C::kSF, C::kSF,
                    q_full);
        for (int j = 0; j < L.count; ++j, ++g) {
          const int st = g % kStages;
          const int use = g / kStages;
          if (use > 0 && !(ok = mbar_wait(kv_empty + st, (use - 1) & 1, abort_flag, &g_error_word, kErrKvEmpty))) break;
          const int kb = key_block(p, L, j);
          mbar_arrive_expect_tx(k_full + st, C::kQKTile + C::kSF);
          tma_load_3d(smem + C::kOffK + st * C::kQKTile, &p.tm_k, k_full + st, 0, kb * 128, bh);
          if (FP4)
            bulk_load(smem + C::kOffSFK + st * C::kSF,
                      p.k_sf + (static_cast<size_t>(bh) * p.nblk + kb) * C::kSF, C::kSF, k_full + st);
          mbar_arrive_expect_tx(v_full + st, C::kVTile);
          tma_load_3d(smem + C::kOffV + st * C::kVTile, &p.tm_v, v_full + st, 0, kb * 128, bh);
          *issued_cnt = g + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t kIdescS = FP4 ? idesc_nvf4(128, 128) : idesc_e4m3(128, 128, false);
      constexpr uint32_t kIdescPV = idesc_e4m3(128, D, true);
      const uint64_t q_desc = make_smem_desc(smem_u32(smem + C::kOffQ), 16, C::kQKSbo, C::kQKSwz);
      int g = 0, it = 0;
      bool ok = true;

      auto issue_pv = [&](int gg, int jj) -> bool {
        const int st = gg % kStages;
        const int buf = gg & 1;
        if (!mbar_wait(p_full + buf, (gg >> 1) & 1, abort_flag, &g_error_word, kErrPFull)) return false;
        if (!mbar_wait(v_full + st, (gg / kStages) & 1, abort_flag, &g_error_word, kErrVFull)) return false;
        tc_fence_after();
        const uint64_t v_desc = make_smem_desc(smem_u32(smem + C::kOffV + st * C::kVTile), 16, C::kVSbo, C::kVSwz);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t a_tmem = tmem + buf * 128 + 64 * (kk >> 1) + 8 * (kk & 1);
          mma_f8f6f4_ts(tmem + C::kColO, a_tmem, v_desc + static_cast<uint64_t>((kk * 32 * D) >> 4), kIdescPV,
                        (jj > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(kv_empty + st);
        mma_commit(o_done);
        *consumed_cnt = gg + 1;
        return true;
      };

      for (int item = blockIdx.x; item < p.num_items && ok; item += gridDim.x, ++it) {
        int bh, qb;
        decode_item(p, item, bh, qb);
        const KList L = key_list(p, qb);
        if (!(ok = mbar_wait(q_full, it & 1, abort_flag, &g_error_word, kErrQFull))) break;
        tc_fence_after();
        if (FP4) {
#pragma unroll
          for (int a = 0; a < D / 64; ++a)
            tmem_cp_32x128_warpx4(tmem + C::kColSFQ + 4 * a,
                                  make_smem_desc(smem_u32(smem + C::kOffSFQ + 512 * a), 128, 128, 0));
        }
        if (L.count == 0) {
          mma_commit(q_empty);
          continue;
        }
        for (int j = 0; j < L.count; ++j, ++g) {
          const int st = g % kStages;
          const int buf = g & 1;
          if (!(ok = mbar_wait(k_full + st, (g / kStages) & 1, abort_flag, &g_error_word, kErrKFull))) break;
          tc_fence_after();
          const uint64_t k_desc =
              make_smem_desc(smem_u32(smem + C::kOffK + st * C::kQKTile), 16, C::kQKSbo, C::kQKSwz);
          const uint32_t s_tmem = tmem + buf * 128;
          if (FP4) {
            const uint32_t sfk = C::kColSFK + buf * C::kSFCols;
#pragma unroll
            for (int a = 0; a < D / 64; ++a)
              tmem_cp_32x128_warpx4(tmem + sfk + 4 * a,
                                    make_smem_desc(smem_u32(smem + C::kOffSFK + st * C::kSF + 512 * a), 128, 128, 0));
#pragma unroll
            for (int kk = 0; kk < C::kKSteps; ++kk)
              mma_nvf4_ss(s_tmem, q_desc + 2 * kk, k_desc + 2 * kk, kIdescS, tmem + C::kColSFQ + 4 * kk,
                          tmem + sfk + 4 * kk, kk > 0 ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < C::kKSteps; ++kk)
              mma_f8f6f4_ss(s_tmem, q_desc + 2 * kk, k_desc + 2 * kk, kIdescS, kk > 0 ? 1u : 0u);
          }
          mma_commit(s_full + buf);
          if (j == L.count - 1) mma_commit(q_empty);
          if (j > 0 && !(ok = issue_pv(g - 1, j - 1))) break;
        }
        if (!ok) break;
        if (!(ok = issue_pv(g - 1, L.count - 1))) break;
      }
      // Drain: every issued MMA completes before tensor memory is released.
      mma_commit(drain);
      uint32_t drained = 0;
      const unsigned long long t0 = globaltimer_ns();
      while (!(drained = mbar_try_wait(smem_u32(drain), 0)) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
      if (!drained) atomicCAS(&g_error_word, 0, kErrDrain);
    }
  } else if (warp >= 4) {
    // -------------------------------------------------------------- softmax
    const int h = (warp - 4) >> 2;           // key / output half
    const int q4 = warp & 3;                 // TMEM lane quarter
    const int row = q4 * 32 + lane;          // query row within the tile
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    int g = 0, it = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.num_items && ok; item += gridDim.x, ++it) {
      int bh, qb;
      decode_item(p, item, bh, qb);
      const KList L = key_list(p, qb);
      float* xl_it = xl + (it & 1) * 256;  // double-buffered across items
      const int qrow = qb * 128 + row;
      float c_fp4 = 0.f, inv_sq = 0.f;
      if (FP4) c_fp4 = p.q_scale[0] * p.k_scale[0] * p.sm_scale_log2;
      else inv_sq = p.sm_scale_log2 / p.q_scale[static_cast<size_t>(bh) * p.nblk + qb];
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < L.count; ++j, ++g) {
        const int buf = g & 1;
        const int kb = key_block(p, L, j);
        bool mine = warp_wait(s_full + buf, (g >> 1) & 1, abort_flag, &g_error_word, kErrSFull);
        float s[64];
        float pmax = -INFINITY;
        if (mine) {
          tc_fence_after();
          uint32_t r0[32], r1[32];
          tmem_ld32(lane_base + buf * 128 + 64 * h, r0);
          tmem_ld32(lane_base + buf * 128 + 64 * h + 32, r1);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            s[i] = __uint_as_float(r0[i]);
            s[32 + i] = __uint_as_float(r1[i]);
          }
          const int key0 = kb * 128 + 64 * h;
          if ((p.causal && kb == qb) || key0 + 64 > p.N) {
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const int key = key0 + i;
              if ((p.causal && key > qrow) || key >= p.N) s[i] = -INFINITY;
            }
          }
          pmax = row_max64(s);
          xmax[(buf * 2 + h) * 128 + row] = pmax;
        }
        ok = softmax_sync_and(mine && ok);
        if (!ok) break;
        const float rawmax = fmaxf(pmax, xmax[(buf * 2 + (h ^ 1)) * 128 + row]);
        const float c = FP4 ? c_fp4 : inv_sq / p.k_scale[static_cast<size_t>(bh) * p.nblk + kb];
        const float m_new = rawmax == -INFINITY ? m : fmaxf(m, rawmax * c);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = (m == m_use) ? 1.f : ex2_approx(m - m_use);
        const float nbias = kLog2_448 - m_use;
        uint32_t pk[16];
        const float psum = exp_pack64<C::kPolyPairs>(s, c, nbias, pk);
        l = l * alpha + psum;
        m = m_new;
        // O correction: rows whose max moved scale O by alpha once PV of the
        // previous tile has landed.
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          if (!warp_wait(o_done, (g - 1) & 1, abort_flag, &g_error_word, kErrODone)) {
            ok = false;
            continue;  // skip the P store; the next tile's barrier ends all warps
          }
          tc_fence_after();
#pragma unroll
          for (int cc = 0; cc < D / 2; cc += 32) {
            uint32_t o[32];
            const uint32_t addr = lane_base + C::kColO + h * (D / 2) + cc;
            tmem_ld32(addr, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(addr, o);
          }
        }
        tmem_st16(lane_base + buf * 128 + 64 * h, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + buf);
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      bool done = true;
      if (L.count > 0) {
        done = warp_wait(o_done, (g - 1) & 1, abort_flag, &g_error_word, kErrODone);
        tc_fence_after();
      }
      xl_it[h * 128 + row] = l;
      ok = softmax_sync_and(done && ok);
      if (!ok) break;
      const float ltot = l + xl_it[(h ^ 1) * 128 + row];
      const float inv_l = ltot > 0.f ? 1.f / ltot : 0.f;
      const bool store = qrow < p.N;
      __nv_bfloat16* orow = p.out + (static_cast<size_t>(bh) * p.N + (store ? qrow : 0)) * D + h * (D / 2);
      const float* vs = p.v_scale + static_cast<size_t>(bh) * D + h * (D / 2);
#pragma unroll
      for (int cc = 0; cc < D / 2; cc += 32) {
        uint32_t o[32];
        if (L.count > 0) {
          tmem_ld32(lane_base + C::kColO + h * (D / 2) + cc, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float a = __uint_as_float(o[2 * i]) * inv_l / __ldg(vs + cc + 2 * i);
          const float b = __uint_as_float(o[2 * i + 1]) * inv_l / __ldg(vs + cc + 2 * i + 1);
          __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
          w[i] = *reinterpret_cast<uint32_t*>(&t);
        }
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (h == 0 && store && p.lse)
        p.lse[static_cast<size_t>(bh) * p.N + qrow] =
            ltot > 0.f ? (m + __log2f(ltot) - kLog2_448) * kLn2 : -INFINITY;
      tc_fence_before();
    }
  }

  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // Bounded drain of TMA loads that were issued but never consumed.
    const int issued = *issued_cnt;
    for (int gg = *consumed_cnt; gg < issued; ++gg) {
      const int st = gg % kStages;
      const uint32_t par = (gg / kStages) & 1;
      const unsigned long long t0 = globaltimer_ns();
      while (!(mbar_try_wait(smem_u32(k_full + st), par) && mbar_try_wait(smem_u32(v_full + st), par)) &&
             globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  return fn;
}

// 3D byte tensor [BH][N][row_bytes] with box [1][128][row_bytes].
bool make_map(CUtensorMap* m, const void* base, int row_bytes, int N, int BH, CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_bytes),
                           static_cast<cuuint64_t>(row_bytes) * static_cast<cuuint64_t>(N)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(row_bytes), 128u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

CUtensorMapSwizzle swizzle_for(int row_bytes) {
  return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

int sm_count() {
  static int n = [] {
    int dev = 0, c = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev);
    return c;
  }();
  return n;
}

template <int D, bool FP4>
cudaError_t launch_t(const AttnArgs& a, cudaStream_t st) {
  using C = Cfg<D, FP4>;
  Params p;
  const int BH = a.B * a.H;
  const int qk_row = C::kQKRow;
  if (!make_map(&p.tm_q, a.q, qk_row, a.N, BH, swizzle_for(qk_row)) ||
      !make_map(&p.tm_k, a.k, qk_row, a.N, BH, swizzle_for(qk_row)) ||
      !make_map(&p.tm_v, a.v, D, a.N, BH, swizzle_for(D)))
    return cudaErrorNotSupported;
  p.q_sf = a.q_sf;
  p.k_sf = a.k_sf;
  p.q_scale = a.q_scale;
  p.k_scale = a.k_scale;
  p.v_scale = a.v_scale;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.row_ptr = a.row_ptr;
  p.col_idx = a.col_idx;
  p.row_order = a.row_order;
  p.N = a.N;
  p.nblk = (a.N + 127) / 128;
  p.BH = BH;
  p.num_items = BH * p.nblk;
  p.causal = a.causal ? 1 : 0;
  p.sparse = a.row_ptr ? 1 : 0;
  p.sm_scale_log2 = a.softmax_scale * 1.4426950408889634f;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, FP4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemRequest);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int grid = p.num_items < sm_count() ? p.num_items : sm_count();
  attn_fwd_kernel<D, FP4><<<grid, kThreads, C::kSmemRequest, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd(const AttnArgs& a, cudaStream_t st) {
  if (a.d == 128) return a.qk_fp4 ? launch_t<128, true>(a, st) : launch_t<128, false>(a, st);
  return a.qk_fp4 ? launch_t<64, true>(a, st) : launch_t<64, false>(a, st);
}

cudaError_t read_device_error(cudaStream_t st, int clear, int* code) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_error_word, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  if (clear && v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_error_word, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  }
  if (code) *code = v;
  return e;
}

}  // namespace fpattn
