// Fused quantized attention forward for sm_100a.
//
// Computes softmax(Q K^T * softmax_scale) V for quantized operands:
//   Q, K: NVFP4 (E2M1 + E4M3 per-16 block scale + FP32 tensor scale), QK^T on
//         the block-scaled FP4 tensor-core MMA (kind::mxf4nvf4), or
//         FP8 E4M3 with one scale per 128-token tile, QK^T on kind::f8f6f4;
//   P:    E4M3 at the fixed scale 1/448 (FPSAttention page, section 3.1);
//   V:    E4M3 with per-channel scales; PV on kind::f8f6f4 with P read
//         straight from tensor memory.
// The PV4 variants quantize P to NVFP4 in the softmax (16-key blocks, the
// tensor amax of P fixed at its bound) and take V in NVFP4 along the
// sequence; PV then runs on kind::mxf4nvf4 with P from tensor memory.
// The online softmax follows the FlashAttention tiling the pages describe
// (FlashAttention-4 article: S and P kept on chip, O accumulated in tensor
// memory, asynchronous pipeline between loads, MMA and softmax). By default
// the reference row max is the exact max of the keys seen so far; O and the
// row sum are rescaled only for rows whose max moved (a warp skips the
// tensor-memory round trip when none of its rows moved), which is exact. A
// threshold tau > 0 moves it only when the max grew by more than tau, with P
// stored at 448 * 2^-tau.
//
// CTA organisation (persistent, one CTA per SM, 512 threads):
//   warp 0        TMA producer: Q once per work item, K/V tiles into a
//                 shared-memory ring, 4 stages deep for FP8 Q/K with E4M3 P
//                 and 3 otherwise (plus block scales)
//   warp 1        tensor-memory allocator; issues O += P V (one thread)
//   warp 2        issues S = Q K^T (one thread)
//   warp 3        idle
//   warps 4-7     softmax warpgroup 0
//   warps 8-11    softmax warpgroup 1
//   warps 12-15   O rescale (correction) and epilogue
// The CTA launches with 128 registers a thread; the warpgroups then take
// 56 (control), 176 (softmax) and 96 (correction) with setmaxnreg.
// With E4M3 P the softmax splits rows: the warp of warpgroup w and quarter q
// owns rows 32q + 16w .. +15 and all 128 keys of every block, two threads a
// row (the tensor-memory 16x64b pattern), so no warp waits on another within
// a block. Its exponentials run 4 of every 16 pairs on an FMA-pipe
// polynomial and the rest on MUFU. With NVFP4 P (PV4) the warpgroups split
// keys instead: one row a thread, 64 keys a warpgroup, and the half-block row
// maxima exchanged per lane through tagged shared-memory words; each keeps
// the row sum of its half and the epilogue adds the two.
// Tensor memory (512 columns): S double buffer at columns 0 and 128 (fp32
// 128x128, buffer = block parity), O at column 256 (d fp32 columns), a ring
// of P buffers (one per ring stage, three with NVFP4 Q/K; E4M3: 32 columns
// each, NVFP4: 16) at 384, then the
// NVFP4 scale vectors (Q, two K tiles; with PV4 also two each of P and V).
// S and P having their own buffers lets the S of a block be issued as soon as
// its buffer's previous tile has been read, independently of the PV of that
// tile; the two MMA kinds are issued by separate threads.
// The epilogue stores bf16 rows with TMA tensor stores: 3-D over [BH][N][d],
// or 5-D over a video's raster grid when the tokens are in tile-major order.
// K and V are loaded with an L2 evict-last policy, Q and the output with
// evict-first. The kernel waits for its stream predecessor (programmatic
// dependent launch) only after its prologue.
// Work items are (batch*head, 128-query block), dealt to the CTAs in orders
// that keep the K/V in flight within the L2: dense runs one head's query
// blocks together; causal runs longest first in L2-sized head groups, or in
// pairs of query blocks head by head (causal_plan); tile-mask runs one head
// after another in the mask's row order.
#include <algorithm>
#include <atomic>
#include <climits>
#include <cfloat>
#include <cstdint>
#include <cstdio>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <mutex>
#include <vector>

#include "fpattn_internal.h"
#include "sm100.cuh"

namespace fpattn {

__device__ int g_error_word = 0;

namespace {

constexpr int kThreads = 512;
// Depth of the K/V shared-memory ring (and of the rings that follow it: O
// rescale hand-off, O done).
// 0 picks per configuration: 4 for FP8 Q/K with E4M3 P (four P buffers fit
// in tensor memory), 3 otherwise (measured: a fourth stage with NVFP4 Q/K,
// where the P buffers stay three, is slower).
#ifndef FPATTN_KV_STAGES
#define FPATTN_KV_STAGES 0
#endif
// Of every 16 exp2 pairs, how many take the FMA-pipe polynomial (the rest
// take MUFU), with NVFP4 and with FP8 Q/K.
#ifndef FPATTN_POLY_FP4
#define FPATTN_POLY_FP4 4
#endif
#ifndef FPATTN_POLY_FP8
#define FPATTN_POLY_FP8 4
#endif
// Per-warpgroup register budgets (setmaxnreg) of the 512-thread CTA, which
// launches with 128 registers a thread: control warps, softmax warps,
// correction warps. 128 * (56 + 96) + 256 * 176 = 64512 <= 65536.
#ifndef FPATTN_REG_SPLIT
#define FPATTN_REG_SPLIT 1
#endif
constexpr bool kRegSplit = FPATTN_REG_SPLIT != 0;
constexpr uint32_t kRegsControl = 56, kRegsSoftmax = 176, kRegsCorrection = 96;
static_assert(128 * (kRegsControl + kRegsCorrection) + 256 * kRegsSoftmax <= 65536, "register split");
// Row-split softmax for E4M3 P: each softmax warp owns 16 rows and all 128
// keys of a block (else each warpgroup owns 64 keys of all 128 rows and the
// two exchange half-row maxima every block).
#ifndef FPATTN_ROW_SPLIT
#define FPATTN_ROW_SPLIT 1
#endif
constexpr bool kRowSplit = FPATTN_ROW_SPLIT != 0;
constexpr float kLog2_448 = 8.807354922057604f;  // log2(448)
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2_6 = 2.584962500721156f;    // log2(6)

// error codes recorded on a wait timeout (which wait gave up)
enum : int {
  kErrQEmpty = 0x101, kErrKvEmpty = 0x102, kErrQFull = 0x201, kErrKFull = 0x202, kErrVFull = 0x203,
  kErrPFull = 0x204, kErrOReady = 0x205, kErrSFull = 0x301, kErrMax = 0x303, kErrFin = 0x304,
  kErrAlpha = 0x305, kErrSFree = 0x306, kErrODone = 0x302, kErrPFree = 0x307, kErrDrain = 0x401
};

// FP4: Q, K in NVFP4 (else E4M3). PV4: P and V in NVFP4 and P V on the
// block-scaled FP4 tensor cores (else E4M3 P and V).
template <int D, bool FP4, bool PV4>
struct Cfg {
  // depth of the K/V ring (and of the rings that follow it)
  static constexpr int kStages = FPATTN_KV_STAGES > 0 ? FPATTN_KV_STAGES : (!FP4 && !PV4 ? 4 : 3);
  static constexpr int kQKRow = FP4 ? D / 2 : D;          // bytes per Q/K row
  static constexpr int kQKTile = 128 * kQKRow;            // bytes per 128-row Q/K tile
  // V tile of one 128-key block: E4M3 [128 keys][D], or NVFP4 transposed
  // [D channels][64 bytes = 128 keys]
  static constexpr int kVTile = PV4 ? D * 64 : 128 * D;
  static constexpr int kSF = FP4 ? 512 * (D / 64) : 0;    // block-scale bytes per 128 rows
  static constexpr int kSFV = PV4 ? 1024 : 0;             // V block scales per key block (2 k-steps)
  static constexpr int kSFP = PV4 ? 1024 : 0;             // P block scales per P buffer
  static constexpr uint32_t kQKSwz = kQKRow == 128 ? 2u : (kQKRow == 64 ? 4u : 6u);
  static constexpr uint32_t kQKSbo = 8 * kQKRow;
  static constexpr uint32_t kVSwz = PV4 ? 4u : (D == 128 ? 2u : 4u);
  static constexpr uint32_t kVSbo = PV4 ? 8 * 64 : 8 * D;
  static constexpr int kKSteps = FP4 ? D / 64 : D / 32;   // MMAs per S tile
  // of the 16 exp2 pairs of a 32-score chunk, how many take the FMA-pipe
  // polynomial (measured best with the row-split softmax and the degree-4
  // polynomial: 4; 3, 5 and 6 were 1-4% slower on the dense workloads)
  static constexpr int kPolyPairs = FP4 ? FPATTN_POLY_FP4 : FPATTN_POLY_FP8;
  static constexpr uint32_t kColO = 256;                  // O: d fp32 columns
  // P buffers, 32 columns each (128 E4M3 keys), as many as K/V stages when
  // tensor memory holds them: the S of block g needs K stage g % kStages,
  // which is refilled only after the PV of block g - kStages has completed,
  // and that PV was the last reader of P buffer g % kPBufs. So a softmax
  // thread that has seen S(g) may overwrite the buffer without a barrier of
  // its own. With fewer P buffers than stages (NVFP4 Q/K at four stages: the
  // scale vectors take the columns of the fourth), the softmax waits for the
  // PV of block g - kPBufs before writing P buffer g % kPBufs.
  static constexpr uint32_t kColP = 384;
  static constexpr uint32_t kPCols = PV4 ? 16 : 32;       // per P buffer: 128 keys of E2M1 or E4M3
  static constexpr int kPBufs =
      kColP + kPCols * kStages + (FP4 ? 3 * 4 * (D / 64) : 0) + (PV4 ? 32 : 0) <= 512 ? kStages : 3;
  static constexpr bool kPWait = kPBufs < kStages;
  static constexpr uint32_t kColSFQ = kColP + kPCols * kPBufs;
  static constexpr uint32_t kSFCols = 4 * (D / 64);
  static constexpr uint32_t kColSFK = kColSFQ + kSFCols;  // + buf * kSFCols
  // P and V block scales of PV4, two buffers of 2 k-steps x 4 columns each
  static constexpr uint32_t kColSFP = kColSFK + (FP4 ? 2 * kSFCols : 0);  // + (g & 1) * 8
  static constexpr uint32_t kColSFV = kColSFP + 16;                       // + (g & 1) * 8
  static_assert(!PV4 || kColSFV + 16 <= 512, "tensor memory columns");
  static_assert(kColP + kPCols * kPBufs + (FP4 ? 3 * kSFCols : 0) <= 512, "tensor memory columns");
  // shared memory layout (offsets from a 1024-byte aligned base)
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQKTile;
  static constexpr int kOffV = kOffK + kStages * kQKTile;
  static constexpr int kOffSFQ = kOffV + kStages * kVTile;
  static constexpr int kOffSFK = kOffSFQ + kSF;
  static constexpr int kOffSFV = kOffSFK + kStages * kSF;   // [stage][1024]
  static constexpr int kOffSFP = kOffSFV + kStages * kSFV;  // [P buffer][1024], written by the softmax
  static constexpr int kOffBar = kOffSFP + kPBufs * kSFP;
  // mbarrier indices (one chain, so the pointers and the count cannot drift)
  static constexpr int kBarQFull = 0, kBarQEmpty = 1, kBarKFull = 2;
  static constexpr int kBarVFull = kBarKFull + kStages, kBarKVEmpty = kBarVFull + kStages;
  static constexpr int kBarSFull = kBarKVEmpty + kStages, kBarSFree = kBarSFull + 2, kBarPFull = kBarSFree + 2;
  static constexpr int kBarOReady = kBarPFull + kPBufs, kBarODone = kBarOReady + kStages;
  static constexpr int kBarDrain = kBarODone + kStages, kBarA = kBarDrain + 2;
  static constexpr int kBarFin = kBarA + 4 * kStages, kBarFinFree = kBarFin + 2;
  static constexpr int kNumBars = kBarFinFree + 2;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffX = (kOffMisc + 64 + 15) & ~15;      // running max, rescale, per-item (l, m)
  static constexpr int kOutWarpBytes = 32 * 2 * D;
  static constexpr int kOffOut =
      (kOffX + 4 * 128 * 8 + (kStages * 128 + 2 * 2 * 2 * 128 + 4 * D) * 4 + 1023) & ~1023;
  static constexpr int kBytes = kOffOut + 4 * kOutWarpBytes;
  // Request at least this much so that a single CTA fits per SM (it takes
  // all 512 tensor-memory columns).
  static constexpr int kSmemRequest = (kBytes + 1024 > 120 * 1024 ? kBytes + 1024 : 120 * 1024);
  static_assert(kSmemRequest <= 227 * 1024, "shared memory per CTA");
};

struct __align__(64) Params {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  // bf16 out, 64 columns x 32 rows per store, 128-byte swizzle: [BH][N][d],
  // or for a video layout [BH][T][Hs][W][d] with a box that covers one
  // 32-row chunk of a tile-major block
  CUtensorMap tm_out;
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const uint8_t* v_sf;  // NVFP4 V block scales [BH][nblk][1024] (PV4)
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  __nv_bfloat16* out;
  float* lse;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const int32_t* row_order;
  int N, nblk, BH;
  int num_items;  // schedule positions: the items, plus the padding of causal head groups
  int nnz;        // tile mask entries (sparse runs)
  int hgroup;     // causal runs: heads scheduled together (longest rows first within a group)
  int gspan;      // causal runs: schedule positions of a full group (items + padding)
  int hpairs;     // causal runs in pairs (else 0): pairs of query blocks per head, ceil(nblk / 2)
  int causal, sparse;
  float sm_scale_log2;
  float tau;           // conditional-rescale threshold, log2 units (0: exact running max)
  float p_log2_scale;  // log2 of the P scale: log2(448) - tau
  TokenMap tmap;  // on: rows are tile-major, out and lse go to raster positions
};

struct KList {
  int begin, count;
};

// Schedule position of this CTA in scheduling round r. Causal runs in pairs
// (p.hpairs > 0): pair (r / 2) * C + CTA, its longer query block on even
// rounds and its shorter one on odd rounds (position 2 * pair + r % 2); every
// pair costs the same, so dealing them round-robin balances the CTAs. Else a
// snake over the C CTAs (forward on even rounds, backward on odd ones), so
// that with items sorted longest first every CTA gets a near-equal share.
__device__ __forceinline__ int sched_item(const Params& p, int r) {
  const int c = static_cast<int>(blockIdx.x), C = static_cast<int>(gridDim.x);
  if (p.hpairs) return (((r >> 1) * C + c) << 1) | (r & 1);
  return r * C + ((r & 1) ? C - 1 - c : c);
}

// Whether schedule position `pos` holds an item. In pairs, the middle block
// of an odd count is its own partner, so its pair has no second item. Causal
// head groups are padded: each group's items are followed by empty positions
// up to a whole number of snake round pairs, so every group is spread evenly
// over the CTAs.
__device__ __forceinline__ bool item_present(const Params& p, int pos) {
  if (p.sparse || !p.causal) return true;
  if (p.hpairs) return (pos & 1) == 0 || 2 * ((pos >> 1) % p.hpairs) + 1 != p.nblk;
  const int grp = pos / p.gspan;
  const int gsz = min(p.hgroup, p.BH - grp * p.hgroup);
  return pos - grp * p.gspan < gsz * p.nblk;
}

// First position at or after round `rnd` that holds an item (rnd advances to
// its round), or a position >= p.num_items when there is none. A CTA's
// positions grow with the round, so every role of the CTA walks the same list.
__device__ __forceinline__ int next_item(const Params& p, int& rnd) {
  int pos = sched_item(p, rnd);
  while (pos < p.num_items && !item_present(p, pos)) pos = sched_item(p, ++rnd);
  return pos;
}

// The tile mask's arrays come from the caller: the host entry points check
// them, and the kernel also keeps every index it derives from them in range
// (a query block outside [0, nblk) is taken as block 0, a row's end is
// clipped to nnz, a key block outside [0, nblk) is loaded as block 0 and
// fully masked), so a malformed mask can give wrong results but never an
// out-of-bounds access.
__device__ __forceinline__ void decode_item(const Params& p, int item, int& bh, int& qb) {
  if (p.sparse) {
    // one head's rows after another, each head's in the mask's row order
    // (longest first): the CTAs in flight share the K/V windows of one or
    // two heads (with every head's same row together, those of all heads
    // passed through the L2 at once: 14.8 against 12.8 ms on the 40-head
    // video workload)
    const int r = item % p.nblk;
    bh = item / p.nblk;
    qb = p.row_order ? p.row_order[r] : r;
    if (static_cast<unsigned>(qb) >= static_cast<unsigned>(p.nblk)) qb = 0;
  } else if (p.hpairs) {
    // pair j of head bh: query blocks nblk - 1 - i (even position) and i
    const int j = item >> 1;
    bh = j / p.hpairs;
    const int i = j - bh * p.hpairs;
    qb = (item & 1) ? i : p.nblk - 1 - i;
  } else if (p.causal) {
    // longest rows first within groups of p.hgroup heads whose K/V fit in
    // part of the L2; the groups follow one another (item_present is true)
    const int grp = item / p.gspan;
    const int r = item - grp * p.gspan;
    const int gsz = min(p.hgroup, p.BH - grp * p.hgroup);
    qb = p.nblk - 1 - r / gsz;
    bh = grp * p.hgroup + r % gsz;
  } else {
    bh = item / p.nblk;             // one head's blocks together: K/V shared in L2
    qb = item % p.nblk;
  }
}

__device__ __forceinline__ KList key_list(const Params& p, int qb) {
  if (p.sparse) {
    const int e0 = min(p.row_ptr[qb + 1], p.nnz);
    const int b = max(0, min(p.row_ptr[qb], e0));
    int e = e0;
    if (p.causal) {
      int n = b;
      while (n < e && p.col_idx[n] <= qb) ++n;
      e = n;
    }
    return {b, e - b};
  }
  return {0, p.causal ? qb + 1 : p.nblk};
}

// Key block j of a query block's list; -1 for an entry outside [0, nblk).
__device__ __forceinline__ int key_block(const Params& p, const KList& L, int j) {
  if (!p.sparse) return j;
  const int kb = p.col_idx[L.begin + j];
  return static_cast<unsigned>(kb) < static_cast<unsigned>(p.nblk) ? kb : -1;
}

// Masks the scores of one 32-key chunk (keys key0..key0+31) that fall past
// the sequence end or, on the causal diagonal, after the query row.
__device__ __forceinline__ void mask_chunk(uint32_t (&r)[32], int key0, int qrow, bool causal_diag, int N) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int key = key0 + i;
    if ((causal_diag && key > qrow) || key >= N) r[i] = 0xff800000u;  // -inf
  }
}

// As mask_chunk for 32 scores of keys key0, key0 + 2, ..., key0 + 62.
__device__ __forceinline__ void mask_chunk2(uint32_t (&r)[32], int key0, int qrow, bool causal_diag, int N) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int key = key0 + 2 * i;
    if ((causal_diag && key > qrow) || key >= N) r[i] = 0xff800000u;  // -inf
  }
}

// The two threads of a row (lanes t and t ^ 2 of the 16x64b pattern) hold
// E4M3 P of keys 8j + {0, 2, 4, 6} (par 0) and 8j + {1, 3, 5, 7} (par 1) in
// pk[j], byte by byte. Afterwards the par-0 thread holds P column 2j (keys
// 8j .. 8j+3) and the par-1 thread column 2j + 1 (keys 8j+4 .. 8j+7), key
// 4k + b in byte b.
__device__ __forceinline__ void pair_columns(uint32_t (&pk)[8], int par) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t other = __shfl_xor_sync(0xffffffffu, pk[j], 2);
    pk[j] = par ? __byte_perm(pk[j], other, 0x3726) : __byte_perm(pk[j], other, 0x5140);
  }
}

// Max of 32 scores: a tree of three-input max instructions.
__device__ __forceinline__ float max32(const uint32_t (&r)[32], float m) {
  float a[4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    a[k] = fmax3(fmax3(__uint_as_float(r[8 * k]), __uint_as_float(r[8 * k + 1]), __uint_as_float(r[8 * k + 2])),
                 fmax3(__uint_as_float(r[8 * k + 3]), __uint_as_float(r[8 * k + 4]), __uint_as_float(r[8 * k + 5])),
                 fmaxf(__uint_as_float(r[8 * k + 6]), __uint_as_float(r[8 * k + 7])));
  return fmax3(fmax3(a[0], a[1], m), a[2], a[3]);
}

// P = 2^(c*s + nbias) for 32 scores (nbias folds -m and log2 448), packed to
// E4M3 four per word (key 4j+b in byte b of pk[j]); returns the sum of the
// unquantized P. kPoly of the 16 pairs take the FMA-pipe polynomial exp2, the
// rest the MUFU ex2, spread evenly so both pipes stay busy.
template <int kPoly>
__device__ __forceinline__ float exp_pack32(const uint32_t (&r)[32], float c, float nbias, uint32_t (&pk)[8]) {
  const uint64_t c2 = f2_pack(c, c), nb2 = f2_pack(nbias, nbias);
  uint64_t acc0 = 0ull, acc1 = 0ull;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), c2, nb2);
    uint64_t pr;
    if (((i * kPoly) % 16) < kPoly) {
      pr = exp2_poly2(x);
    } else {
      float x0, x1;
      f2_unpack(x, x0, x1);
      pr = f2_pack(ex2_approx(x0), ex2_approx(x1));
    }
    if (i & 1) acc1 = f2_add(acc1, pr);
    else acc0 = f2_add(acc0, pr);
    float p0, p1;
    f2_unpack(pr, p0, p1);
    const uint32_t h = cvt_e4m3x2(p0, p1);
    if (i & 1) pk[i >> 1] |= h << 16;
    else pk[i >> 1] = h;
  }
  float lo, hi;
  f2_unpack(f2_add(acc0, acc1), lo, hi);
  return lo + hi;
}

// NVFP4 P for 32 scores: two 16-key blocks, each with an E4M3 block scale
// taken from its largest P. This is the NVFP4 recipe with P's tensor amax fixed
// at its bound: in units where P carries the factor 448 * 2^-tau, as nbias
// gives it, sb = E4M3(P_max) and the codes are E2M1(6 P / dec(sb)). The
// 6 / dec(sb) is folded into the block's exponent bias, so each exp2 lands on
// the E2M1 grid directly. A block whose scale underflows to 0 keeps the plain
// bias; its P are then far below the smallest E2M1 step and encode as 0.
// Returns the sum of the unquantized P (in nbias units) for the row sum.
// pk: key 8j + b in nibble b of pk[j]; sfw receives the two scale bytes at
// byte positions shift and shift + 1.
template <int kPoly>
__device__ __forceinline__ float exp_pack32_fp4(const uint32_t (&r)[32], float c, float nbias, uint32_t (&pk)[4],
                                                uint32_t& sfw, int shift) {
  const uint64_t c2 = f2_pack(c, c);
  float total = 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t* rb = r + 16 * h;
    const float bm =
        fmax3(fmax3(fmax3(__uint_as_float(rb[0]), __uint_as_float(rb[1]), __uint_as_float(rb[2])),
                    fmax3(__uint_as_float(rb[3]), __uint_as_float(rb[4]), __uint_as_float(rb[5])),
                    fmax3(__uint_as_float(rb[6]), __uint_as_float(rb[7]), __uint_as_float(rb[8]))),
              fmax3(__uint_as_float(rb[9]), __uint_as_float(rb[10]), __uint_as_float(rb[11])),
              fmax3(fmax3(__uint_as_float(rb[12]), __uint_as_float(rb[13]), __uint_as_float(rb[14])),
                    __uint_as_float(rb[15]), -INFINITY));
    const uint32_t sb = cvt_e4m3x2(ex2_approx(fmaf(bm, c, nbias)), 0.f) & 0xFFu;
    const float dec = e4m3_to_float(sb);
    const float bias = sb ? nbias + (kLog2_6 - __log2f(dec)) : nbias;
    const float back = sb ? dec * (1.f / 6.f) : 1.f;  // from the E2M1 grid back to P
    const uint64_t nb2 = f2_pack(bias, bias);
    uint64_t acc = 0ull;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int q = 8 * h + i;  // pair of keys 2q, 2q + 1 of the chunk
      const uint64_t x = f2_fma(f2_pack(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1])), c2, nb2);
      uint64_t pr;
      if (((q * kPoly) % 16) < kPoly) {
        pr = exp2_poly2(x);
      } else {
        float x0, x1;
        f2_unpack(x, x0, x1);
        pr = f2_pack(ex2_approx(x0), ex2_approx(x1));
      }
      acc = f2_add(acc, pr);
      float p0, p1;
      f2_unpack(pr, p0, p1);
      const uint32_t byte = cvt_e2m1x2(p0, p1);
      if ((q & 3) == 0) pk[q >> 2] = byte;
      else pk[q >> 2] |= byte << (8 * (q & 3));
    }
    float lo, hi;
    f2_unpack(acc, lo, hi);
    total += (lo + hi) * back;
    sfw |= sb << (8 * (shift + h));
  }
  return total;
}

// Every lane polls the barrier (one broadcast shared-memory access per poll),
// so the warp never diverges around the wait.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* err, int code) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, err, code));
}

// Polls a shared-memory word until its high half equals tag, then returns
// its low half (a float) in val. A 64-bit aligned store is single-copy
// atomic, so the value and its tag arrive together. Bounded like mbar_wait.
__device__ __forceinline__ bool tagged_wait(const volatile unsigned long long* slot, uint32_t tag, float& val,
                                            volatile int* abort, int* err, int code) {
  unsigned long long v, t0 = 0;
  for (uint32_t it = 0;; ++it) {
    v = *slot;
    if (static_cast<uint32_t>(v >> 32) == tag) break;
    if ((it & 63u) == 63u) {
      if (*abort) return false;
      const unsigned long long now = globaltimer_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > kWaitTimeoutNs) {
        atomicCAS(err, 0, code);
        *abort = 1;
        return false;
      }
    }
  }
  val = __uint_as_float(static_cast<uint32_t>(v));
  return true;
}

// Lane 0 arrives once all lanes of the warp are past this point.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

template <int D, bool FP4, bool PV4>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ Params p) {
  using C = Cfg<D, FP4, PV4>;
  constexpr int kStages = C::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars + C::kBarQFull;
  uint64_t* q_empty = bars + C::kBarQEmpty;
  uint64_t* k_full = bars + C::kBarKFull;      // [stage]
  uint64_t* v_full = bars + C::kBarVFull;      // [stage]
  uint64_t* kv_empty = bars + C::kBarKVEmpty;  // [stage], 2 arrivals: S issuer (K), PV issuer (V)
  uint64_t* s_full = bars + C::kBarSFull;      // [buffer]
  uint64_t* s_free = bars + C::kBarSFree;      // [buffer], 8 arrivals: softmax warps read S
  uint64_t* p_full = bars + C::kBarPFull;      // [g % kPBufs], 8 arrivals: softmax warps wrote P
  // Rings whose two sides may drift apart are kStages deep. A block's S needs
  // its K/V stage, which is released only when PV of the block kStages back has
  // completed, so in these rings no producer laps its consumer and no waiter is
  // ever more than one phase behind the phase it waits for (the condition for
  // a parity wait to be exact).
  uint64_t* o_ready = bars + C::kBarOReady;    // [g % kStages], 4 arrivals: correction warps
  uint64_t* o_done = bars + C::kBarODone;      // [g % kStages]: PV of block g completed
  uint64_t* drain = bars + C::kBarDrain;       // [2]: PV issuer, S issuer
  uint64_t* a_bar = bars + C::kBarA;           // [quarter][g % kStages]: rescale factor published (warpgroup g % 2)
  uint64_t* fin_bar = bars + C::kBarFin;       // [item parity], 8 arrivals: per-item (l, m) published
  uint64_t* fin_free = bars + C::kBarFinFree;  // [item parity], 4 arrivals: correction warps read them
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  volatile int* issued_cnt = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);
  volatile int* consumed_cnt = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 12);
  // [block parity][warpgroup][128]: half-block row max, tag g + 1 in the high word
  volatile unsigned long long* xs = reinterpret_cast<volatile unsigned long long*>(smem + C::kOffX);
  float* ax = reinterpret_cast<float*>(smem + C::kOffX + 4 * 128 * 8);  // [kStages][128] O rescale factor
  float* fin = ax + kStages * 128;                              // [2 items][2 wg][2 (l, m)][128]
  float* inv_vs = fin + 2 * 2 * 2 * 128;                        // [correction warp][d]: 1 / V scale

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(v_full + s, 1);
      mbar_init(kv_empty + s, 2);  // S issuer (K read) and PV issuer (V read)
    }
    for (int s = 0; s < kStages; ++s) mbar_init(o_ready + s, 4);
    for (int b = 0; b < C::kPBufs; ++b) {
      mbar_init(p_full + b, 8);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(s_free + b, 8);
      mbar_init(fin_bar + b, 8);
      mbar_init(fin_free + b, 4);
    }
    for (int s = 0; s < kStages; ++s) mbar_init(o_done + s, 1);
    mbar_init(drain, 1);
    mbar_init(drain + 1, 1);
    // rescale factors: both warps of a quarter publish every block (row
    // split), or the two warpgroups take turns (half-key loop)
    for (int i = 0; i < 4 * kStages; ++i) mbar_init(a_bar + i, kRowSplit && !PV4 ? 2 : 1);
    *abort_flag = 0;
    *issued_cnt = 0;
    *consumed_cnt = 0;
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < 4 * 128; i += kThreads) xs[i] = 0ull;
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
  // the prologue above touches no global memory; from here on the stream
  // predecessor's results are read
  griddep_wait();
  if (warp < 4) {
  if (kRegSplit && !PV4) reg_dealloc<kRegsControl>();
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      // K and V blocks are read by every query block of their head; Q once
      const uint64_t keep = l2_policy_evict_last(), stream = l2_policy_evict_first();
      int g = 0, it = 0;
      bool ok = true;
      for (int rnd = 0, item = next_item(p, rnd); item < p.num_items && ok; ++rnd, item = next_item(p, rnd), ++it) {
        int bh, qb;
        decode_item(p, item, bh, qb);
        const KList L = key_list(p, qb);
        if (it > 0) ok = mbar_wait(q_empty, (it - 1) & 1, abort_flag, &g_error_word, kErrQEmpty);
        if (!ok) break;
        mbar_arrive_expect_tx(q_full, C::kQKTile + C::kSF);
        tma_load_3d_hint(smem + C::kOffQ, &p.tm_q, q_full, 0, qb * 128, bh, stream);
        if (FP4)
          bulk_load_hint(smem + C::kOffSFQ, p.q_sf + (static_cast<size_t>(bh) * p.nblk + qb) * C::kSF, C::kSF,
                         q_full, stream);
        for (int j = 0; j < L.count; ++j, ++g) {
          const int st = g % kStages;
          const int use = g / kStages;
          if (use > 0 && !(ok = mbar_wait(kv_empty + st, (use - 1) & 1, abort_flag, &g_error_word, kErrKvEmpty)))
            break;
          const int kb = max(key_block(p, L, j), 0);
          mbar_arrive_expect_tx(k_full + st, C::kQKTile + C::kSF);
          tma_load_3d_hint(smem + C::kOffK + st * C::kQKTile, &p.tm_k, k_full + st, 0, kb * 128, bh, keep);
          if (FP4)
            bulk_load_hint(smem + C::kOffSFK + st * C::kSF,
                           p.k_sf + (static_cast<size_t>(bh) * p.nblk + kb) * C::kSF, C::kSF, k_full + st, keep);
          mbar_arrive_expect_tx(v_full + st, C::kVTile + C::kSFV);
          if (PV4) {
            tma_load_3d_hint(smem + C::kOffV + st * C::kVTile, &p.tm_v, v_full + st, kb * 64, 0, bh, keep);
            bulk_load_hint(smem + C::kOffSFV + st * C::kSFV,
                           p.v_sf + (static_cast<size_t>(bh) * p.nblk + kb) * C::kSFV, C::kSFV, v_full + st, keep);
          } else {
            tma_load_3d_hint(smem + C::kOffV + st * C::kVTile, &p.tm_v, v_full + st, 0, kb * 128, bh, keep);
          }
          *issued_cnt = g + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ PV issuer
    if (lane == 0) {
      constexpr uint32_t kIdescPV = PV4 ? idesc_nvf4(128, D) : idesc_e4m3(128, D, true);
      int g = 0;
      bool ok = true;
      for (int rnd = 0, item = next_item(p, rnd); item < p.num_items && ok; ++rnd, item = next_item(p, rnd)) {
        int bh, qb;
        decode_item(p, item, bh, qb);
        const KList L = key_list(p, qb);
        for (int j = 0; j < L.count; ++j, ++g) {
          // O += P V once P is in TMEM, O has been rescaled and V has landed.
          const int st = g % kStages;
          const int pb = g % C::kPBufs;
          if (!(ok = mbar_wait(p_full + pb, (g / C::kPBufs) & 1, abort_flag, &g_error_word, kErrPFull))) break;
          if (!(ok = mbar_wait(o_ready + st, (g / kStages) & 1, abort_flag, &g_error_word, kErrOReady))) break;
          if (!(ok = mbar_wait(v_full + st, (g / kStages) & 1, abort_flag, &g_error_word, kErrVFull))) break;
          tc_fence_after();
          const uint64_t v_desc =
              make_smem_desc(smem_u32(smem + C::kOffV + st * C::kVTile), 16, C::kVSbo, C::kVSwz);
          if (PV4) {
            // block scales of P (written by the softmax) and of V into tensor
            // memory, then two K = 64 block-scaled MMAs with P from tensor memory
            const uint32_t sb = (g & 1) * 8;
#pragma unroll
            for (int a = 0; a < 2; ++a) {
              tmem_cp_32x128_warpx4(tmem + C::kColSFP + sb + 4 * a,
                                    make_smem_desc(smem_u32(smem + C::kOffSFP + pb * C::kSFP + 512 * a), 128, 128, 0));
              tmem_cp_32x128_warpx4(tmem + C::kColSFV + sb + 4 * a,
                                    make_smem_desc(smem_u32(smem + C::kOffSFV + st * C::kSFV + 512 * a), 128, 128, 0));
            }
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
              mma_nvf4_ts(tmem + C::kColO, tmem + C::kColP + pb * C::kPCols + 8 * kk, v_desc + 2 * kk, kIdescPV,
                          tmem + C::kColSFP + sb + 4 * kk, tmem + C::kColSFV + sb + 4 * kk,
                          (j > 0 || kk > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f8f6f4_ts(tmem + C::kColO, tmem + C::kColP + pb * 32 + 8 * kk,
                            v_desc + static_cast<uint64_t>((kk * 32 * D) >> 4), kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(kv_empty + st);
          mma_commit(o_done + st);
          *consumed_cnt = g + 1;
        }
      }
      // Drain: every issued MMA completes before tensor memory is released.
      mma_commit(drain);
      uint32_t drained = 0;
      const unsigned long long t0 = globaltimer_ns();
      while (!(drained = mbar_try_wait(smem_u32(drain), 0)) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
      if (!drained) atomicCAS(&g_error_word, 0, kErrDrain);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------- S issuer
    if (lane == 0) {
      constexpr uint32_t kIdescS = FP4 ? idesc_nvf4(128, 128) : idesc_e4m3(128, 128, false);
      const uint64_t q_desc = make_smem_desc(smem_u32(smem + C::kOffQ), 16, C::kQKSbo, C::kQKSwz);
      int g = 0, it = 0;
      bool ok = true;
      for (int rnd = 0, item = next_item(p, rnd); item < p.num_items && ok; ++rnd, item = next_item(p, rnd), ++it) {
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
        for (int j = 0; j < L.count; ++j, ++g) {
          // S = Q K^T into buffer g % 2 once K has landed and the owner
          // warpgroup has read the buffer's previous tile.
          const int st = g % kStages;
          const int buf = g & 1;
          if (!(ok = mbar_wait(k_full + st, (g / kStages) & 1, abort_flag, &g_error_word, kErrKFull))) break;
          if (g >= 2 && !(ok = mbar_wait(s_free + buf, ((g >> 1) - 1) & 1, abort_flag, &g_error_word, kErrSFree)))
            break;
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
          mma_commit(kv_empty + st);
        }
        if (!ok) break;
        mma_commit(q_empty);  // all S of the item issued: Q (and its scales) may be replaced
      }
      mma_commit(drain + 1);
      uint32_t drained = 0;
      const unsigned long long t0 = globaltimer_ns();
      while (!(drained = mbar_try_wait(smem_u32(drain + 1), 0)) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
      if (!drained) atomicCAS(&g_error_word, 0, kErrDrain);
    }
  }
  } else if (warp < 12 && kRowSplit && !PV4) {
    // ------------------------------------------------ softmax (row split)
    // Warp (warpgroup w, quarter q) owns rows 32q + 16w .. 32q + 16w + 15 of
    // the query tile and all 128 keys of every block: thread t takes row
    // 32q + 16w + t/4 + 8 (t & 1) and the keys of parity (t >> 1) & 1, 64
    // scores read from tensor memory once (the 16x64b access pattern; the
    // partner thread of the row is t ^ 2). The two threads of a row combine their maxima with
    // one shuffle and keep partial row sums, so no warp waits on another: the
    // two warps of an SM sub-partition run their blocks independently, and
    // one's exponentials fill the other's latencies.
    if (kRegSplit) reg_alloc<kRegsSoftmax>();
    const int w = (warp - 4) >> 2;
    const int q4 = warp & 3;
    const int par = (lane >> 1) & 1;
    const int row = q4 * 32 + w * 16 + (lane >> 2) + 8 * (lane & 1);
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32 + w * 16) << 16;
    int g = 0, it = 0;
    bool ok = true;
    for (int rnd = 0, item = next_item(p, rnd); item < p.num_items && ok; ++rnd, item = next_item(p, rnd), ++it) {
      int bh, qb;
      decode_item(p, item, bh, qb);
      const KList L = key_list(p, qb);
      const int qrow = qb * 128 + row;
      float c_fp4 = 0.f, inv_sq = 0.f;
      if (FP4) c_fp4 = p.q_scale[0] * p.k_scale[0] * p.sm_scale_log2;
      else inv_sq = p.sm_scale_log2 / p.q_scale[static_cast<size_t>(bh) * p.nblk + qb];
      float l = 0.f, m_ref = -INFINITY;
      // FP8 K tile scales are read one block ahead
      float ks_next = (!FP4 && L.count > 0)
                          ? __ldg(p.k_scale + static_cast<size_t>(bh) * p.nblk + max(key_block(p, L, 0), 0))
                          : 1.f;
      for (int j = 0; j < L.count && ok; ++j, ++g) {
        const int kb_raw = key_block(p, L, j);
        const int kb = max(kb_raw, 0);
        const int buf = g & 1;
        const float ks = ks_next;
        if (!FP4 && j + 1 < L.count)
          ks_next = __ldg(p.k_scale + static_cast<size_t>(bh) * p.nblk + max(key_block(p, L, j + 1), 0));
        ok = warp_wait(s_full + buf, (g >> 1) & 1, abort_flag, &g_error_word, kErrSFull);
        tc_fence_after();
        uint32_t r0[32], r1[32];
        const uint32_t s_addr = tmem + lane_off + buf * 128;
        tmem_ld16x64b_x32(s_addr, r0);       // keys 2i + par
        tmem_ld16x64b_x32(s_addr + 64, r1);  // keys 64 + 2i + par
        tmem_wait_ld(r0);
        tmem_wait_ld(r1);
        tc_fence_before();
        warp_arrive(s_free + buf);
        const int key0 = kb * 128 + par;
        const bool diag = p.causal && kb == qb;
        if (diag || (kb + 1) * 128 > p.N || kb_raw < 0) {
          // an invalid mask entry masks every key of its block
          const int lim = kb_raw < 0 ? 0 : p.N;
          mask_chunk2(r0, key0, qrow, diag, lim);
          mask_chunk2(r1, key0 + 64, qrow, diag, lim);
        }
        const float own = max32(r1, max32(r0, -INFINITY));
        const float rawmax = fmaxf(own, __shfl_xor_sync(0xffffffffu, own, 2));
        const float c = FP4 ? c_fp4 : inv_sq / ks;
        // reference max and rescale factor: as in the half-key loop below
        const float m_prev = m_ref;
        const float cand = rawmax == -INFINITY ? m_prev : fmaxf(m_prev, rawmax * c);
        const float m_new = (m_prev == -INFINITY || cand - m_prev > p.tau) ? cand : m_prev;
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = m_prev == m_new ? 1.f : ex2_approx(m_prev - m_use);
        // both warps of the quarter publish their 16 rows' factors every block
        if (par == 0) ax[(g % kStages) * 128 + row] = alpha;
        warp_arrive(a_bar + q4 * kStages + g % kStages);
        l *= alpha;
        m_ref = m_new;
        const float nbias = p.p_log2_scale - m_use;
        const int pb = g % C::kPBufs;
        if (C::kPWait && g >= C::kPBufs) {
          // P buffer pb was last read by the PV of block g - kPBufs
          const int gp = g - C::kPBufs;
          ok = warp_wait(o_done + gp % kStages, (gp / kStages) & 1, abort_flag, &g_error_word, kErrPFree) && ok;
          tc_fence_after();
        }
        // P: each thread packs its keys 8j + par + {0, 2, 4, 6}; the pair
        // swaps halves so that the even thread holds P column 2j (keys
        // 8j .. 8j + 3) and the odd one column 2j + 1, the columns the 16x64b
        // store writes from them.
        const uint32_t p_addr = tmem + lane_off + C::kColP + pb * 32;
        uint32_t pk[8];
        float psum = exp_pack32<C::kPolyPairs>(r0, c, nbias, pk);
        pair_columns(pk, par);
        tmem_st16x64b_x8(p_addr, pk);
        psum += exp_pack32<C::kPolyPairs>(r1, c, nbias, pk);
        pair_columns(pk, par);
        tmem_st16x64b_x8(p_addr + 16, pk);
        l += psum;
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(p_full + pb);
      }
      if (!ok) break;
      // per-item (l, m) of the row for the epilogue, in the first half's
      // slot; the second half's slot is empty (l = 0)
      const float lrow = l + __shfl_xor_sync(0xffffffffu, l, 2);
      if (it >= 2 && !(ok = warp_wait(fin_free + (it & 1), ((it >> 1) - 1) & 1, abort_flag, &g_error_word,
                                      kErrFin)))
        break;
      if (par == 0) {
        fin[(((it & 1) * 2 + 0) * 2 + 0) * 128 + row] = lrow;
        fin[(((it & 1) * 2 + 0) * 2 + 1) * 128 + row] = m_ref;
        fin[(((it & 1) * 2 + 1) * 2 + 0) * 128 + row] = 0.f;
        fin[(((it & 1) * 2 + 1) * 2 + 1) * 128 + row] = -INFINITY;
      }
      warp_arrive(fin_bar + (it & 1));
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------- softmax
    if (kRegSplit && !PV4) reg_alloc<kRegsSoftmax>();
    // Both warpgroups work on every key block: warpgroup w takes keys
    // 64w..64w+63 of it. Thread (warp quarter q, lane t) owns query row
    // 32q + t; its 64 scores are read from tensor memory once and stay in
    // registers. The two halves' row maxima are exchanged per lane through a
    // tagged shared-memory word, so each thread holds the exact running max
    // of its row without any chain between blocks.
    const int w = (warp - 4) >> 2;
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    int g = 0, it = 0;
    bool ok = true;
    for (int rnd = 0, item = next_item(p, rnd); item < p.num_items && ok; ++rnd, item = next_item(p, rnd), ++it) {
      int bh, qb;
      decode_item(p, item, bh, qb);
      const KList L = key_list(p, qb);
      const int qrow = qb * 128 + row;
      float c_fp4 = 0.f, inv_sq = 0.f;
      if (FP4) c_fp4 = p.q_scale[0] * p.k_scale[0] * p.sm_scale_log2;
      else inv_sq = p.sm_scale_log2 / p.q_scale[static_cast<size_t>(bh) * p.nblk + qb];
      float l = 0.f, m_ref = -INFINITY;
      for (int j = 0; j < L.count && ok; ++j, ++g) {
        const int kb_raw = key_block(p, L, j);
        const int kb = max(kb_raw, 0);
        const int buf = g & 1;
        // A failed wait raises the abort flag; the block then runs to its end
        // on whatever the buffers hold (every later wait returns at once) and
        // the loop stops after it.
        ok = warp_wait(s_full + buf, (g >> 1) & 1, abort_flag, &g_error_word, kErrSFull);
        tc_fence_after();
        uint32_t r0[32], r1[32];
        const uint32_t s_addr = tmem + lane_off + buf * 128 + 64 * w;
        tmem_ld32(s_addr, r0);
        tmem_ld32(s_addr + 32, r1);
        tmem_wait_ld(r0);
        tmem_wait_ld(r1);
        // both halves are in registers: the buffer may take the next S
        tc_fence_before();
        warp_arrive(s_free + buf);
        const int key0 = kb * 128 + 64 * w;
        const bool diag = p.causal && kb == qb;
        if (diag || (kb + 1) * 128 > p.N || kb_raw < 0) {
          // an invalid mask entry masks every key of its block
          const int lim = kb_raw < 0 ? 0 : p.N;
          mask_chunk(r0, key0, qrow, diag, lim);
          mask_chunk(r1, key0 + 32, qrow, diag, lim);
        }
        const float half_max = max32(r1, max32(r0, -INFINITY));
        // exchange the half maxima (tag g + 1; slots alternate by block parity)
        xs[(buf * 2 + w) * 128 + row] =
            (static_cast<unsigned long long>(g + 1) << 32) | __float_as_uint(half_max);
        float other_max;
        const bool got = tagged_wait(xs + (buf * 2 + (w ^ 1)) * 128 + row, static_cast<uint32_t>(g + 1), other_max,
                                     abort_flag, &g_error_word, kErrMax);
        ok = __all_sync(0xffffffffu, got) && ok;
        const float rawmax = w == 0 ? fmaxf(half_max, other_max) : fmaxf(other_max, half_max);
        const float c = FP4 ? c_fp4 : inv_sq / p.k_scale[static_cast<size_t>(bh) * p.nblk + kb];
        // m_ref: reference max (-inf while every key so far is masked). It
        // moves to the running max only when that exceeds it by more than tau
        // (log2 units; tau = 0: the exact running max), and P then reaches at
        // most 2^tau, which the P scale 448 * 2^-tau absorbs. m_use: the
        // offset the exponentials use (0 while m_ref is -inf).
        const float m_prev = m_ref;
        const float cand = rawmax == -INFINITY ? m_prev : fmaxf(m_prev, rawmax * c);
        const float m_new = (m_prev == -INFINITY || cand - m_prev > p.tau) ? cand : m_prev;
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        // Rescale factor of O and of the row sum; a row that has seen no key
        // yet (m_prev = -inf) has O = 0 and l = 0, scaled by 2^-inf = 0.
        const float alpha = m_prev == m_new ? 1.f : ex2_approx(m_prev - m_use);
        // the two warpgroups take turns publishing it, which keeps their
        // per-block work equal
        if (w == (g & 1)) {
          ax[(g % kStages) * 128 + row] = alpha;
          warp_arrive(a_bar + q4 * kStages + g % kStages);
        }
        l *= alpha;
        m_ref = m_new;
        // P = 2^(c s - m + log2 448) -> E4M3, this half's 16 columns of P
        // buffer g % kPBufs.
        const float nbias = p.p_log2_scale - m_use;
        const int pb = g % C::kPBufs;
        if (C::kPWait && g >= C::kPBufs) {
          // P buffer pb was last read by the PV of block g - kPBufs
          const int gp = g - C::kPBufs;
          ok = warp_wait(o_done + gp % kStages, (gp / kStages) & 1, abort_flag, &g_error_word, kErrPFree) && ok;
          tc_fence_after();
        }
        float psum;
        if (PV4) {
          // NVFP4 P: this half's 64 keys are one K = 64 step of the P V
          // product: 8 columns of E2M1 and 4 block scales, which go through
          // shared memory (in the tensor-core scale layout) to the PV issuer.
          const uint32_t p_addr = tmem + lane_off + C::kColP + pb * C::kPCols + 8 * w;
          uint32_t pk0[4], pk1[4], sfw = 0u;
          psum = exp_pack32_fp4<C::kPolyPairs>(r0, c, nbias, pk0, sfw, 0);
          tmem_st4(p_addr, pk0);
          psum += exp_pack32_fp4<C::kPolyPairs>(r1, c, nbias, pk1, sfw, 2);
          tmem_st4(p_addr + 4, pk1);
          reinterpret_cast<uint32_t*>(smem + C::kOffSFP + pb * C::kSFP + 512 * w)[(row & 31) * 4 + (row >> 5)] = sfw;
          fence_proxy_async_shared();
        } else {
          const uint32_t p_addr = tmem + lane_off + C::kColP + pb * 32 + 16 * w;
          uint32_t pk0[8], pk1[8];
          psum = exp_pack32<C::kPolyPairs>(r0, c, nbias, pk0);
          tmem_st8(p_addr, pk0);
          psum += exp_pack32<C::kPolyPairs>(r1, c, nbias, pk1);
          tmem_st8(p_addr + 8, pk1);
        }
        l += psum;
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(p_full + pb);
      }
      if (!ok) break;
      // per-item (l, m) of this warpgroup's half of the keys for the epilogue
      if (it >= 2 && !(ok = warp_wait(fin_free + (it & 1), ((it >> 1) - 1) & 1, abort_flag, &g_error_word,
                                      kErrFin)))
        break;
      fin[(((it & 1) * 2 + w) * 2 + 0) * 128 + row] = l;
      fin[(((it & 1) * 2 + w) * 2 + 1) * 128 + row] = m_ref;
      warp_arrive(fin_bar + (it & 1));
    }
  } else {
    // ------------------------------------------------- correction, epilogue
    if (kRegSplit && !PV4) reg_dealloc<kRegsCorrection>();
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t o_base = tmem + (static_cast<uint32_t>(q4 * 32) << 16) + C::kColO;
    int g = 0, it = 0;
    bool ok = true;
    for (int rnd = 0, item = next_item(p, rnd); item < p.num_items && ok; ++rnd, item = next_item(p, rnd), ++it) {
      int bh, qb;
      decode_item(p, item, bh, qb);
      const KList L = key_list(p, qb);
      // this head's V scales, loaded now so their latency hides behind the
      // item's blocks (lane t holds channels t, t + 32, ...)
      // (NVFP4 V: every channel takes 6 / s_t, the P scale's 1/2688 against
      // the 1/448 the row sum is kept in)
      float vsv[D / 32];
#pragma unroll
      for (int i = 0; i < D / 32; ++i)
        vsv[i] = PV4 ? __fdiv_rn(6.f, __ldg(p.v_scale))
                     : __ldg(p.v_scale + static_cast<size_t>(bh) * D + lane + 32 * i);
      for (int j = 0; j < L.count; ++j, ++g) {
        const int slot = g % kStages;
        if (!(ok = warp_wait(a_bar + q4 * kStages + slot, (g / kStages) & 1, abort_flag, &g_error_word, kErrAlpha)))
          break;
        const float alpha = ax[slot * 128 + row];
        // Rows whose running max moved scale O by alpha, once PV of the
        // previous block has landed (block 0 overwrites O instead).
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          if (!(ok = warp_wait(o_done + (g - 1) % kStages, ((g - 1) / kStages) & 1, abort_flag, &g_error_word,
                               kErrODone)))
            break;
          tc_fence_after();
          const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
          for (int cc = 0; cc < D; cc += 32) {
            uint32_t o[32];
            tmem_ld32(o_base + cc, o);
            tmem_wait_ld(o);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const uint64_t v = f2_mul(f2_pack(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), a2);
              float lo, hi;
              f2_unpack(v, lo, hi);
              o[2 * i] = __float_as_uint(lo);
              o[2 * i + 1] = __float_as_uint(hi);
            }
            tmem_st32(o_base + cc, o);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        warp_arrive(o_ready + slot);
      }
      if (!ok) break;
      // epilogue: combine the two warpgroups' row sums, normalize, store
      if (!(ok = warp_wait(fin_bar + (it & 1), (it >> 1) & 1, abort_flag, &g_error_word, kErrFin))) break;
      const float* f = fin + (it & 1) * 512;
      const float l0 = f[0 * 128 + row], m0 = f[1 * 128 + row];
      const float l1 = f[2 * 128 + row], m1 = f[3 * 128 + row];
      warp_arrive(fin_free + (it & 1));
      const float m = fmaxf(m0, m1);
      const float ltot = (l0 > 0.f ? l0 * ex2_approx(m0 - m) : 0.f) + (l1 > 0.f ? l1 * ex2_approx(m1 - m) : 0.f);
      const float inv_l = ltot > 0.f ? 1.f / ltot : 0.f;
      if (L.count > 0) {
        if (!(ok = warp_wait(o_done + (g - 1) % kStages, ((g - 1) / kStages) & 1, abort_flag, &g_error_word,
                             kErrODone)))
          break;
        tc_fence_after();
      }
      const int qrow = qb * 128 + row;
      const bool store = qrow < p.N;
      // per-channel 1 / V scale in the warp's own shared-memory slice (read
      // back as broadcasts)
      float* rv = inv_vs + q4 * D;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) rv[lane + 32 * i] = __frcp_rn(vsv[i]);
      // the staging tile's previous contents must have been read out
      if (lane == 0) bulk_wait_read();
      __syncwarp();
      // Each thread writes its bf16 row into the warp's staging tiles (32 rows
      // x 64 columns each, 16-byte granule g of row r at g ^ (r % 8): the
      // tensor map's 128-byte swizzle, free of bank conflicts); one thread
      // then stores them with the tensor engine, which also clips rows >= N.
      // The next item's first PV overwrites O, so this epilogue is on the
      // critical path only until O has been read.
      uint8_t* tile = smem + C::kOffOut + q4 * C::kOutWarpBytes;
#pragma unroll 2
      for (int cc = 0; cc < D; cc += 16) {
        uint32_t o[16];
        if (L.count > 0) {
          tmem_ld16(o_base + cc, o);
          tmem_wait_ld(o);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = 0u;
        }
        uint32_t wd[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          __nv_bfloat162 t = __floats2bfloat162_rn(__uint_as_float(o[2 * i]) * inv_l * rv[cc + 2 * i],
                                                  __uint_as_float(o[2 * i + 1]) * inv_l * rv[cc + 2 * i + 1]);
          wd[i] = *reinterpret_cast<uint32_t*>(&t);
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int col = cc + 8 * k;
          const int gr = (col & 63) >> 3;
          uint4* dst = reinterpret_cast<uint4*>(tile + (col >> 6) * 4096 + lane * 128 + ((gr ^ (lane & 7)) << 4));
          *dst = make_uint4(wd[4 * k], wd[4 * k + 1], wd[4 * k + 2], wd[4 * k + 3]);
        }
      }
      fence_proxy_async_shared();
      __syncwarp();
      if (lane == 0) {
        if (p.tmap.on) {
          // the warp's 32 rows form one box of the raster grid; its first
          // row is the box's corner
          int t0, h0, w0;
          tile_major_coords(p.tmap, static_cast<uint32_t>(qb * 128 + q4 * 32), t0, h0, w0);
#pragma unroll
          for (int h = 0; h < D / 64; ++h) tma_store_5d(&p.tm_out, tile + h * 4096, h * 64, w0, h0, t0, bh);
        } else {
          const uint64_t stream = l2_policy_evict_first();  // written once, read by no one here
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
            tma_store_3d_hint(&p.tm_out, tile + h * 4096, h * 64, qb * 128 + q4 * 32, bh, stream);
        }
        bulk_commit();
      }
      if (store && p.lse)
        p.lse[static_cast<size_t>(bh) * p.N + to_raster(p.tmap, qrow)] =
            ltot > 0.f ? (m + __log2f(ltot) - p.p_log2_scale) * kLn2 : -INFINITY;
      tc_fence_before();
    }
    if (lane == 0) bulk_wait_all();
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
  griddep_launch_dependents();
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

bool make_out_map(CUtensorMap* m, void* base, int d, int N, int BH) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(d) * 2 * static_cast<cuuint64_t>(N)};
  cuuint32_t box[3] = {64u, 32u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [BH][T][Hs][W][d] with a box of 64 channels x one 32-row chunk.
bool make_out_map_video(CUtensorMap* m, void* base, int d, const VideoLayout& v, int BH) {
  EncodeTiledFn enc = get_encoder();
  int bw, bh, bt;
  if (!enc || !video_chunk_box(v, bw, bh, bt)) return false;
  const cuuint64_t row = static_cast<cuuint64_t>(d) * 2;
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(v.W), static_cast<cuuint64_t>(v.Hs),
                        static_cast<cuuint64_t>(v.T), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[4] = {row, row * v.W, row * v.W * v.Hs, row * v.W * v.Hs * v.T};
  cuuint32_t box[5] = {64u, static_cast<cuuint32_t>(bw), static_cast<cuuint32_t>(bh), static_cast<cuuint32_t>(bt),
                       1u};
  cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

CUtensorMapSwizzle swizzle_for(int row_bytes) {
  return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// NVFP4 V, transposed: bytes [BH][D][nkb * 64] with box [1][D][64] (one
// 128-key block of every channel), 64-byte swizzle.
bool make_map_vt(CUtensorMap* m, const void* base, int D, int nkb, int BH) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  const cuuint64_t pitch = static_cast<cuuint64_t>(nkb) * 64;
  cuuint64_t dims[3] = {pitch, static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {pitch, pitch * static_cast<cuuint64_t>(D)};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(D), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool FP4, bool PV4>
cudaError_t launch_t(const AttnArgs& a, cudaStream_t st) {
  using C = Cfg<D, FP4, PV4>;
  Params p;
  const int BH = a.B * a.H;
  const int qk_row = C::kQKRow;
  const int nkb = (a.N + 127) / 128;
  if (!make_map(&p.tm_q, a.q, qk_row, a.N, BH, swizzle_for(qk_row)) ||
      !make_map(&p.tm_k, a.k, qk_row, a.N, BH, swizzle_for(qk_row)) ||
      !(PV4 ? make_map_vt(&p.tm_v, a.v, D, nkb, BH) : make_map(&p.tm_v, a.v, D, a.N, BH, swizzle_for(D))))
    return cudaErrorNotSupported;
  if (a.video) {
    if (!make_out_map_video(&p.tm_out, a.out, D, *a.video, BH)) return cudaErrorNotSupported;
    p.tmap = make_token_map(a.video->T, a.video->Hs, a.video->W, a.video->tt, a.video->th, a.video->tw);
  } else {
    if (!make_out_map(&p.tm_out, a.out, D, a.N, BH)) return cudaErrorNotSupported;
    p.tmap = TokenMap{};
  }
  p.q_sf = a.q_sf;
  p.k_sf = a.k_sf;
  p.v_sf = a.v_sf;
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
  const int sms = device_sm_count();
  const int grid = p.num_items < sms ? p.num_items : sms;
  p.hgroup = BH;
  p.gspan = p.num_items;
  p.hpairs = 0;
  if (p.causal && !p.sparse) {
    CausalPlan cp;
    causal_plan(BH, a.N, D, FP4, PV4, grid, &cp);
    p.hgroup = cp.hgroup;
    p.gspan = cp.gspan;
    p.hpairs = cp.hpairs;
    p.num_items = cp.num_items;
  }
  p.nnz = a.nnz;
  p.sm_scale_log2 = a.softmax_scale * 1.4426950408889634f;
  p.tau = a.rescale_threshold;
  p.p_log2_scale = kLog2_448 - a.rescale_threshold;
  // The shared-memory opt-in is a per-device attribute of the kernel: set it
  // once on each device this process launches on.
  static std::atomic<unsigned long long> configured[(kMaxDevices + 63) / 64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const bool cacheable = dev >= 0 && dev < kMaxDevices;
  const unsigned long long bit = cacheable ? 1ull << (dev % 64) : 0ull;
  if (!cacheable || !(configured[cacheable ? dev / 64 : 0].load(std::memory_order_acquire) & bit)) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, FP4, PV4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemRequest);
    if (e != cudaSuccess) return e;
    if (cacheable) configured[dev / 64].fetch_or(bit, std::memory_order_acq_rel);
  }
  if (kRegSplit && !PV4) {
    // The per-warpgroup budgets add up to the 128 registers a thread the
    // kernel must launch with; with fewer, the softmax warps' increase could
    // never be granted, so such a build is refused instead of launched.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attn_fwd_kernel<D, FP4, PV4>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * kThreads < static_cast<int>(128 * (kRegsControl + kRegsCorrection) + 256 * kRegsSoftmax))
      return cudaErrorInvalidConfiguration;
  }
  const cudaError_t e = launch_pdl(attn_fwd_kernel<D, FP4, PV4>, dim3(grid), dim3(kThreads), C::kSmemRequest, st, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

// L2 share for the K/V of one causal head group: 32 MiB of the 126 MB L2 (the
// LLM prefill's 37-head groups read each K/V byte from DRAM once; with all
// 128 heads in flight, five times).
#ifndef FPATTN_CAUSAL_GROUP_MB
#define FPATTN_CAUSAL_GROUP_MB 32
#endif
constexpr double kCausalGroupBytes = FPATTN_CAUSAL_GROUP_MB * 1024.0 * 1024.0;
// 0 keeps every causal launch on the longest-first order
#ifndef FPATTN_CAUSAL_PAIRS
#define FPATTN_CAUSAL_PAIRS 1
#endif

namespace {

// Schedule positions of a causal head group of n items: rounded up to whole
// pairs of snake rounds over `grid` CTAs.
long long padded_span(long long n, int grid) {
  const long long pair = 2LL * grid;
  return (n + pair - 1) / pair * pair;
}

// Makespan of the causal snake schedule with heads in groups of g (padded
// unless one group holds every head), in 128x128 blocks with one block of
// per-item cost added; `load` is scratch for the per-CTA sums.
double causal_makespan(int BH, int nblk, int g, int grid, std::vector<double>& load) {
  load.assign(grid, 0.0);
  long long pos = 0;
  for (int g0 = 0; g0 < BH; g0 += g) {
    const int gsz = std::min(g, BH - g0);
    const long long n = static_cast<long long>(gsz) * nblk;
    for (long long r = 0; r < n; ++r) {
      const long long at = pos + r;
      const long long rnd = at / grid;
      const int c = static_cast<int>(at % grid);
      load[(rnd & 1) ? grid - 1 - c : c] += static_cast<double>(nblk - r / gsz) + 1.0;
    }
    pos += g >= BH ? n : padded_span(n, grid);
  }
  return *std::max_element(load.begin(), load.end());
}

// Heads per group of the causal schedule. Longest rows first over all heads
// puts the same query block of every head in flight at once, so the K/V of
// all heads pass through the L2 together. Groups whose K and V (codes and
// scales, kv_head bytes a head) fit in kCausalGroupBytes keep that
// working set in L2; a group size is taken only if its padded schedule is
// within 0.5% of the ungrouped one's balance (modelled on the host), else all
// heads form one group.
int causal_head_group(int BH, int nblk, int grid, double kv_head) {
  const double budget = kCausalGroupBytes;
  if (budget <= 0.0 || kv_head <= 0.0) return BH;
  const double fit = budget / kv_head;
  if (fit >= BH) return BH;
  const int gmax = fit < 1.0 ? 1 : static_cast<int>(fit);
  std::vector<double> load;
  const double base = causal_makespan(BH, nblk, BH, grid, load);
  int best = BH;
  double best_m = base * 1.005;
  // at most 64 sizes, largest first, and about 2^21 modelled items in all
  // (a few milliseconds of host time, once per shape); a smaller group must
  // beat a larger one by 0.1% to be taken
  const long long items = static_cast<long long>(BH) * nblk;
  const int budget_sizes = static_cast<int>(std::max(1LL, std::min(64LL, (1LL << 21) / std::max(1LL, items))));
  for (int g = gmax, tried = 0; g >= 1 && tried < budget_sizes; --g, ++tried) {
    const double m = causal_makespan(BH, nblk, g, grid, load);
    if (m <= best_m && (best == BH || m < best_m * 0.999)) {
      best = g;
      best_m = m;
    }
  }
  return best;
}

}  // namespace

// Paired order for the causal launch, if its modelled makespan is within
// 1.5% of the ungrouped snake's; returns false (plan untouched) otherwise.
static bool causal_pairs(int BH, int nblk, int grid, CausalPlan* plan) {
  const int hp = (nblk + 1) / 2;
  const long long pairs = static_cast<long long>(BH) * hp;
  if (2 * pairs > INT_MAX / 2) return false;
  std::vector<double> load;
  const double base = causal_makespan(BH, nblk, BH, grid, load);
  load.assign(grid, 0.0);
  for (long long j = 0; j < pairs; ++j) {
    const int i = static_cast<int>(j % hp);
    const int lo = i, hi = nblk - 1 - i;
    load[j % grid] += (hi + 2.0) + (hi != lo ? lo + 2.0 : 0.0);
  }
  if (*std::max_element(load.begin(), load.end()) > base * 1.015) return false;
  plan->hpairs = hp;
  plan->num_items = static_cast<int>(2 * pairs);
  return true;
}

// Which order a causal launch takes, as measured on the sequence sweep
// (B*H*N = 2^22 tokens, H = 32) against the plain longest-first snake:
// - NVFP4 Q/K with at most 32 query blocks: L2-sized head groups (+3% to
//   +8% at N <= 2048, neutral at 4096; LLM prefill reads its K/V once).
//   With FP8 Q/K the groups were 5-12% slower at N = 1024-2048, so FP8 keeps
//   the snake.
// - d = 128 with at least 32 query blocks and K/V beyond the whole L2 (four
//   shares): pairs (+8% to +23% from N = 4096 up). At d = 64 the pairs were
//   1.5-2.5% slower, and with fewer blocks 7-23% slower.
static void causal_plan_uncached(int BH, int N, int D, bool qk_fp4, bool pv_fp4, int grid, CausalPlan* plan) {
  const int nblk = (N + 127) / 128;
  plan->hgroup = BH;
  plan->gspan = BH * nblk;
  plan->hpairs = 0;
  plan->num_items = BH * nblk;
  if (BH < 1 || nblk < 1 || grid < 1) return;
  // K codes and block scales, V codes: the bytes of one head's keys
  const double kv_head = static_cast<double>(N) * ((qk_fp4 ? D / 2.0 + D / 16.0 : D) + (pv_fp4 ? D / 2.0 : D));
  if (qk_fp4 && nblk <= 32) {
    const int g = causal_head_group(BH, nblk, grid, kv_head);
    if (g < BH) {
      const long long span = padded_span(static_cast<long long>(g) * nblk, grid);
      const int rest = BH % g;
      const long long total =
          (BH / g) * span + (rest ? padded_span(static_cast<long long>(rest) * nblk, grid) : 0);
      if (total > INT_MAX / 2) return;  // keep positions in int range: one group, no padding
      plan->hgroup = g;
      plan->gspan = static_cast<int>(span);
      plan->num_items = static_cast<int>(total);
      return;
    }
  }
  if (FPATTN_CAUSAL_PAIRS && D == 128 && nblk >= 32 && BH * kv_head > 4 * kCausalGroupBytes)
    causal_pairs(BH, nblk, grid, plan);
}

// The plans of the last 64 shapes are kept: modelling one takes host time
// (about 30 ns per modelled item: a few milliseconds for the head groups,
// whose search is capped, and for the pairs linear in B*H*N/128, far below
// the launch's own time, which grows with the square of N); a launch of the
// same shape needs none.
void causal_plan(int BH, int N, int D, bool qk_fp4, bool pv_fp4, int grid, CausalPlan* plan) {
  struct Entry {
    int BH, N, D, flags, grid;
    CausalPlan plan;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  const int flags = (qk_fp4 ? 1 : 0) | (pv_fp4 ? 2 : 0);
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& e : cache)
      if (e.BH == BH && e.N == N && e.D == D && e.flags == flags && e.grid == grid) {
        *plan = e.plan;
        return;
      }
  }
  causal_plan_uncached(BH, N, D, qk_fp4, pv_fp4, grid, plan);
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() >= 64) cache.erase(cache.begin());
  cache.push_back(Entry{BH, N, D, flags, grid, *plan});
}

cudaError_t launch_attn_fwd(const AttnArgs& a, cudaStream_t st) {
  if (a.pv_fp4) {
    if (a.d == 128) return a.qk_fp4 ? launch_t<128, true, true>(a, st) : launch_t<128, false, true>(a, st);
    return a.qk_fp4 ? launch_t<64, true, true>(a, st) : launch_t<64, false, true>(a, st);
  }
  if (a.d == 128) return a.qk_fp4 ? launch_t<128, true, false>(a, st) : launch_t<128, false, false>(a, st);
  return a.qk_fp4 ? launch_t<64, true, false>(a, st) : launch_t<64, false, false>(a, st);
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
