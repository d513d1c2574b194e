// Stage 4-5 of In-context Sparse Attention: both attention paths and the
// write-back, as one persistent tcgen05 kernel.
//
// Method: "Lightning Unified Video Editing via In-Context Sparse Attention",
// papernotes.org notes, Key design 2 and the flowchart:
//  * exact path (sharp query blocks): S = Q K_new^T / sqrt(D), P = exp(S),
//    l += rowsum(P), O += P V_new, O /= l, by online softmax over all keys of
//    K_new = [K_src ; kept context blocks];
//  * block-wise 0th-order Taylor path (flat query blocks): each block j of
//    K_new stands in as b * exp(q . Kc_j / sqrt(D)) paired with Vc_j. Every
//    block holds b keys, so the weight b cancels between numerator and
//    denominator and the path is softmax(q Kc_new^T / sqrt(D)) Vc_new: the same
//    online-softmax attention, against the n_new pooled rows instead of L_new
//    keys. The paperlayer.ai summary, section 3 (Taylor Sparse Attention),
//    gives the O(L_Q D) cost per query block that this reaches;
//  * each output row is written at its original token position (each query
//    block takes exactly one path, so there is nothing to merge).
// When b does not divide L_src or L_ctx, the last block of either part is
// short. K_new still takes b rows per block; the rows past a short block's keys
// are masked. A short block's pooled row carries log2(len / b) on its exponent,
// so that in the Taylor path it weighs its own length (the weight no longer
// cancels for it). Query rows are addressed by block start, and only a block's
// own rows are stored. Such calls are run by this kernel, not the CTA-pair one.
//
// Design for sm_100a (prior art on the pages is Triton / TileLang on Hopper):
//  * one CTA per SM (persistent), 12 warps: warp 0 issues TMA loads, warp 1
//    owns TMEM and issues tcgen05.mma from one thread (warps 2-3 idle), warps
//    4-7 and 8-11 are two softmax warpgroups, one per 128-row query tile; each
//    softmax thread owns one query row and keeps its 128 scores in registers
//    (setmaxnreg moves registers from warpgroup 0 to them);
//  * P is written and released in two halves (keys 0-63, then 64-127), and the
//    P V MMAs of a half start as soon as it is released;
//  * a work item is up to two 128-row query tiles of one head (four blocks
//    when b = 64), both walking the same K/V tiles, so every K/V tile is
//    loaded once for 256 query rows;
//  * TMEM: S_t at columns [128 t, 128 t + 128), O_t at [256 + 128 t, ...);
//    P_t is written over S_t (bf16 pairs, or fp32 for tf32) and fed to the
//    P V MMA straight from TMEM;
//  * MMA order per K/V tile j: PV0_j, S0_{j+1}, PV1_j, S1_{j+1}, so the tensor
//    core works on one tile while the softmax warps work on the other;
//  * lazy rescaling: the running max only moves when it grows by more than
//    2^8, and only then is the O row rescaled in TMEM by its own thread;
//  * exact items come first in the static schedule and Taylor items after.
//
// The same kernel, instantiated with NS = true, computes Taylor query blocks
// with some key blocks kept exact (the no-sparsity ratio alpha_ns of
// papernotes.org, Key design 3; Key design 2 gives the two kinds of terms and
// their one softmax). Each query block u has its own set E_u of k_ns blocks of
// K_new. An item (the Taylor blocks of two query tiles) walks first the pooled
// rows of K_new, each weighted by b (a log2(b) bias on its exponent) and masked
// for the row's own E_u, then the key tiles of the union of its blocks' E_u in
// ascending block order. The K/V tiles are loaded once for both query tiles,
// but a query tile takes part (S and P V MMAs, softmax) only in the key tiles
// that hold one of its own blocks' E_u, and a tile that sits out a key tile gets
// the S of its next one at once, so the two tiles' softmax steps overlap. Inside
// a key tile every row masks the blocks outside its own E_u.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <float.h>

#include "exp2_poly.cuh"
#include "isa_internal.h"
#include "ptx.cuh"
#include "tensor_map.cuh"

namespace isa {
namespace {

// One softmax thread per query row holds all 128 scores of its row. (Two threads
// per row, exchanging partial maxima through shared memory, measured slower:
// 6.05 ms against 4.78 ms for the attention kernel at the 32K-token workload.)
constexpr int kThreads = 384;  // warpgroup 0 (TMA, MMA) + one softmax warpgroup per query tile
// Register budget: the kernel is compiled for 168 registers a thread at launch
// (384 x 168 = 64512 of the SM's 65536). Warpgroup 0 (TMA + MMA warps) gives
// registers back and the two softmax warpgroups take them:
// 128 x 88 + 256 x 208 = 64512, the same total, so the increase never waits.
// The launcher checks the compiled count before every launch.
constexpr int kLaunchRegs = 168;
constexpr int kLowRegs = 88;
constexpr int kHighRegs = 208;
static_assert(128 * kLowRegs + 256 * kHighRegs <= kThreads * kLaunchRegs, "register split exceeds the launch budget");
constexpr int kCols = 128;  // scores per softmax thread
constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per K/V tile
// The running row maximum only moves (and O is rescaled) when a tile's maximum
// exceeds it by more than this many powers of two; P then stays below 2^this.
#ifndef ISA_RESCALE_LOG2
#define ISA_RESCALE_LOG2 8
#endif
constexpr float kRescaleThreshold = (float)ISA_RESCALE_LOG2;
// Share of the exponentials computed by the FMA-pipe polynomial instead of ex2:
// pair i of a row goes to the polynomial when (i % kPolyDen) < kPolyNum. On B200
// the softmax is bound by instruction issue, not by the ex2 unit, so the
// polynomial's extra instructions cost more than they save: measured at the
// 32K-token workload, the attention kernel takes 4.78 ms with no polynomial
// share, 5.07 ms with 1/4 and 5.44 ms with 1/2. It stays available here.
#ifndef ISA_POLY_NUM
#define ISA_POLY_NUM 0
#endif
#ifndef ISA_POLY_DEN
#define ISA_POLY_DEN 4
#endif
constexpr int kPolyNum = ISA_POLY_NUM;
constexpr int kPolyDen = ISA_POLY_DEN;

struct AttnParams {
  const int32_t* route;
  void* out;
  uint32_t* err;
  float* lse;          // optional [BH, N] (plain path only): natural log of each row's softmax denominator
  float taylor_ln_b;   // ln(b): the Taylor rows' weight b, dropped from their exponents, back in their lse
  const uint32_t* nsmask;  // NS: [BH, n_q, ns_words] exact key blocks of every query block
  int ns_words;            // NS: ceil(n_new / 32)
  int npt;                 // NS: K/V tiles of the pooled rows, ceil(n_new / 128)
  float bias_log2;         // NS: log2(b), the weight of a pooled row in the exponent
  // Short blocks (b does not divide L_src or L_ctx). Block j of K_new takes rows [j b, j b + b),
  // the rows past a short block's length are masked; a pooled row weighs its block's length.
  const int32_t* sel;      // [BH, k] kept context blocks (the short last one can only be the last kept)
  int k, n_src, n_ctx, L_srcp, len_src_last, len_ctx_last, ragged;
  float src_last_bias, ctx_last_bias;  // log2(len / b) / scale_log2: raw-score offsets of short pooled rows
  int BH, N, b, L_src, n_q, n_exact, n_flat, L_new, n_new;
  int bpt;       // blocks per 128-row tile (128 / b)
  int bpi;       // blocks per item (2 tiles)
  int items_e;   // exact items per head
  int items_t;   // Taylor items per head
  int total;     // all items
  float scale_log2;
};

// First token of query block i (source blocks from 0, context blocks from L_src) and its length.
__device__ __forceinline__ int qblock_start(const AttnParams& p, int i) {
  return i < p.n_src ? i * p.b : p.L_src + (i - p.n_src) * p.b;
}
__device__ __forceinline__ int qblock_len(const AttnParams& p, int i) {
  return i == p.n_src - 1 ? p.len_src_last : (i == p.n_q - 1 ? p.len_ctx_last : p.b);
}
// Whether head bh keeps the short last context block, which is then the last block of K_new.
__device__ __forceinline__ bool short_ctx_kept(const AttnParams& p, int bh) {
  return p.len_ctx_last < p.b && p.k > 0 && __ldg(p.sel + (size_t)bh * p.k + p.k - 1) == p.n_ctx - 1;
}
// Keys held by block j of K_new (b unless it is a short block).
__device__ __forceinline__ int new_block_len(const AttnParams& p, int j, bool ctx_short) {
  return j == p.n_src - 1 ? p.len_src_last : (ctx_short && j == p.n_new - 1 ? p.len_ctx_last : p.b);
}

struct Bars {
  uint64_t q_full[2];
  uint64_t q_empty;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], p_half[2][2], o_done[2];  // p_half[t][k]: P of keys 64k..64k+63 written
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  // NS: query tiles taking part in the K/V tile of each stage (bit t = tile t), written by
  // the producer before it arms k_full of the stage, read by the MMA issuer after that wait
  uint32_t stage_tiles[2];
};

template <typename T, int D>
struct Cfg {
  static constexpr int E = sizeof(T);
  static constexpr bool kTf32 = (E == 4);
  static constexpr int RB = D * E;              // bytes per row
  static constexpr int NCH = RB / 128;          // 128-byte swizzle chunks per row
  static constexpr int CH_STRIDE = kBM * 128;   // bytes between chunks of a 128-row tile
  static constexpr int TILE = kBM * RB;         // bytes of one 128-row tile
  static constexpr int BOX_X = 128 / E;         // elements per 128-byte chunk row
  static constexpr int KS_QK = RB / 32;         // UMMA K-steps of Q K^T (32 bytes each)
  static constexpr int PV_K = 32 / E;           // keys per P V UMMA
  static constexpr int KS_PV = kBN / PV_K;
  static constexpr int STAGES = 2;
  static constexpr uint32_t FMT = kTf32 ? 2u : 1u;
  static constexpr uint32_t IDESC_QK = umma_idesc(FMT, kBM, kBN, 0, 0);
  // bf16: V tiles as stored ([keys][D], MN-major B). tf32 takes B K-major only,
  // so fp32 inputs load tiles of V^T ([D][keys], 32-key chunks of 128 bytes).
  static constexpr bool kVT = kTf32;
  static constexpr int VT_CH_STRIDE = D * 128;  // bytes between 32-key chunks of a V^T tile
  static constexpr uint32_t IDESC_PV = umma_idesc(FMT, kBM, D, 0, kVT ? 0u : 1u);
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = 2 * TILE;
  static constexpr int OFF_V = OFF_K + STAGES * TILE;
  static constexpr int OFF_BAR = OFF_V + STAGES * TILE;
  static constexpr int SMEM_USED = OFF_BAR + (int)sizeof(Bars);
  // padded above half of the SM's shared memory so that exactly one CTA (and one
  // 512-column TMEM allocation) lives on each SM
  static constexpr int SMEM_ALLOC = (SMEM_USED + 1024 > 120 * 1024 ? SMEM_USED + 1024 : 120 * 1024);
  static_assert(NCH >= 1 && NCH <= 2, "row of 128 or 256 bytes");
  static_assert(D % 32 == 0, "D multiple of 32");
};

struct Item {
  int bh, kind, nblk, ntiles, nkv, last_valid;
  int nu;  // NS: blocks in the union of the item's exact key blocks
  int blk0, blk1, blk2, blk3;  // query blocks of the item (repeats of blk0 past nblk)
  __device__ __forceinline__ int blk(int u) const { return u == 0 ? blk0 : u == 1 ? blk1 : u == 2 ? blk2 : blk3; }
};

// NS: word `wd` of the union of the exact-block bitmasks of the item's query blocks
// (blocks past nblk repeat blk0, so all loads are issued unconditionally and at once)
__device__ __forceinline__ uint32_t union_word(const AttnParams& p, const Item& it, int wd) {
  const uint32_t* m = p.nsmask + (size_t)it.bh * p.n_q * p.ns_words + wd;
  uint32_t x = __ldg(m + (size_t)it.blk0 * p.ns_words) | __ldg(m + (size_t)it.blk1 * p.ns_words);
  if (p.bpi > 2) x |= __ldg(m + (size_t)it.blk2 * p.ns_words) | __ldg(m + (size_t)it.blk3 * p.ns_words);
  return x;
}

// NS: walks the union of an item's exact key blocks in ascending order. Callers ask
// for at most it.nu blocks; past the end it returns block 0. (Walking the blocks that
// only one query tile keeps in alternation, so that consecutive K/V tiles belong to
// different tiles, measured slower: 6.35 ms against 5.99 ms for the attention stage
// at the 32K-token workload with alpha_ns = 0.0625, on one box.)
struct BlockCursor {
  int wd = -1;
  uint32_t bits = 0;
  __device__ __forceinline__ int next(const AttnParams& p, const Item& it) {
    while (bits == 0 && wd + 1 < p.ns_words) bits = union_word(p, it, ++wd);
    if (bits == 0) return 0;
    const int j = __ffs(bits) - 1;
    bits &= bits - 1;
    return 32 * wd + j;
  }
};

// NS: blocks of exact K/V tile j (the next 128 / b blocks of the union); bk1 is the
// second 64-key block when b = 64, or -1 (b = 128, or past the end of the union).
struct KeyTile {
  int bk0, bk1;
};
__device__ __forceinline__ KeyTile next_key_tile(const AttnParams& p, const Item& it, BlockCursor& cur, int j) {
  KeyTile kt;
  kt.bk0 = cur.next(p, it);
  kt.bk1 = (p.b == 64 && 2 * (j - p.npt) + 1 < it.nu) ? cur.next(p, it) : -1;
  return kt;
}
__device__ __forceinline__ bool has_block(const uint32_t* mask, int bk) {
  return bk >= 0 && ((__ldg(mask + (bk >> 5)) >> (bk & 31)) & 1u) != 0u;
}

// NS: whether query tile t of the item keeps a block of the K/V tile (any of its query blocks)
__device__ __forceinline__ bool tile_keeps(const AttnParams& p, const Item& it, int t, const KeyTile& kt) {
  const int u0 = t * p.bpt, u1 = min(it.nblk, u0 + p.bpt);
  for (int u = u0; u < u1; ++u) {
    const uint32_t* m = p.nsmask + ((size_t)it.bh * p.n_q + it.blk(u)) * p.ns_words;
    if (has_block(m, kt.bk0) || has_block(m, kt.bk1)) return true;
  }
  return false;
}

template <bool NS>
__device__ __forceinline__ Item decode_item(const AttnParams& p, int g) {
  Item it;
  int count, base, pp;
  if (g < p.BH * p.items_e) {
    it.bh = g / p.items_e;
    pp = g - it.bh * p.items_e;
    it.kind = 0;
    count = p.n_exact;
    base = 0;
  } else {
    const int g2 = g - p.BH * p.items_e;
    it.bh = g2 / p.items_t;
    pp = g2 - it.bh * p.items_t;
    it.kind = 1;
    count = p.n_flat;
    base = p.n_exact;
  }
  const int32_t* lst = p.route + (size_t)it.bh * p.n_q + base;
  const int first = pp * p.bpi;
  it.nblk = min(p.bpi, count - first);
  it.blk0 = __ldg(lst + first);
  it.blk1 = it.nblk > 1 ? __ldg(lst + first + 1) : it.blk0;
  it.blk2 = it.nblk > 2 ? __ldg(lst + first + 2) : it.blk0;
  it.blk3 = it.nblk > 3 ? __ldg(lst + first + 3) : it.blk0;
  it.ntiles = (it.nblk + p.bpt - 1) / p.bpt;
  if constexpr (NS) {
    // pooled rows, then the union of the exact blocks, 128 / b blocks per K/V tile
    // (four words of every query block's mask per round, all loads issued before any is used;
    // blocks past nblk repeat blk0, so OR-ing them changes nothing)
    const uint32_t* m = p.nsmask + (size_t)it.bh * p.n_q * p.ns_words;
    const uint32_t *m0 = m + (size_t)it.blk0 * p.ns_words, *m1 = m + (size_t)it.blk1 * p.ns_words;
    const uint32_t *m2 = m + (size_t)it.blk2 * p.ns_words, *m3 = m + (size_t)it.blk3 * p.ns_words;
    const bool four = p.bpi > 2;
    int nu = 0;
    for (int wd = 0; wd < p.ns_words; wd += 4) {
      uint32_t x[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int w = min(wd + i, p.ns_words - 1);
        x[i] = __ldg(m0 + w) | __ldg(m1 + w);
        if (four) x[i] |= __ldg(m2 + w) | __ldg(m3 + w);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) nu += wd + i < p.ns_words ? __popc(x[i]) : 0;
    }
    it.nu = nu;
    it.nkv = p.npt + (nu + p.bpt - 1) / p.bpt;
    it.last_valid = p.n_new - kBN * (p.npt - 1);  // of the last pooled tile
  } else {
    const int rows = it.kind == 0 ? p.L_new : p.n_new;
    it.nu = 0;
    it.nkv = (rows + kBN - 1) / kBN;
    it.last_valid = rows - kBN * (it.nkv - 1);
  }
  return it;
}


__device__ __forceinline__ bool aborted(const Bars* b) {
  return *reinterpret_cast<const volatile int*>(&b->abort_flag) != 0;
}
__device__ __forceinline__ void raise_abort(Bars* b, uint32_t* err, uint32_t code) {
  atomicOr(err, code);
  *reinterpret_cast<volatile int*>(&b->abort_flag) = 1;
}

// All 32 lanes wait on the barrier; the result is the same in every lane and the
// warp is converged on return (the TMEM moves that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(Bars* b, uint64_t* bar, uint32_t parity, uint32_t* err) {
  bool ok = mbar_wait_or_abort(bar, parity, &b->abort_flag);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) raise_abort(b, err, kErrSoftmax);
  tc_fence_after();
  return ok;
}

// -inf on the scores of the K/V tile columns whose K_new rows (tile rows from `base`) lie in [lo, hi)
__device__ __forceinline__ void mask_key_rows(uint32_t (&r)[kCols], int base, int lo, int hi) {
  if (hi <= base || lo >= base + kBN) return;  // the same for every thread of the CTA
#pragma unroll
  for (int i = 0; i < kCols; ++i)
    if (base + i >= lo && base + i < hi) r[i] = 0xff800000u;
}
// Adds `delta` to the raw score of the column holding pooled row `col` (tile rows from `base`)
__device__ __forceinline__ void add_col_bias(uint32_t (&r)[kCols], int base, int col, float delta) {
  const int c = col - base;
  if (c < 0 || c >= kBN) return;
#pragma unroll
  for (int i = 0; i < kCols; ++i)
    if (i == c) r[i] = __float_as_uint(__uint_as_float(r[i]) + delta);
}

template <typename T>
__device__ __forceinline__ void store_row_chunk(T* dst, const float* v);  // 32 values

template <>
__device__ __forceinline__ void store_row_chunk<__nv_bfloat16>(__nv_bfloat16* dst, const float* v) {
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    pk[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
}
template <>
__device__ __forceinline__ void store_row_chunk<float>(float* dst, const float* v) {
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 8; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

template <typename T, int D, bool NS>
__global__ void __launch_bounds__(kThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_ksel, const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_vsel, const __grid_constant__ CUtensorMap tm_kcn,
                     const __grid_constant__ CUtensorMap tm_vcn, const AttnParams p) {
  using C = Cfg<T, D>;
  static_assert(!NS || !C::kVT, "exact key blocks inside the Taylor path need bf16 tiles");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  Bars* bars = reinterpret_cast<Bars*>(smem + C::OFF_BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->q_full[t], 1);
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_half[t][0], 128);
      mbar_init(&bars->p_half[t][1], 128);
      mbar_init(&bars->o_done[t], 1);
    }
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_ksel);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_vsel);
    tma_prefetch_desc(&tm_kcn);
    tma_prefetch_desc(&tm_vcn);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp < 4) regs_dealloc<kLowRegs>();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t kv_it = 0, n_local = 0, k_issued = 0, v_issued = 0, q_arm0 = 0, q_arm1 = 0;
      bool ok = true;
      for (int g = blockIdx.x; g < p.total && ok; g += gridDim.x, ++n_local) {
        const Item it = decode_item<NS>(p, g);
        if (n_local > 0 && !mbar_wait(&bars->q_empty, (n_local - 1) & 1)) {
          raise_abort(bars, p.err, kErrProducer);
          ok = false;
          break;
        }
        for (int t = 0; t < it.ntiles; ++t) {
          mbar_arrive_expect_tx(&bars->q_full[t], C::TILE);
          if (t == 0) ++q_arm0; else ++q_arm1;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int r = 64 * h;
            int u = t * p.bpt + r / p.b;
            if (u >= it.nblk) u = t * p.bpt;  // missing block: load a valid one, rows are not stored
            const int y = qblock_start(p, it.blk(u)) + (r % p.b);  // rows past a short block: not stored
#pragma unroll
            for (int c = 0; c < C::NCH; ++c)
              tma_load_3d(sQ + t * C::TILE + c * C::CH_STRIDE + h * 8192, &tm_q, &bars->q_full[t], c * C::BOX_X,
                          y, it.bh);
          }
        }
        BlockCursor cur;
        for (int j = 0; j < it.nkv; ++j, ++kv_it) {
          if (aborted(bars)) { ok = false; break; }
          const int st = kv_it % C::STAGES;
          const uint32_t ph = (kv_it / C::STAGES) & 1;
          // rows of K_new (or of the pooled rows) of the tile's two 64-row halves
          int hrow0 = j * kBN, hrow1 = j * kBN + 64;
          bool new_rows = it.kind == 0;
          uint32_t tiles = 3u;  // NS: query tiles taking part in this K/V tile
          if constexpr (NS) {
            if (j >= p.npt) {
              new_rows = true;
              const KeyTile kt = next_key_tile(p, it, cur, j);
              tiles = (tile_keeps(p, it, 0, kt) ? 1u : 0u) | (it.ntiles > 1 && tile_keeps(p, it, 1, kt) ? 2u : 0u);
              if (p.b == 128) {
                hrow0 = kt.bk0 * 128;
                hrow1 = hrow0 + 64;
              } else {
                hrow0 = kt.bk0 * 64;
                hrow1 = (kt.bk1 >= 0 ? kt.bk1 : kt.bk0) * 64;  // missing second block: loaded, masked
              }
            }
          }
          // K tile
          if (!mbar_wait(&bars->k_empty[st], ph ^ 1)) { raise_abort(bars, p.err, kErrProducer); ok = false; break; }
          if constexpr (NS) *reinterpret_cast<volatile uint32_t*>(&bars->stage_tiles[st]) = tiles;
          mbar_arrive_expect_tx(&bars->k_full[st], C::TILE);
          ++k_issued;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int r0 = h ? hrow1 : hrow0;
            const CUtensorMap* map;
            int y;
            if (new_rows) {
              if (r0 < p.L_srcp) { map = &tm_k; y = r0; } else { map = &tm_ksel; y = r0 - p.L_srcp; }
            } else {
              map = &tm_kcn; y = r0;
            }
#pragma unroll
            for (int c = 0; c < C::NCH; ++c)
              tma_load_3d(sK + st * C::TILE + c * C::CH_STRIDE + h * 8192, map, &bars->k_full[st], c * C::BOX_X,
                          y, it.bh);
          }
          // V tile
          if (!mbar_wait(&bars->v_empty[st], ph ^ 1)) { raise_abort(bars, p.err, kErrProducer); ok = false; break; }
          mbar_arrive_expect_tx(&bars->v_full[st], C::TILE);
          ++v_issued;
          if constexpr (C::kVT) {
            // V^T tile: 4 chunks of 32 keys x D rows (tm_v / tm_vcn hold V_new^T / Vc_new^T here)
            const CUtensorMap* map = it.kind == 0 ? &tm_v : &tm_vcn;
#pragma unroll
            for (int c = 0; c < 4; ++c)
              tma_load_3d(sV + st * C::TILE + c * C::VT_CH_STRIDE, map, &bars->v_full[st], j * kBN + 32 * c, 0,
                          it.bh);
          } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int r0 = h ? hrow1 : hrow0;
              const CUtensorMap* map;
              int y;
              if (new_rows) {
                if (r0 < p.L_srcp) { map = &tm_v; y = r0; } else { map = &tm_vsel; y = r0 - p.L_srcp; }
              } else {
                map = &tm_vcn; y = r0;
              }
#pragma unroll
              for (int c = 0; c < C::NCH; ++c)
                tma_load_3d(sV + st * C::TILE + c * C::CH_STRIDE + h * 8192, map, &bars->v_full[st],
                            c * C::BOX_X, y, it.bh);
            }
          }
        }
      }
      if (!ok) {
        // let every copy this thread started land before the CTA can leave
        if (q_arm0) mbar_wait(&bars->q_full[0], (q_arm0 - 1) & 1);
        if (q_arm1) mbar_wait(&bars->q_full[1], (q_arm1 - 1) & 1);
        for (uint32_t s = 0; s < (uint32_t)C::STAGES; ++s) {
          // tiles issued into stage s so far: those with index = s (mod STAGES)
          const uint32_t ka = k_issued > s ? (k_issued - s + C::STAGES - 1) / C::STAGES : 0;
          const uint32_t va = v_issued > s ? (v_issued - s + C::STAGES - 1) / C::STAGES : 0;
          if (ka) mbar_wait(&bars->k_full[s], (ka - 1) & 1);
          if (va) mbar_wait(&bars->v_full[s], (va - 1) & 1);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop with warp-uniform values; one elected lane issues each
    // tensor-core instruction.
    {
      const uint32_t tmem = __shfl_sync(0xffffffffu, *reinterpret_cast<volatile uint32_t*>(&bars->tmem_base), 0);
      uint32_t kv_it = 0, q_cnt0 = 0, q_cnt1 = 0, pv_cnt0 = 0, pv_cnt1 = 0;
      bool ok = true;
      // descriptor low words of the operand bases; every K-step adds a compile-time offset
      constexpr uint32_t HI = desc_hi_sw128(1024);
      const uint32_t q_lo0 = desc_lo(smem_addr(sQ), 16), q_lo1 = desc_lo(smem_addr(sQ + C::TILE), 16);
      const uint32_t k_lo0 = desc_lo(smem_addr(sK), 16), k_lo1 = desc_lo(smem_addr(sK + C::TILE), 16);
      const uint32_t v_lbo = C::kVT ? 16u : (uint32_t)C::CH_STRIDE;
      const uint32_t v_lo0 = desc_lo(smem_addr(sV), v_lbo), v_lo1 = desc_lo(smem_addr(sV + C::TILE), v_lbo);
      const uint32_t t_s0 = tmem, t_s1 = tmem + 128, t_o0 = tmem + 256, t_o1 = tmem + 384;
      auto issue_s = [&](uint32_t d, uint32_t qa, uint32_t ka) {
#pragma unroll
        for (int s = 0; s < C::KS_QK; ++s) {
          constexpr uint32_t dummy = 0;
          (void)dummy;
          const uint32_t off = (uint32_t)(((s / 4) * C::CH_STRIDE + (s % 4) * 32) >> 4);
          umma_ss_lo_warp<C::kTf32>(d, qa + off, ka + off, HI, C::IDESC_QK, s > 0 ? 1u : 0u);
        }
      };
      // P V over keys [64 half, 64 half + 64) of the tile
      auto issue_pv = [&](uint32_t d, uint32_t pa, uint32_t va, uint32_t acc, int half) {
#pragma unroll
        for (int s = half * C::KS_PV / 2; s < (half + 1) * C::KS_PV / 2; ++s) {
          const uint32_t off = C::kVT ? (uint32_t)(((s / 4) * C::VT_CH_STRIDE + (s % 4) * 32) >> 4)
                                      : (uint32_t)((s * C::PV_K * 128) >> 4);
          umma_ts_lo_warp<C::kTf32>(d, pa + s * 8, va + off, HI, C::IDESC_PV, (acc | (uint32_t)s) != 0 ? 1u : 0u);
        }
      };
      auto wait_or_abort = [&](uint64_t* bar, uint32_t par) -> bool {
        const bool got = mbar_wait_or_abort(bar, par, &bars->abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) raise_abort(bars, p.err, kErrMma);
          ok = false;
          return false;
        }
        tc_fence_after();
        return true;
      };
      for (int g = blockIdx.x; g < p.total && ok; g += gridDim.x) {
        const Item it = decode_item<NS>(p, g);
        const bool two = it.ntiles > 1;
        if (!wait_or_abort(&bars->q_full[0], q_cnt0 & 1)) break;
        ++q_cnt0;
        if (two) {
          if (!wait_or_abort(&bars->q_full[1], q_cnt1 & 1)) break;
          ++q_cnt1;
        }
        // NS: the query tiles taking part in this step and the next (the first K/V tile holds
        // pooled rows, in which every query tile takes part)
        bool pc0 = true, pc1 = two;
        // S_t for the first K/V tile
        {
          const uint32_t st = kv_it % C::STAGES;
          if (!wait_or_abort(&bars->k_full[st], (kv_it / C::STAGES) & 1)) break;
          const uint32_t ka = st ? k_lo1 : k_lo0;
          issue_s(t_s0, q_lo0, ka);
          umma_commit_warp(&bars->s_full[0]);
          if (two) {
            issue_s(t_s1, q_lo1, ka);
            umma_commit_warp(&bars->s_full[1]);
          }
          umma_commit_warp(&bars->k_empty[st]);
          if (it.nkv == 1) umma_commit_warp(&bars->q_empty);
        }
        for (int j = 0; j < it.nkv; ++j, ++kv_it) {
          const uint32_t st = kv_it % C::STAGES;
          const bool more = (j + 1 < it.nkv);
          const uint32_t st1 = (kv_it + 1) % C::STAGES;
          bool pn0 = more, pn1 = more && two;  // NS: read from the stage once it is full
          if constexpr (NS) {
            // A tile that sits out this K/V tile but takes part in the next one gets its S for
            // the next tile now, without waiting for the other tile's P (its own S/P columns
            // were consumed by its last P V, issued earlier).
            if (more) {
              if (!wait_or_abort(&bars->k_full[st1], ((kv_it + 1) / C::STAGES) & 1)) break;
              const uint32_t tiles =
                  __shfl_sync(0xffffffffu, *reinterpret_cast<volatile uint32_t*>(&bars->stage_tiles[st1]), 0);
              pn0 = (tiles & 1u) != 0u;
              pn1 = two && (tiles & 2u) != 0u;
              const uint32_t ka1 = st1 ? k_lo1 : k_lo0;
              if (!pc0 && pn0) {
                issue_s(t_s0, q_lo0, ka1);
                umma_commit_warp(&bars->s_full[0]);
              }
              if (!pc1 && pn1) {
                issue_s(t_s1, q_lo1, ka1);
                umma_commit_warp(&bars->s_full[1]);
              }
            }
          }
          if (!wait_or_abort(&bars->v_full[st], (kv_it / C::STAGES) & 1)) break;
          const uint32_t va = st ? v_lo1 : v_lo0;
          const uint32_t ka1 = st1 ? k_lo1 : k_lo0;
          const uint32_t acc = j > 0 ? 1u : 0u;
          // tile 0: P0 V_j in two halves (each as soon as its P is written), then S0 of the next K/V tile
          if (!NS || pc0) {
            if (!wait_or_abort(&bars->p_half[0][0], pv_cnt0 & 1)) break;
            issue_pv(t_o0, t_s0, va, acc, 0);
            if (!wait_or_abort(&bars->p_half[0][1], pv_cnt0 & 1)) break;
            issue_pv(t_o0, t_s0, va, 1u, 1);
            umma_commit_warp(&bars->o_done[0]);
            ++pv_cnt0;
          }
          if (more) {
            if (!NS && !wait_or_abort(&bars->k_full[st1], ((kv_it + 1) / C::STAGES) & 1)) break;
            if (!NS || (pc0 && pn0)) {
              issue_s(t_s0, q_lo0, ka1);
              umma_commit_warp(&bars->s_full[0]);
            }
          }
          // tile 1
          if (NS ? pc1 : two) {
            if (!wait_or_abort(&bars->p_half[1][0], pv_cnt1 & 1)) break;
            issue_pv(t_o1, t_s1, va, acc, 0);
            if (!wait_or_abort(&bars->p_half[1][1], pv_cnt1 & 1)) break;
            issue_pv(t_o1, t_s1, va, 1u, 1);
            umma_commit_warp(&bars->o_done[1]);
            ++pv_cnt1;
          }
          if (NS ? (pc1 && pn1) : (two && more)) {
            issue_s(t_s1, q_lo1, ka1);
            umma_commit_warp(&bars->s_full[1]);
          }
          if (more) {
            umma_commit_warp(&bars->k_empty[st1]);
            if (j + 2 == it.nkv) umma_commit_warp(&bars->q_empty);
          }
          umma_commit_warp(&bars->v_empty[st]);
          pc0 = pn0;
          pc1 = pn1;
        }
      }
      // every MMA issued by this thread completes before TMEM can be released
      umma_commit_warp(&bars->drain);
      mbar_wait(&bars->drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    regs_alloc<kHighRegs>();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(&bars->tmem_base);
    const int t = (warp - 4) >> 2;           // query tile of this warpgroup
    const int wl = warp & 3;                 // TMEM lane quarter
    const int row = wl * 32 + lane;          // row inside the 128-row tile
    const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
    const uint32_t t_s = tmem + lane_off + t * 128;        // this row's scores, then its P
    const uint32_t t_p = t_s;
    const uint32_t t_o = tmem + lane_off + 256 + t * 128;  // this row's O
    uint32_t s_cnt = 0, pv_cnt = 0;
    bool ok = true;
    T* out = static_cast<T*>(p.out);
    for (int g = blockIdx.x; g < p.total && ok; g += gridDim.x) {
      const Item it = decode_item<NS>(p, g);
      if (t >= it.ntiles) continue;
      float m = -FLT_MAX, l = 0.f;
      // NS: this row's query block and its exact-block bitmask
      BlockCursor cur;
      const uint32_t* own = nullptr;
      if constexpr (NS) {
        const int u = t * p.bpt + row / p.b;
        own = p.nsmask + ((size_t)it.bh * p.n_q + it.blk(u < it.nblk ? u : 0)) * p.ns_words;
      }
      // short blocks: whether this head keeps the short last context block (the last of K_new)
      const bool cs = p.ragged ? short_ctx_kept(p, it.bh) : false;
      for (int j = 0; j < it.nkv; ++j) {
        bool keep0 = true, keep1 = true;  // NS: this row keeps the K/V tile's first / second 64 keys
        int len0 = 64, len1 = 64;         // NS: keys held by the tile's first / second 64 rows
        if constexpr (NS) {
          if (j >= p.npt) {
            const KeyTile kt = next_key_tile(p, it, cur, j);
            if (!tile_keeps(p, it, t, kt)) continue;  // no row of this tile keeps the K/V tile
            keep0 = has_block(own, kt.bk0);
            keep1 = p.b == 128 ? keep0 : has_block(own, kt.bk1);
            if (p.ragged) {
              const int l0 = new_block_len(p, kt.bk0, cs);
              if (p.b == 128) {
                len0 = min(l0, 64);
                len1 = max(l0 - 64, 0);
              } else {
                len0 = l0;
                len1 = kt.bk1 >= 0 ? new_block_len(p, kt.bk1, cs) : 0;
              }
            }
          }
        }
        if (!warp_wait(bars, &bars->s_full[t], s_cnt & 1, p.err)) { ok = false; break; }
        ++s_cnt;
        uint32_t r[kCols];
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) tmem_ld32(t_s + 32 * c, r + 32 * c);
        tmem_ld_wait<kCols>(r);
        float bias = 0.f;  // log2 of the weight of this tile's keys
        if constexpr (NS) {
          constexpr uint32_t kNegInf = 0xff800000u;
          if (j < p.npt) {
            // pooled rows: weight b, the row's own exact blocks and the rows past n_new masked
            bias = p.bias_log2;
            const int lim = j == p.npt - 1 ? it.last_valid : kBN;
#pragma unroll
            for (int c = 0; c < kCols / 32; ++c) {
              const int wd = (kCols / 32) * j + c;
              const uint32_t mw = wd < p.ns_words ? __ldg(own + wd) : 0u;
#pragma unroll
              for (int i = 0; i < 32; ++i)
                r[32 * c + i] = (((mw >> i) & 1u) != 0u || 32 * c + i >= lim) ? kNegInf : r[32 * c + i];
            }
            if (p.ragged) {  // a short block's pooled row weighs its own length
              if (p.len_src_last < p.b) add_col_bias(r, j * kBN, p.n_src - 1, p.src_last_bias);
              if (cs) add_col_bias(r, j * kBN, p.n_new - 1, p.ctx_last_bias);
            }
          } else {
            // exact blocks of the union: keep those in the row's own set (and, in a short
            // block, only its keys)
#pragma unroll
            for (int i = 0; i < kCols; ++i)
              r[i] = ((i < kCols / 2 ? keep0 : keep1) && (i & 63) < (i < kCols / 2 ? len0 : len1)) ? r[i] : kNegInf;
          }
        } else {
          if (j == it.nkv - 1 && it.last_valid < kBN) {  // ragged last K/V tile (uniform branch)
#pragma unroll
            for (int i = 0; i < kCols; ++i)
              if (i >= it.last_valid) r[i] = __float_as_uint(-INFINITY);
          }
          if (p.ragged) {
            if (it.kind == 0) {
              // exact path: the padding rows of the short source block and of a kept short
              // context block (the last block of K_new)
              mask_key_rows(r, j * kBN, p.L_src, p.L_srcp);
              if (cs) mask_key_rows(r, j * kBN, p.L_new - (p.b - p.len_ctx_last), p.L_new);
            } else {
              // Taylor path: a short block's pooled row weighs its own length
              if (p.len_src_last < p.b) add_col_bias(r, j * kBN, p.n_src - 1, p.src_last_bias);
              if (cs) add_col_bias(r, j * kBN, p.n_new - 1, p.ctx_last_bias);
            }
          }
        }
        // row max of the raw scores: 8 independent chains of 3-input max
        float mc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) mc[c] = __uint_as_float(r[c]);
#pragma unroll
        for (int i = 8; i < kCols; i += 16) {
#pragma unroll
          for (int c = 0; c < 8; ++c) mc[c] = fmax3(mc[c], __uint_as_float(r[i + c]), __uint_as_float(r[i + 8 + c]));
        }
        const float raw_max = fmaxf(fmax3(mc[0], mc[1], mc[2]), fmax3(fmax3(mc[3], mc[4], mc[5]), mc[6], mc[7]));
        const float mx = raw_max * p.scale_log2 + bias;
        // lazy max: move it only when the tile's max exceeds it by more than 2^8
        const bool need = (j > 0) && (mx > m + kRescaleThreshold);
        const float alpha = need ? ex2_approx(m - mx) : 1.0f;
        if (j == 0 || need) m = mx;
        // O holds P V up to tile j-1 (complete: this tile's S was committed after it);
        // rows whose max moved are rescaled in place before any P of tile j is
        // released. TMEM moves are warp-collective, so the whole warp takes this step
        // when any of its rows needs it (alpha = 1 for the others).
        if (__any_sync(0xffffffffu, need)) {
          if (!warp_wait(bars, &bars->o_done[t], (pv_cnt - 1) & 1, p.err)) { ok = false; break; }
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(t_o + 32 * c, o);
            tmem_ld_wait<32>(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(t_o + 32 * c, o);
          }
        }
        // p = 2^(s * scale - m), in pairs (pairs with i % kPolyDen < kPolyNum on the FMA
        // pipe, the rest on ex2). P is written and released in two halves (keys 0-63,
        // then 64-127) so that the P V MMAs can start on the first half.
        // NS: a row with no unmasked key yet has m = -inf and all its entries -inf (p = 0)
        const float nm = (NS && m == -INFINITY) ? 0.f : bias - m;
        const uint64_t sc2 = pack2(p.scale_log2, p.scale_log2), nm2 = pack2(nm, nm);
        uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
          for (int i = half * kCols / 4; i < (half + 1) * kCols / 4; ++i) {
            const uint64_t x = ffma2(static_cast<uint64_t>(r[2 * i]) | (static_cast<uint64_t>(r[2 * i + 1]) << 32), sc2,
                                     nm2);
            uint64_t e;
            if (i % kPolyDen < kPolyNum) e = exp2_poly2(x);
            else e = pack2(ex2_approx(lo2(x)), ex2_approx(hi2(x)));
            acc[i & 3] = fadd2(acc[i & 3], e);
            if constexpr (sizeof(T) == 2) {
              __nv_bfloat162 hv = __floats2bfloat162_rn(lo2(e), hi2(e));
              r[i] = *reinterpret_cast<uint32_t*>(&hv);
            } else {
              r[2 * i] = static_cast<uint32_t>(e);
              r[2 * i + 1] = static_cast<uint32_t>(e >> 32);
            }
          }
          // this half's P: bf16 pairs in kCols/4 columns, or fp32 in kCols/2 columns
          constexpr int kPCols = sizeof(T) == 2 ? kCols / 4 : kCols / 2;
#pragma unroll
          for (int c = 0; c < kPCols / 32; ++c) {
            const int col = half * kPCols + 32 * c;
            tmem_st32(t_p + col, r + col);
          }
          static_assert(kPCols % 32 == 0, "P columns");
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&bars->p_half[t][half]);
        }
        // bf16: the P V MMA multiplies the bf16 p, the row sum takes the fp32 p except that the
        // tile's largest p enters as its bf16 value when it exceeds 1. With the lazy maximum a
        // row's dominant keys have p in (1, 2^8] (only in tiles whose maximum exceeds m), which
        // bf16 rounds by up to 2^-9: left in the sum, that mismatch between numerator and
        // denominator would scale the whole output row by it. (A key that set m has p = 1.)
        float corr = 0.f;
        if constexpr (sizeof(T) == 2) {
          if (mx > m) {
            const float em = ex2_approx(fmaf(raw_max, p.scale_log2, nm));  // the largest p, as computed above
            corr = __bfloat162float(__float2bfloat16_rn(em)) - em;
          }
        }
        const uint64_t a2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
        l = l * alpha + ((lo2(a2) + hi2(a2)) + corr);
        ++pv_cnt;
      }
      if (!ok) break;
      // epilogue: O / (l_half0 + l_half1) for this half's columns, at the row's original token position
      const float inv_l = 1.0f / l;
      if (!warp_wait(bars, &bars->o_done[t], (pv_cnt - 1) & 1, p.err)) { ok = false; break; }
      const int u = t * p.bpt + row / p.b;
      const int qb = it.blk(u < it.nblk ? u : 0);
      const bool store = (u < it.nblk) && (row % p.b) < qblock_len(p, qb);  // rows past a short block: none
      const size_t token = (size_t)qblock_start(p, qb) + (row % p.b);
      T* dst = out + ((size_t)it.bh * p.N + token) * D;
      if (!NS && p.lse && store)  // m and log2(l) are base 2; the weight b is not in the Taylor exponents
        p.lse[(size_t)it.bh * p.N + token] =
            (m + __log2f(l)) * 0.6931471805599453f + (it.kind == 1 ? p.taylor_ln_b : 0.f);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + 32 * c, o);
        tmem_ld_wait<32>(o);
        float* f = reinterpret_cast<float*>(o);
#pragma unroll
        for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(o[i]) * inv_l;
        if (store) store_row_chunk<T>(dst + 32 * c, f);
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(*reinterpret_cast<volatile uint32_t*>(&bars->tmem_base), 512);
  }
}

template <typename T, int D, bool NS>
cudaError_t launch_t(const void* q, const void* k, const void* v, void* out, const Plan& pl, const Work& w,
                     cudaStream_t s, int* n_ctas) {
  using C = Cfg<T, D>;
  AttnParams p{};
  p.route = w.route;
  p.lse = NS ? nullptr : w.lse;
  p.taylor_ln_b = logf((float)pl.b);
  p.out = out;
  p.err = w.ctrl;
  p.BH = pl.BH;
  p.N = pl.N;
  p.b = pl.b;
  p.L_src = pl.L_src;
  p.n_q = pl.n_q;
  p.n_exact = pl.n_exact;
  p.n_flat = pl.n_flat;
  p.L_new = pl.L_new;
  p.n_new = pl.n_new;
  p.bpt = kBM / pl.b;
  p.bpi = 2 * p.bpt;
  p.items_e = NS ? 0 : (pl.n_exact + p.bpi - 1) / p.bpi;  // NS: Taylor items only
  p.items_t = (pl.n_flat + p.bpi - 1) / p.bpi;
  p.total = pl.BH * (p.items_e + p.items_t);
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  p.nsmask = w.nsmask;
  p.ns_words = pl.ns_words;
  p.sel = w.sel;
  p.k = pl.k;
  p.n_src = pl.n_src;
  p.n_ctx = pl.n_ctx;
  p.L_srcp = pl.L_srcp;
  p.len_src_last = pl.len_src_last;
  p.len_ctx_last = pl.len_ctx_last;
  p.ragged = pl.ragged;
  p.src_last_bias = log2f((float)pl.len_src_last / (float)pl.b) / p.scale_log2;
  p.ctx_last_bias = log2f((float)pl.len_ctx_last / (float)pl.b) / p.scale_log2;
  p.npt = (pl.n_new + kBN - 1) / kBN;
  p.bias_log2 = log2f((float)pl.b);
  if (NS && (pl.k_ns <= 0 || w.nsmask == nullptr)) return cudaErrorInvalidValue;
  if (n_ctas) *n_ctas = 0;
  if (p.total == 0) return cudaSuccess;

  const int E = sizeof(T);
  CUtensorMap tq, tk, tks, tv, tvs, tkc, tvc;
  const bool has_sel = pl.k > 0;
  bool ok = make_map(&tq, q, E, D, pl.N, pl.BH) && make_map(&tk, k, E, D, pl.N, pl.BH) &&
            make_map(&tks, has_sel ? w.ksel : k, E, D, has_sel ? pl.k * pl.b : pl.N, pl.BH) &&
            make_map(&tkc, w.kcn, E, D, pl.n_new, pl.BH);
  if (C::kVT) {
    // V_new^T [BH][D][L_new] and Vc_new^T [BH][D][n_new]: rows are D, the inner axis is the key
    ok = ok && make_map_t(&tv, w.vtn, pl.L_new, pl.L_new, D, pl.BH) &&
         make_map_t(&tvc, w.vct, pl.n_new, vct_ld(pl), D, pl.BH);
    tvs = tv;
  } else {
    ok = ok && make_map(&tv, v, E, D, pl.N, pl.BH) &&
         make_map(&tvs, has_sel ? w.vsel : v, E, D, has_sel ? pl.k * pl.b : pl.N, pl.BH) &&
         make_map(&tvc, w.vcn, E, D, pl.n_new, pl.BH);
  }
  if (!ok) return cudaErrorInvalidValue;

  auto kern = attention_kernel<T, D, NS>;
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  // the warpgroup register split is only safe with the launch count it was sized for
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidKernelImage;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  int grid = device_sm_count();
  if (grid > p.total) grid = p.total;
  kern<<<grid, kThreads, C::SMEM_ALLOC, s>>>(tq, tk, tks, tv, tvs, tkc, tvc, p);
  if (n_ctas) *n_ctas = grid;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const void* q, const void* k, const void* v, void* out, const Plan& p, const Work& w,
                             cudaStream_t s, int* n_ctas) {
  if (p.dt == 0) return p.D == 128 ? launch_t<__nv_bfloat16, 128, false>(q, k, v, out, p, w, s, n_ctas)
                                   : launch_t<__nv_bfloat16, 64, false>(q, k, v, out, p, w, s, n_ctas);
  if (p.D == 64) return launch_t<float, 64, false>(q, k, v, out, p, w, s, n_ctas);
  return cudaErrorNotSupported;
}

cudaError_t launch_attention_ns(const void* q, const void* k, const void* v, void* out, const Plan& p,
                                const Work& w, cudaStream_t s) {
  if (p.dt != 0) return cudaErrorNotSupported;
  return p.D == 128 ? launch_t<__nv_bfloat16, 128, true>(q, k, v, out, p, w, s, nullptr)
                    : launch_t<__nv_bfloat16, 64, true>(q, k, v, out, p, w, s, nullptr);
}

}  // namespace isa
