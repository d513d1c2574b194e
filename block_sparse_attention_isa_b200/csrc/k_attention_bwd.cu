// Backward pass of In-context Sparse Attention (trainable ISA) for bf16 inputs with D = 128.
//
// Method: "Lightning Unified Video Editing via In-Context Sparse Attention". The
// papernotes.org notes (overview; Key design 2) and the paperlayer.ai summary
// (appendix H) train through ISA with forward and backward kernels, without
// spelling the backward out. The reading taken here: the discrete decisions of
// the forward pass (kept context blocks, routing) are held fixed, and the
// gradient flows through everything else:
//  * an exact-path row q attends to every key of K_new = [K_src ; kept blocks]:
//    P = exp(q K_new^T / sqrt(D) - lse), dP = dO V_new^T, dS = P (dP - delta)
//    with delta = rowsum(dO * O), dq = dS K_new / sqrt(D), dK_new += dS^T q /
//    sqrt(D), dV_new += P^T dO;
//  * a Taylor-path row q attends to the pooled rows Kc_j, Vc_j of K_new's blocks
//    with weight b (Key design 2), the same formulas over the pooled rows; the
//    gradient of a block mean spreads dKc_j / b and dVc_j / b over the block's b
//    rows;
//  * dK_new and dV_new rows go back to K and V: source rows in place, the rows of
//    a kept context block at that block's position; other context rows get 0.
//
// Two kernels, one template (sm_100a, tcgen05, TMA), both "row-stationary":
//  * dQ (kDKDV = false): an item is 128 query rows of one head (exact or Taylor
//    rows); it walks the keys in 64-key tiles: S = Q K^T and T = dO V^T into
//    TMEM, then one softmax thread per query row forms P and dS and writes dS
//    back into TMEM as bf16, and dQ += dS K accumulates in TMEM;
//  * dK/dV (kDKDV = true): an item is 128 key rows of one head (rows of K_new
//    for the exact path, pooled rows for the Taylor path); it walks the query
//    rows of that path in 64-row tiles: S^T = K Q^T and T^T = V dO^T, then one
//    thread per key row forms P^T and dS^T (with the queries' lse and delta
//    staged in shared memory), and dV += P^T dO, dK += dS^T Q accumulate in TMEM.
// Every operand has the layout of one in the forward kernels: A tiles are
// [rows][D] K-major, the score MMAs take the column tile K-major, the
// accumulating MMAs take P / dS from TMEM and the column tile as an MN-major B.
// TMEM: S and T double-buffered (columns [0,128) and [128,256)), accumulators at
// [256, 384) (dV or dQ) and [384, 512) (dK). Warp 0 issues the TMA loads, warp 1
// the MMAs (one thread), warps 4-7 and 8-11 are two elementwise warpgroups that
// take alternate column tiles (one S/T buffer each), so that two tiles' chains
// of TMEM loads, exponentials and TMEM stores are in flight at once; while they
// work, the tensor core computes the next tiles' S and T and the accumulating
// MMAs of the tiles already done.
// Every wait is bounded; a timeout sets the workspace error word and stops the CTA.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <float.h>

#include "exp2_poly.cuh"
#include "isa_internal.h"
#include "ptx.cuh"
#include "tensor_map.cuh"

namespace isa {
namespace {

constexpr int kThreads = 384;   // warp 0 TMA, warp 1 MMA, warps 4-7 and 8-11 the two elementwise warpgroups
// Register split: warpgroup 0 (TMA, MMA) gives registers back, the elementwise warpgroups take them
// (384 x 168 at launch = 128 x 88 + 256 x 208).
constexpr int kLaunchRegs = 168;
constexpr int kLowRegs = 88;
constexpr int kHighRegs = 208;
static_assert(128 * kLowRegs + 256 * kHighRegs <= kThreads * kLaunchRegs, "register split exceeds the launch budget");
constexpr int kD = 128;
constexpr int kBM = 128;                 // rows of an item
constexpr int kBN = 64;                  // columns of a tile
constexpr int kStages = 4;
constexpr int kATile = kBM * kD * 2;     // 32 KB
constexpr int kACh = kBM * 128;          // bytes between the two 128-byte chunks of an A tile
constexpr int kBTile = kBN * kD * 2;     // 16 KB
constexpr int kBCh = kBN * 128;          // bytes between the two chunks of a column tile
constexpr int kStat = kBN * 4;           // 64 floats
constexpr int kStageBytes = 2 * kBTile + 1024;  // column tiles, then lse and delta of the 64 queries (padded)
constexpr uint32_t kIdescS = umma_idesc(1u, kBM, kBN, 0, 0);
constexpr uint32_t kIdescAcc = umma_idesc(1u, kBM, kD, 0, 1);
constexpr float kLog2e = 1.4426950408889634f;

struct BwdParams {
  const int32_t* route;   // [BH, n_q]: exact blocks, then Taylor blocks
  const int32_t* sel;     // [BH, k]
  const float* lse;       // [BH, N] natural log of each row's softmax denominator (forward)
  const float* delta;     // [BH, N] rowsum(dO * O)
  void* dq;               // dQ kernel: [BH, N, D] bf16
  void* dk;               // dK/dV exact: [BH, N, D] bf16
  void* dv;
  float* dkc;             // [BH, n_new, D] fp32: the Taylor path's dKc (dK/dV Taylor adds, exact reads)
  float* dvc;
  uint32_t* err;
  int BH, N, b, L_src, n_q, n_exact, n_flat, L_new, n_new, k;
  int kind_split;         // items [0, kind_split) are exact-path items, the rest Taylor-path items
  int items_e, items_t;   // items per head of each kind
  int chunks;             // dK/dV Taylor: column ranges per row tile (partial sums added atomically)
  int total;
  float scale_log2;       // log2(e) / sqrt(D)
  float inv_sqrt_d;
  float log2_b;           // the Taylor rows' weight b, dropped from their exponents
};

constexpr int kRing = 4;

struct Bars {
  uint64_t a_full, a_empty;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], p_full[2];
  uint64_t acc_full, acc_empty;
  uint64_t drain;
  // Work items from the per-launch counter (exact items first, then Taylor items), published by
  // the producer lane: item_full (1 arrival), item_free (the issuer and the 256 elementwise threads).
  uint64_t item_full[kRing];
  uint64_t item_free[kRing];
  int item_ring[kRing];  // item index, or -1 past the last
  uint32_t tmem_base;
  int abort_flag;
};

constexpr int kOffA1 = 0;
constexpr int kOffA2 = kATile;
constexpr int kOffB = 2 * kATile;
constexpr int kOffBar = kOffB + kStages * kStageBytes;
constexpr int kSmemAlloc = kOffBar + (int)sizeof(Bars) + 1024;
static_assert(kSmemAlloc <= 227 * 1024, "shared memory");
static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled tiles");

__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// One work item: the head, the path (0 exact, 1 Taylor), the first row of the item and its
// column tiles [c_begin, c_end).
struct Item {
  int bh, kind, row0, c_begin, c_end, rows;  // rows: valid rows of the item
};

template <bool kDKDV>
__device__ __forceinline__ Item decode_item(const BwdParams& p, int g) {
  Item it;
  int local;
  if (g < p.kind_split) {
    it.kind = 0;
    it.bh = g / p.items_e;
    local = g - it.bh * p.items_e;
  } else {
    it.kind = 1;
    const int g2 = g - p.kind_split;
    it.bh = g2 / p.items_t;
    local = g2 - it.bh * p.items_t;
  }
  if constexpr (kDKDV) {
    // rows: 128 rows of K_new (exact) or of the pooled rows (Taylor); columns: the path's query rows
    const int chunks = it.kind == 0 ? 1 : p.chunks;
    const int tile = local / chunks, chunk = local - tile * chunks;
    it.row0 = tile * kBM;
    const int all_rows = it.kind == 0 ? p.L_new : p.n_new;
    it.rows = min(kBM, all_rows - it.row0);
    const int ncols = ((it.kind == 0 ? p.n_exact : p.n_flat) * p.b) / kBN;
    it.c_begin = (int)(((long long)ncols * chunk) / chunks);
    it.c_end = (int)(((long long)ncols * (chunk + 1)) / chunks);
  } else {
    // rows: 128 query rows of the path (local-th tile of its block list); columns: keys
    it.row0 = local * kBM;
    const int all_rows = (it.kind == 0 ? p.n_exact : p.n_flat) * p.b;
    it.rows = min(kBM, all_rows - it.row0);
    it.c_begin = 0;
    it.c_end = ((it.kind == 0 ? p.L_new : p.n_new) + kBN - 1) / kBN;
  }
  return it;
}

// Token of the r-th query row of a path's block list (rows of a block are consecutive tokens).
__device__ __forceinline__ int path_token(const BwdParams& p, int bh, int kind, int r) {
  const int32_t* lst = p.route + (size_t)bh * p.n_q + (kind == 0 ? 0 : p.n_exact);
  return __ldg(lst + r / p.b) * p.b + (r % p.b);
}

__device__ __forceinline__ void raise_abort(Bars* b, uint32_t* err, uint32_t code) {
  atomicOr(err, code);
  *reinterpret_cast<volatile int*>(&b->abort_flag) = 1;
}
__device__ __forceinline__ bool aborted(const Bars* b) {
  return *reinterpret_cast<const volatile int*>(&b->abort_flag) != 0;
}
// All 32 lanes wait; the warp is converged on return.
__device__ __forceinline__ bool warp_wait(Bars* b, uint64_t* bar, uint32_t parity, uint32_t* err) {
  bool ok = mbar_wait_or_abort(bar, parity, &b->abort_flag);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && (threadIdx.x & 31) == 0) raise_abort(b, err, kErrSoftmax);
  tc_fence_after();
  return ok;
}

__device__ __forceinline__ void store_bf16_32(__nv_bfloat16* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    d[i] = make_uint4(bf16x2(v[8 * i], v[8 * i + 1]), bf16x2(v[8 * i + 2], v[8 * i + 3]),
                      bf16x2(v[8 * i + 4], v[8 * i + 5]), bf16x2(v[8 * i + 6], v[8 * i + 7]));
}

template <bool kDKDV>
__global__ void __launch_bounds__(kThreads, 1)
    attention_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_ksel, const __grid_constant__ CUtensorMap tm_vsel,
                         const __grid_constant__ CUtensorMap tm_kcn, const __grid_constant__ CUtensorMap tm_vcn,
                         const BwdParams p, uint32_t* next) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA1 = smem + kOffA1;
  uint8_t* sA2 = smem + kOffA2;
  uint8_t* sB = smem + kOffB;
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->a_full, 1);
    mbar_init(&bars->a_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->p_full[b], 128);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, 256);
    mbar_init(&bars->drain, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&bars->item_full[i], 1);
      mbar_init(&bars->item_free[i], 257);
    }
    bars->abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_ksel);
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
      uint32_t n_items = 0, tile_it = 0;
      bool ok = true;
      // 64 rows of K_new (or the pooled rows) starting at r into dst (two 128-byte chunks)
      auto load_keys = [&](uint8_t* dst, int ch, int kind, bool values, int bh, int r, uint64_t* bar) {
        const CUtensorMap* map;
        int y = r;
        if (kind == 1) {
          map = values ? &tm_vcn : &tm_kcn;
        } else if (r < p.L_src) {
          map = values ? &tm_v : &tm_k;
        } else {
          map = values ? &tm_vsel : &tm_ksel;
          y = r - p.L_src;
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) tma_load_3d(dst + c * ch, map, bar, c * 64, y, bh);
      };
      // 64 query rows (of Q or dO) of the path, from its r-th row, into dst
      auto load_queries = [&](uint8_t* dst, int ch, bool grad, int bh, int kind, int r, uint64_t* bar) {
        const int all = (kind == 0 ? p.n_exact : p.n_flat) * p.b;
        const int tok = path_token(p, bh, kind, r < all ? r : 0);  // missing rows: a copy, never stored
#pragma unroll
        for (int c = 0; c < 2; ++c) tma_load_3d(dst + c * ch, grad ? &tm_do : &tm_q, bar, c * 64, tok, bh);
      };
      for (uint32_t n = 0; ok; ++n) {
        const uint32_t slot = n % kRing;
        if (n >= kRing && !mbar_wait(&bars->item_free[slot], ((n / kRing) - 1) & 1)) {
          raise_abort(bars, p.err, kErrProducer);
          ok = false;
          break;
        }
        int g = (int)atomicAdd(next, 1u);
        if (g >= p.total) g = -1;
        *reinterpret_cast<volatile int*>(&bars->item_ring[slot]) = g;
        mbar_arrive(&bars->item_full[slot]);
        if (g < 0) break;
        const Item it = decode_item<kDKDV>(p, g);
        if (it.c_end <= it.c_begin) continue;  // nothing to accumulate (every role skips it)
        if (n_items > 0 && !mbar_wait(&bars->a_empty, (n_items - 1) & 1)) {
          raise_abort(bars, p.err, kErrProducer);
          ok = false;
          break;
        }
        ++n_items;
        mbar_arrive_expect_tx(&bars->a_full, 2 * kATile);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if constexpr (kDKDV) {
            load_keys(sA1 + h * 8192, kACh, it.kind, false, it.bh, it.row0 + 64 * h, &bars->a_full);
            load_keys(sA2 + h * 8192, kACh, it.kind, true, it.bh, it.row0 + 64 * h, &bars->a_full);
          } else {
            load_queries(sA1 + h * 8192, kACh, false, it.bh, it.kind, it.row0 + 64 * h, &bars->a_full);
            load_queries(sA2 + h * 8192, kACh, true, it.bh, it.kind, it.row0 + 64 * h, &bars->a_full);
          }
        }
        for (int j = it.c_begin; j < it.c_end && ok; ++j, ++tile_it) {
          if (aborted(bars)) { ok = false; break; }
          const int st = tile_it % kStages;
          if (!mbar_wait(&bars->kv_empty[st], ((tile_it / kStages) & 1) ^ 1)) {
            raise_abort(bars, p.err, kErrProducer);
            ok = false;
            break;
          }
          uint8_t* b1 = sB + st * kStageBytes;
          uint8_t* b2 = b1 + kBTile;
          float* stat = reinterpret_cast<float*>(b2 + kBTile);
          if constexpr (kDKDV) {
            mbar_arrive_expect_tx(&bars->kv_full[st], 2 * kBTile + 2 * kStat);
            load_queries(b1, kBCh, false, it.bh, it.kind, j * kBN, &bars->kv_full[st]);
            load_queries(b2, kBCh, true, it.bh, it.kind, j * kBN, &bars->kv_full[st]);
            // the 64 queries are consecutive tokens of one block (b is 64 or 128)
            const size_t tok = (size_t)it.bh * p.N + path_token(p, it.bh, it.kind, j * kBN);
            bulk_load(stat, p.lse + tok, kStat, &bars->kv_full[st]);
            bulk_load(stat + kBN, p.delta + tok, kStat, &bars->kv_full[st]);
          } else {
            mbar_arrive_expect_tx(&bars->kv_full[st], 2 * kBTile);
            load_keys(b1, kBCh, it.kind, false, it.bh, j * kBN, &bars->kv_full[st]);
            load_keys(b2, kBCh, it.kind, true, it.bh, j * kBN, &bars->kv_full[st]);
          }
        }
      }
      if (!ok) {
        // let the copies this thread started land before the CTA leaves
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 2000000ull) {
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
      constexpr uint32_t HI = desc_hi_sw128(1024);
      const uint32_t a1_lo = desc_lo(smem_addr(sA1), 16), a2_lo = desc_lo(smem_addr(sA2), 16);
      uint32_t n_items = 0, tile_it = 0, ct = 0;
      bool ok = true;
      auto wait = [&](uint64_t* bar, uint32_t par) -> bool {
        const bool got = mbar_wait_or_abort(bar, par, &bars->abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) raise_abort(bars, p.err, kErrMma);
          ok = false;
          return false;
        }
        tc_fence_after();
        return true;
      };
      // D (M 128 x N 64) = A (128 x 128, K-major) * B^T (64 x 128, K-major)
      auto issue_score = [&](uint32_t d, uint32_t a_lo, uint32_t b_lo) {
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const uint32_t oa = (uint32_t)(((s / 4) * kACh + (s % 4) * 32) >> 4);
          const uint32_t ob = (uint32_t)(((s / 4) * kBCh + (s % 4) * 32) >> 4);
          umma_ss_lo_warp<false>(d, a_lo + oa, b_lo + ob, HI, kIdescS, s > 0 ? 1u : 0u);
        }
      };
      // D (128 x 128) (+)= X (TMEM, 128 x 64 bf16) * B (64 x 128, MN-major)
      auto issue_acc = [&](uint32_t d, uint32_t x_tmem, uint32_t b_lo, uint32_t acc) {
#pragma unroll
        for (int s = 0; s < kBN / 16; ++s)
          umma_ts_lo_warp<false>(d, x_tmem + s * 8, b_lo + (uint32_t)((s * 16 * 128) >> 4), HI, kIdescAcc,
                            (acc | (uint32_t)s) != 0 ? 1u : 0u);
      };
      const uint32_t t_s = tmem, t_t = tmem + 128, t_acc0 = tmem + 256, t_acc1 = tmem + 384;
      for (uint32_t n = 0; ok; ++n) {
        const uint32_t slot = n % kRing;
        if (!wait(&bars->item_full[slot], (n / kRing) & 1)) break;
        const int g = __shfl_sync(0xffffffffu, *reinterpret_cast<volatile int*>(&bars->item_ring[slot]), 0);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->item_free[slot]);
        if (g < 0) break;
        const Item it = decode_item<kDKDV>(p, g);
        if (it.c_end <= it.c_begin) continue;
        if (!wait(&bars->a_full, n_items & 1)) break;
        const uint32_t item_ix = n_items++;
        const int nc = it.c_end - it.c_begin;
        uint32_t prev_st = 0;
        for (int jj = 0; jj <= nc; ++jj) {
          if (jj < nc) {
            // S and T of tile jj into buffer ct & 1 (its last reader, the accumulating MMAs of
            // tile jj - 2, was issued earlier by this thread)
            const uint32_t st = tile_it % kStages;
            if (!wait(&bars->kv_full[st], (tile_it / kStages) & 1)) break;
            const uint32_t b1 = desc_lo(smem_addr(sB + st * kStageBytes), 16);
            const uint32_t b2 = desc_lo(smem_addr(sB + st * kStageBytes + kBTile), 16);
            const uint32_t bf = ct & 1;
            issue_score(t_s + bf * kBN, a1_lo, b1);
            issue_score(t_t + bf * kBN, a2_lo, b2);
            umma_commit_warp(&bars->s_full[bf]);
            if (jj == nc - 1) umma_commit_warp(&bars->a_empty);
          }
          if (jj > 0) {
            // the accumulating MMAs of tile jj - 1 once its P and dS are in TMEM
            const uint32_t cp = ct - 1, bf = cp & 1;
            if (!wait(&bars->p_full[bf], (cp >> 1) & 1)) break;
            // the accumulators are free once the epilogue of the previous item has read them
            if (jj == 1 && item_ix > 0 && !wait(&bars->acc_empty, (item_ix - 1) & 1)) break;
            const uint32_t b1 = desc_lo(smem_addr(sB + prev_st * kStageBytes), (uint32_t)kBCh);
            const uint32_t b2 = desc_lo(smem_addr(sB + prev_st * kStageBytes + kBTile), (uint32_t)kBCh);
            const uint32_t acc = jj > 1 ? 1u : 0u;
            if constexpr (kDKDV) {
              issue_acc(t_acc0, t_s + bf * kBN, b2, acc);  // dV += P^T dO
              issue_acc(t_acc1, t_t + bf * kBN, b1, acc);  // dK += dS^T Q
            } else {
              issue_acc(t_acc0, t_t + bf * kBN, b1, acc);  // dQ += dS K
            }
            umma_commit_warp(&bars->kv_empty[prev_st]);
          }
          if (jj < nc) {
            prev_st = tile_it % kStages;
            ++tile_it;
            ++ct;
          }
        }
        if (!ok) break;
        umma_commit_warp(&bars->acc_full);
      }
      // every MMA issued by this thread completes before TMEM can be released
      umma_commit_warp(&bars->drain);
      mbar_wait(&bars->drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ elementwise + epilogue
    // Warpgroup w takes the column tiles in S/T buffer w (tiles ct with ct % 2 == w), so the two
    // work on consecutive tiles at once; both then write half of the item's epilogue.
    regs_alloc<kHighRegs>();
    const int w = (warp - 4) >> 2;
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(&bars->tmem_base);
    const int wl = warp & 3;
    const int row = wl * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
    const uint32_t t_s = tmem + lane_off, t_t = tmem + lane_off + 128;
    const uint32_t t_acc0 = tmem + lane_off + 256, t_acc1 = tmem + lane_off + 384;
    uint32_t n_items = 0, tile_it = 0, ct = 0;
    bool ok = true;
    const uint64_t sc2 = pack2(p.scale_log2, p.scale_log2);
    for (uint32_t n = 0; ok; ++n) {
      const uint32_t slot = n % kRing;
      if (!warp_wait(bars, &bars->item_full[slot], (n / kRing) & 1, p.err)) { ok = false; break; }
      const int g = *reinterpret_cast<volatile int*>(&bars->item_ring[slot]);
      mbar_arrive(&bars->item_free[slot]);
      if (g < 0) break;
      const Item it = decode_item<kDKDV>(p, g);
      const int nc = it.c_end - it.c_begin;
      const float path_off = it.kind == 1 ? p.log2_b : 0.f;  // the Taylor exponents omit the weight b
      // dQ: this query row's statistics (row stats); dK/dV: per column, from shared memory
      float l2r = 0.f, dr = 0.f;
      int tok_row = 0;
      if constexpr (!kDKDV) {
        const int r = it.row0 + row;
        tok_row = path_token(p, it.bh, it.kind, r < it.row0 + it.rows ? r : it.row0);
        const size_t ix = (size_t)it.bh * p.N + tok_row;
        l2r = __ldg(p.lse + ix) * kLog2e - path_off;
        dr = __ldg(p.delta + ix);
      }
      const int ncols_valid = kDKDV ? 0 : (it.kind == 0 ? p.L_new : p.n_new);
      for (int jj = 0; jj < nc; ++jj, ++ct, ++tile_it) {
        const uint32_t bf = ct & 1;
        if ((int)bf != w) continue;  // the other warpgroup's tile
        if (!warp_wait(bars, &bars->s_full[bf], (ct >> 1) & 1, p.err)) { ok = false; break; }
        uint32_t s[kBN], t[kBN];
        tmem_ld32(t_s + bf * kBN, s);
        tmem_ld32(t_s + bf * kBN + 32, s + 32);
        tmem_ld32(t_t + bf * kBN, t);
        tmem_ld32(t_t + bf * kBN + 32, t + 32);
        tmem_ld_wait<kBN>(s);
        tmem_ld_wait<kBN>(t);
        uint32_t pw[kBN / 2], dw[kBN / 2];
        if constexpr (kDKDV) {
          const float* stat = reinterpret_cast<const float*>(sB + (tile_it % kStages) * kStageBytes + 2 * kBTile);
          // columns are queries: P^T = 2^(S^T c - lse2_col), dS^T = P^T (T^T - delta_col)
#pragma unroll
          for (int i = 0; i < kBN / 2; i += 2) {
            const float4 l4 = *reinterpret_cast<const float4*>(stat + 2 * i);
            const float4 d4 = *reinterpret_cast<const float4*>(stat + kBN + 2 * i);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int ii = i + h;
              const float la = h ? l4.z : l4.x, lb = h ? l4.w : l4.y;
              const float da = h ? d4.z : d4.x, db = h ? d4.w : d4.y;
              const uint64_t nl = pack2(path_off - la * kLog2e, path_off - lb * kLog2e);
              const uint64_t x = ffma2(pack2(__uint_as_float(s[2 * ii]), __uint_as_float(s[2 * ii + 1])), sc2, nl);
              const float e0 = ex2_approx(lo2(x)), e1 = ex2_approx(hi2(x));
              const uint64_t ds = fmul2(pack2(e0, e1), fadd2(pack2(__uint_as_float(t[2 * ii]),
                                                                    __uint_as_float(t[2 * ii + 1])),
                                                              pack2(-da, -db)));
              pw[ii] = bf16x2(e0, e1);
              dw[ii] = bf16x2(lo2(ds), hi2(ds));
            }
          }
        } else {
          // columns are keys: P = 2^(S c - lse2_row), dS = P (T - delta_row); keys past the end are 0
          const int base = (it.c_begin + jj) * kBN;
          const uint64_t nl = pack2(-l2r, -l2r), nd = pack2(-dr, -dr);
          const bool tail = base + kBN > ncols_valid;
#pragma unroll
          for (int i = 0; i < kBN / 2; ++i) {
            const uint64_t x = ffma2(pack2(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1])), sc2, nl);
            float e0 = ex2_approx(lo2(x)), e1 = ex2_approx(hi2(x));
            if (tail) {
              if (base + 2 * i >= ncols_valid) e0 = 0.f;
              if (base + 2 * i + 1 >= ncols_valid) e1 = 0.f;
            }
            const uint64_t ds = fmul2(pack2(e0, e1), fadd2(pack2(__uint_as_float(t[2 * i]), __uint_as_float(t[2 * i + 1])), nd));
            pw[i] = bf16x2(e0, e1);
            dw[i] = bf16x2(lo2(ds), hi2(ds));
          }
        }
        // P over S's columns, dS over T's columns (bf16 pairs), then hand both to the MMA issuer
        tmem_st32(t_s + bf * kBN, pw);
        tmem_st32(t_t + bf * kBN, dw);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_full[bf]);
      }
      if (!ok) break;
      if (nc > 0) {
        if (!warp_wait(bars, &bars->acc_full, n_items & 1, p.err)) { ok = false; break; }
        ++n_items;
      }
      // ---------------------------------------------------------------- epilogue
      if constexpr (kDKDV) {
        const int r = it.row0 + row;  // row of K_new (exact) or pooled row (Taylor)
        const bool valid = row < it.rows;
        // warpgroup 0 writes dV (accumulator 0), warpgroup 1 dK (accumulator 1, times 1/sqrt(D))
        const uint32_t t_acc = w == 0 ? t_acc0 : t_acc1;
        const float scl = w == 0 ? 1.0f : p.inv_sqrt_d;
        if (it.kind == 1) {
          // Taylor: add this column range's partial dKc / dVc (several chunks share a row tile)
          if (nc == 0) continue;  // (not reached: every chunk holds a column tile)
          float* dst = (w == 0 ? p.dvc : p.dkc) + ((size_t)it.bh * p.n_new + r) * kD;
#pragma unroll 1
          for (int c = 0; c < kD / 32; ++c) {
            uint32_t a[32];
            tmem_ld32(t_acc + 32 * c, a);
            tmem_ld_wait<32>(a);
            if (valid) {
#pragma unroll
              for (int i = 0; i < 32; ++i) atomicAdd(dst + 32 * c + i, __uint_as_float(a[i]) * scl);
            }
          }
        } else {
          // exact: row r of K_new back to its token; plus the Taylor path's spread of its block
          int tok = -1;
          if (valid) {
            if (r < p.L_src) {
              tok = r;
            } else {
              const int rr = r - p.L_src;
              tok = p.L_src + __ldg(p.sel + (size_t)it.bh * p.k + rr / p.b) * p.b + rr % p.b;
            }
          }
          const int blk = r / p.b;
          const float inv_b = 1.0f / (float)p.b;
          const float* spread = (w == 0 ? p.dvc : p.dkc);
          if (spread) spread += ((size_t)it.bh * p.n_new + blk) * kD;
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(w == 0 ? p.dv : p.dk) +
                               ((size_t)it.bh * p.N + (tok < 0 ? 0 : tok)) * kD;
#pragma unroll 1
          for (int c = 0; c < kD / 32; ++c) {
            float f[32];
            if (nc > 0) {
              uint32_t a[32];
              tmem_ld32(t_acc + 32 * c, a);
              tmem_ld_wait<32>(a);
#pragma unroll
              for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(a[i]) * scl;
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) f[i] = 0.f;
            }
            if (tok >= 0) {
              if (spread) {
#pragma unroll
                for (int i = 0; i < 32; ++i) f[i] += __ldg(spread + 32 * c + i) * inv_b;
              }
              store_bf16_32(dst + 32 * c, f);
            }
          }
        }
      } else {
        // dQ: the row's gradient at its token (rows past the item's last block are copies)
        const bool valid = row < it.rows;
        __nv_bfloat16* dq = static_cast<__nv_bfloat16*>(p.dq) + ((size_t)it.bh * p.N + tok_row) * kD;
        // warpgroup w writes columns [64 w, 64 w + 64)
#pragma unroll 1
        for (int c = 2 * w; c < 2 * w + 2; ++c) {
          uint32_t a0[32];
          tmem_ld32(t_acc0 + 32 * c, a0);
          tmem_ld_wait<32>(a0);
          float f[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(a0[i]) * p.inv_sqrt_d;
          if (valid) store_bf16_32(dq + 32 * c, f);
        }
      }
      if (nc > 0) {
        tc_fence_before();
        mbar_arrive(&bars->acc_empty);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(*reinterpret_cast<volatile uint32_t*>(&bars->tmem_base), 512);
  }
}

// delta[row] = sum_d dO[row, d] * O[row, d] (fp32), one warp per row.
__global__ void bwd_delta_kernel(const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ out,
                                 float* __restrict__ delta, size_t rows) {
  const int lane = threadIdx.x & 31;
  const size_t warps = (size_t)gridDim.x * (blockDim.x >> 5);
  for (size_t r = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const uint2 a = *reinterpret_cast<const uint2*>(dout + r * kD + 4 * lane);
    const uint2 o = *reinterpret_cast<const uint2*>(out + r * kD + 4 * lane);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o);
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float2 x = __bfloat1622float2(a2[i]), y = __bfloat1622float2(o2[i]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
#pragma unroll
    for (int o_ = 16; o_ > 0; o_ >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o_);
    if (lane == 0) delta[r] = acc;
  }
}

template <bool kDKDV>
cudaError_t launch_bwd(const void* q, const void* k, const void* v, const void* dout, const Plan& pl, const Work& w,
                       BwdParams p, uint32_t* next, cudaStream_t s) {
  p.total = p.kind_split + pl.BH * p.items_t;
  if (p.total == 0) return cudaSuccess;
  CUtensorMap tq, tdo, tk, tv, tks, tvs, tkc, tvc;
  const bool has_sel = pl.k > 0;
  const int sel_rows = has_sel ? pl.k * pl.b : pl.N;
  const bool ok = make_map(&tq, q, 2, kD, pl.N, pl.BH, 64) && make_map(&tdo, dout, 2, kD, pl.N, pl.BH, 64) &&
                  make_map(&tk, k, 2, kD, pl.N, pl.BH, 64) && make_map(&tv, v, 2, kD, pl.N, pl.BH, 64) &&
                  make_map(&tks, has_sel ? w.ksel : k, 2, kD, sel_rows, pl.BH, 64) &&
                  make_map(&tvs, has_sel ? w.vsel : v, 2, kD, sel_rows, pl.BH, 64) &&
                  make_map(&tkc, w.kcn, 2, kD, pl.n_new, pl.BH, 64) &&
                  make_map(&tvc, w.vcn, 2, kD, pl.n_new, pl.BH, 64);
  if (!ok) return cudaErrorInvalidValue;
  auto kern = attention_bwd_kernel<kDKDV>;
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidKernelImage;  // the register split needs this count
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
  if (e != cudaSuccess) return e;
  int grid = device_sm_count();
  if (grid > p.total) grid = p.total;
  kern<<<grid, kThreads, kSmemAlloc, s>>>(tq, tdo, tk, tv, tks, tvs, tkc, tvc, p, next);
  return cudaGetLastError();
}

}  // namespace

bool backward_supported(const Plan& p) { return p.dt == 0 && p.D == kD && !p.ragged && p.k_ns == 0; }

size_t backward_workspace_bytes(const Plan& p) {
  auto a = [](size_t x) { return (x + 255) & ~size_t(255); };
  return a(sizeof(float) * (size_t)p.BH * p.N) + 2 * a(sizeof(float) * (size_t)p.BH * p.n_new * p.D);
}

cudaError_t launch_backward(const void* q, const void* k, const void* v, const void* out, const float* lse,
                            const void* dout, void* dq, void* dk, void* dv, const Plan& pl, const Work& w,
                            void* bwd_ws, cudaStream_t s) {
  auto a = [](size_t x) { return (x + 255) & ~size_t(255); };
  char* base = static_cast<char*>(bwd_ws);
  float* delta = reinterpret_cast<float*>(base);
  float* dkc = reinterpret_cast<float*>(base + a(sizeof(float) * (size_t)pl.BH * pl.N));
  float* dvc = reinterpret_cast<float*>(reinterpret_cast<char*>(dkc) + a(sizeof(float) * (size_t)pl.BH * pl.n_new * pl.D));
  const size_t rows = (size_t)pl.BH * pl.N;
  const size_t row_bytes = (size_t)pl.D * 2;
  cudaError_t e;
  // unkept context rows get no gradient; kept rows are overwritten by the dK/dV kernel
  if ((e = cudaMemsetAsync(dk, 0, rows * row_bytes, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dv, 0, rows * row_bytes, s)) != cudaSuccess) return e;
  if (pl.n_flat > 0) {
    if ((e = cudaMemsetAsync(dkc, 0, sizeof(float) * (size_t)pl.BH * pl.n_new * pl.D, s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dvc, 0, sizeof(float) * (size_t)pl.BH * pl.n_new * pl.D, s)) != cudaSuccess) return e;
  }
  {
    const int threads = 256;
    size_t blocks = (rows + 7) / 8;
    const size_t cap = (size_t)device_sm_count() * 16;
    if (blocks > cap) blocks = cap;
    bwd_delta_kernel<<<(unsigned)blocks, threads, 0, s>>>(static_cast<const __nv_bfloat16*>(dout),
                                                          static_cast<const __nv_bfloat16*>(out), delta, rows);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  BwdParams p{};
  p.route = w.route;
  p.sel = w.sel;
  p.lse = lse;
  p.delta = delta;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.err = w.ctrl;
  if ((e = cudaMemsetAsync(w.ctrl + kCtrlBwdNext, 0, 3 * sizeof(uint32_t), s)) != cudaSuccess) return e;
  p.BH = pl.BH;
  p.N = pl.N;
  p.b = pl.b;
  p.L_src = pl.L_src;
  p.n_q = pl.n_q;
  p.n_exact = pl.n_exact;
  p.n_flat = pl.n_flat;
  p.L_new = pl.L_new;
  p.n_new = pl.n_new;
  p.k = pl.k;
  p.scale_log2 = kLog2e / sqrtf((float)kD);
  p.inv_sqrt_d = 1.0f / sqrtf((float)kD);
  p.log2_b = log2f((float)pl.b);
  // dQ: 128-row query tiles of each path
  {
    BwdParams d = p;
    d.items_e = (pl.n_exact * pl.b + kBM - 1) / kBM;
    d.items_t = (pl.n_flat * pl.b + kBM - 1) / kBM;
    d.kind_split = pl.BH * d.items_e;
    d.chunks = 1;
    if ((e = launch_bwd<false>(q, k, v, dout, pl, w, d, w.ctrl + kCtrlBwdNext, s)) != cudaSuccess) return e;
  }
  // dK/dV of the Taylor path over the pooled rows: column ranges split so that the grid fills
  // the GPU, partial sums added into dKc / dVc
  if (pl.n_flat > 0) {
    BwdParams d = p;
    d.dkc = dkc;
    d.dvc = dvc;
    d.items_e = 0;
    const int row_tiles = (pl.n_new + kBM - 1) / kBM;
    const int ncols = pl.n_flat * pl.b / kBN;
    int chunks = (2 * device_sm_count() + pl.BH * row_tiles - 1) / (pl.BH * row_tiles);
    if (chunks > ncols) chunks = ncols;
    if (chunks < 1) chunks = 1;
    d.chunks = chunks;
    d.items_t = row_tiles * chunks;
    d.kind_split = 0;
    if ((e = launch_bwd<true>(q, k, v, dout, pl, w, d, w.ctrl + kCtrlBwdNext + 1, s)) != cudaSuccess) return e;
  }
  // dK/dV of the exact path over the rows of K_new, plus the Taylor spread, written to dK / dV
  {
    BwdParams d = p;
    d.dkc = pl.n_flat > 0 ? dkc : nullptr;
    d.dvc = pl.n_flat > 0 ? dvc : nullptr;
    d.items_e = (pl.L_new + kBM - 1) / kBM;
    d.items_t = 0;
    d.kind_split = pl.BH * d.items_e;
    d.chunks = 1;
    if ((e = launch_bwd<true>(q, k, v, dout, pl, w, d, w.ctrl + kCtrlBwdNext + 2, s)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace isa
