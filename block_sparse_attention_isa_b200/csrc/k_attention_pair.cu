// Stage 4-5 of In-context Sparse Attention (both attention paths and the
// write-back) for bf16 inputs with D = 128, on pairs of CTAs that share every
// tensor-core operation.
//
// Method: "Lightning Unified Video Editing via In-Context Sparse Attention",
// papernotes.org notes, Key design 2 and the flowchart: the exact path is online
// softmax attention of a sharp query block over all keys of
// K_new = [K_src ; kept context blocks]; the block-wise 0th-order Taylor path
// replaces each block j of K_new by b * exp(q . Kc_j / sqrt(D)) paired with Vc_j,
// and since every block holds b keys the weight b cancels, leaving
// softmax(q Kc_new^T / sqrt(D)) Vc_new: the same attention against the n_new
// pooled rows. Each output row is written at its original token position.
//
// Why pairs. With one CTA per SM, every 256 query rows re-read their head's whole
// K_new / V_new from L2 (22.5 GB per call at the 32K-token workload). A
// tcgen05.mma with cta_group::2 computes M = 256 rows on two SMs: each CTA holds
// its own 128 query rows of A and HALF of B. Here each CTA loads 64 of the 128
// keys of every K tile and 64 of the 128 columns of every V tile, so per query
// row the pair moves half the K/V bytes from L2 and reads half the B operand
// bytes from shared memory (the Q K^T MMA, M = 256 and N = 128, then reads 6 KB
// of shared memory per 64 cycles on each SM, under the 128 B/clk it can take).
//
// Structure (each CTA of the pair: 12 warps, one CTA per SM):
//  * warp 0 issues the TMA loads of this CTA's halves; the loads of both CTAs
//    signal the leader CTA's "full" barriers, which the leader arms with the
//    byte count of both halves;
//  * warp 1 of the leader issues every MMA: the whole warp runs the loop with
//    warp-uniform values and one elected lane issues each instruction (the MMAs
//    go out in one order, from one lane at a time); completions are committed
//    to the barriers of both CTAs at once (multicast commit);
//  * warps 4-7 and 8-11 are two softmax warpgroups per CTA, one per query-tile
//    slot: slot t of a work item is tile 2t in the leader and tile 2t + 1 in the
//    peer (a slot with no tile for the peer gives it a copy of the leader's tile,
//    computed and not stored). One thread per query row; every softmax thread of
//    both CTAs arrives on the leader's "P written" barrier;
//  * K/V tiles of 128 keys in 4-stage rings; TMEM of each CTA: slot t owns one
//    128-column S buffer at [128 t, 128 t + 128) and O_t at [256 + 128 t, ...);
//    P_j is written over S_j as bf16 pairs (its first 64 columns) and read by the
//    P V MMA straight from TMEM;
//  * per slot, the MMA issuer sends P V_j and then S of tile j + 1 into the same
//    buffer (one thread's MMAs run in issue order, so S_{j+1} is written only
//    after P V_j has read P_j); the order per K/V tile is P0 V_j, S0 of j + 1,
//    P1 V_j, S1 of j + 1, so while slot 0's softmax works on tile j + 1 the
//    tensor core runs slot 1's P V and S, and the two softmax warpgroups stay
//    staggered instead of sharing the ex2 units at the same time;
//  * the softmax writes P in two halves of 64 keys and signals each, so the P V
//    MMAs of the first half run while the second half is exponentiated;
//  * work items from a per-call counter, exact items first and Taylor items
//    after: the leader's producer takes each index and publishes it to both CTAs'
//    roles through a ring in shared memory, so a pair that finishes its exact
//    items early fills the end with the cheap Taylor items;
//  * lazy rescaling (the running max moves only when it grows by more than 2^8);
//    one pair of exponentials in eight on the FMA-pipe polynomial (exp2_poly.cuh);
//  * every wait is bounded; on a timeout the CTA flags an error in the device
//    error word and in the abort flags of both CTAs, lets its copies land,
//    meets its peer at a cluster barrier and frees TMEM.
// Short last blocks (b does not divide L_src or L_ctx): K_new still gives every
// block b rows, so the source part of K_new ends at n_src * b; the exact path
// masks the rows past a short block's keys (the source part's padding and the
// tail of a kept short context block), the Taylor path adds log2(len / b) to the
// exponent of a short block's pooled row so that it weighs its own length, and
// query rows are read and written by block start, only a block's own rows stored.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <float.h>

#include "exp2_poly.cuh"
#include "isa_internal.h"
#include "pair_ptx.cuh"
#include "ptx.cuh"
#include "tensor_map.cuh"

namespace isa {
namespace {

constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kLowRegs = 88;
constexpr int kHighRegs = 208;
static_assert(128 * kLowRegs + 256 * kHighRegs <= kThreads * kLaunchRegs, "register split exceeds the launch budget");
constexpr int kD = 128;
constexpr int kBM = 128;            // query rows per tile (per CTA)
constexpr int kBN = 128;            // keys per K/V tile (per pair)
constexpr int kCols = kBN;          // scores per softmax thread and K/V tile
#ifndef ISA_PAIR_STAGES
#define ISA_PAIR_STAGES 4
#endif
constexpr int kStages = ISA_PAIR_STAGES;  // K/V ring: stage i holds this CTA's halves of the K and V tile i
constexpr int kRB = kD * 2;         // bytes per row
constexpr int kQCh = kBM * 128;     // bytes between the two 128-byte chunks of a Q tile
constexpr int kQTile = kBM * kRB;   // 32 KB
constexpr int kKRows = kBN / 2;     // keys of each K tile held by one CTA
constexpr int kKCh = kKRows * 128;  // bytes between the chunks of a K half-tile
constexpr int kKHalf = kKRows * kRB;  // 16 KB
constexpr int kVRows = 64;            // keys per V copy (a copy never straddles the seam of K_new)
constexpr int kVHalf = kBN * 128;     // 16 KB: 128 keys x this CTA's 64 columns
constexpr uint32_t kIdescQK = umma_idesc(1u, 256, kBN, 0, 0);
constexpr uint32_t kIdescPV = umma_idesc(1u, 256, kD, 0, 1);
constexpr float kRescaleThreshold = 8.0f;
constexpr int kRing = 4;  // work items published ahead by the leader's producer
constexpr int kItemFreeArrivals = 1 + 256 + 1 + 256;
// Share of the exponentials computed by the FMA-pipe polynomial (exp2_poly.cuh) instead of
// ex2: pair i of a row goes to the polynomial when (i % kPolyDen) < kPolyNum. One pair in eight
// measured 1.5-2.5 % faster than none; two in eight slower again.
#ifndef ISA_PAIR_POLY_NUM
#define ISA_PAIR_POLY_NUM 1
#endif
#ifndef ISA_PAIR_POLY_DEN
#define ISA_PAIR_POLY_DEN 8
#endif
constexpr int kPolyNum = ISA_PAIR_POLY_NUM;
constexpr int kPolyDen = ISA_PAIR_POLY_DEN;

// Scalars and the pointers every call uses. (The two pointers that only some instances read travel
// in PairExtra: with them in this struct, ptxas spilled registers in every instance.)
struct PairParams {
  const int32_t* route;
  void* out;
  uint32_t* err;
  float taylor_ln_b;   // ln(b): the Taylor rows' weight b, dropped from their exponents, back in their lse
  // short blocks (a kept short block is the last one kept)
  int k, n_src, L_srcp, len_src_last, len_ctx_last, ragged;
  float src_last_bias, ctx_last_bias;  // log2(len / b) / scale_log2: raw-score offsets of short pooled rows
  int BH, N, b, L_src, n_q, n_exact, n_flat, L_new, n_new;
  int bpt;      // blocks per 128-row tile (128 / b)
  int bpi;      // blocks per work item (4 tiles)
  int items_e;  // exact items per head
  int items_t;  // Taylor items per head
  int total;    // all items
  float scale_log2;
};

struct PairExtra {
  float* lse;          // kLse: [BH, N] natural log of each row's softmax denominator
  const int32_t* sel;  // kRagged: [BH, k] kept context blocks
  uint32_t* next;      // per-call work counter (zeroed with the control words)
};

struct Bars {
  uint64_t q_full[2];    // leader: Q of slot t in both CTAs
  uint64_t q_empty[2];   // slot t's S MMAs of the item are complete
  uint64_t kv_full[kStages];   // leader: both CTAs' K and V halves of the stage
  uint64_t kv_empty[kStages];  // the MMAs reading the stage are complete
  uint64_t s_full[2];     // [slot]: S of the slot's next K/V tile (and every earlier MMA of it) complete
  uint64_t p_full[2][2];  // leader: [slot][half], one arrival per softmax thread of both CTAs
  uint64_t o_done[2];     // [slot]: the P V MMAs of the slot's item are complete
  uint64_t drain;         // leader: every MMA is complete
  // Work items, taken by the leader's producer from the per-call counter and published to both
  // CTAs through a ring: item_full in each CTA (1 arrival), item_free in the leader (the
  // leader's issuer and softmax threads, the peer's producer and softmax threads).
  uint64_t item_full[kRing];
  uint64_t item_free[kRing];
  int item_ring[kRing];  // item index, or -1 past the last
  uint32_t tmem_base;
  int abort_flag;
};

constexpr int kOffQ = 0;
constexpr int kOffK = 2 * kQTile;
constexpr int kOffV = kOffK + kStages * kKHalf;
constexpr int kOffBar = kOffV + kStages * kVHalf;
constexpr int kSmemAlloc = kOffBar + (int)sizeof(Bars) + 1024;
static_assert(kSmemAlloc <= 227 * 1024, "shared memory");

// First token of query block i (source blocks from 0, context blocks from L_src) and its length.
__device__ __forceinline__ int qblock_start(const PairParams& p, int i) {
  return i < p.n_src ? i * p.b : p.L_src + (i - p.n_src) * p.b;
}
__device__ __forceinline__ int qblock_len(const PairParams& p, int i) {
  return i == p.n_src - 1 ? p.len_src_last : (i == p.n_q - 1 ? p.len_ctx_last : p.b);
}
// Whether head bh keeps the short last context block, which is then the last block of K_new.
__device__ __forceinline__ bool short_ctx_kept(const PairParams& p, const int32_t* sel, int bh) {
  return p.len_ctx_last < p.b && p.k > 0 && __ldg(sel + (size_t)bh * p.k + p.k - 1) == p.n_q - p.n_src - 1;
}
// -inf for the key rows [lo, hi) of the K/V tile starting at row `base` (uniform per tile).
__device__ __forceinline__ void mask_key_rows(uint32_t (&r)[kCols], int base, int lo, int hi) {
  if (hi <= base || lo >= base + kBN) return;
#pragma unroll
  for (int i = 0; i < kCols; ++i)
    if (base + i >= lo && base + i < hi) r[i] = 0xff800000u;
}
// Adds `delta` to the raw score of the column holding pooled row `col` (tile rows from `base`).
__device__ __forceinline__ void add_col_bias(uint32_t (&r)[kCols], int base, int col, float delta) {
  const int c = col - base;
  if (c < 0 || c >= kBN) return;
#pragma unroll
  for (int i = 0; i < kCols; ++i)
    if (i == c) r[i] = __float_as_uint(__uint_as_float(r[i]) + delta);
}

// Cluster-scope acquire wait (the peer CTA's item ring is written and signalled by the leader's
// producer), bounded like mbar_wait_or_abort.
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_acq_cluster_or_abort(uint64_t* bar, uint32_t parity, const int* abort) {
  const uint32_t a = smem_addr(bar);
  if (mbar_try_wait_acq_cluster(a, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait_acq_cluster(a, parity)) return true;
    if (*reinterpret_cast<const volatile int*>(abort) != 0) return false;
    if (global_timer_ns() - t0 > kWaitTimeoutNs) return false;
  }
}
__device__ __forceinline__ void arrive_cluster_release(uint32_t addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}

struct Item {
  int bh, kind, nblk, ntiles, nslots, nkv, last_valid;
  const int32_t* lst;
  __device__ __forceinline__ int blk(int u) const { return __ldg(lst + u); }
};

__device__ __forceinline__ Item decode_item(const PairParams& p, int g) {
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
  const int first = pp * p.bpi;
  it.lst = p.route + (size_t)it.bh * p.n_q + base + first;
  it.nblk = min(p.bpi, count - first);
  it.ntiles = (it.nblk + p.bpt - 1) / p.bpt;
  it.nslots = (it.ntiles + 1) / 2;
  const int rows = it.kind == 0 ? p.L_new : p.n_new;
  it.nkv = (rows + kBN - 1) / kBN;
  it.last_valid = rows - kBN * (it.nkv - 1);
  return it;
}

// Record the error and stop both CTAs of the pair.
__device__ __noinline__ void raise_abort(Bars* b, uint32_t* err, uint32_t code) {
  atomicOr(err, code);
  *reinterpret_cast<volatile int*>(&b->abort_flag) = 1;
  store_cluster_u32(map_to(&b->abort_flag, cluster_rank() ^ 1u), 1u);
}

// All 32 lanes wait on a local barrier; the warp is converged on return.
__device__ __forceinline__ bool warp_wait(Bars* b, uint64_t* bar, uint32_t parity, uint32_t* err) {
  bool ok = mbar_wait_or_abort(bar, parity, &b->abort_flag);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) raise_abort(b, err, kErrSoftmax);
  tc_fence_after();
  return ok;
}

__device__ __forceinline__ void store_row_chunk(__nv_bfloat16* dst, const float* v) {  // 32 values
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

// kRagged: the call has a short last block (block starts, masks, length weights); kLse: write each
// row's lse. Whole-block calls without lse run code with neither.
template <bool kRagged, bool kLse>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attention_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_ksel, const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_vsel, const __grid_constant__ CUtensorMap tm_kcn,
                          const __grid_constant__ CUtensorMap tm_vcn, const PairParams p,
                          const PairExtra x) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sK = smem + kOffK;
  uint8_t* sV = smem + kOffV;
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->q_full[t], 1);
      mbar_init(&bars->q_empty[t], 1);
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->o_done[t], 1);
      for (int h = 0; h < 2; ++h) mbar_init(&bars->p_full[t][h], 256);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&bars->item_full[i], 1);
      mbar_init(&bars->item_free[i], kItemFreeArrivals);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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
  if (warp == 1) {  // the same warp in both CTAs allocates the pair's TMEM
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(&bars->tmem_base)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_warp();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();

  // A kernel launched after this one with programmatic serialization (the mixed Taylor kernel)
  // may take SMs as soon as CTAs of this grid exit.
  asm volatile("griddepcontrol.launch_dependents;");

  if (warp < 4) regs_dealloc<kLowRegs>();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t q_full_l = map_to(&bars->q_full[0], 0);
      const uint32_t kv_full_l = map_to(&bars->kv_full[0], 0);
      uint32_t kv_it = 0, q_loads0 = 0, q_loads1 = 0;
      bool ok = true;
      // Items in counter order: all exact items, then the (much cheaper) Taylor items, so a pair
      // that finishes its exact work early fills the end with Taylor items.
      for (uint32_t n = 0; ok; ++n) {
        const uint32_t slot = n % kRing;
        int g;
        if (rank == 0) {
          if (n >= kRing && !mbar_wait(&bars->item_free[slot], ((n / kRing) - 1) & 1)) {
            raise_abort(bars, p.err, kErrProducer);
            ok = false;
            break;
          }
          g = (int)atomicAdd(x.next, 1u);
          if (g >= p.total) g = -1;
          *reinterpret_cast<volatile int*>(&bars->item_ring[slot]) = g;
          store_cluster_u32(map_to(&bars->item_ring[slot], 1), (uint32_t)g);
          mbar_arrive(&bars->item_full[slot]);
          arrive_cluster_release(map_to(&bars->item_full[slot], 1));
        } else {
          if (!mbar_wait_acq_cluster_or_abort(&bars->item_full[slot], (n / kRing) & 1, &bars->abort_flag)) {
            raise_abort(bars, p.err, kErrProducer);
            ok = false;
            break;
          }
          g = *reinterpret_cast<volatile int*>(&bars->item_ring[slot]);
          arrive_cluster_release(map_to(&bars->item_free[slot], 0));
        }
        if (g < 0) break;
        const Item it = decode_item(p, g);
        for (int t = 0; t < it.nslots; ++t) {
          // slot t's Q buffer is free once the S MMAs of the last item that used it are complete
          const uint32_t prior = t == 0 ? q_loads0 : q_loads1;
          if (prior > 0 && !mbar_wait(&bars->q_empty[t], (prior - 1) & 1)) {
            raise_abort(bars, p.err, kErrProducer);
            ok = false;
            break;
          }
          if (t == 0) ++q_loads0; else ++q_loads1;
          if (rank == 0) mbar_arrive_expect_tx(&bars->q_full[t], 2 * kQTile);
          int ut = 2 * t + (int)rank;
          if (ut >= it.ntiles) ut = 2 * t;  // no tile for the peer in this slot: a copy, not stored
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int r = 64 * h;
            int u = ut * p.bpt + r / p.b;
            if (u >= it.nblk) u = ut * p.bpt;  // missing block of a partial tile: rows are not stored
            // rows past a short block: loaded, not stored
            const int y = (kRagged ? qblock_start(p, it.blk(u)) : it.blk(u) * p.b) + (r % p.b);
#pragma unroll
            for (int c = 0; c < 2; ++c)
              tma_load_pair(sQ + t * kQTile + c * kQCh + h * 8192, &tm_q, q_full_l + 8u * t, c * 64, y, it.bh);
          }
        }
        for (int j = 0; j < it.nkv && ok; ++j, ++kv_it) {
          if (*reinterpret_cast<volatile int*>(&bars->abort_flag)) { ok = false; break; }
          const int r0 = j * kBN;
          const int st = kv_it % kStages;
          if (!mbar_wait(&bars->kv_empty[st], ((kv_it / kStages) & 1) ^ 1)) {
            raise_abort(bars, p.err, kErrProducer);
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&bars->kv_full[st], 2 * (kKHalf + kVHalf));
          const uint32_t bar = kv_full_l + 8u * st;
          // K: this CTA's 64 keys of the tile (64 keys never straddle the seam of K_new's source
          // part, which ends at n_src * b, a multiple of 64)
          {
            const int rk = r0 + (int)rank * kKRows;
            const CUtensorMap* map;
            int y;
            if (it.kind == 0) {
              if (rk < p.L_srcp) { map = &tm_k; y = rk; } else { map = &tm_ksel; y = rk - p.L_srcp; }
            } else {
              map = &tm_kcn; y = rk;
            }
#pragma unroll
            for (int c = 0; c < 2; ++c) tma_load_pair(sK + st * kKHalf + c * kKCh, map, bar, c * 64, y, it.bh);
          }
          // V: all 128 keys in two copies of 64, this CTA's 64 columns
#pragma unroll
          for (int h = 0; h < kBN / kVRows; ++h) {
            const int rv = r0 + h * kVRows;
            const CUtensorMap* map;
            int y;
            if (it.kind == 0) {
              if (rv < p.L_srcp) { map = &tm_v; y = rv; } else { map = &tm_vsel; y = rv - p.L_srcp; }
            } else {
              map = &tm_vcn; y = rv;
            }
            tma_load_pair(sV + st * kVHalf + h * kVRows * 128, map, bar, (int)rank * 64, y, it.bh);
          }
        }
      }
      if (!ok) {
        // the copies this thread started signal the leader's barriers, which this CTA cannot
        // wait on; give them time to land (copies complete in microseconds) before leaving
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 2000000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader CTA only)
    // The whole warp runs the issue loop with warp-uniform values and one elected lane issues
    // each tensor-core instruction (issued from a single-lane branch, every MMA took about 60
    // cycles of the issuing thread, as long as the MMA itself). The MMAs of both slots go out
    // in a fixed order per K/V tile j:
    // P0 V_j, S0 of tile j + 1, P1 V_j, S1 of tile j + 1. Slot 1's S completes one slot's
    // worth of tensor work after slot 0's, so the two softmax warpgroups stay staggered:
    // each exponentiates mostly while the tensor core runs the other slot's MMAs, rather
    // than both at once on the shared ex2 units.
    if (rank == 0) {
      const uint32_t tmem = __shfl_sync(0xffffffffu, *reinterpret_cast<volatile uint32_t*>(&bars->tmem_base), 0);
      uint32_t kv_base = 0, q_cnt[2] = {0, 0}, p_seq[2] = {0, 0};
      bool ok = true;
      constexpr uint32_t HI = desc_hi_sw128(1024);
      const uint32_t k_lo = desc_lo(smem_addr(sK), 16);
      const uint32_t v_lo = desc_lo(smem_addr(sV), (uint32_t)kVHalf);
      // S_t = Q_t K^T for the K tile in stage st (rows of both CTAs, keys of both halves)
      auto issue_s = [&](int t, uint32_t st) {
        const uint32_t q_lo = desc_lo(smem_addr(sQ + t * kQTile), 16);
        const uint32_t kb = k_lo + ((st * kKHalf) >> 4);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const uint32_t qo = (uint32_t)(((s / 4) * kQCh + (s % 4) * 32) >> 4);
          const uint32_t ko = (uint32_t)(((s / 4) * kKCh + (s % 4) * 32) >> 4);
          mma_ss_pair_warp(tmem + 128 * t, q_lo + qo, kb + ko, HI, kIdescQK, s > 0 ? 1u : 0u);
        }
        commit_pair_warp(&bars->s_full[t]);
      };
      // O_t (+)= P V over keys [64 h, 64 h + 64) of the V tile in stage st, P (of each CTA, from its
      // own TMEM) in slot t's S buffer columns [32 h, 32 h + 32)
      auto issue_pv = [&](int t, uint32_t st, uint32_t acc, int h) {
        const uint32_t vb = v_lo + ((st * kVHalf) >> 4);
#pragma unroll
        for (int s = 4 * h; s < 4 * h + 4; ++s)
          mma_ts_pair_warp(tmem + 256 + 128 * t, tmem + 128 * t + s * 8, vb + (uint32_t)((s * 16 * 128) >> 4), HI,
                      kIdescPV, (acc | (uint32_t)s) != 0 ? 1u : 0u);
      };
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
      for (uint32_t n = 0; ok; ++n) {
        const uint32_t slot = n % kRing;
        if (!wait(&bars->item_full[slot], (n / kRing) & 1)) break;
        const int g = __shfl_sync(0xffffffffu, *reinterpret_cast<volatile int*>(&bars->item_ring[slot]), 0);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->item_free[slot]);
        if (g < 0) break;
        const Item it = decode_item(p, g);
        const int ns = it.nslots;
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (t < ns && ok && wait(&bars->q_full[t], q_cnt[t] & 1)) ++q_cnt[t];
        if (!ok) break;
        // S of the first K/V tile for every slot
        {
          const uint32_t st0 = kv_base % kStages;
          if (!wait(&bars->kv_full[st0], (kv_base / kStages) & 1)) break;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (t >= ns) break;
            issue_s(t, st0);
            if (it.nkv == 1) commit_pair_warp(&bars->q_empty[t]);
          }
        }
        for (int j = 0; j < it.nkv && ok; ++j) {
          const uint32_t idx = kv_base + j, st = idx % kStages;
          const bool more = j + 1 < it.nkv;
          const uint32_t idx1 = idx + 1, st1 = idx1 % kStages;
          // the K/V stage of tile j + 1 first (normally long full)
          if (more && !wait(&bars->kv_full[st1], (idx1 / kStages) & 1)) break;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (t >= ns) break;
            if (!wait(&bars->p_full[t][0], p_seq[t] & 1)) break;
            issue_pv(t, st, j > 0 ? 1u : 0u, 0);
            if (!wait(&bars->p_full[t][1], p_seq[t] & 1)) break;
            issue_pv(t, st, 1u, 1);
            ++p_seq[t];
            if (more) {
              issue_s(t, st1);
              if (j + 2 == it.nkv) commit_pair_warp(&bars->q_empty[t]);
            } else {
              commit_pair_warp(&bars->o_done[t]);
            }
          }
          if (!ok) break;
          commit_pair_warp(&bars->kv_empty[st]);
        }
        kv_base += it.nkv;
      }
      // every MMA completes before either CTA can release TMEM or leave
      commit_pair_warp(&bars->drain);
      mbar_wait(&bars->drain, 0);
      __syncwarp();
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue (both CTAs)
    regs_alloc<kHighRegs>();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(&bars->tmem_base);
    const int t = (warp - 4) >> 2;  // slot of this warpgroup
    const int wl = warp & 3;        // TMEM lane quarter
    const int row = wl * 32 + lane; // row inside this CTA's 128-row tile
    const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
    const uint32_t t_s = tmem + lane_off + t * 128;
    const uint32_t t_o = tmem + lane_off + 256 + t * 128;
    const uint32_t p_full_l = map_to(&bars->p_full[t][0], 0);  // the leader's P barriers of this slot
    uint32_t seq = 0, items = 0;
    bool ok = true;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
    const uint32_t item_free_l = map_to(&bars->item_free[0], 0);
    for (uint32_t n = 0; ok; ++n) {
      const uint32_t slot = n % kRing;
      {
        bool got = rank == 0 ? mbar_wait_or_abort(&bars->item_full[slot], (n / kRing) & 1, &bars->abort_flag)
                             : mbar_wait_acq_cluster_or_abort(&bars->item_full[slot], (n / kRing) & 1,
                                                              &bars->abort_flag);
        got = __all_sync(0xffffffffu, got);
        if (!got) {
          if (lane == 0) raise_abort(bars, p.err, kErrSoftmax);
          ok = false;
          break;
        }
      }
      const int g = *reinterpret_cast<volatile int*>(&bars->item_ring[slot]);
      if (rank == 0) mbar_arrive(&bars->item_free[slot]);
      else arrive_cluster_release(item_free_l + 8u * slot);
      if (g < 0) break;
      const Item it = decode_item(p, g);
      if (t >= it.nslots) continue;
      const bool cs = kRagged ? short_ctx_kept(p, x.sel, it.bh) : false;
      float m = -FLT_MAX, l = 0.f;
      for (int j = 0; j < it.nkv; ++j, ++seq) {
        // S_j complete implies P V_{j-1} complete (the issuer sent it first), so O may be rescaled
        if (!warp_wait(bars, &bars->s_full[t], seq & 1, p.err)) { ok = false; break; }
        uint32_t r[kCols];
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) tmem_ld32(t_s + 32 * c, r + 32 * c);
        tmem_ld_wait<kCols>(r);
        if (j == it.nkv - 1 && it.last_valid < kBN) {  // ragged last K/V tile (uniform branch)
#pragma unroll
          for (int i = 0; i < kCols; ++i)
            if (i >= it.last_valid) r[i] = __float_as_uint(-INFINITY);
        }
        if constexpr (kRagged) {  // (the first tile always holds a key of block 0)
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
        // row max: 8 independent chains of 3-input max over the 128 scores
        float mc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
          mc[c] = fmax3(__uint_as_float(r[c]), __uint_as_float(r[8 + c]), __uint_as_float(r[16 + c]));
#pragma unroll
        for (int q = 24; q + 8 < kCols; q += 16)
#pragma unroll
          for (int c = 0; c < 8; ++c) mc[c] = fmax3(mc[c], __uint_as_float(r[q + c]), __uint_as_float(r[q + 8 + c]));
#pragma unroll
        for (int c = 0; c < 8; ++c) mc[c] = fmaxf(mc[c], __uint_as_float(r[kCols - 8 + c]));
        const float raw_max = fmax3(fmax3(mc[0], mc[1], mc[2]), fmax3(mc[3], mc[4], mc[5]), fmaxf(mc[6], mc[7]));
        const float mx = raw_max * p.scale_log2;
        const bool need = (j > 0) && (mx > m + kRescaleThreshold);
        const float alpha = need ? ex2_approx(m - mx) : 1.0f;
        if (j == 0 || need) m = mx;
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int c = 0; c < kD / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(t_o + 32 * c, o);
            tmem_ld_wait<32>(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(t_o + 32 * c, o);
          }
        }
        // The P V MMA multiplies the bf16 p; the row sum takes the fp32 p, except that the tile's
        // largest p enters as its bf16 value when it exceeds 1. With the lazy maximum a row's
        // dominant keys have p in (1, 2^8] (only in tiles whose maximum exceeds m), which bf16
        // rounds by up to 2^-9: left in the sum, that mismatch between numerator and denominator
        // would scale the whole output row by it. (A key that set m has p = 1 exactly.)
        // p = 2^(s * scale - m) in pairs, written over this tile's S buffer as bf16 pairs, 64 keys
        // (32 columns) at a time, each half signalled to the MMA issuer as soon as it is in TMEM
        const uint64_t sc2 = pack2(p.scale_log2, p.scale_log2), nm2 = pack2(-m, -m);
        uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int i = 32 * h; i < 32 * h + 32; ++i) {
            const uint64_t x =
                ffma2(static_cast<uint64_t>(r[2 * i]) | (static_cast<uint64_t>(r[2 * i + 1]) << 32), sc2, nm2);
            const uint64_t e =
                (i % kPolyDen < kPolyNum) ? exp2_poly2(x) : pack2(ex2_approx(lo2(x)), ex2_approx(hi2(x)));
            acc[i & 3] = fadd2(acc[i & 3], e);
            __nv_bfloat162 hv = __floats2bfloat162_rn(lo2(e), hi2(e));
            r[i] = *reinterpret_cast<uint32_t*>(&hv);
          }
          tmem_st32(t_s + 32 * h, r + 32 * h);
          tmem_st_wait();
          tc_fence_before();
          arrive_cluster(p_full_l + 8u * h);
        }
        float corr = 0.f;
        if (mx > m) {
          const float em = ex2_approx(fmaf(raw_max, p.scale_log2, -m));  // the largest p, as computed above
          corr = __bfloat162float(__float2bfloat16_rn(em)) - em;
        }
        const uint64_t a2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
        l = l * alpha + ((lo2(a2) + hi2(a2)) + corr);
      }
      if (!ok) break;
      // epilogue: O / l at the row's original token position
      const float inv_l = 1.0f / l;
      if (!warp_wait(bars, &bars->o_done[t], items & 1, p.err)) { ok = false; break; }
      ++items;
      const int ut = 2 * t + (int)rank;
      const int u = ut * p.bpt + row / p.b;
      const int qb = it.blk((ut < it.ntiles && u < it.nblk) ? u : 0);
      const bool store = (ut < it.ntiles) && (u < it.nblk) && (!kRagged || (row % p.b) < qblock_len(p, qb));
      const size_t token = (size_t)(kRagged ? qblock_start(p, qb) : qb * p.b) + (row % p.b);
      __nv_bfloat16* dst = out + ((size_t)it.bh * p.N + token) * kD;
      if constexpr (kLse) {
        // log of the row's denominator: m and log2(l) are base 2 (a short pooled row's length is
        // already in its exponent, the weight b is not)
        if (store)
          x.lse[(size_t)it.bh * p.N + token] =
              (m + __log2f(l)) * 0.6931471805599453f + (it.kind == 1 ? p.taylor_ln_b : 0.f);
      }
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + 32 * c, o);
        tmem_ld_wait<32>(o);
        float* f = reinterpret_cast<float*>(o);
#pragma unroll
        for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(o[i]) * inv_l;
        if (store) store_row_chunk(dst + 32 * c, f);
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  cluster_sync_warp();  // both CTAs done with TMEM, shared memory and the leader's barriers
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(
                     *reinterpret_cast<volatile uint32_t*>(&bars->tmem_base)),
                 "r"(512)
                 : "memory");
  }
}

}  // namespace

// The build checks that the kernel compiled to kLaunchRegs registers per thread, which its
// warpgroup register split needs. A library built some other way that got another count runs its
// calls on the single-CTA kernel instead (the launcher below refuses to launch it).
bool attention_pair_regs_ok() {
  static int cached[64] = {0};  // 0 unknown, 1 ok, 2 not ok
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!cached[dev]) {
    cudaFuncAttributes fa;
    bool ok = true;
    const void* kernels[4] = {(const void*)attention_pair_kernel<false, false>,
                              (const void*)attention_pair_kernel<false, true>,
                              (const void*)attention_pair_kernel<true, false>,
                              (const void*)attention_pair_kernel<true, true>};
    for (const void* k : kernels) ok = ok && cudaFuncGetAttributes(&fa, k) == cudaSuccess && fa.numRegs == kLaunchRegs;
    cached[dev] = ok ? 1 : 2;
  }
  return cached[dev] == 1;
}

bool attention_pair_supported(const Plan& p) { return p.dt == 0 && p.D == kD && attention_pair_regs_ok(); }

cudaError_t launch_attention_pair(const void* q, const void* k, const void* v, void* out, const Plan& pl,
                                  const Work& w, cudaStream_t s, int* n_ctas) {
  PairParams p{};
  p.route = w.route;
  p.out = out;
  p.err = w.ctrl;
  p.taylor_ln_b = logf((float)pl.b);
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
  p.n_src = pl.n_src;
  p.L_srcp = pl.L_srcp;
  p.len_src_last = pl.len_src_last;
  p.len_ctx_last = pl.len_ctx_last;
  p.ragged = pl.ragged;
  p.bpt = kBM / pl.b;
  p.bpi = 4 * p.bpt;
  p.items_e = (pl.n_exact + p.bpi - 1) / p.bpi;
  p.items_t = (pl.n_flat + p.bpi - 1) / p.bpi;
  p.total = pl.BH * (p.items_e + p.items_t);
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
  p.src_last_bias = log2f((float)pl.len_src_last / (float)pl.b) / p.scale_log2;
  p.ctx_last_bias = log2f((float)pl.len_ctx_last / (float)pl.b) / p.scale_log2;
  if (n_ctas) *n_ctas = 0;
  if (p.total == 0) return cudaSuccess;

  CUtensorMap tq, tk, tks, tv, tvs, tkc, tvc;
  const bool has_sel = pl.k > 0;
  const int sel_rows = has_sel ? pl.k * pl.b : pl.N;
  const bool ok = make_map(&tq, q, 2, kD, pl.N, pl.BH, 64) && make_map(&tk, k, 2, kD, pl.N, pl.BH, kKRows) &&
                  make_map(&tks, has_sel ? w.ksel : k, 2, kD, sel_rows, pl.BH, kKRows) &&
                  make_map(&tkc, w.kcn, 2, kD, pl.n_new, pl.BH, kKRows) &&
                  make_map(&tv, v, 2, kD, pl.N, pl.BH, kVRows) &&
                  make_map(&tvs, has_sel ? w.vsel : v, 2, kD, sel_rows, pl.BH, kVRows) &&
                  make_map(&tvc, w.vcn, 2, kD, pl.n_new, pl.BH, kVRows);
  if (!ok) return cudaErrorInvalidValue;

  auto kern = pl.ragged ? (w.lse ? attention_pair_kernel<true, true> : attention_pair_kernel<true, false>)
                        : (w.lse ? attention_pair_kernel<false, true> : attention_pair_kernel<false, false>);
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidKernelImage;  // the register split needs this count
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
  if (e != cudaSuccess) return e;
  // as many CTA pairs as can be resident at once (one CTA per SM), at most one per work item
  static int cached_pairs[64] = {0};  // the same for every instance (same block, shared memory, cluster)
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  int pairs = dev >= 0 && dev < 64 ? cached_pairs[dev] : 0;
  if (pairs <= 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (device_sm_count() / 2), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemAlloc;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if ((e = cudaOccupancyMaxActiveClusters(&pairs, kern, &cfg)) != cudaSuccess) return e;
    if (pairs <= 0) return cudaErrorLaunchOutOfResources;
    if (dev >= 0 && dev < 64) cached_pairs[dev] = pairs;
  }
  if (pairs > p.total) pairs = p.total;
  kern<<<2 * pairs, kThreads, kSmemAlloc, s>>>(tq, tk, tks, tv, tvs, tkc, tvc, p,
                                                PairExtra{w.lse, w.sel, w.ctrl + kCtrlPairNext});
  if (n_ctas) *n_ctas = 2 * pairs;
  return cudaGetLastError();
}

}  // namespace isa
