// Backward pass of In-context Sparse Attention (bf16, D = 128) on pairs of CTAs that share every
// tensor-core operation.
//
// The arithmetic is that of k_attention_bwd.cu (same method, same reading: the forward's
// decisions held fixed; the dQ kernel walks the keys of a path for its query rows, the dK/dV
// kernel walks a path's query rows for its key rows; S and T are recomputed in both). The
// difference is the shape of the work: a tcgen05.mma with cta_group::2 computes M = 256 rows on
// two SMs, each CTA holding its own 128 rows of A and HALF of every column tile of B:
//  * for the score MMAs (S = A1 B1^T, T = A2 B2^T, N = 64 columns), each CTA loads 32 of the
//    64 columns (their full D);
//  * for the accumulating MMAs (acc += X B, K = 64 columns, N = D = 128), each CTA loads all 64
//    columns but only its half of D (64 of the 128 features).
// So per row the pair streams half the column bytes from L2 that a single CTA does, and each
// CTA's tensor core reads half the B operand bytes from shared memory: with N = 64 a single
// CTA's score MMAs are bound by shared-memory reads (67 % of the MMA rate), a pair's are not.
// Column tiles are loaded in both layouts (the column data is read once per layout).
//
// Roles (each CTA of the pair, 12 warps): warp 0 issues this CTA's TMA loads, which signal the
// leader CTA's barriers (the leader arms them with both CTAs' bytes); warp 1 of the leader issues
// every MMA and commits to both CTAs' barriers at once; warps 4-7 and 8-11 are two elementwise
// warpgroups per CTA that take alternate column tiles (one S/T buffer each), one thread per row,
// and arrive on the leader's barriers; both write half of the epilogue. TMEM per CTA: S and T
// double-buffered at columns [0, 256), accumulators at [256, 384) and [384, 512). Every wait is
// bounded; a timeout flags the error word and both CTAs' abort flags, lets the CTA's copies land,
// meets the peer at the final cluster barrier and frees TMEM.
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
constexpr int kBM = 128;                  // rows per CTA (256 per pair)
constexpr int kBN = 64;                   // columns per tile (per pair)
constexpr int kStages = 4;
constexpr int kATile = kBM * kD * 2;      // 32 KB: [2 chunks][128 rows][128 B]
constexpr int kACh = kBM * 128;
constexpr int kBsTile = 32 * kD * 2;      // 8 KB: this CTA's 32 columns, all of D: [2 chunks][32 rows][128 B]
constexpr int kBsCh = 32 * 128;
constexpr int kBaTile = kBN * 128;        // 8 KB: all 64 columns, this CTA's 64 features: [64 rows][128 B]
constexpr int kStat = kBN * 4;
// stage: B1 score layout, B2 score layout, B1 accumulate layout, B2 accumulate layout, lse + delta
constexpr int kOffB1s = 0, kOffB2s = kBsTile, kOffB1a = 2 * kBsTile, kOffB2a = 2 * kBsTile + kBaTile;
constexpr int kOffStat = 2 * kBsTile + 2 * kBaTile;
constexpr int kStageBytes = kOffStat + 1024;
constexpr uint32_t kIdescS = umma_idesc(1u, 256, kBN, 0, 0);
constexpr uint32_t kIdescAcc = umma_idesc(1u, 256, kD, 0, 1);
constexpr float kLog2e = 1.4426950408889634f;

struct PairBwdParams {
  const int32_t* route;
  const int32_t* sel;
  const float* lse;
  const float* delta;
  void* dq;
  void* dk;
  void* dv;
  float* dkc;
  float* dvc;
  uint32_t* err;
  int BH, N, b, L_src, n_q, n_exact, n_flat, L_new, n_new, k;
  int kind_split, items_e, items_t, chunks, total;
  float scale_log2, inv_sqrt_d, log2_b;
};

struct Bars {
  uint64_t a_full, a_empty;
  uint64_t kv_full[kStages], kv_empty[kStages], st_full[kStages];
  uint64_t s_full[2], p_full[2];
  uint64_t acc_full, acc_empty;
  uint64_t drain;
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
__device__ __forceinline__ void store_bf16_32(__nv_bfloat16* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    d[i] = make_uint4(bf16x2(v[8 * i], v[8 * i + 1]), bf16x2(v[8 * i + 2], v[8 * i + 3]),
                      bf16x2(v[8 * i + 4], v[8 * i + 5]), bf16x2(v[8 * i + 6], v[8 * i + 7]));
}

// A work item of the pair: head, path (0 exact, 1 Taylor), first row of the pair's 256, the
// column tiles [c_begin, c_end) and the rows the path has from row0 on.
struct Item {
  int bh, kind, row0, c_begin, c_end, rows;
};

template <bool kDKDV>
__device__ __forceinline__ Item decode_item(const PairBwdParams& p, int g) {
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
    const int chunks = it.kind == 0 ? 1 : p.chunks;
    const int tile = local / chunks, chunk = local - tile * chunks;
    it.row0 = tile * 2 * kBM;
    it.rows = (it.kind == 0 ? p.L_new : p.n_new) - it.row0;
    const int ncols = ((it.kind == 0 ? p.n_exact : p.n_flat) * p.b) / kBN;
    it.c_begin = (int)(((long long)ncols * chunk) / chunks);
    it.c_end = (int)(((long long)ncols * (chunk + 1)) / chunks);
  } else {
    it.row0 = local * 2 * kBM;
    it.rows = (it.kind == 0 ? p.n_exact : p.n_flat) * p.b - it.row0;
    it.c_begin = 0;
    it.c_end = ((it.kind == 0 ? p.L_new : p.n_new) + kBN - 1) / kBN;
  }
  return it;
}

__device__ __forceinline__ int path_token(const PairBwdParams& p, int bh, int kind, int r) {
  const int32_t* lst = p.route + (size_t)bh * p.n_q + (kind == 0 ? 0 : p.n_exact);
  return __ldg(lst + r / p.b) * p.b + (r % p.b);
}

__device__ __noinline__ void raise_abort(Bars* b, uint32_t* err, uint32_t code) {
  atomicOr(err, code);
  *reinterpret_cast<volatile int*>(&b->abort_flag) = 1;
  store_cluster_u32(map_to(&b->abort_flag, cluster_rank() ^ 1u), 1u);
}
__device__ __forceinline__ bool aborted(const Bars* b) {
  return *reinterpret_cast<const volatile int*>(&b->abort_flag) != 0;
}
__device__ __forceinline__ bool warp_wait(Bars* b, uint64_t* bar, uint32_t parity, uint32_t* err) {
  bool ok = mbar_wait_or_abort(bar, parity, &b->abort_flag);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && (threadIdx.x & 31) == 0) raise_abort(b, err, kErrSoftmax);
  tc_fence_after();
  return ok;
}

template <bool kDKDV>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attention_bwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                              const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                              const __grid_constant__ CUtensorMap tm_ksel, const __grid_constant__ CUtensorMap tm_vsel,
                              const __grid_constant__ CUtensorMap tm_kcn, const __grid_constant__ CUtensorMap tm_vcn,
                              const PairBwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA1 = smem + kOffA1;
  uint8_t* sA2 = smem + kOffA2;
  uint8_t* sB = smem + kOffB;
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    mbar_init(&bars->a_full, 1);
    mbar_init(&bars->a_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
      mbar_init(&bars->st_full[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->p_full[b], 256);  // leader: one warpgroup of each CTA
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, 512);    // leader: both warpgroups of both CTAs
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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

  if (warp < 4) regs_dealloc<kLowRegs>();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t a_full_l = map_to(&bars->a_full, 0);
      const uint32_t kv_full_l = map_to(&bars->kv_full[0], 0);
      uint32_t n_items = 0, tile_it = 0;
      bool ok = true;
      // `rows` rows of K_new (or the pooled rows) from r, 32 rows per box, into dst: chunks c
      // (128 bytes of features each) from chunk c0 on, `nch` of them, at dst + c * ch
      auto load_keys = [&](uint8_t* dst, int ch, int c0, int nch, int kind, bool values, int bh, int r, int rows,
                           uint32_t bar) {
        for (int q4 = 0; q4 < rows / 32; ++q4) {
          const int rr = r + 32 * q4;
          const CUtensorMap* map;
          int y = rr;
          if (kind == 1) {
            map = values ? &tm_vcn : &tm_kcn;
          } else if (rr < p.L_src) {
            map = values ? &tm_v : &tm_k;
          } else {
            map = values ? &tm_vsel : &tm_ksel;
            y = rr - p.L_src;
          }
          for (int c = 0; c < nch; ++c)
            tma_load_pair(dst + c * ch + q4 * 4096, map, bar, (c0 + c) * 64, y, bh);
        }
      };
      // `rows` query rows of a path (Q or dO) from its r-th row, 32 per box (the 32 rows of a box
      // are consecutive tokens of one block; rows past the path's end load a copy, never stored)
      auto load_queries = [&](uint8_t* dst, int ch, int c0, int nch, bool grad, int bh, int kind, int r, int rows,
                              uint32_t bar) {
        const int all = (kind == 0 ? p.n_exact : p.n_flat) * p.b;
        for (int q4 = 0; q4 < rows / 32; ++q4) {
          const int rr = r + 32 * q4;
          const int tok = path_token(p, bh, kind, rr < all ? rr : 0);
          for (int c = 0; c < nch; ++c)
            tma_load_pair(dst + c * ch + q4 * 4096, grad ? &tm_do : &tm_q, bar, (c0 + c) * 64, tok, bh);
        }
      };
      for (int g = pair; g < p.total && ok; g += npairs) {
        const Item it = decode_item<kDKDV>(p, g);
        if (it.c_end <= it.c_begin) continue;  // nothing to accumulate (every role skips it)
        if (n_items > 0 && !mbar_wait(&bars->a_empty, (n_items - 1) & 1)) {
          raise_abort(bars, p.err, kErrProducer);
          ok = false;
          break;
        }
        ++n_items;
        if (rank == 0) mbar_arrive_expect_tx(&bars->a_full, 2 * 2 * kATile);
        const int my_row = it.row0 + kBM * (int)rank;
        if constexpr (kDKDV) {
          load_keys(sA1, kACh, 0, 2, it.kind, false, it.bh, my_row, kBM, a_full_l);
          load_keys(sA2, kACh, 0, 2, it.kind, true, it.bh, my_row, kBM, a_full_l);
        } else {
          load_queries(sA1, kACh, 0, 2, false, it.bh, it.kind, my_row, kBM, a_full_l);
          load_queries(sA2, kACh, 0, 2, true, it.bh, it.kind, my_row, kBM, a_full_l);
        }
        for (int j = it.c_begin; j < it.c_end && ok; ++j, ++tile_it) {
          if (aborted(bars)) { ok = false; break; }
          const int st = tile_it % kStages;
          if (!mbar_wait(&bars->kv_empty[st], ((tile_it / kStages) & 1) ^ 1)) {
            raise_abort(bars, p.err, kErrProducer);
            ok = false;
            break;
          }
          uint8_t* stg = sB + st * kStageBytes;
          const uint32_t bar = kv_full_l + 8u * st;
          const int c0 = j * kBN;
          if constexpr (kDKDV) {
            // columns are queries: score layouts (this CTA's 32 queries, all of D), accumulate
            // layouts (all 64 queries, this CTA's half of D); lse and delta of the 64 queries
            // (the 64 queries of a tile are consecutive tokens of one block: b is 64 or 128)
            if (rank == 0) mbar_arrive_expect_tx(&bars->kv_full[st], 2 * (2 * kBsTile + 2 * kBaTile));
            const int tok = path_token(p, it.bh, it.kind, c0);
            const int my_tok = tok + 32 * (int)rank;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              tma_load_pair(stg + kOffB1s + c * kBsCh, &tm_q, bar, c * 64, my_tok, it.bh);
              tma_load_pair(stg + kOffB2s + c * kBsCh, &tm_do, bar, c * 64, my_tok, it.bh);
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              tma_load_pair(stg + kOffB1a + h * 4096, &tm_q, bar, (int)rank * 64, tok + 32 * h, it.bh);
              tma_load_pair(stg + kOffB2a + h * 4096, &tm_do, bar, (int)rank * 64, tok + 32 * h, it.bh);
            }
            const size_t ix = (size_t)it.bh * p.N + tok;
            float* stat = reinterpret_cast<float*>(stg + kOffStat);
            mbar_arrive_expect_tx(&bars->st_full[st], 2 * kStat);
            bulk_load(stat, p.lse + ix, kStat, &bars->st_full[st]);
            bulk_load(stat + kBN, p.delta + ix, kStat, &bars->st_full[st]);
          } else {
            // columns are keys: K in both layouts, V in the score layout
            if (rank == 0) mbar_arrive_expect_tx(&bars->kv_full[st], 2 * (2 * kBsTile + kBaTile));
            load_keys(stg + kOffB1s, kBsCh, 0, 2, it.kind, false, it.bh, c0 + 32 * (int)rank, 32, bar);
            load_keys(stg + kOffB2s, kBsCh, 0, 2, it.kind, true, it.bh, c0 + 32 * (int)rank, 32, bar);
            load_keys(stg + kOffB1a, 0, (int)rank, 1, it.kind, false, it.bh, c0, kBN, bar);
          }
        }
      }
      if (!ok) {
        // the copies this thread started signal the leader's barriers, which this CTA cannot
        // wait on; give them time to land before leaving
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 2000000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader CTA only)
    if (rank == 0 && lane == 0) {
      const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(&bars->tmem_base);
      constexpr uint32_t HI = desc_hi_sw128(1024);
      const uint32_t a1_lo = desc_lo(smem_addr(sA1), 16), a2_lo = desc_lo(smem_addr(sA2), 16);
      uint32_t n_items = 0, tile_it = 0, ct = 0;
      bool ok = true;
      auto wait = [&](uint64_t* bar, uint32_t par) -> bool {
        if (!mbar_wait_or_abort(bar, par, &bars->abort_flag)) {
          raise_abort(bars, p.err, kErrMma);
          ok = false;
          return false;
        }
        tc_fence_after();
        return true;
      };
      // D (256 x 64) = A (this CTA's 128 rows of each) * B^T (each CTA's 32 of the 64 columns)
      auto issue_score = [&](uint32_t d, uint32_t a_lo, uint32_t b_lo) {
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const uint32_t oa = (uint32_t)(((s / 4) * kACh + (s % 4) * 32) >> 4);
          const uint32_t ob = (uint32_t)(((s / 4) * kBsCh + (s % 4) * 32) >> 4);
          mma_ss_pair(d, a_lo + oa, b_lo + ob, HI, kIdescS, s > 0 ? 1u : 0u);
        }
      };
      // D (256 x 128) (+)= X (TMEM, 64 columns as bf16) * B (64 x each CTA's 64 of D, MN-major)
      auto issue_acc = [&](uint32_t d, uint32_t x_tmem, uint32_t b_lo, uint32_t acc) {
#pragma unroll
        for (int s = 0; s < kBN / 16; ++s)
          mma_ts_pair(d, x_tmem + s * 8, b_lo + (uint32_t)((s * 16 * 128) >> 4), HI, kIdescAcc,
                      (acc | (uint32_t)s) != 0 ? 1u : 0u);
      };
      const uint32_t t_s = tmem, t_t = tmem + 128, t_acc0 = tmem + 256, t_acc1 = tmem + 384;
      for (int g = pair; g < p.total && ok; g += npairs) {
        const Item it = decode_item<kDKDV>(p, g);
        if (it.c_end <= it.c_begin) continue;
        if (!wait(&bars->a_full, n_items & 1)) break;
        const uint32_t item_ix = n_items++;
        const int nc = it.c_end - it.c_begin;
        uint32_t prev_st = 0;
        for (int jj = 0; jj <= nc; ++jj) {
          if (jj < nc) {
            const uint32_t st = tile_it % kStages;
            if (!wait(&bars->kv_full[st], (tile_it / kStages) & 1)) break;
            const uint32_t base = smem_addr(sB + st * kStageBytes);
            const uint32_t bf = ct & 1;
            issue_score(t_s + bf * kBN, a1_lo, desc_lo(base + kOffB1s, 16));
            issue_score(t_t + bf * kBN, a2_lo, desc_lo(base + kOffB2s, 16));
            commit_pair(&bars->s_full[bf]);
            if (jj == nc - 1) commit_pair(&bars->a_empty);
          }
          if (jj > 0) {
            const uint32_t cp = ct - 1, bf = cp & 1;
            if (!wait(&bars->p_full[bf], (cp >> 1) & 1)) break;
            if (jj == 1 && item_ix > 0 && !wait(&bars->acc_empty, (item_ix - 1) & 1)) break;
            const uint32_t base = smem_addr(sB + prev_st * kStageBytes);
            const uint32_t acc = jj > 1 ? 1u : 0u;
            if constexpr (kDKDV) {
              issue_acc(t_acc0, t_s + bf * kBN, desc_lo(base + kOffB2a, (uint32_t)kBaTile), acc);  // dV += P^T dO
              issue_acc(t_acc1, t_t + bf * kBN, desc_lo(base + kOffB1a, (uint32_t)kBaTile), acc);  // dK += dS^T Q
            } else {
              issue_acc(t_acc0, t_t + bf * kBN, desc_lo(base + kOffB1a, (uint32_t)kBaTile), acc);  // dQ += dS K
            }
            commit_pair(&bars->kv_empty[prev_st]);
          }
          if (jj < nc) {
            prev_st = tile_it % kStages;
            ++tile_it;
            ++ct;
          }
        }
        if (!ok) break;
        commit_pair(&bars->acc_full);
      }
      // every MMA this thread issued completes before either CTA can release TMEM or leave
      commit_pair(&bars->drain);
      mbar_wait(&bars->drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ elementwise + epilogue (both CTAs)
    regs_alloc<kHighRegs>();
    const int w = (warp - 4) >> 2;  // warpgroup: the column tiles in S/T buffer w
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(&bars->tmem_base);
    const int wl = warp & 3;
    const int row = wl * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
    const uint32_t t_s = tmem + lane_off, t_t = tmem + lane_off + 128;
    const uint32_t t_acc0 = tmem + lane_off + 256, t_acc1 = tmem + lane_off + 384;
    const uint32_t p_full_l = map_to(&bars->p_full[0], 0);
    const uint32_t acc_empty_l = map_to(&bars->acc_empty, 0);
    uint32_t n_items = 0, tile_it = 0, ct = 0;
    bool ok = true;
    const uint64_t sc2 = pack2(p.scale_log2, p.scale_log2);
    for (int g = pair; g < p.total && ok; g += npairs) {
      const Item it = decode_item<kDKDV>(p, g);
      const int nc = it.c_end - it.c_begin;
      const float path_off = it.kind == 1 ? p.log2_b : 0.f;  // the Taylor exponents omit the weight b
      const int my = kBM * (int)rank + row;                  // this thread's row among the pair's 256
      const bool valid = my < it.rows;
      float l2r = 0.f, dr = 0.f;
      int tok_row = 0;
      if constexpr (!kDKDV) {
        tok_row = path_token(p, it.bh, it.kind, it.row0 + (valid ? my : 0));
        const size_t ix = (size_t)it.bh * p.N + tok_row;
        l2r = __ldg(p.lse + ix) * kLog2e - path_off;
        dr = __ldg(p.delta + ix);
      }
      const int ncols_valid = kDKDV ? 0 : (it.kind == 0 ? p.L_new : p.n_new);
      for (int jj = 0; jj < nc; ++jj, ++ct, ++tile_it) {
        const uint32_t bf = ct & 1;
        if ((int)bf != w) continue;  // the other warpgroup's tile
        if (!warp_wait(bars, &bars->s_full[bf], (ct >> 1) & 1, p.err)) { ok = false; break; }
        const uint32_t st = tile_it % kStages;
        if constexpr (kDKDV) {
          if (!warp_wait(bars, &bars->st_full[st], (tile_it / kStages) & 1, p.err)) { ok = false; break; }
        }
        if constexpr (kDKDV) {
          // in two halves of 32 columns (keys of this row against 32 queries each), so that
          // S, T, P and dS of only half a tile are live at a time
          const float* stat = reinterpret_cast<const float*>(sB + st * kStageBytes + kOffStat);
#pragma unroll 1
          for (int h2 = 0; h2 < 2; ++h2) {
            uint32_t s[32], t[32];
            tmem_ld32(t_s + bf * kBN + 32 * h2, s);
            tmem_ld32(t_t + bf * kBN + 32 * h2, t);
            tmem_ld_wait<32>(s);
            tmem_ld_wait<32>(t);
            uint32_t pw[16], dw[16];
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
              const float4 l4 = *reinterpret_cast<const float4*>(stat + 32 * h2 + 2 * i);
              const float4 d4 = *reinterpret_cast<const float4*>(stat + kBN + 32 * h2 + 2 * i);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int ii = i + h;
                const float la = h ? l4.z : l4.x, lb = h ? l4.w : l4.y;
                const float da = h ? d4.z : d4.x, db = h ? d4.w : d4.y;
                const uint64_t nl = pack2(path_off - la * kLog2e, path_off - lb * kLog2e);
                const uint64_t x =
                    ffma2(pack2(__uint_as_float(s[2 * ii]), __uint_as_float(s[2 * ii + 1])), sc2, nl);
                const float e0 = ex2_approx(lo2(x)), e1 = ex2_approx(hi2(x));
                const uint64_t ds = fmul2(pack2(e0, e1), fadd2(pack2(__uint_as_float(t[2 * ii]),
                                                                      __uint_as_float(t[2 * ii + 1])),
                                                                pack2(-da, -db)));
                pw[ii] = bf16x2(e0, e1);
                dw[ii] = bf16x2(lo2(ds), hi2(ds));
              }
            }
            // P over S's columns, dS over T's columns: bf16 pairs, 16 columns per half
            tmem_st16(t_s + bf * kBN + 16 * h2, pw);
            tmem_st16(t_t + bf * kBN + 16 * h2, dw);
          }
        } else {
          uint32_t s[kBN], t[kBN];
          tmem_ld32(t_s + bf * kBN, s);
          tmem_ld32(t_s + bf * kBN + 32, s + 32);
          tmem_ld32(t_t + bf * kBN, t);
          tmem_ld32(t_t + bf * kBN + 32, t + 32);
          tmem_ld_wait<kBN>(s);
          tmem_ld_wait<kBN>(t);
          uint32_t pw[kBN / 2], dw[kBN / 2];
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
            const uint64_t ds =
                fmul2(pack2(e0, e1), fadd2(pack2(__uint_as_float(t[2 * i]), __uint_as_float(t[2 * i + 1])), nd));
            pw[i] = bf16x2(e0, e1);
            dw[i] = bf16x2(lo2(ds), hi2(ds));
          }
          tmem_st32(t_s + bf * kBN, pw);
          tmem_st32(t_t + bf * kBN, dw);
        }
        tmem_st_wait();
        tc_fence_before();
        arrive_cluster(p_full_l + 8u * bf);
      }
      if (!ok) break;
      if (nc > 0) {
        if (!warp_wait(bars, &bars->acc_full, n_items & 1, p.err)) { ok = false; break; }
        ++n_items;
      }
      // ---------------------------------------------------------------- epilogue
      if constexpr (kDKDV) {
        const int r = it.row0 + my;  // row of K_new (exact) or pooled row (Taylor)
        const uint32_t t_acc = w == 0 ? t_acc0 : t_acc1;  // warpgroup 0: dV, warpgroup 1: dK
        const float scl = w == 0 ? 1.0f : p.inv_sqrt_d;
        if (it.kind == 1) {
          if (nc > 0) {
            float* dst = (w == 0 ? p.dvc : p.dkc) + ((size_t)it.bh * p.n_new + (valid ? r : 0)) * kD;
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
          }
        } else {
          int tok = -1;
          if (valid) {
            if (r < p.L_src) {
              tok = r;
            } else {
              const int rr = r - p.L_src;
              tok = p.L_src + __ldg(p.sel + (size_t)it.bh * p.k + rr / p.b) * p.b + rr % p.b;
            }
          }
          const int blk = (valid ? r : 0) / p.b;
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
        // dQ: warpgroup w writes features [64 w, 64 w + 64) of the row
        __nv_bfloat16* dq = static_cast<__nv_bfloat16*>(p.dq) + ((size_t)it.bh * p.N + tok_row) * kD;
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
        arrive_cluster(acc_empty_l);
      }
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

template <bool kDKDV>
cudaError_t launch_pair_t(const void* q, const void* k, const void* v, const void* dout, const Plan& pl,
                          const Work& w, PairBwdParams p, cudaStream_t s) {
  p.total = p.kind_split + pl.BH * p.items_t;
  if (p.total == 0) return cudaSuccess;
  CUtensorMap tq, tdo, tk, tv, tks, tvs, tkc, tvc;
  const bool has_sel = pl.k > 0;
  const int sel_rows = has_sel ? pl.k * pl.b : pl.N;
  const bool ok = make_map(&tq, q, 2, kD, pl.N, pl.BH, 32) && make_map(&tdo, dout, 2, kD, pl.N, pl.BH, 32) &&
                  make_map(&tk, k, 2, kD, pl.N, pl.BH, 32) && make_map(&tv, v, 2, kD, pl.N, pl.BH, 32) &&
                  make_map(&tks, has_sel ? w.ksel : k, 2, kD, sel_rows, pl.BH, 32) &&
                  make_map(&tvs, has_sel ? w.vsel : v, 2, kD, sel_rows, pl.BH, 32) &&
                  make_map(&tkc, w.kcn, 2, kD, pl.n_new, pl.BH, 32) &&
                  make_map(&tvc, w.vcn, 2, kD, pl.n_new, pl.BH, 32);
  if (!ok) return cudaErrorInvalidValue;
  auto kern = attention_bwd_pair_kernel<kDKDV>;
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidKernelImage;  // the register split needs this count
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc)) != cudaSuccess)
    return e;
  static int cached_pairs[64] = {0};
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
  kern<<<2 * pairs, kThreads, kSmemAlloc, s>>>(tq, tdo, tk, tv, tks, tvs, tkc, tvc, p);
  return cudaGetLastError();
}

}  // namespace

bool backward_pair_regs_ok() {
  static int cached[64] = {0};  // 0 unknown, 1 ok, 2 not ok
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!cached[dev]) {
    cudaFuncAttributes fa;
    const bool ok = cudaFuncGetAttributes(&fa, attention_bwd_pair_kernel<false>) == cudaSuccess &&
                    fa.numRegs == kLaunchRegs &&
                    cudaFuncGetAttributes(&fa, attention_bwd_pair_kernel<true>) == cudaSuccess &&
                    fa.numRegs == kLaunchRegs;
    cached[dev] = ok ? 1 : 2;
  }
  return cached[dev] == 1;
}

// dQ (both paths), dK/dV of the Taylor path (column ranges split, partial sums added
// atomically) and dK/dV of the exact path with the Taylor spread, on CTA pairs.
cudaError_t launch_backward_pair(const void* q, const void* k, const void* v, const void* dout, const Plan& pl,
                                 const Work& w, const float* lse, const float* delta, void* dq, void* dk, void* dv,
                                 float* dkc, float* dvc, cudaStream_t s) {
  PairBwdParams p{};
  p.route = w.route;
  p.sel = w.sel;
  p.lse = lse;
  p.delta = delta;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
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
  p.k = pl.k;
  p.scale_log2 = kLog2e / sqrtf((float)kD);
  p.inv_sqrt_d = 1.0f / sqrtf((float)kD);
  p.log2_b = log2f((float)pl.b);
  cudaError_t e;
  {
    PairBwdParams d = p;
    d.items_e = (pl.n_exact * pl.b + 2 * kBM - 1) / (2 * kBM);
    d.items_t = (pl.n_flat * pl.b + 2 * kBM - 1) / (2 * kBM);
    d.kind_split = pl.BH * d.items_e;
    d.chunks = 1;
    if ((e = launch_pair_t<false>(q, k, v, dout, pl, w, d, s)) != cudaSuccess) return e;
  }
  if (pl.n_flat > 0) {
    PairBwdParams d = p;
    d.dkc = dkc;
    d.dvc = dvc;
    d.items_e = 0;
    const int row_tiles = (pl.n_new + 2 * kBM - 1) / (2 * kBM);
    const int ncols = pl.n_flat * pl.b / kBN;
    int chunks = (device_sm_count() + pl.BH * row_tiles - 1) / (pl.BH * row_tiles);
    if (chunks > ncols) chunks = ncols;
    if (chunks < 1) chunks = 1;
    d.chunks = chunks;
    d.items_t = row_tiles * chunks;
    d.kind_split = 0;
    if ((e = launch_pair_t<true>(q, k, v, dout, pl, w, d, s)) != cudaSuccess) return e;
  }
  {
    PairBwdParams d = p;
    d.dkc = pl.n_flat > 0 ? dkc : nullptr;
    d.dvc = pl.n_flat > 0 ? dvc : nullptr;
    d.items_e = (pl.L_new + 2 * kBM - 1) / (2 * kBM);
    d.items_t = 0;
    d.kind_split = pl.BH * d.items_e;
    d.chunks = 1;
    if ((e = launch_pair_t<true>(q, k, v, dout, pl, w, d, s)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace isa
