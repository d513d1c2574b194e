// Taylor query blocks with exactly computed key blocks (the no-sparsity ratio alpha_ns > 0) for
// bf16 inputs with D = 128 and b = 128, on one CTA per SM with split-K over two warpgroups.
//
// Method: "Lightning Unified Video Editing via In-Context Sparse Attention", papernotes.org
// notes, Key designs 2 and 3: inside a flat (Taylor) query block i, the k_ns = ceil(alpha_ns *
// n_new) key blocks of K_new with the largest coarse scores are computed key by key
// (S = q K_j^T / sqrt(D), l += rowsum(P), O += P V_j), every other block through its pooled
// row with its length as weight (l += P^c * b, O += P^c Vc_j * b), one softmax over both kinds
// of terms. The blocks of each query block were chosen by the routing kernel (its ascending
// list `nsel` and bitmask `nsmask`).
//
// Why this design. A Taylor query block's key set is its own: the pooled rows (its own exact
// blocks masked) and its k_ns exact blocks, which neighbouring query blocks share only in part
// (about 13 % at the 32K-token workload). So a 128-row query tile cannot share its key tiles
// with another tile, and one tile's chain of S MMA -> softmax -> P V MMA would leave the tensor
// core idle most of the time. Here both softmax warpgroups work on the SAME query tile: the
// item's key tiles (pooled tiles first, then the exact blocks in ascending order) alternate
// between them, each warpgroup keeps its own running maximum, sum and O accumulator, and at
// the end of the item warpgroup 0 merges the two softmax states:
//   O = (O_0 2^(m_0 - M) + O_1 2^(m_1 - M)) / (l_0 2^(m_0 - M) + l_1 2^(m_1 - M)), M = max(m_0, m_1).
// While one warpgroup exponentiates its tile, the tensor core runs the other's S and P V.
// TMEM: S_0 [0, 128), S_1 [128, 256), O_0 [256, 384), O_1 [384, 512). K and V of a key tile
// share one stage of a 3-stage ring. Every wait is bounded.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <float.h>

#include "exp2_poly.cuh"
#include "isa_internal.h"
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
constexpr int kB = 128;        // block size (one query block = one 128-row tile)
constexpr int kBN = 128;       // keys per K/V tile
constexpr int kCols = 128;     // scores per softmax thread and tile
constexpr int kStages = 3;
constexpr int kTile = 128 * kD * 2;   // 32 KB
constexpr int kCh = 128 * 128;        // bytes between the two 128-byte chunks of a tile
constexpr uint32_t kIdescQK = umma_idesc(1u, 128, kBN, 0, 0);
constexpr uint32_t kIdescPV = umma_idesc(1u, 128, kD, 0, 1);
constexpr float kRescaleThreshold = 8.0f;
constexpr int kRing = 4;  // work items published ahead by the producer

struct MixParams {
  const int32_t* route;    // [BH, n_q]: exact blocks, then Taylor blocks
  const int32_t* nsel;     // [BH, n_q, k_ns]: each query block's exact K_new blocks, ascending
  const uint32_t* nsmask;  // [BH, n_q, ns_words]: the same as a bitmask over K_new's blocks
  void* out;
  uint32_t* err;
  uint32_t* next;          // per-call work counter (zeroed with the control words)
  int BH, N, n_q, n_src, n_exact, n_flat, n_new, k_ns, ns_words, npt;
  float scale_log2;
  float bias_log2;         // log2(b): a pooled row's weight b in the exponent
};

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t o_free;         // warpgroup 0 has read both O accumulators of the item (128 arrivals)
  uint64_t st_full;        // warpgroup 1 has written m1, l1 of the item (128 arrivals)
  uint64_t st_read;        // warpgroup 0 has read them (128 arrivals)
  uint64_t drain;
  uint64_t item_full[kRing];  // the producer has published the item in the slot
  uint64_t item_free[kRing];  // the issuer (1) and the softmax threads (256) have read it
  int item_ring[kRing];       // item index, or -1 past the last
  uint32_t tmem_base;
  int abort_flag;
  float m1[128], l1[128];  // warpgroup 1's softmax state per row, for the merge
};

constexpr int kOffQ = 0;
constexpr int kOffKV = kTile;  // stage s: K at kOffKV + s * 2 * kTile, V right after it
constexpr int kOffBar = kOffKV + kStages * 2 * kTile;
constexpr int kSmemAlloc = kOffBar + (int)sizeof(Bars) + 1024;
static_assert(kSmemAlloc <= 227 * 1024, "shared memory");

struct Item {
  int bh, blk, nkv;
};
__device__ __forceinline__ Item decode_item(const MixParams& p, int g) {
  Item it;
  it.bh = g / p.n_flat;
  it.blk = __ldg(p.route + (size_t)it.bh * p.n_q + p.n_exact + (g - it.bh * p.n_flat));
  it.nkv = p.npt + p.k_ns;
  return it;
}
// K_new block of key tile j >= npt of the item
__device__ __forceinline__ int exact_block(const MixParams& p, const Item& it, int j) {
  return __ldg(p.nsel + ((size_t)it.bh * p.n_q + it.blk) * p.k_ns + (j - p.npt));
}

__device__ __forceinline__ bool aborted(const Bars* b) {
  return *reinterpret_cast<const volatile int*>(&b->abort_flag) != 0;
}
__device__ __noinline__ void raise_abort(Bars* b, uint32_t* err, uint32_t code) {
  atomicOr(err, code);
  *reinterpret_cast<volatile int*>(&b->abort_flag) = 1;
}
__device__ __forceinline__ bool warp_wait(Bars* b, uint64_t* bar, uint32_t parity, uint32_t* err) {
  bool ok = mbar_wait_or_abort(bar, parity, &b->abort_flag);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && (threadIdx.x & 31) == 0) raise_abort(b, err, kErrSoftmax);
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

__global__ void __launch_bounds__(kThreads, 1)
    attention_mixed_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_ksel, const __grid_constant__ CUtensorMap tm_v,
                           const __grid_constant__ CUtensorMap tm_vsel, const __grid_constant__ CUtensorMap tm_kcn,
                           const __grid_constant__ CUtensorMap tm_vcn, const MixParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sKV = smem + kOffKV;
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = p.BH * p.n_flat;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bars->s_full[w], 1);
      mbar_init(&bars->p_full[w], 128);
      mbar_init(&bars->o_done[w], 1);
    }
    mbar_init(&bars->o_free, 128);
    mbar_init(&bars->st_full, 128);
    mbar_init(&bars->st_read, 128);
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
      uint32_t n_items = 0, kv_it = 0;
      bool ok = true;
      // Items come from a per-call counter (a CTA that starts late, on an SM freed late by the
      // kernel before, takes fewer), published to the other roles through the ring.
      for (uint32_t n = 0; ok; ++n, ++n_items) {
        const uint32_t slot = n % kRing;
        if (n >= kRing && !mbar_wait(&bars->item_free[slot], ((n / kRing) - 1) & 1)) {
          raise_abort(bars, p.err, kErrProducer);
          ok = false;
          break;
        }
        int g = (int)atomicAdd(p.next, 1u);
        if (g >= total) g = -1;
        *reinterpret_cast<volatile int*>(&bars->item_ring[slot]) = g;
        mbar_arrive(&bars->item_full[slot]);
        if (g < 0) break;
        const Item it = decode_item(p, g);
        if (n_items > 0 && !mbar_wait(&bars->q_empty, (n_items - 1) & 1)) {
          raise_abort(bars, p.err, kErrProducer);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bars->q_full, kTile);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int c = 0; c < 2; ++c)
            tma_load_3d(sQ + c * kCh + h * 8192, &tm_q, &bars->q_full, c * 64, it.blk * kB + 64 * h, it.bh);
        for (int j = 0; j < it.nkv && ok; ++j, ++kv_it) {
          if (aborted(bars)) { ok = false; break; }
          const int st = kv_it % kStages;
          if (!mbar_wait(&bars->kv_empty[st], ((kv_it / kStages) & 1) ^ 1)) {
            raise_abort(bars, p.err, kErrProducer);
            ok = false;
            break;
          }
          const CUtensorMap *mk, *mv;
          int y;
          if (j < p.npt) {  // pooled rows of K_new (rows past n_new read as zeros, masked)
            mk = &tm_kcn;
            mv = &tm_vcn;
            y = j * kBN;
          } else {  // an exact block of K_new: a source block in place, or a gathered context block
            const int e = exact_block(p, it, j);
            if (e < p.n_src) {
              mk = &tm_k;
              mv = &tm_v;
              y = e * kB;
            } else {
              mk = &tm_ksel;
              mv = &tm_vsel;
              y = (e - p.n_src) * kB;
            }
          }
          uint8_t* sK = sKV + st * 2 * kTile;
          uint8_t* sV = sK + kTile;
          mbar_arrive_expect_tx(&bars->kv_full[st], 2 * kTile);
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              tma_load_3d(sK + c * kCh + h * 8192, mk, &bars->kv_full[st], c * 64, y + 64 * h, it.bh);
              tma_load_3d(sV + c * kCh + h * 8192, mv, &bars->kv_full[st], c * 64, y + 64 * h, it.bh);
            }
        }
      }
      if (!ok) {
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
      const uint32_t q_lo = desc_lo(smem_addr(sQ), 16);
      uint32_t n_items = 0, kv_it = 0;
      uint32_t pv_par = 0;  // bit w: parity of the number of P V groups issued for warpgroup w
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
      // S_w = Q K^T for the K tile of stage st
      auto issue_s = [&](int w, uint32_t st) {
        const uint32_t k_lo = desc_lo(smem_addr(sKV + st * 2 * kTile), 16);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const uint32_t off = (uint32_t)(((s / 4) * kCh + (s % 4) * 32) >> 4);
          umma_ss_lo_warp<false>(tmem + 128 * w, q_lo + off, k_lo + off, HI, kIdescQK, s > 0 ? 1u : 0u);
        }
        umma_commit_warp(&bars->s_full[w]);
      };
      // O_w (+)= P_w V for the V tile of stage st
      auto issue_pv = [&](int w, uint32_t st, uint32_t acc) {
        const uint32_t v_lo = desc_lo(smem_addr(sKV + st * 2 * kTile + kTile), (uint32_t)kCh);
#pragma unroll
        for (int s = 0; s < kBN / 16; ++s)
          umma_ts_lo_warp<false>(tmem + 256 + 128 * w, tmem + 128 * w + s * 8, v_lo + (uint32_t)((s * 16 * 128) >> 4), HI,
                            kIdescPV, (acc | (uint32_t)s) != 0 ? 1u : 0u);
        umma_commit_warp(&bars->o_done[w]);
        pv_par ^= 1u << w;
      };
      for (uint32_t n = 0; ok; ++n, ++n_items) {
        const uint32_t slot = n % kRing;
        if (!wait(&bars->item_full[slot], (n / kRing) & 1)) break;
        const int g = __shfl_sync(0xffffffffu, *reinterpret_cast<volatile int*>(&bars->item_ring[slot]), 0);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->item_free[slot]);
        if (g < 0) break;
        const Item it = decode_item(p, g);
        if (!wait(&bars->q_full, n_items & 1)) break;
        // S of the first two key tiles (one per warpgroup)
        for (int j = 0; j < 2 && j < it.nkv; ++j) {
          const uint32_t idx = kv_it + j, st = idx % kStages;
          if (!wait(&bars->kv_full[st], (idx / kStages) & 1)) break;
          issue_s(j & 1, st);
          if (j == it.nkv - 1) umma_commit_warp(&bars->q_empty);
        }
        if (!ok) break;
        // the O accumulators of the previous item have been read by the merge
        if (n_items > 0 && !wait(&bars->o_free, (n_items - 1) & 1)) break;
        for (int j = 0; j < it.nkv; ++j) {
          const int w = j & 1;
          const uint32_t idx = kv_it + j, st = idx % kStages;
          // P V of tile j once its P is written, then S of tile j + 2 into the buffer it read
          if (!wait(&bars->p_full[w], (pv_par >> w) & 1u)) break;
          issue_pv(w, st, j >= 2 ? 1u : 0u);
          umma_commit_warp(&bars->kv_empty[st]);
          if (j + 2 < it.nkv) {
            const uint32_t idx2 = idx + 2, st2 = idx2 % kStages;
            if (!wait(&bars->kv_full[st2], (idx2 / kStages) & 1)) break;
            issue_s(w, st2);
            if (j + 3 == it.nkv) umma_commit_warp(&bars->q_empty);
          }
        }
        kv_it += it.nkv;
      }
      umma_commit_warp(&bars->drain);
      mbar_wait(&bars->drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax (two warpgroups) + merge
    regs_alloc<kHighRegs>();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(&bars->tmem_base);
    const int w = (warp - 4) >> 2;  // warpgroup: key tiles j with j % 2 == w
    const int wl = warp & 3;
    const int row = wl * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
    const uint32_t t_s = tmem + lane_off + 128 * w;
    const uint32_t t_o = tmem + lane_off + 256 + 128 * w;
    uint32_t n_items = 0, s_cnt = 0, pv_cnt = 0, pv_all[2] = {0, 0};
    bool ok = true;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
    constexpr uint32_t kNegInf = 0xff800000u;
    for (uint32_t n = 0; ok; ++n, ++n_items) {
      const uint32_t slot = n % kRing;
      if (!warp_wait(bars, &bars->item_full[slot], (n / kRing) & 1, p.err)) { ok = false; break; }
      const int g = *reinterpret_cast<volatile int*>(&bars->item_ring[slot]);
      mbar_arrive(&bars->item_free[slot]);
      if (g < 0) break;
      const Item it = decode_item(p, g);
      const uint32_t* own = p.nsmask + ((size_t)it.bh * p.n_q + it.blk) * p.ns_words;
      float m = -INFINITY, l = 0.f;
      int nmine = 0;
      for (int j = w; j < it.nkv; j += 2, ++nmine) {
        if (!warp_wait(bars, &bars->s_full[w], s_cnt & 1, p.err)) { ok = false; break; }
        ++s_cnt;
        uint32_t r[kCols];
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) tmem_ld32(t_s + 32 * c, r + 32 * c);
        tmem_ld_wait<kCols>(r);
        float bias = 0.f;  // log2 of the weight of this tile's keys
        if (j < p.npt) {
          // pooled rows: weight b, the row's own exact blocks and the rows past n_new masked
          bias = p.bias_log2;
          const int lim = min(kBN, p.n_new - j * kBN);
#pragma unroll
          for (int c = 0; c < kCols / 32; ++c) {
            const int wd = (kCols / 32) * j + c;
            const uint32_t mw = wd < p.ns_words ? __ldg(own + wd) : 0u;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              r[32 * c + i] = (((mw >> i) & 1u) != 0u || 32 * c + i >= lim) ? kNegInf : r[32 * c + i];
          }
        }
        float mc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) mc[c] = __uint_as_float(r[c]);
#pragma unroll
        for (int i = 8; i < kCols; i += 16) {
#pragma unroll
          for (int c = 0; c < 8; ++c) mc[c] = fmax3(mc[c], __uint_as_float(r[i + c]), __uint_as_float(r[i + 8 + c]));
        }
        const float raw_max =
            fmaxf(fmax3(mc[0], mc[1], mc[2]), fmax3(fmax3(mc[3], mc[4], mc[5]), mc[6], mc[7]));
        const float mx = raw_max * p.scale_log2 + bias;
        // lazy maximum: it moves only when the tile's maximum exceeds it by more than 2^8
        const bool need = (nmine > 0) && (mx > m + kRescaleThreshold);
        const float alpha = need ? ex2_approx(m - mx) : 1.0f;
        if (nmine == 0 || need) m = mx;
        if (__any_sync(0xffffffffu, need)) {
          // O_w holds P V up to this warpgroup's previous tile: complete before it is rescaled
          if (!warp_wait(bars, &bars->o_done[w], (pv_cnt - 1) & 1, p.err)) { ok = false; break; }
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
        // a row with no unmasked key yet has m = -inf: its p are 0 (offset 0, scores -inf)
        const float nm = (m == -INFINITY) ? 0.f : bias - m;
        // the tile's largest p enters the row sum as its bf16 value when it exceeds 1 (the P V
        // MMA multiplies the bf16 p; with the lazy maximum the dominant keys' p lie in (1, 2^8])
        float corr = 0.f;
        if (mx > m) {
          const float em = ex2_approx(fmaf(raw_max, p.scale_log2, nm));
          corr = __bfloat162float(__float2bfloat16_rn(em)) - em;
        }
        const uint64_t sc2 = pack2(p.scale_log2, p.scale_log2), nm2 = pack2(nm, nm);
        uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < kCols / 2; ++i) {
          const uint64_t x = ffma2(static_cast<uint64_t>(r[2 * i]) | (static_cast<uint64_t>(r[2 * i + 1]) << 32), sc2,
                                   nm2);
          const uint64_t e = pack2(ex2_approx(lo2(x)), ex2_approx(hi2(x)));
          acc[i & 3] = fadd2(acc[i & 3], e);
          __nv_bfloat162 hv = __floats2bfloat162_rn(lo2(e), hi2(e));
          r[i] = *reinterpret_cast<uint32_t*>(&hv);
        }
#pragma unroll
        for (int c = 0; c < kCols / 64; ++c) tmem_st32(t_s + 32 * c, r + 32 * c);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_full[w]);
        ++pv_cnt;
        const uint64_t a2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
        l = l * alpha + ((lo2(a2) + hi2(a2)) + corr);
      }
      if (!ok) break;
      // ---------------------------------------------------------------- merge of the two states
      // (the handshakes between the warpgroups are bounded mbarrier waits, so that one that gave
      // up cannot leave the other waiting)
      pv_all[w] += (uint32_t)nmine;
      const int n1 = it.nkv / 2;  // tiles of warpgroup 1 in this item
      pv_all[1 - w] += (uint32_t)((w == 0) ? n1 : it.nkv - n1);
      if (w == 1) {
        // m1, l1 of the previous item have been read
        if (n_items > 0 && !warp_wait(bars, &bars->st_read, (n_items - 1) & 1, p.err)) { ok = false; break; }
        bars->m1[row] = m;
        bars->l1[row] = l;
        mbar_arrive(&bars->st_full);
      } else {
        if (!warp_wait(bars, &bars->st_full, n_items & 1, p.err)) { ok = false; break; }
        const float m1 = bars->m1[row], l1 = bars->l1[row];
        mbar_arrive(&bars->st_read);
        // the last P V of each warpgroup (and so every earlier one) is complete
        if (!warp_wait(bars, &bars->o_done[0], (pv_all[0] - 1) & 1, p.err)) { ok = false; break; }
        if (n1 > 0 && !warp_wait(bars, &bars->o_done[1], (pv_all[1] - 1) & 1, p.err)) { ok = false; break; }
        const float M = fmaxf(m, m1);
        const float a0 = (m == -INFINITY) ? 0.f : ex2_approx(m - M);
        const float a1 = (n1 == 0 || m1 == -INFINITY) ? 0.f : ex2_approx(m1 - M);
        const float inv = 1.0f / (l * a0 + l1 * a1);
        const float c0 = a0 * inv, c1 = a1 * inv;
        __nv_bfloat16* dst = out + ((size_t)it.bh * p.N + (size_t)it.blk * kB + row) * kD;
        const uint32_t t_o0 = tmem + lane_off + 256, t_o1 = tmem + lane_off + 384;
#pragma unroll 1
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t o0[32], o1[32];
          tmem_ld32(t_o0 + 32 * c, o0);
          tmem_ld32(t_o1 + 32 * c, o1);
          tmem_ld_wait<32>(o0);
          tmem_ld_wait<32>(o1);
          float f[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            f[i] = __uint_as_float(o0[i]) * c0 + (n1 > 0 ? __uint_as_float(o1[i]) * c1 : 0.f);
          store_row_chunk(dst + 32 * c, f);
        }
        tc_fence_before();
        mbar_arrive(&bars->o_free);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(*reinterpret_cast<volatile uint32_t*>(&bars->tmem_base), 512);
  }
  // This grid may start before the attention kernel launched ahead of it has finished (it takes
  // the SMs that kernel frees); it does not read that kernel's output, but it finishes only after
  // it, so that stream order holds for the work after both.
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace

bool attention_mixed_supported(const Plan& p) {
  return p.dt == 0 && p.D == kD && p.b == kB && !p.ragged && p.k_ns > 0;
}

cudaError_t launch_attention_mixed(const void* q, const void* k, const void* v, void* out, const Plan& pl,
                                   const Work& w, cudaStream_t s) {
  MixParams p{};
  p.route = w.route;
  p.nsel = w.nsel;
  p.nsmask = w.nsmask;
  p.out = out;
  p.err = w.ctrl;
  p.next = w.ctrl + kCtrlMixedNext;
  p.BH = pl.BH;
  p.N = pl.N;
  p.n_q = pl.n_q;
  p.n_src = pl.n_src;
  p.n_exact = pl.n_exact;
  p.n_flat = pl.n_flat;
  p.n_new = pl.n_new;
  p.k_ns = pl.k_ns;
  p.ns_words = pl.ns_words;
  p.npt = (pl.n_new + kBN - 1) / kBN;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
  p.bias_log2 = log2f((float)pl.b);
  const int total = pl.BH * pl.n_flat;
  if (total == 0) return cudaSuccess;
  CUtensorMap tq, tk, tks, tv, tvs, tkc, tvc;
  const bool has_sel = pl.k > 0;
  const int sel_rows = has_sel ? pl.k * pl.b : pl.N;
  const bool ok = make_map(&tq, q, 2, kD, pl.N, pl.BH, 64) && make_map(&tk, k, 2, kD, pl.N, pl.BH, 64) &&
                  make_map(&tks, has_sel ? w.ksel : k, 2, kD, sel_rows, pl.BH, 64) &&
                  make_map(&tv, v, 2, kD, pl.N, pl.BH, 64) &&
                  make_map(&tvs, has_sel ? w.vsel : v, 2, kD, sel_rows, pl.BH, 64) &&
                  make_map(&tkc, w.kcn, 2, kD, pl.n_new, pl.BH, 64) &&
                  make_map(&tvc, w.vcn, 2, kD, pl.n_new, pl.BH, 64);
  if (!ok) return cudaErrorInvalidValue;
  auto kern = attention_mixed_kernel;
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidKernelImage;  // the register split needs this count
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc)) != cudaSuccess)
    return e;
  int grid = device_sm_count();
  if (grid > total) grid = total;
  // Programmatic dependent launch: the CTAs may start on the SMs the preceding attention kernel
  // frees (that kernel allows it at its start) instead of after its last CTA.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemAlloc;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tq, tk, tks, tv, tvs, tkc, tvc, p);
}

}  // namespace isa
