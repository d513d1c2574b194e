// Stages 1-2 of In-context Sparse Attention in one launch: block-mean pooling
// of Q, K, V, the coarse score map over the source query blocks, its mean
// over the query axis on the context columns, and the per-head top-k of the
// context blocks.
//
// Method: "Lightning Unified Video Editing via In-Context Sparse Attention",
// papernotes.org notes, Key design 1 (Context Pre-Selection), and the
// paperlayer.ai summary, section 2 (Pooling Attention) and section 3
// (Pre-Selection):
//   Qc, Kc, Vc = means over blocks of b tokens (source blocks from token 0,
//     context blocks from token L_src; the last block of either part may be
//     short, and its mean is over its own tokens),
//   S_coarse[i, :] = softmax_j(Qc_i . Kc_j / sqrt(D)) for source blocks i,
//   score[c] = mean_i S_coarse[i, n_src + c],
//   sel = the k largest scores (ties by lower index), stored ascending.
//
// One persistent cooperative launch, one CTA per SM, 256 threads:
//  * phase 1 (HBM-bound): pooling units (head, block) are dealt round-robin to
//    the CTAs; each unit's Q, K and V blocks (b contiguous rows each, fewer in a
//    short last block) arrive in
//    a ring of shared-memory stages by 1-D TMA bulk copies, so several units
//    are in flight per SM while the previous one is reduced (fp32 sums, 4-byte
//    words, conflict-free shared-memory reads);
//  * a grid barrier (all block means written);
//  * phase 2: scoring items (head, 48 source rows, or 16 when n_q > 512) are
//    dealt round-robin; each computes its rows of S_coarse (CUDA cores, fp32;
//    the key blocks pass through shared memory in double-buffered chunks of
//    64), their softmax, and the
//    rows' sum on every context column, written as a partial. The last item of
//    a head to finish adds the partials in a fixed order (deterministic), then
//    runs the top-k as a shared-memory bitonic sort.
// Every wait is bounded and reports through the error word.
#include <cuda_bf16.h>
#include <float.h>

#include "block_sort.cuh"
#include "isa_internal.h"
#include "ptx.cuh"

namespace isa {
namespace {

// Up to this many context blocks the top-k splits by counted ranks (n comparisons per block),
// above it by a bitonic sort.
constexpr int kRankSplitMax = 512;

// 16-byte global -> shared copies that complete asynchronously (groups committed and awaited).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int n>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(n) : "memory"); }

constexpr int kThreads = 256;
constexpr int kKeys = 64;                  // pooled key blocks per shared-memory chunk in phase 2
constexpr int kGroups = kThreads / kKeys;  // phase-2 row groups (R / kGroups rows per thread)
// Source query blocks per scoring item: 48 (three items per head at the 32K-token workload, so
// all items run in one round) while the item's scores, 48 x n_q floats, fit in shared memory;
// 16 above that.
constexpr int kRowsLarge = 48;
constexpr int kRowsSmall = 16;
constexpr int kLargeMaxNq = 512;
static_assert(kRowsLarge % kGroups == 0 && kRowsSmall % kGroups == 0, "rows per group");
inline int rows_per_item(int n_q) { return n_q <= kLargeMaxNq ? kRowsLarge : kRowsSmall; }
constexpr int kStageBudget = 192 * 1024;   // shared memory for the phase-1 ring
constexpr int kMaxStages = 8;

template <typename T, int D, int BLK>
struct PoolCfg {
  static constexpr int E = sizeof(T);
  static constexpr int TENSOR_BYTES = BLK * D * E;          // one block of one tensor
  static constexpr int STAGE_BYTES = 3 * TENSOR_BYTES;
  static constexpr int STAGES = (kStageBudget / STAGE_BYTES) < kMaxStages ? (kStageBudget / STAGE_BYTES) : kMaxStages;
  static constexpr int WPR = D * E / 4;                     // 4-byte words per row
  static constexpr int RG = kThreads / WPR;                 // row groups
  static constexpr int FPW = 4 / E;                         // floats per word
  static constexpr int RED_FLOATS = 3 * RG * D;             // phase-1 reduction scratch
  static_assert(kThreads % WPR == 0 && BLK % RG == 0, "layout");
  static_assert(STAGES >= 2, "at least two stages");
};

int score_scratch_floats(const Plan& p, int D, int R) {
  const int P = next_pow2(p.n_ctx < 1 ? 1 : p.n_ctx);
  return R * D + 2 * kKeys * (D + 4) + R * p.n_q + p.n_ctx + 2 * P + next_pow2(p.k < 1 ? 1 : p.k);
}

template <typename T>
__device__ __forceinline__ void add_word(float* acc, uint32_t u);
template <>
__device__ __forceinline__ void add_word<__nv_bfloat16>(float* acc, uint32_t u) {
  acc[0] += __uint_as_float(u << 16);
  acc[1] += __uint_as_float(u & 0xffff0000u);
}
template <>
__device__ __forceinline__ void add_word<float>(float* acc, uint32_t u) {
  acc[0] += __uint_as_float(u);
}

__device__ __forceinline__ bool grid_barrier(uint32_t* counter, uint32_t* err) {
  __syncthreads();
  __shared__ int s_ok;
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(counter, 1u);
    const uint64_t t0 = global_timer_ns();
    int ok = 1;
    while (true) {
      uint32_t c;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(c) : "l"(counter) : "memory");
      if (c >= gridDim.x) break;
      if (global_timer_ns() - t0 > kWaitTimeoutNs) {
        atomicOr(err, kErrPool);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

template <typename T, int D, int BLK, int R>
__global__ void __launch_bounds__(kThreads, 1) pool_score_topk_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                                      const T* __restrict__ v, Plan p, Work w) {
  using C = PoolCfg<T, D, BLK>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  float* red = reinterpret_cast<float*>(full + kMaxStages);
  const int tid = threadIdx.x, G = gridDim.x, g = blockIdx.x;
  const int n_units = p.BH * p.n_q;
  const T* src[3] = {q, k, v};

  // ---- phase 1: block means --------------------------------------------------------
  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) mbar_init(&full[s], 1);
    mbar_fence_init();
  }
  __syncthreads();
  auto issue = [&](int u, int s) {  // thread 0: the three blocks of unit u into stage s
    const int bh = u / p.n_q, blk = u - bh * p.n_q;
    // a block's rows are contiguous; the last block of the source or the context part may
    // be short (its row count times D * E stays a multiple of 16 bytes)
    const size_t off = ((size_t)bh * p.N + (size_t)block_start(p, blk)) * D;
    const uint32_t bytes = (uint32_t)block_len(p, blk) * D * C::E;
    uint8_t* dst = smem + s * C::STAGE_BYTES;
    mbar_arrive_expect_tx(&full[s], 3 * bytes);
    for (int t = 0; t < 3; ++t) bulk_load(dst + t * C::TENSOR_BYTES, src[t] + off, bytes, &full[s]);
  };
  const int my_units = g < n_units ? (n_units - g + G - 1) / G : 0;
  int issued = 0;  // thread 0: units whose copies were started (unit i goes to stage i % STAGES)
  if (tid == 0)
    for (int i = 0; i < C::STAGES && i < my_units; ++i, ++issued) issue(g + i * G, i);
  const int wd = tid % C::WPR, rg = tid / C::WPR;
  bool ok = true;
  for (int i = 0; i < my_units; ++i) {
    const int s = i % C::STAGES, u = g + i * G;
    const int bh = u / p.n_q, blk = u - bh * p.n_q;
    int good = mbar_wait(&full[s], (i / C::STAGES) & 1) ? 1 : 0;
    if (!__syncthreads_and(good)) {
      if (tid == 0) atomicOr(&w.ctrl[kCtrlError], kErrPool);
      ok = false;
      break;
    }
    const uint32_t* base = reinterpret_cast<const uint32_t*>(smem + s * C::STAGE_BYTES);
    const int len = block_len(p, blk);  // rows of this block (BLK unless it is a short last block)
#pragma unroll
    for (int t = 0; t < 3; ++t) {
      float acc[C::FPW];
#pragma unroll
      for (int f = 0; f < C::FPW; ++f) acc[f] = 0.f;
      const uint32_t* tb = base + t * (C::TENSOR_BYTES / 4);
#pragma unroll 8
      for (int r = rg; r < len; r += C::RG) add_word<T>(acc, tb[r * C::WPR + wd]);
#pragma unroll
      for (int f = 0; f < C::FPW; ++f) red[(t * C::RG + rg) * D + wd * C::FPW + f] = acc[f];
    }
    __syncthreads();  // stage s fully read; partial sums in `red`
    if (tid == 0 && i + C::STAGES < my_units) {
      fence_proxy_async_smem();
      issue(g + (i + C::STAGES) * G, s);
      ++issued;
    }
    const float inv_len = 1.0f / (float)len;
    for (int e = tid; e < 3 * D; e += kThreads) {
      const int t = e / D, c = e - t * D;
      float sum = 0.f;
#pragma unroll
      for (int r = 0; r < C::RG; ++r) sum += red[(t * C::RG + r) * D + c];
      float* dst = (t == 0 ? w.qc : t == 1 ? w.kc : w.vc) + ((size_t)bh * p.n_q + blk) * D;
      dst[c] = sum * inv_len;
    }
    __syncthreads();  // `red` free for the next unit
  }
  if (!ok) {
    // let this CTA's outstanding copies land before leaving: wait for the last
    // phase armed on every stage
    if (tid == 0)
      for (int st = 0; st < C::STAGES && st < issued; ++st) {
        const int armed = (issued - st + C::STAGES - 1) / C::STAGES;
        mbar_wait(&full[st], (armed - 1) & 1);
      }
    return;
  }

  // ---- grid barrier: every block mean is written --------------------------------------
  if (!grid_barrier(&w.ctrl[kCtrlGridBarrier], &w.ctrl[kCtrlError])) return;

  // ---- phase 2: coarse scores, context-column partial sums, top-k ----------------------
  const int n_q = p.n_q, n_src = p.n_src, n_ctx = p.n_ctx;
  const int n_chunks = (n_src + R - 1) / R;
  constexpr int KS = D + 4;                         // key row stride: 4-word skew between rows
  float* qcs = reinterpret_cast<float*>(smem);      // [R][D]
  float* ks = qcs + R * D;                          // [2][kKeys][KS]: double-buffered key chunks
  float* lg = ks + 2 * kKeys * KS;                  // [R][n_q]
  float* cs = lg + R * n_q;                         // [n_ctx]
  const int P = next_pow2(n_ctx < 1 ? 1 : n_ctx);
  float* skey = cs + n_ctx;                         // [P]
  int32_t* sidx = reinterpret_cast<int32_t*>(skey + P);
  int32_t* ssel = sidx + P;
  const float scale = 1.0f / sqrtf((float)D);
  const int lane = tid & 31, warp = tid >> 5;
  __shared__ int s_last;
  for (int item = g; item < p.BH * n_chunks; item += G) {
    const int bh = item / n_chunks, chunk = item - bh * n_chunks;
    const int i0 = chunk * R, nr = min(R, n_src - i0);
    const float* Qc = w.qc + (size_t)bh * n_q * D;
    const float* Kc = w.kc + (size_t)bh * n_q * D;
    __syncthreads();
    for (int e = tid; e < R * (D / 4); e += kThreads) {
      const int r = e / (D / 4), d4 = e - r * (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < nr) v = __ldcg(reinterpret_cast<const float4*>(Qc + (size_t)(i0 + r) * D) + d4);
      *reinterpret_cast<float4*>(qcs + r * D + 4 * d4) = v;
    }
    // the key blocks pass through shared memory in chunks of kKeys, double-buffered: the next
    // chunk is copied (cp.async, 16 bytes a thread at a time) while this one is scored; thread
    // (key kj, row group rg) accumulates R / kGroups scores, summing over d in order
    constexpr int RPG = R / kGroups;
    const int kj = tid % kKeys, rg = tid / kKeys;
    const int n_kc = (n_q + kKeys - 1) / kKeys;
    auto stage_chunk = [&](int c) {
      float* dstb = ks + (c & 1) * kKeys * KS;
      const int j0 = c * kKeys;
      for (int e = tid; e < kKeys * (D / 4); e += kThreads) {
        const int jj = e / (D / 4), d4 = e - jj * (D / 4);
        if (j0 + jj < n_q) cp_async16(dstb + jj * KS + 4 * d4, Kc + (size_t)(j0 + jj) * D + 4 * d4);
      }
      cp_async_commit();
    };
    stage_chunk(0);
    for (int c = 0; c < n_kc; ++c) {
      if (c + 1 < n_kc) {
        stage_chunk(c + 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();  // chunk c (and, the first time, the query rows) visible to every thread
      float a[RPG];
#pragma unroll
      for (int r = 0; r < RPG; ++r) a[r] = 0.f;
      const float* kr = ks + (c & 1) * kKeys * KS + kj * KS;
#pragma unroll 4
      for (int d4 = 0; d4 < D / 4; ++d4) {
        const float4 kv = *reinterpret_cast<const float4*>(kr + 4 * d4);
#pragma unroll
        for (int r = 0; r < RPG; ++r) {
          const float4 qv = *reinterpret_cast<const float4*>(qcs + (rg * RPG + r) * D + 4 * d4);
          a[r] = fmaf(qv.x, kv.x, a[r]);
          a[r] = fmaf(qv.y, kv.y, a[r]);
          a[r] = fmaf(qv.z, kv.z, a[r]);
          a[r] = fmaf(qv.w, kv.w, a[r]);
        }
      }
      const int j = c * kKeys + kj;
      if (j < n_q) {
#pragma unroll
        for (int r = 0; r < RPG; ++r)
          if (rg * RPG + r < nr) lg[(rg * RPG + r) * n_q + j] = a[r] * scale;
      }
      __syncthreads();  // chunk c consumed: its buffer is refilled with chunk c + 2 next round
    }
    for (int r = warp; r < nr; r += kThreads / 32) {  // row softmax, one warp per row
      float* row = lg + r * n_q;
      float m = -FLT_MAX;
      for (int j = lane; j < n_q; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float sum = 0.f;
      for (int j = lane; j < n_q; j += 32) sum += expf(row[j] - m);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      const float inv = 1.0f / sum;
      __syncwarp();
      for (int c = lane; c < n_ctx; c += 32) row[n_src + c] = expf(row[n_src + c] - m) * inv;
    }
    __syncthreads();
    float* part = w.partial + ((size_t)bh * n_chunks + chunk) * n_ctx;
    for (int c = tid; c < n_ctx; c += kThreads) {
      float sum = 0.f;
      for (int r = 0; r < nr; ++r) sum += lg[r * n_q + n_src + c];
      part[c] = sum;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&w.ctr_pool[bh], 1u) == (unsigned)(n_chunks - 1));
    __syncthreads();
    if (!s_last) continue;
    __threadfence();
    // this head is complete: context scores in a fixed order, then the top-k
    const float inv_src = 1.0f / (float)n_src;
    for (int c = tid; c < P; c += kThreads) {
      if (c < n_ctx) {
        float sum = 0.f;
        for (int ch = 0; ch < n_chunks; ++ch) sum += __ldcg(w.partial + ((size_t)bh * n_chunks + ch) * n_ctx + c);
        const float sc = sum * inv_src;
        w.colscore[(size_t)bh * n_ctx + c] = sc;
        skey[c] = sc;
        sidx[c] = c;
      } else {
        skey[c] = -FLT_MAX;
        sidx[c] = 0x7fffffff - (c - n_ctx);
      }
    }
    const int kk = p.k;
    if (n_ctx <= kRankSplitMax) {
      // the kk best context blocks by counted ranks (ties to the lower index), ascending
      rank_split<true>(skey, n_ctx, kk, sidx, w.sel + (size_t)bh * kk, nullptr);
      continue;
    }
    bitonic_sort_pairs<true>(skey, sidx, P);
    if (kk > 0) {
      const int PK = next_pow2(kk);
      for (int i = tid; i < PK; i += kThreads) ssel[i] = i < kk ? sidx[i] : 0x7fffffff;
      bitonic_sort_int(ssel, PK);
      for (int i = tid; i < kk; i += kThreads) w.sel[(size_t)bh * kk + i] = ssel[i];
    }
  }
}

template <typename T, int D, int BLK, int R>
cudaError_t launch_r(const void* q, const void* k, const void* v, const Plan& p, const Work& w, cudaStream_t s) {
  using C = PoolCfg<T, D, BLK>;
  const size_t ring = (size_t)C::STAGES * C::STAGE_BYTES + sizeof(uint64_t) * kMaxStages + sizeof(float) * C::RED_FLOATS;
  const size_t score = sizeof(float) * (size_t)score_scratch_floats(p, D, R);
  const size_t smem = ring > score ? ring : score;
  auto kern = pool_score_topk_kernel<T, D, BLK, R>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  int grid = device_sm_count() * per_sm;
  // the grid barrier needs every CTA resident at once: cooperative launch guarantees it
  Plan pp = p;
  Work ww = w;
  const T* qq = static_cast<const T*>(q);
  const T* kk = static_cast<const T*>(k);
  const T* vv = static_cast<const T*>(v);
  void* args[] = {&qq, &kk, &vv, &pp, &ww};
  return cudaLaunchCooperativeKernel(reinterpret_cast<void*>(kern), dim3(grid), dim3(kThreads), args, smem, s);
}

template <typename T, int D, int BLK>
cudaError_t launch_t(const void* q, const void* k, const void* v, const Plan& p, const Work& w, cudaStream_t s) {
  return rows_per_item(p.n_q) == kRowsLarge ? launch_r<T, D, BLK, kRowsLarge>(q, k, v, p, w, s)
                                            : launch_r<T, D, BLK, kRowsSmall>(q, k, v, p, w, s);
}

}  // namespace

size_t pool_partial_floats(const Plan& p) {
  const int R = rows_per_item(p.n_q);
  return (size_t)p.BH * ((p.n_src + R - 1) / R) * p.n_ctx;
}

cudaError_t launch_pool_score_topk(const void* q, const void* k, const void* v, const Plan& p, const Work& w,
                                   cudaStream_t s) {
  if (p.dt == 0) {
    if (p.D == 128) return p.b == 128 ? launch_t<__nv_bfloat16, 128, 128>(q, k, v, p, w, s)
                                      : launch_t<__nv_bfloat16, 128, 64>(q, k, v, p, w, s);
    return p.b == 128 ? launch_t<__nv_bfloat16, 64, 128>(q, k, v, p, w, s)
                      : launch_t<__nv_bfloat16, 64, 64>(q, k, v, p, w, s);
  }
  if (p.D != 64) return cudaErrorNotSupported;  // float32 inputs are supported with D = 64 only
  return p.b == 128 ? launch_t<float, 64, 128>(q, k, v, p, w, s) : launch_t<float, 64, 64>(q, k, v, p, w, s);
}

}  // namespace isa
