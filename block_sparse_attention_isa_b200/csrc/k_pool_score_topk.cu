// Stages 1-2 of In-context Sparse Attention in one launch: block-mean pooling
// of Q, K, V, the coarse score map over the source query blocks, its mean
// over the query axis on the context columns, and the per-head top-k of the
// context blocks.
//
// Method: "Lightning Unified Video Editing via In-Context Sparse Attention",
// papernotes.org notes, Key design 1 (Context Pre-Selection), and the
// paperlayer.ai summary, section 2 (Pooling Attention) and section 3
// (Pre-Selection).
//
// Grid (n_q, B*H), 256 threads. Each CTA pools one block of b tokens of Q, K
// and V with 16-byte vector loads (all loads of a thread issued before any
// use, fp32 sums). The last CTA to finish a head (atomic counter after a
// __threadfence) then scores that head:
//   S_coarse[i, :] = softmax_j(Qc_i . Kc_j / sqrt(D)) for source blocks i,
//   score[c] = mean_i S_coarse[i, n_src + c],
//   sel = the k largest scores (ties by lower index), stored ascending.
// Work per head is n_src * n_q * D multiply-adds on the CUDA cores; the pooling
// pass itself is bound by HBM (it reads Q, K and V once).
#include <cuda_bf16.h>
#include <float.h>

#include "block_sort.cuh"
#include "isa_internal.h"

namespace isa {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerChunk = 8;  // source query blocks scored per pass

template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ static void add(float* acc, const uint4& u) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  }
};
template <>
struct Vec16<float> {
  static constexpr int n = 4;
  __device__ static void add(float* acc, const uint4& u) {
    acc[0] += __uint_as_float(u.x);
    acc[1] += __uint_as_float(u.y);
    acc[2] += __uint_as_float(u.z);
    acc[3] += __uint_as_float(u.w);
  }
};

template <int D>
size_t score_smem_bytes(const Plan& p) {
  const int P = next_pow2(p.n_ctx < 1 ? 1 : p.n_ctx);
  return sizeof(float) * (size_t)(kRowsPerChunk * D + kRowsPerChunk * p.n_q + p.n_ctx) +
         (sizeof(float) + sizeof(int32_t)) * (size_t)P + sizeof(int32_t) * (size_t)next_pow2(p.k < 1 ? 1 : p.k);
}

template <typename T, int D, int BLK>
__global__ void __launch_bounds__(kThreads) pool_score_topk_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                                   const T* __restrict__ v, Plan p, Work w) {
  extern __shared__ __align__(16) float smem[];
  constexpr int VEC = Vec16<T>::n;
  constexpr int TPR = D / VEC;           // threads per row
  constexpr int RPP = kThreads / TPR;    // rows per pass
  constexpr int PASSES = BLK / RPP;
  static_assert(BLK % RPP == 0, "block size must be a multiple of the rows per pass");

  const int blk = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int col0 = (tid % TPR) * VEC, r0 = tid / TPR;
  const size_t base = ((size_t)bh * p.N + (size_t)blk * BLK) * D + col0;

  // ---- stage 1a: block means of Q, K, V ---------------------------------------------
  float acc[3][VEC];
#pragma unroll
  for (int t = 0; t < 3; ++t)
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[t][i] = 0.f;
  {
    uint4 buf[3][PASSES];
#pragma unroll
    for (int s = 0; s < PASSES; ++s) {
      const size_t off = base + (size_t)(r0 + s * RPP) * D;
      buf[0][s] = __ldcs(reinterpret_cast<const uint4*>(q + off));
      buf[1][s] = __ldcs(reinterpret_cast<const uint4*>(k + off));
      buf[2][s] = __ldcs(reinterpret_cast<const uint4*>(v + off));
    }
#pragma unroll
    for (int s = 0; s < PASSES; ++s)
#pragma unroll
      for (int t = 0; t < 3; ++t) Vec16<T>::add(acc[t], buf[t][s]);
  }
  float* red = smem;  // [3][RPP][D]
#pragma unroll
  for (int t = 0; t < 3; ++t)
#pragma unroll
    for (int i = 0; i < VEC; ++i) red[(t * RPP + r0) * D + col0 + i] = acc[t][i];
  __syncthreads();
  const float inv_b = 1.0f / (float)BLK;
  for (int e = tid; e < 3 * D; e += kThreads) {
    const int t = e / D, c = e % D;
    float s = 0.f;
#pragma unroll 4
    for (int r = 0; r < RPP; ++r) s += red[(t * RPP + r) * D + c];
    float* dst = (t == 0 ? w.qc : t == 1 ? w.kc : w.vc) + ((size_t)bh * p.n_q + blk) * D;
    dst[c] = s * inv_b;
  }

  // ---- last CTA of this head scores it ----------------------------------------------
  __shared__ int s_last;
  __threadfence();  // make this thread's block means visible device-wide before the count
  __syncthreads();
  if (tid == 0) {
    const unsigned prev = atomicAdd(&w.ctr_pool[bh], 1u);
    s_last = (prev == (unsigned)(p.n_q - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  const int n_q = p.n_q, n_src = p.n_src, n_ctx = p.n_ctx;
  float* qcs = smem;                              // [R][D]
  float* lg = qcs + kRowsPerChunk * D;            // [R][n_q]
  float* cs = lg + kRowsPerChunk * n_q;           // [n_ctx]
  const int P = next_pow2(n_ctx < 1 ? 1 : n_ctx);
  float* skey = cs + n_ctx;                       // [P]
  int32_t* sidx = reinterpret_cast<int32_t*>(skey + P);  // [P]
  int32_t* ssel = sidx + P;                       // [next_pow2(k)]
  const float* Qc = w.qc + (size_t)bh * n_q * D;
  const float* Kc = w.kc + (size_t)bh * n_q * D;
  const float scale = 1.0f / sqrtf((float)D);
  const int lane = tid & 31, warp = tid >> 5;

  for (int c = tid; c < n_ctx; c += kThreads) cs[c] = 0.f;
  for (int i0 = 0; i0 < n_src; i0 += kRowsPerChunk) {
    const int nr = min(kRowsPerChunk, n_src - i0);
    __syncthreads();
    for (int e = tid; e < kRowsPerChunk * D; e += kThreads) {
      const int r = e / D;
      qcs[e] = r < nr ? __ldcg(Qc + (size_t)(i0 + r) * D + (e % D)) : 0.f;
    }
    __syncthreads();
    for (int j = tid; j < n_q; j += kThreads) {
      float a[kRowsPerChunk];
#pragma unroll
      for (int r = 0; r < kRowsPerChunk; ++r) a[r] = 0.f;
      const float4* kr = reinterpret_cast<const float4*>(Kc + (size_t)j * D);
#pragma unroll 4
      for (int d4 = 0; d4 < D / 4; ++d4) {
        const float4 kv = __ldcg(kr + d4);
#pragma unroll
        for (int r = 0; r < kRowsPerChunk; ++r) {
          const float4 qv = *reinterpret_cast<const float4*>(qcs + r * D + 4 * d4);
          a[r] = fmaf(qv.x, kv.x, a[r]);
          a[r] = fmaf(qv.y, kv.y, a[r]);
          a[r] = fmaf(qv.z, kv.z, a[r]);
          a[r] = fmaf(qv.w, kv.w, a[r]);
        }
      }
#pragma unroll
      for (int r = 0; r < kRowsPerChunk; ++r)
        if (r < nr) lg[r * n_q + j] = a[r] * scale;
    }
    __syncthreads();
    // row softmax, one warp per row; only the context columns are kept
    for (int r = warp; r < nr; r += kThreads / 32) {
      float* row = lg + r * n_q;
      float m = -FLT_MAX;
      for (int j = lane; j < n_q; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float s = 0.f;
      for (int j = lane; j < n_q; j += 32) s += expf(row[j] - m);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const float inv = 1.0f / s;
      __syncwarp();
      for (int c = lane; c < n_ctx; c += 32) row[n_src + c] = expf(row[n_src + c] - m) * inv;
    }
    __syncthreads();
    for (int c = tid; c < n_ctx; c += kThreads) {
      float s = cs[c];
      for (int r = 0; r < nr; ++r) s += lg[r * n_q + n_src + c];
      cs[c] = s;
    }
  }
  __syncthreads();
  const float inv_src = 1.0f / (float)n_src;
  for (int c = tid; c < P; c += kThreads) {
    if (c < n_ctx) {
      const float sc = cs[c] * inv_src;
      w.colscore[(size_t)bh * n_ctx + c] = sc;
      skey[c] = sc;
      sidx[c] = c;
    } else {
      skey[c] = -FLT_MAX;
      sidx[c] = 0x7fffffff - (c - n_ctx);
    }
  }
  bitonic_sort_pairs<true>(skey, sidx, P);
  // the k winners, re-sorted by block index
  const int kk = p.k;
  if (kk > 0) {
    const int PK = next_pow2(kk);
    for (int i = tid; i < PK; i += kThreads) ssel[i] = i < kk ? sidx[i] : 0x7fffffff;
    bitonic_sort_int(ssel, PK);
    for (int i = tid; i < kk; i += kThreads) w.sel[(size_t)bh * kk + i] = ssel[i];
  }
}

template <typename T, int D, int BLK>
cudaError_t launch_t(const void* q, const void* k, const void* v, const Plan& p, const Work& w, cudaStream_t s) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int RPP = kThreads / (D / VEC);
  const size_t pool_bytes = sizeof(float) * 3 * RPP * D;
  const size_t smem = pool_bytes > score_smem_bytes<D>(p) ? pool_bytes : score_smem_bytes<D>(p);
  auto kern = pool_score_topk_kernel<T, D, BLK>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(p.n_q, p.BH);
  kern<<<grid, kThreads, smem, s>>>(static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
                                    p, w);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool_score_topk(const void* q, const void* k, const void* v, const Plan& p, const Work& w,
                                   cudaStream_t s) {
  if (p.dt == 0) {
    if (p.D == 128) return p.b == 128 ? launch_t<__nv_bfloat16, 128, 128>(q, k, v, p, w, s)
                                      : launch_t<__nv_bfloat16, 128, 64>(q, k, v, p, w, s);
    return p.b == 128 ? launch_t<__nv_bfloat16, 64, 128>(q, k, v, p, w, s)
                      : launch_t<__nv_bfloat16, 64, 64>(q, k, v, p, w, s);
  }
  if (p.D == 128) return p.b == 128 ? launch_t<float, 128, 128>(q, k, v, p, w, s)
                                    : launch_t<float, 128, 64>(q, k, v, p, w, s);
  return p.b == 128 ? launch_t<float, 64, 128>(q, k, v, p, w, s) : launch_t<float, 64, 64>(q, k, v, p, w, s);
}

}  // namespace isa
