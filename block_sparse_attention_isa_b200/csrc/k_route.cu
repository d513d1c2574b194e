// Stage 3 of In-context Sparse Attention: query sharpness and routing.
//
// Method: "Lightning Unified Video Editing via In-Context Sparse Attention",
// papernotes.org notes, Key design 3 (grouped computation by query
// sharpness): M_i = Var(softmax(Qc_i Kc^T)), read from the pooling scores;
// query blocks are sorted by M_i and split by the flat ratio alpha_f. The
// paperlayer.ai summary, section 3 (Grouped Computation), gives the same.
//
// Readings: Kc here is the pooled blocks of K_new (source blocks, then the
// kept context blocks in ascending order), scores are scaled by 1/sqrt(D), the
// variance is the population variance sum_j (p_j - 1/n)^2 / n (two-pass form,
// free of the cancellation of sum p^2/n - 1/n^2), and the n_flat blocks of
// LOWEST sharpness (ties by lower index) take the Taylor path.
//
// Grid (ceil(n_q / 8), B*H), 256 threads. Each CTA scores 8 query blocks
// against all n_new pooled key blocks and writes their M_i; it also writes
// its share of the pooled K_new / V_new rows in the attention kernel's element
// type. The last CTA of a head sorts (M_i, i), then writes the route list:
// exact blocks ascending followed by Taylor blocks ascending.
#include <cuda_bf16.h>
#include <float.h>

#include "block_sort.cuh"
#include "isa_internal.h"

namespace isa {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 8;  // query blocks per CTA

__device__ __forceinline__ void store_elem(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void store_elem(float* p, float x) { *p = x; }

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) route_kernel(Plan p, Work w) {
  extern __shared__ __align__(16) float smem[];
  const int bh = blockIdx.y, i0 = blockIdx.x * kRows, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int n_q = p.n_q, n_src = p.n_src, n_new = p.n_new;
  const int nr = min(kRows, n_q - i0);
  const float* Qc = w.qc + (size_t)bh * n_q * D;
  const float* Kc = w.kc + (size_t)bh * n_q * D;
  const float* Vc = w.vc + (size_t)bh * n_q * D;
  const int32_t* sel = w.sel + (size_t)bh * p.k;
  float* qcs = smem;                 // [kRows][D]
  float* lg = qcs + kRows * D;       // [kRows][n_new]
  __shared__ int s_last;

  for (int e = tid; e < kRows * D; e += kThreads) {
    const int r = e / D;
    qcs[e] = r < nr ? Qc[(size_t)(i0 + r) * D + (e % D)] : 0.f;
  }
  __syncthreads();
  const float scale = 1.0f / sqrtf((float)D);
  for (int j = tid; j < n_new; j += kThreads) {
    const int src = j < n_src ? j : n_src + sel[j - n_src];
    const float4* kr = reinterpret_cast<const float4*>(Kc + (size_t)src * D);
    float a[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) a[r] = 0.f;
#pragma unroll 4
    for (int d4 = 0; d4 < D / 4; ++d4) {
      const float4 kv = kr[d4];
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const float4 qv = *reinterpret_cast<const float4*>(qcs + r * D + 4 * d4);
        a[r] = fmaf(qv.x, kv.x, a[r]);
        a[r] = fmaf(qv.y, kv.y, a[r]);
        a[r] = fmaf(qv.z, kv.z, a[r]);
        a[r] = fmaf(qv.w, kv.w, a[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      if (r < nr) lg[r * n_new + j] = a[r] * scale;
  }
  __syncthreads();
  const float inv_n = 1.0f / (float)n_new;
  for (int r = warp; r < nr; r += kThreads / 32) {
    const float* row = lg + r * n_new;
    float m = -FLT_MAX;
    for (int j = lane; j < n_new; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float s = 0.f;
    for (int j = lane; j < n_new; j += 32) s += expf(row[j] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float inv = 1.0f / s;
    float v = 0.f;
    for (int j = lane; j < n_new; j += 32) {
      const float d = expf(row[j] - m) * inv - inv_n;
      v = fmaf(d, d, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) w.sharp[(size_t)bh * n_q + i0 + r] = v * inv_n;
  }

  // pooled K_new / V_new rows for the Taylor path, in the MMA element type
  T* kcn = static_cast<T*>(w.kcn) + (size_t)bh * n_new * D;
  T* vcn = static_cast<T*>(w.vcn) + (size_t)bh * n_new * D;
  for (int j = blockIdx.x; j < n_new; j += gridDim.x) {
    const int src = j < n_src ? j : n_src + sel[j - n_src];
    for (int d = tid; d < D; d += kThreads) {
      store_elem(kcn + (size_t)j * D + d, Kc[(size_t)src * D + d]);
      store_elem(vcn + (size_t)j * D + d, Vc[(size_t)src * D + d]);
    }
  }

  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&w.ctr_route[bh], 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  const int P = next_pow2(n_q);
  float* key = smem;                                       // [P]
  int32_t* idx = reinterpret_cast<int32_t*>(key + P);      // [P]
  int32_t* lst = idx + P;                                  // [P]
  for (int i = tid; i < P; i += kThreads) {
    key[i] = i < n_q ? __ldcg(w.sharp + (size_t)bh * n_q + i) : FLT_MAX;
    idx[i] = i < n_q ? i : 0x7fffffff - (i - n_q);
  }
  bitonic_sort_pairs<false>(key, idx, P);
  const int n_flat = p.n_flat, n_exact = p.n_exact;
  int32_t* route = w.route + (size_t)bh * n_q;
  // exact part: ranks n_flat .. n_q-1, re-sorted by block index
  if (n_exact > 0) {
    const int PE = next_pow2(n_exact);
    for (int i = tid; i < PE; i += kThreads) lst[i] = i < n_exact ? idx[n_flat + i] : 0x7fffffff;
    bitonic_sort_int(lst, PE);
    for (int i = tid; i < n_exact; i += kThreads) route[i] = lst[i];
    __syncthreads();
  }
  if (n_flat > 0) {
    const int PF = next_pow2(n_flat);
    for (int i = tid; i < PF; i += kThreads) lst[i] = i < n_flat ? idx[i] : 0x7fffffff;
    bitonic_sort_int(lst, PF);
    for (int i = tid; i < n_flat; i += kThreads) route[n_exact + i] = lst[i];
  }
}

template <typename T, int D>
cudaError_t launch_t(const Plan& p, const Work& w, cudaStream_t s) {
  const int P = next_pow2(p.n_q);
  size_t a = sizeof(float) * (size_t)(kRows * D + kRows * p.n_new);
  size_t b = (sizeof(float) + 2 * sizeof(int32_t)) * (size_t)P;
  const size_t smem = a > b ? a : b;
  auto kern = route_kernel<T, D>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((p.n_q + kRows - 1) / kRows, p.BH);
  kern<<<grid, kThreads, smem, s>>>(p, w);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const Plan& p, const Work& w, cudaStream_t s) {
  if (p.dt == 0) return p.D == 128 ? launch_t<__nv_bfloat16, 128>(p, w, s) : launch_t<__nv_bfloat16, 64>(p, w, s);
  return p.D == 128 ? launch_t<float, 128>(p, w, s) : launch_t<float, 64>(p, w, s);
}

}  // namespace isa
