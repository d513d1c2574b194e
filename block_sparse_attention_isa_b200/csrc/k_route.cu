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
// Grid (ceil(n_q / R), B*H), 256 threads, R = 32 query blocks per CTA (16 when
// n_new is above 1024). The CTA keeps its R pooled query rows in shared memory
// and streams the gathered pooled keys of K_new through shared memory in
// chunks of 64 (rows padded so that the 32 keys a warp reads fall in distinct
// banks); thread (key, row group) accumulates R / 4 scores. It writes the M_i of
// its rows, and its share of the pooled K_new / V_new rows in the attention
// kernel's element type. The last CTA of a head sorts (M_i, i), then writes the
// route list: exact blocks ascending followed by Taylor blocks ascending.
//
// With k_ns > 0 (the no-sparsity ratio alpha_ns of papernotes.org, Key design 3)
// each row also picks the k_ns blocks of K_new with the largest coarse scores
// (ties to the lower index) from the same scores: the k_ns-th largest score is
// found by a bitwise search over order-preserving integer keys (32 counting
// passes over the row, held in registers when n_new <= 256), then the blocks
// above it and the first equal ones are written as an ascending list and as a
// bitmask over K_new's blocks.
#include <cuda_bf16.h>
#include <float.h>

#include "block_sort.cuh"
#include "isa_internal.h"

namespace isa {
namespace {

constexpr int kThreads = 256;
constexpr int kKeys = 64;     // pooled keys per shared-memory chunk
constexpr int kGroups = kThreads / kKeys;  // row groups
// Up to this many query blocks the routing splits by counted ranks (n comparisons per block),
// above it by bitonic sorts.
constexpr int kRankSplitMax = 512;

__device__ __forceinline__ void store_elem(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void store_elem(float* p, float x) { *p = x; }

// Unsigned key with the order of the float (-0 folded into +0; no NaN inputs).
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The k_ns largest entries of one row (ties to the lower index), by one warp:
// ascending list into nsel[k_ns], bitmask into nsmask[ceil(n / 32)]. Rows of up to
// 32 * KPL entries keep their keys in registers (entry lane + 32 i in key[i]).
template <int KPL>
__device__ __forceinline__ void select_row_blocks_reg(const float* row, int n, int k_ns, int lane, int32_t* nsel,
                                                      uint32_t* nsmask) {
  uint32_t key[KPL];  // 0 past the end: every real key is above 0
#pragma unroll
  for (int i = 0; i < KPL; ++i) key[i] = lane + 32 * i < n ? order_key(row[lane + 32 * i]) : 0u;
  uint32_t t = 0;  // grows to the key of the k_ns-th largest entry
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = t | (1u << bit);
    int c = 0;
#pragma unroll
    for (int i = 0; i < KPL; ++i) c += key[i] >= cand ? 1 : 0;
    if (__reduce_add_sync(0xffffffffu, c) >= k_ns) t = cand;
  }
  int above = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) above += key[i] > t ? 1 : 0;
  int eq_left = k_ns - __reduce_add_sync(0xffffffffu, above);
  int pos = 0;
  const uint32_t below = (1u << lane) - 1u;
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    if (32 * i >= n) break;
    const bool eq = key[i] == t;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const bool take = key[i] > t || (eq && __popc(eqm & below) < eq_left);
    eq_left = max(0, eq_left - __popc(eqm));
    const uint32_t tm = __ballot_sync(0xffffffffu, take);
    if (lane == 0) nsmask[i] = tm;
    if (take) nsel[pos + __popc(tm & below)] = lane + 32 * i;
    pos += __popc(tm);
  }
}

// The same for rows of any length, reading the keys from shared memory on every pass.
__device__ __forceinline__ void select_row_blocks(const float* row, int n, int k_ns, int lane, int32_t* nsel,
                                                  uint32_t* nsmask) {
  uint32_t t = 0;  // grows to the key of the k_ns-th largest entry
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = t | (1u << bit);
    int c = 0;
    for (int j = lane; j < n; j += 32) c += order_key(row[j]) >= cand ? 1 : 0;
    c = __reduce_add_sync(0xffffffffu, c);
    if (c >= k_ns) t = cand;
  }
  int above = 0;
  for (int j = lane; j < n; j += 32) above += order_key(row[j]) > t ? 1 : 0;
  above = __reduce_add_sync(0xffffffffu, above);
  int eq_left = k_ns - above;  // entries equal to the threshold still to take, lowest index first
  int pos = 0;
  const uint32_t below = (1u << lane) - 1u;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < n ? order_key(row[j]) : 0u;
    const bool eq = j < n && key == t;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const bool take = (j < n && key > t) || (eq && __popc(eqm & below) < eq_left);
    eq_left = max(0, eq_left - __popc(eqm));
    const uint32_t tm = __ballot_sync(0xffffffffu, take);
    if (lane == 0) nsmask[j0 >> 5] = tm;
    if (take) nsel[pos + __popc(tm & below)] = j;
    pos += __popc(tm);
  }
}

template <int D>
__host__ __device__ constexpr int key_stride() { return D + 4; }  // floats; 4-word skew between consecutive key rows

template <typename T, int D, int R>
__global__ void __launch_bounds__(kThreads) route_kernel(Plan p, Work w) {
  constexpr int KS = key_stride<D>();
  constexpr int RPG = R / kGroups;  // rows per thread
  static_assert(R % kGroups == 0, "rows per group");
  extern __shared__ __align__(16) float smem[];
  const int bh = blockIdx.y, i0 = blockIdx.x * R, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int n_q = p.n_q, n_src = p.n_src, n_new = p.n_new;
  const int nr = min(R, n_q - i0);
  const float* Qc = w.qc + (size_t)bh * n_q * D;
  const float* Kc = w.kc + (size_t)bh * n_q * D;
  const float* Vc = w.vc + (size_t)bh * n_q * D;
  const int32_t* sel = w.sel + (size_t)bh * p.k;
  float* qs = smem;              // [R][D]
  float* ks = qs + R * D;        // [kKeys][KS]
  float* lg = ks + kKeys * KS;   // [R][n_new]
  __shared__ int s_last;

  for (int e = tid; e < R * (D / 4); e += kThreads) {
    const int r = e / (D / 4), d4 = e - r * (D / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < nr) v = __ldcg(reinterpret_cast<const float4*>(Qc + (size_t)(i0 + r) * D) + d4);
    *reinterpret_cast<float4*>(qs + r * D + 4 * d4) = v;
  }
  const float scale = 1.0f / sqrtf((float)D);
  const int kk = tid % kKeys, rg = tid / kKeys;
  for (int j0 = 0; j0 < n_new; j0 += kKeys) {
    __syncthreads();  // the previous chunk is consumed (and the query rows are in place)
    for (int e = tid; e < kKeys * (D / 4); e += kThreads) {
      const int jj = e / (D / 4), d4 = e - jj * (D / 4);
      const int j = j0 + jj;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < n_new) {
        const int src = j < n_src ? j : n_src + sel[j - n_src];
        v = __ldcg(reinterpret_cast<const float4*>(Kc + (size_t)src * D) + d4);
      }
      *reinterpret_cast<float4*>(ks + jj * KS + 4 * d4) = v;
    }
    __syncthreads();
    float a[RPG];
#pragma unroll
    for (int r = 0; r < RPG; ++r) a[r] = 0.f;
    const float* kr = ks + kk * KS;
#pragma unroll 4
    for (int d4 = 0; d4 < D / 4; ++d4) {
      const float4 kv = *reinterpret_cast<const float4*>(kr + 4 * d4);
#pragma unroll
      for (int r = 0; r < RPG; ++r) {
        const float4 qv = *reinterpret_cast<const float4*>(qs + (rg * RPG + r) * D + 4 * d4);
        a[r] = fmaf(qv.x, kv.x, a[r]);
        a[r] = fmaf(qv.y, kv.y, a[r]);
        a[r] = fmaf(qv.z, kv.z, a[r]);
        a[r] = fmaf(qv.w, kv.w, a[r]);
      }
    }
    const int j = j0 + kk;
    if (j < n_new) {
#pragma unroll
      for (int r = 0; r < RPG; ++r)
        if (rg * RPG + r < nr) lg[(rg * RPG + r) * n_new + j] = a[r] * scale;
    }
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
  if (p.k_ns > 0) {
#pragma unroll 1
    for (int r = warp; r < nr; r += kThreads / 32) {
      const size_t gi = (size_t)bh * n_q + i0 + r;
      if (n_new <= 256)
        select_row_blocks_reg<8>(lg + r * n_new, n_new, p.k_ns, lane, w.nsel + gi * p.k_ns,
                                 w.nsmask + gi * p.ns_words);
      else
        select_row_blocks(lg + r * n_new, n_new, p.k_ns, lane, w.nsel + gi * p.k_ns, w.nsmask + gi * p.ns_words);
    }
  }

  // pooled K_new / V_new rows for the Taylor path, in the MMA element type
  T* kcn = static_cast<T*>(w.kcn) + (size_t)bh * n_new * D;
  T* vcn = static_cast<T*>(w.vcn) + (size_t)bh * n_new * D;
  for (int e = tid + blockIdx.x * kThreads; e < n_new * D; e += gridDim.x * kThreads) {
    const int j = e / D, d = e - j * D;
    const int src = j < n_src ? j : n_src + sel[j - n_src];
    store_elem(kcn + e, Kc[(size_t)src * D + d]);
    store_elem(vcn + e, Vc[(size_t)src * D + d]);
  }

  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&w.ctr_route[bh], 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  const int n_flat = p.n_flat, n_exact = p.n_exact;
  int32_t* route = w.route + (size_t)bh * n_q;
  if (n_q <= kRankSplitMax) {
    // rank of every (M_i, i) among all, then one scan: Taylor blocks (the n_flat lowest) and exact
    // blocks, each in ascending block order
    float* key = smem;
    int32_t* scratch = reinterpret_cast<int32_t*>(key + n_q);
    for (int i = tid; i < n_q; i += kThreads) key[i] = __ldcg(w.sharp + (size_t)bh * n_q + i);
    rank_split<false>(key, n_q, n_flat, scratch, route + n_exact, route);
    return;
  }
  const int P = next_pow2(n_q);
  float* key = smem;                                       // [P]
  int32_t* idx = reinterpret_cast<int32_t*>(key + P);      // [P]
  int32_t* lst = idx + P;                                  // [P]
  for (int i = tid; i < P; i += kThreads) {
    key[i] = i < n_q ? __ldcg(w.sharp + (size_t)bh * n_q + i) : FLT_MAX;
    idx[i] = i < n_q ? i : 0x7fffffff - (i - n_q);
  }
  bitonic_sort_pairs<false>(key, idx, P);
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

template <typename T, int D, int R>
cudaError_t launch_r(const Plan& p, const Work& w, cudaStream_t s) {
  const int P = next_pow2(p.n_q);
  const size_t a = sizeof(float) * (size_t)(R * D + kKeys * key_stride<D>() + R * p.n_new);
  const size_t b = (sizeof(float) + 2 * sizeof(int32_t)) * (size_t)P;
  const size_t smem = a > b ? a : b;
  auto kern = route_kernel<T, D, R>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((p.n_q + R - 1) / R, p.BH);
  kern<<<grid, kThreads, smem, s>>>(p, w);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_t(const Plan& p, const Work& w, cudaStream_t s) {
  // 32 query blocks per CTA; 16 when the scores of 32 rows would not fit in shared memory
  return p.n_new <= 1024 ? launch_r<T, D, 32>(p, w, s) : launch_r<T, D, 16>(p, w, s);
}

}  // namespace

cudaError_t launch_route(const Plan& p, const Work& w, cudaStream_t s) {
  if (p.dt == 0) return p.D == 128 ? launch_t<__nv_bfloat16, 128>(p, w, s) : launch_t<__nv_bfloat16, 64>(p, w, s);
  return p.D == 128 ? launch_t<float, 128>(p, w, s) : launch_t<float, 64>(p, w, s);
}

}  // namespace isa
