// Shared-memory bitonic sorts used by the per-head top-k and routing steps.
#pragma once
#include <cstdint>

namespace isa {

// Sort P (a power of two) (key, idx) pairs in shared memory, all threads of the block taking part.
// Order: key descending when kDescending, else ascending; equal keys by idx ascending.
// Entries beyond the live range must be padded with keys that sort last and distinct idx values.
template <bool kDescending>
__device__ void bitonic_sort_pairs(float* key, int32_t* idx, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int i = threadIdx.x; i < P; i += blockDim.x) {
        const int j = i ^ stride;
        if (j <= i) continue;
        const float ki = key[i], kj = key[j];
        const int32_t ii = idx[i], ij = idx[j];
        // "j before i" in the target order?
        const bool j_first = kDescending ? (kj > ki || (kj == ki && ij < ii)) : (kj < ki || (kj == ki && ij < ii));
        const bool up = (i & size) == 0;  // this sub-sequence is sorted in the target order
        if (up == j_first) {
          key[i] = kj; key[j] = ki;
          idx[i] = ij; idx[j] = ii;
        }
      }
    }
  }
  __syncthreads();
}

// Sort P (a power of two) int32 values ascending in shared memory.
__device__ inline void bitonic_sort_int(int32_t* v, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int i = threadIdx.x; i < P; i += blockDim.x) {
        const int j = i ^ stride;
        if (j <= i) continue;
        const int32_t a = v[i], c = v[j];
        const bool up = (i & size) == 0;
        if (up == (c < a)) { v[i] = c; v[j] = a; }
      }
    }
  }
  __syncthreads();
}

// In-place exclusive prefix sum of v[0, n) in shared memory, each thread summing a contiguous run of
// ceil(n / blockDim.x) entries; all threads of the block take part.
__device__ inline void block_exclusive_scan(int32_t* v, int n) {
  __shared__ int32_t warp_tot[32];
  const int nt = blockDim.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = (nt + 31) >> 5;
  const int per = (n + nt - 1) / nt;
  const int b0 = threadIdx.x * per;
  __syncthreads();  // v is complete
  int32_t local = 0;
  for (int k = 0; k < per; ++k)
    if (b0 + k < n) local += v[b0 + k];
  int32_t x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int32_t t = lane < nwarps ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_tot[lane] = t;
  }
  __syncthreads();
  int32_t base = (warp > 0 ? warp_tot[warp - 1] : 0) + x - local;
  for (int k = 0; k < per; ++k) {
    if (b0 + k < n) {
      const int32_t f = v[b0 + k];
      v[b0 + k] = base;
      base += f;
    }
  }
  __syncthreads();
}

// Split the n entries (key[i], index i) of shared memory into the `cnt` that rank first in the
// order (key descending when kDescending, else ascending; equal keys by lower index) and the
// rest, and write each part's indices in ascending order: first[0, cnt) and rest[0, n - cnt)
// (global or shared memory; rest may be NULL). Each entry's rank is counted against all n keys, then one block
// scan places it. `scratch` is shared memory for n int32. All threads of the block take part.
// (For a few hundred entries this takes a handful of barriers where a bitonic sort of the
// pairs followed by sorts of both parts takes about a hundred.)
template <bool kDescending>
__device__ void rank_split(const float* key, int n, int cnt, int32_t* scratch, int32_t* first, int32_t* rest) {
  __syncthreads();  // key is complete
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float ki = key[i];
    int r = 0;
    for (int j = 0; j < n; ++j) {
      const float kj = key[j];
      r += (kDescending ? (kj > ki) : (kj < ki)) || (kj == ki && j < i);
    }
    scratch[i] = r < cnt ? 1 : 0;
  }
  __syncthreads();
  // each thread keeps the flags of its scan run (n <= 8 * blockDim.x), which the scan overwrites
  int32_t flags[8];
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int b0 = threadIdx.x * per;
  for (int k = 0; k < per && k < 8; ++k) flags[k] = b0 + k < n ? scratch[b0 + k] : 0;
  block_exclusive_scan(scratch, n);
  for (int k = 0; k < per && k < 8; ++k) {
    const int i = b0 + k;
    if (i >= n) break;
    const int pf = scratch[i];  // first-part entries before i
    if (flags[k]) first[pf] = i;
    else if (rest) rest[i - pf] = i;
  }
  __syncthreads();
}

__host__ __device__ inline int next_pow2(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

}  // namespace isa
