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

__host__ __device__ inline int next_pow2(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

}  // namespace isa
