// fp32 inputs only: V_new and the pooled V_new rows, transposed to [D, rows].
//
// The tf32 tensor-core MMA takes its B operand K-major only (an MN-major B
// returns zeros), so for fp32 inputs the P V product needs V with the key axis
// contiguous. This kernel writes V_new^T = [V_src ; V_sel]^T and Vc_new^T once
// per call; the attention kernel then loads K-major tiles of them with TMA.
// bf16 inputs never take this step (their P V MMA reads V as it is).
#include "isa_internal.h"

namespace isa {
namespace {

constexpr int kTile = 32;

__global__ void __launch_bounds__(256) transpose_v_kernel(const float* __restrict__ v, Plan p, Work w) {
  __shared__ float tile[kTile][kTile + 1];
  const int bh = blockIdx.z, d0 = blockIdx.y * kTile;
  const int tiles_new = (p.L_new + kTile - 1) / kTile;
  const bool pooled = (int)blockIdx.x >= tiles_new;
  const int r0 = (pooled ? (int)blockIdx.x - tiles_new : (int)blockIdx.x) * kTile;
  const int rows = pooled ? p.n_new : p.L_new;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  for (int i = ty; i < kTile; i += 8) {
    const int r = r0 + i;
    float x = 0.f;
    if (r < rows) {
      const float* src;
      if (pooled) src = static_cast<const float*>(w.vcn) + ((size_t)bh * p.n_new + r) * p.D;
      // K_new rows: the source part (read in place; rows L_src .. L_srcp - 1 of it are
      // padding, masked by the attention kernel, and may lie past N), then the kept
      // blocks, b rows each
      else if (r < p.L_srcp) src = r < p.N ? v + ((size_t)bh * p.N + r) * p.D : nullptr;
      else src = static_cast<const float*>(w.vsel) + ((size_t)bh * p.k * p.b + (r - p.L_srcp)) * p.D;
      x = src ? src[d0 + tx] : 0.f;
    }
    tile[i][tx] = x;
  }
  __syncthreads();
  float* dst = pooled ? w.vct : w.vtn;
  const int ld = pooled ? vct_ld(p) : p.L_new;
  for (int i = ty; i < kTile; i += 8) {
    const int r = r0 + tx;
    if (r < rows) dst[((size_t)bh * p.D + d0 + i) * ld + r] = tile[tx][i];
  }
}

}  // namespace

cudaError_t launch_transpose_v(const void* v, const Plan& p, const Work& w, cudaStream_t s) {
  if (p.dt != 1) return cudaSuccess;
  dim3 grid((p.L_new + kTile - 1) / kTile + (p.n_new + kTile - 1) / kTile, p.D / kTile, p.BH);
  transpose_v_kernel<<<grid, 256, 0, s>>>(static_cast<const float*>(v), p, w);
  return cudaGetLastError();
}

}  // namespace isa
