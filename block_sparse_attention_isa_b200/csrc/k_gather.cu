// Stage 2b of In-context Sparse Attention: gather the kept context blocks of
// K and V into a compact buffer, so that K_new = [K_src ; K_sel] and
// V_new = [V_src ; V_sel] (the source part is read in place by the attention
// kernel and never copied).
//
// Method: "Lightning Unified Video Editing via In-Context Sparse Attention",
// papernotes.org notes, Key design 1: gather + concat rebuild K_new, V_new of
// length L_src + alpha_s * L_ctx.
//
// A context block of b rows is one contiguous run of b * D elements, so each
// CTA moves one chunk of it with a pair of 1-D TMA bulk copies: global ->
// shared (completion on an mbarrier), then shared -> global (bulk group).
// Pure HBM traffic: 2 (K and V) x k x b x D elements read and written per head.
// Every kept block takes b rows of K_sel / V_sel; when the last context block is
// short (b does not divide L_ctx) and kept, its rows past its length are written
// as zeros, so that the attention kernel's masked keys meet finite values.
#include "isa_internal.h"
#include "ptx.cuh"

namespace isa {
namespace {

constexpr uint32_t kChunk = 16384;  // bytes per CTA

__global__ void __launch_bounds__(32) gather_kernel(const char* __restrict__ k, const char* __restrict__ v,
                                                    char* __restrict__ ksel, char* __restrict__ vsel, Plan p,
                                                    Work w) {
  __shared__ __align__(128) char buf[kChunk];
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const int chunk = blockIdx.x, c = blockIdx.y;
  const int bh = blockIdx.z >> 1, which = blockIdx.z & 1;
  const size_t row_bytes = (size_t)p.D * p.elem;
  const size_t blk_bytes = (size_t)p.b * row_bytes;
  const size_t off = (size_t)chunk * kChunk;
  if (off >= blk_bytes) return;
  const uint32_t bytes = (uint32_t)((blk_bytes - off) < kChunk ? (blk_bytes - off) : kChunk);
  const int src_blk = w.sel[(size_t)bh * p.k + c];
  const size_t valid = (size_t)(src_blk == p.n_ctx - 1 ? p.len_ctx_last : p.b) * row_bytes;
  // bytes of this chunk that hold rows of the block (a multiple of the 128-byte-or-more row)
  const uint32_t load = off >= valid ? 0u : (uint32_t)((valid - off) < bytes ? (valid - off) : bytes);
  const char* src = (which ? v : k) + ((size_t)bh * p.N + p.L_src + (size_t)src_blk * p.b) * row_bytes + off;
  char* dst = (which ? vsel : ksel) + ((size_t)bh * p.k + c) * blk_bytes + off;

  for (uint32_t i = load; i < bytes; i += 16) *reinterpret_cast<uint4*>(buf + i) = make_uint4(0u, 0u, 0u, 0u);
  if (load > 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
    mbar_arrive_expect_tx(&bar, load);
    bulk_load(buf, src, load, &bar);
    if (!mbar_wait(&bar, 0)) {
      atomicOr(&w.ctrl[0], kErrGather);
      // the load may still land; give it the same bound once more before leaving
      mbar_wait(&bar, 0);
      return;
    }
  }
  fence_proxy_async_smem();
  bulk_store(dst, buf, bytes);
  bulk_commit();
  bulk_wait_all();
}

}  // namespace

cudaError_t launch_gather(const void* k, const void* v, const Plan& p, const Work& w, cudaStream_t s) {
  if (p.k == 0) return cudaSuccess;
  const size_t blk_bytes = (size_t)p.b * p.D * p.elem;
  dim3 grid((unsigned)((blk_bytes + kChunk - 1) / kChunk), p.k, 2 * p.BH);
  gather_kernel<<<grid, 32, 0, s>>>(static_cast<const char*>(k), static_cast<const char*>(v),
                                    static_cast<char*>(w.ksel), static_cast<char*>(w.vsel), p, w);
  return cudaGetLastError();
}

}  // namespace isa
