// Allocation-free entry point: the pooling + coarse-score + context top-k
// kernel with its scratch memory in a fixed device array instead of a
// caller-provided workspace.
//
// Why: some callers cannot allocate device memory. Plugin hosts of inference
// runtimes often hand an operator only its input and output buffers and keep
// every other byte of device memory to themselves, and latency-critical serving
// loops may forbid cudaMalloc because it can synchronise the device. Such
// callers can still ask which context blocks the pass would keep.
//
// How: the block means of Q, K and V, the per-item partial sums, the control
// words and the per-head completion counters live in `g_scratch`, a file-scope
// __device__ array of kScratchBytes. Every GPU that
// loads this library holds that array until the process exits. Host code must
// not pass the symbol itself to a kernel (on the host it names a host-side
// stand-in); the device address is looked up once per device with
// cudaGetSymbolAddress and cached. The cache does not survive cudaDeviceReset.
//
// The kernel's bounded waits report a give-up in the error word at the start of
// the array; isa_select_context_noalloc_status synchronises the stream and reads
// and clears that word, so that a call that timed out is not taken for a good one.
#include <mutex>

#include "../../include/isa.h"
#include "isa_internal.h"

namespace isa {
namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;  // 32 MiB per device
__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Device address of g_scratch on the current device, or NULL when no call has looked it up yet.
int scratch_address_if_known(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(ISA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return set_error(ISA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  *out = g_scratch_addr[dev];
  return ISA_OK;
}

// Device address of g_scratch on the current device (looked up on first use).
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(ISA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return set_error(ISA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_scratch);
    if (e != cudaSuccess || !ptr)
      return set_error(ISA_ERR_CUDA, "cudaGetSymbolAddress of the fixed scratch array: %s", cudaGetErrorString(e));
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return ISA_OK;
}

}  // namespace
}  // namespace isa

using namespace isa;

extern "C" int isa_select_context_noalloc(const void* q, const void* k, const void* v, int B, int H, int L_src,
                                          int L_ctx, int D, int b, float alpha_s, isa_dtype dt, int32_t* sel,
                                          float* colscore, void* stream) {
  Plan p;
  int rc = build_plan(B, H, L_src, L_ctx, D, b, alpha_s, 0.0f, (int)dt, &p);
  if (rc != ISA_OK) return rc;
  if (!q || !k || !v) return set_error(ISA_ERR_ARG, "q, k and v must not be NULL");
  if (!sel || !colscore) return set_error(ISA_ERR_ARG, "sel and colscore must not be NULL");
  {
    // the pooling kernel reads the inputs with bulk copies, which need 16-byte aligned addresses
    const void* ptrs[3] = {q, k, v};
    const char* names[3] = {"q", "k", "v"};
    for (int i = 0; i < 3; ++i)
      if (reinterpret_cast<uintptr_t>(ptrs[i]) & 15)
        return set_error(ISA_ERR_ARG, "%s must be 16-byte aligned (device address %p)", names[i], ptrs[i]);
    if ((reinterpret_cast<uintptr_t>(sel) & 3) || (reinterpret_cast<uintptr_t>(colscore) & 3))
      return set_error(ISA_ERR_ARG, "sel and colscore must be 4-byte aligned");
  }
  const size_t BH = (size_t)p.BH;
  const size_t ctrl_bytes = align256(sizeof(uint32_t) * kCtrlWords);
  const size_t ctr_bytes = align256(sizeof(uint32_t) * BH);
  const size_t pooled_bytes = align256(sizeof(float) * BH * p.n_q * p.D);
  const size_t partial_bytes = align256(sizeof(float) * pool_partial_floats(p));
  const size_t need = ctrl_bytes + ctr_bytes + 3 * pooled_bytes + partial_bytes;
  if (need > kScratchBytes)
    return set_error(ISA_ERR_UNSUPPORTED,
                     "these sizes need %zu bytes of scratch; the fixed array of the allocation-free entry point "
                     "holds %zu (3 * B*H * (N/b) * D * 4 bytes plus counters must fit)",
                     need, kScratchBytes);
  void* base = nullptr;
  if ((rc = scratch_address(&base)) != ISA_OK) return rc;
  char* c = static_cast<char*>(base);
  Work w{};
  w.ctrl = reinterpret_cast<uint32_t*>(c);
  w.ctr_pool = reinterpret_cast<uint32_t*>(c + ctrl_bytes);
  w.qc = reinterpret_cast<float*>(c + ctrl_bytes + ctr_bytes);
  w.kc = reinterpret_cast<float*>(c + ctrl_bytes + ctr_bytes + pooled_bytes);
  w.vc = reinterpret_cast<float*>(c + ctrl_bytes + ctr_bytes + 2 * pooled_bytes);
  w.partial = reinterpret_cast<float*>(c + ctrl_bytes + ctr_bytes + 3 * pooled_bytes);
  w.colscore = colscore;
  w.sel = sel;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the array keeps the previous call's contents: the control words (error word,
  // grid barrier) and the per-head counters must start at zero
  cudaError_t e = cudaMemsetAsync(c, 0, ctrl_bytes + ctr_bytes, s);
  if (e != cudaSuccess) return set_error(ISA_ERR_CUDA, "clearing the scratch counters: %s", cudaGetErrorString(e));
  e = launch_pool_score_topk(q, k, v, p, w, s);
  if (e != cudaSuccess) return set_error(ISA_ERR_CUDA, "pool/score/top-k launch: %s", cudaGetErrorString(e));
  return ISA_OK;
}

extern "C" int isa_select_context_noalloc_status(void* stream) {
  void* base = nullptr;
  int rc = scratch_address_if_known(&base);
  if (rc != ISA_OK) return rc;
  if (!base) return ISA_OK;  // no call has run on this device
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return set_error(ISA_ERR_CUDA, "synchronising the stream: %s", cudaGetErrorString(e));
  uint32_t word = 0;
  e = cudaMemcpy(&word, static_cast<uint32_t*>(base) + kCtrlError, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return set_error(ISA_ERR_CUDA, "reading the error word: %s", cudaGetErrorString(e));
  if (word) {
    e = cudaMemset(static_cast<uint32_t*>(base) + kCtrlError, 0, sizeof(word));
    if (e != cudaSuccess) return set_error(ISA_ERR_CUDA, "clearing the error word: %s", cudaGetErrorString(e));
    return set_error(ISA_ERR_TIMEOUT, "the allocation-free selection kernel's wait timed out (error word 0x%x)",
                     word);
  }
  return ISA_OK;
}
