// Internal types shared by the ISA kernels and the C-ABI layer.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace isa {

// Sizes of one call, all derived on the host from the arguments.
struct Plan {
  int B, H, BH, N, D, b, L_src, L_ctx;
  int n_q;     // n_src + n_ctx query blocks (also key blocks)
  int n_src;   // ceil(L_src / b): source blocks from token 0, the last one possibly short
  int n_ctx;   // ceil(L_ctx / b): context blocks from token L_src, the last one possibly short
  int k;       // kept context blocks
  int n_new;   // n_src + k blocks in K_new
  int L_new;   // n_new * b rows of K_new: every block takes b rows, a short one padded (masked)
  int L_srcp;  // n_src * b: rows of the source part of K_new (rows L_src .. L_srcp - 1 masked)
  int len_src_last;  // tokens of the last source block (b when b divides L_src)
  int len_ctx_last;  // tokens of the last context block (b when b divides L_ctx)
  int ragged;  // 1 when b does not divide L_src or L_ctx
  int n_flat;  // query blocks on the Taylor path
  int n_exact; // n_q - n_flat query blocks on the exact path
  int dt;      // 0 = bf16, 1 = fp32
  int elem;    // bytes per element
  int k_ns;    // key blocks of K_new computed exactly inside each Taylor query block (0: plain Taylor path)
  int ns_words;  // 32-bit words of one query block's exact-key-block bitmask (ceil(n_new / 32))
};

// First token of block i (source blocks from 0, context blocks from L_src) and its length.
__host__ __device__ inline int block_start(const Plan& p, int i) {
  return i < p.n_src ? i * p.b : p.L_src + (i - p.n_src) * p.b;
}
__host__ __device__ inline int block_len(const Plan& p, int i) {
  return i == p.n_src - 1 ? p.len_src_last : (i == p.n_q - 1 ? p.len_ctx_last : p.b);
}

// Row length of the transposed pooled V rows (fp32 inputs): n_new rounded up to 4
// floats so that the rows start on 16-byte boundaries, as TMA requires.
__host__ __device__ inline int vct_ld(const Plan& p) { return (p.n_new + 3) & ~3; }

// Views into the caller's workspace (all 256-byte aligned).
struct Work {
  uint32_t* ctrl;        // [kCtrlWords]: error word, spare words
  uint32_t* ctr_pool;    // [BH] scoring items finished per head (pooling kernel)
  uint32_t* ctr_route;   // [BH] CTAs of the routing grid finished per head
  float* qc;             // [BH, n_q, D] block means of Q (fp32)
  float* kc;             // [BH, n_q, D]
  float* vc;             // [BH, n_q, D]
  float* colscore;       // [BH, n_ctx] context-block scores
  float* partial;        // [BH, ceil(n_src/16), n_ctx] per-item context-column sums (pooling kernel)
  int32_t* sel;          // [BH, max(k,1)] kept context blocks, ascending
  float* sharp;          // [BH, n_q] query-block sharpness M_i
  int32_t* route;        // [BH, n_q] exact blocks ascending, then Taylor blocks ascending
  void* kcn;             // [BH, n_new, D] pooled K_new blocks in the MMA element type
  void* vcn;             // [BH, n_new, D]
  void* ksel;            // [BH, k*b, D] gathered context keys
  void* vsel;            // [BH, k*b, D]
  float* vtn;            // fp32 inputs only: [BH, D, L_new] V_new transposed
  float* vct;            // fp32 inputs only: [BH, D, vct_ld] pooled V_new rows transposed
  int32_t* nsel;         // k_ns > 0 only: [BH, n_q, k_ns] exactly computed K_new blocks of each query block, ascending
  uint32_t* nsmask;      // k_ns > 0 only: [BH, n_q, ns_words] the same blocks as a bitmask over K_new's blocks
  float* lse;            // optional, caller memory (not workspace): [BH, N] per-row log-sum-exp written by the
                         // attention kernels (training forward); NULL to skip
};

constexpr int kCtrlWords = 64;
constexpr int kStageEvents = 5;  // before pooling, after pooling, gather, routing, attention
constexpr int kMaxBlocks = 2048;  // max n_q supported by the per-head sorts

// Error-word bits written by kernels when a bounded wait gives up.
enum : uint32_t {
  kErrProducer = 1u << 0,
  kErrMma = 1u << 1,
  kErrSoftmax = 1u << 2,
  kErrGather = 1u << 3,
  kErrSelftest = 1u << 4,
  kErrPool = 1u << 5,
};

// Control words at the start of the workspace (cleared on every call).
enum : int {
  kCtrlError = 0,
  kCtrlGridBarrier = 1,
  kCtrlMixedNext = 2,  // next work item of the mixed Taylor kernel (dynamic schedule)
  kCtrlPairNext = 3,   // next work item of the CTA-pair attention kernel (dynamic schedule)
  kCtrlBwdNext = 4,    // [3]: next work item of the three backward launches (dynamic schedule)
};

// Floats of the pooling kernel's per-item partial sums for these sizes.
size_t pool_partial_floats(const Plan& p);

size_t workspace_layout(const Plan& p, Work* w, char* base);

// Argument checks and block counts shared by the entry points (same rules and
// messages as isa_forward_ex); returns ISA_OK or an error code.
int build_plan(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, float alpha_f, int dt, Plan* p,
               float alpha_ns = 0.0f);
// Sets the thread-local message returned by isa_last_error() and returns `code`.
int set_error(int code, const char* fmt, ...);

cudaError_t launch_pool_score_topk(const void* q, const void* k, const void* v, const Plan& p, const Work& w,
                                   cudaStream_t s);
cudaError_t launch_gather(const void* k, const void* v, const Plan& p, const Work& w, cudaStream_t s);
cudaError_t launch_route(const Plan& p, const Work& w, cudaStream_t s);
cudaError_t launch_transpose_v(const void* v, const Plan& p, const Work& w, cudaStream_t s);
cudaError_t launch_attention(const void* q, const void* k, const void* v, void* out, const Plan& p,
                             const Work& w, cudaStream_t s, int* n_ctas_out);
// Attention on pairs of CTAs (bf16, D = 128): same contract as launch_attention.
bool attention_pair_supported(const Plan& p);
cudaError_t launch_attention_pair(const void* q, const void* k, const void* v, void* out, const Plan& p,
                                  const Work& w, cudaStream_t s, int* n_ctas);
// Taylor query blocks with exactly computed key blocks (k_ns > 0, bf16): one query block per
// work item, keys = the pooled K_new rows (weight b, the block's exact blocks masked) followed
// by the keys of its exact blocks, in one online softmax.
cudaError_t launch_attention_ns(const void* q, const void* k, const void* v, void* out, const Plan& p,
                                const Work& w, cudaStream_t s);
// The same for bf16, D = 128, b = 128 and whole blocks: one query block per work item, the two
// softmax warpgroups on alternate key tiles of it, their softmax states merged at the end.
bool attention_mixed_supported(const Plan& p);
cudaError_t launch_attention_mixed(const void* q, const void* k, const void* v, void* out, const Plan& p,
                                   const Work& w, cudaStream_t s);

// Backward pass (bf16, D = 128, whole blocks, alpha_ns = 0): whether these sizes are supported,
// the scratch it needs beyond the forward's workspace, and the launch sequence (delta pass, dQ,
// dK/dV of the Taylor path over the pooled rows, dK/dV of the exact path plus the Taylor spread).
bool backward_supported(const Plan& p);
size_t backward_workspace_bytes(const Plan& p);
cudaError_t launch_backward(const void* q, const void* k, const void* v, const void* out, const float* lse,
                            const void* dout, void* dq, void* dk, void* dv, const Plan& pl, const Work& w,
                            void* bwd_ws, cudaStream_t s);

// One thread waits on an mbarrier that nothing arrives on; the bounded wait gives
// up after `timeout_ms` and sets kErrSelftest in err[0].
cudaError_t launch_wait_selftest(uint32_t* err, int timeout_ms, cudaStream_t s);
// y_poly[i] = the attention softmax's polynomial 2^x[i]; y_ref[i] = CUDA's exp2f(x[i]).
cudaError_t launch_exp2_selftest(const float* x, float* y_poly, float* y_ref, int n, cudaStream_t s);

// Number of SMs of the current device (cached per device).
int device_sm_count();

}  // namespace isa
