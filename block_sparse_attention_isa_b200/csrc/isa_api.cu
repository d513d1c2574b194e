// C ABI of the In-context Sparse Attention forward pass: argument checks,
// block counts, workspace layout and the stream-ordered launch sequence
//   pool + coarse score + top-k  ->  gather  ->  sharpness + routing  ->  attention.
// See include/isa.h for the contract of every entry point.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/isa.h"
#include "isa_internal.h"

namespace isa {

namespace {
thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(ISA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Kept context blocks: ceil(alpha_s * n_ctx) with a 1e-4 guard on the float ratio.
int kept_blocks(float alpha_s, int n_ctx) {
  const double x = (double)alpha_s * (double)n_ctx;
  long kk = (long)std::ceil(x - 1e-4);
  if (kk < 0) kk = 0;
  if (kk > n_ctx) kk = n_ctx;
  return (int)kk;
}
// Taylor query blocks: floor(alpha_f * n_q) with a 1e-4 guard on the float ratio.
int flat_blocks(float alpha_f, int n_q) {
  const double x = (double)alpha_f * (double)n_q;
  long n = (long)std::floor(x + 1e-4);
  if (n < 0) n = 0;
  if (n > n_q) n = n_q;
  return (int)n;
}

bool ratio_ok(float a) { return !std::isnan(a) && a >= 0.0f && a <= 1.0f; }

// Exactly computed key blocks per Taylor query block: ceil(alpha_ns * n_new) with a 1e-4 guard.
int no_sparse_blocks(float alpha_ns, int n_new) {
  if (!(alpha_ns > 0.0f)) return 0;
  return kept_blocks(alpha_ns, n_new);
}

int make_plan(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, float alpha_f, int dt, Plan* p,
              float alpha_ns = 0.0f) {
  if (B <= 0 || H <= 0) return fail(ISA_ERR_ARG, "B and H must be positive (B=%d H=%d)", B, H);
  if (L_src <= 0 || L_ctx <= 0) return fail(ISA_ERR_ARG, "L_src and L_ctx must be positive (%d, %d)", L_src, L_ctx);
  if (!ratio_ok(alpha_s) || !ratio_ok(alpha_f))
    return fail(ISA_ERR_ARG, "alpha_s and alpha_f must lie in [0, 1] (%g, %g)", (double)alpha_s, (double)alpha_f);
  if (!ratio_ok(alpha_ns)) return fail(ISA_ERR_ARG, "alpha_ns must lie in [0, 1] (%g)", (double)alpha_ns);
  if (dt != ISA_BF16 && dt != ISA_F32) return fail(ISA_ERR_UNSUPPORTED, "unknown dtype %d", dt);
  if (D != 64 && D != 128) return fail(ISA_ERR_UNSUPPORTED, "D must be 64 or 128 (got %d)", D);
  if (b != 64 && b != 128) return fail(ISA_ERR_UNSUPPORTED, "block size b must be 64 or 128 (got %d)", b);
  if (dt == ISA_F32 && D != 64) return fail(ISA_ERR_UNSUPPORTED, "float32 inputs need D = 64");
  const long long N = (long long)L_src + L_ctx;
  if (N > (1ll << 30)) return fail(ISA_ERR_UNSUPPORTED, "N too large");
  const long long BH = (long long)B * H;
  if (BH > 65535) return fail(ISA_ERR_UNSUPPORTED, "B*H must be at most 65535");
  // the source and the context part each end in a block of at most b tokens
  const long long n_src = (L_src + (long long)b - 1) / b, n_ctx = (L_ctx + (long long)b - 1) / b;
  const long long n_q_ll = n_src + n_ctx;
  if (n_q_ll > kMaxBlocks)
    return fail(ISA_ERR_UNSUPPORTED, "the block count must be at most %d (got %lld)", kMaxBlocks, n_q_ll);
  const int n_q = (int)n_q_ll;
  p->B = B;
  p->H = H;
  p->BH = (int)BH;
  p->N = (int)N;
  p->D = D;
  p->b = b;
  p->L_src = L_src;
  p->L_ctx = L_ctx;
  p->n_q = n_q;
  p->n_src = (int)n_src;
  p->n_ctx = (int)n_ctx;
  p->k = kept_blocks(alpha_s, p->n_ctx);
  p->n_new = p->n_src + p->k;
  p->L_new = p->n_new * b;
  p->L_srcp = p->n_src * b;
  p->len_src_last = L_src - (p->n_src - 1) * b;
  p->len_ctx_last = L_ctx - (p->n_ctx - 1) * b;
  p->ragged = (L_src % b || L_ctx % b) ? 1 : 0;
  p->n_flat = flat_blocks(alpha_f, n_q);
  p->n_exact = n_q - p->n_flat;
  p->dt = dt;
  p->elem = dt == ISA_BF16 ? 2 : 4;
  p->k_ns = no_sparse_blocks(alpha_ns, p->n_new);
  p->ns_words = (p->n_new + 31) / 32;
  if (p->k_ns > 0 && dt != ISA_BF16)
    return fail(ISA_ERR_UNSUPPORTED, "alpha_ns > 0 needs bfloat16 inputs");
  return ISA_OK;
}

bool overlaps(const void* a, const void* b, size_t bytes) {
  const char* x = static_cast<const char*>(a);
  const char* y = static_cast<const char*>(b);
  return x < y + bytes && y < x + bytes;
}
// [a, a + na) and [b, b + nb) share a byte
bool overlaps2(const void* a, size_t na, const void* b, size_t nb) {
  const char* x = static_cast<const char*>(a);
  const char* y = static_cast<const char*>(b);
  return x < y + nb && y < x + na;
}

}  // namespace

int build_plan(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, float alpha_f, int dt, Plan* p,
               float alpha_ns) {
  return make_plan(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, dt, p, alpha_ns);
}

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

size_t workspace_layout(const Plan& p, Work* w, char* base) {
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* r = base ? base + off : nullptr;
    off += align256(bytes);
    return r;
  };
  const size_t BH = p.BH;
  Work t{};
  t.ctrl = reinterpret_cast<uint32_t*>(take(sizeof(uint32_t) * (kCtrlWords + 2 * BH)));
  if (base) {
    t.ctr_pool = t.ctrl + kCtrlWords;
    t.ctr_route = t.ctr_pool + BH;
  }
  t.qc = reinterpret_cast<float*>(take(sizeof(float) * BH * p.n_q * p.D));
  t.kc = reinterpret_cast<float*>(take(sizeof(float) * BH * p.n_q * p.D));
  t.vc = reinterpret_cast<float*>(take(sizeof(float) * BH * p.n_q * p.D));
  t.colscore = reinterpret_cast<float*>(take(sizeof(float) * BH * p.n_ctx));
  t.partial = reinterpret_cast<float*>(take(sizeof(float) * pool_partial_floats(p)));
  t.sel = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * BH * (p.k > 0 ? p.k : 1)));
  t.sharp = reinterpret_cast<float*>(take(sizeof(float) * BH * p.n_q));
  t.route = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * BH * p.n_q));
  t.kcn = take((size_t)p.elem * BH * p.n_new * p.D);
  t.vcn = take((size_t)p.elem * BH * p.n_new * p.D);
  t.ksel = take((size_t)p.elem * BH * (p.k > 0 ? p.k : 1) * p.b * p.D);
  t.vsel = take((size_t)p.elem * BH * (p.k > 0 ? p.k : 1) * p.b * p.D);
  if (p.dt == ISA_F32) {
    t.vtn = reinterpret_cast<float*>(take(sizeof(float) * BH * p.D * p.L_new));
    t.vct = reinterpret_cast<float*>(take(sizeof(float) * BH * p.D * vct_ld(p)));
  }
  if (p.k_ns > 0) {
    t.nsel = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * BH * p.n_q * p.k_ns));
    t.nsmask = reinterpret_cast<uint32_t*>(take(sizeof(uint32_t) * BH * p.n_q * p.ns_words));
  }
  if (w) *w = t;
  return off;
}

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

namespace {

// Optional CUDA events recorded between the stages of the next forward calls on
// this host thread (set by isa_set_stage_events; used for live per-kernel timing).
thread_local cudaEvent_t g_stage_events[kStageEvents] = {};
thread_local bool g_stage_events_on = false;

inline cudaError_t mark(int i, cudaStream_t s) {
  return g_stage_events_on ? cudaEventRecord(g_stage_events[i], s) : cudaSuccess;
}

// The CTA-pair attention kernel runs every call it supports (bf16, D = 128), whole blocks or
// short last blocks alike; the single-CTA kernel runs D = 64 and float32.
bool use_pair_kernel(const Plan& p) { return attention_pair_supported(p); }

// keep_error: leave the error word as it is (a later element of a variable-length batch must not
// clear what an earlier one reported)
int run_forward(const void* q, const void* k, const void* v, const Plan& p, void* out, int32_t* dbg_sel,
                int32_t* dbg_route, void* workspace, size_t workspace_bytes, cudaStream_t s, bool keep_error = false,
                float* lse = nullptr) {
  const size_t need = workspace_layout(p, nullptr, nullptr);
  if (!workspace) return fail(ISA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
  if (workspace_bytes < need)
    return fail(ISA_ERR_WORKSPACE, "workspace too small: %zu bytes given, %zu needed", workspace_bytes, need);
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return fail(ISA_ERR_WORKSPACE, "workspace not 256-byte aligned");
  Work w;
  workspace_layout(p, &w, static_cast<char*>(workspace));
  w.lse = lse;
  static_assert(kCtrlError == 0, "the error word is the first control word");
  const int skip = keep_error ? 1 : 0;
  cudaError_t e = cudaMemsetAsync(w.ctrl + skip, 0, sizeof(uint32_t) * (kCtrlWords - skip + 2 * (size_t)p.BH), s);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the workspace counters");
  if ((e = mark(0, s)) != cudaSuccess) return cuda_fail(e, "recording a stage event");
  if ((e = launch_pool_score_topk(q, k, v, p, w, s)) != cudaSuccess) return cuda_fail(e, "pool/score/top-k launch");
  if ((e = mark(1, s)) != cudaSuccess) return cuda_fail(e, "recording a stage event");
  if ((e = launch_gather(k, v, p, w, s)) != cudaSuccess) return cuda_fail(e, "gather launch");
  if ((e = mark(2, s)) != cudaSuccess) return cuda_fail(e, "recording a stage event");
  if ((e = launch_route(p, w, s)) != cudaSuccess) return cuda_fail(e, "routing launch");
  if ((e = launch_transpose_v(v, p, w, s)) != cudaSuccess) return cuda_fail(e, "V transpose launch");
  if ((e = mark(3, s)) != cudaSuccess) return cuda_fail(e, "recording a stage event");
  {
    // with alpha_ns > 0 the Taylor query blocks go to their own launch; the first one then
    // takes the exact items only (its plan has no flat blocks; the route lists are unchanged)
    Plan pe = p;
    if (p.k_ns > 0) pe.n_flat = 0;
    e = use_pair_kernel(pe) ? launch_attention_pair(q, k, v, out, pe, w, s, nullptr)
                                     : launch_attention(q, k, v, out, pe, w, s, nullptr);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    if (p.k_ns > 0 && p.n_flat > 0) {
      e = attention_mixed_supported(p) ? launch_attention_mixed(q, k, v, out, p, w, s)
                                       : launch_attention_ns(q, k, v, out, p, w, s);
      if (e != cudaSuccess) return cuda_fail(e, "mixed Taylor attention launch");
    }
  }
  if ((e = mark(4, s)) != cudaSuccess) return cuda_fail(e, "recording a stage event");
  if (dbg_sel && p.k > 0) {
    e = cudaMemcpyAsync(dbg_sel, w.sel, sizeof(int32_t) * (size_t)p.BH * p.k, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "copying dbg_sel");
  }
  if (dbg_route) {
    e = cudaMemcpyAsync(dbg_route, w.route, sizeof(int32_t) * (size_t)p.BH * p.n_q, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "copying dbg_route");
  }
  return ISA_OK;
}

int check_io(const void* q, const void* k, const void* v, const void* out, const Plan& p) {
  if (!q || !k || !v || !out) return fail(ISA_ERR_ARG, "q, k, v and out must not be NULL");
  const size_t bytes = (size_t)p.BH * p.N * p.D * p.elem;
  if (overlaps(out, q, bytes) || overlaps(out, k, bytes) || overlaps(out, v, bytes))
    return fail(ISA_ERR_ARG, "out must not overlap q, k or v");
  return ISA_OK;
}

// Device buffers are read and written by bulk and tensor copies, which need 16-byte
// aligned addresses: a misaligned pointer is an argument error, not a launch.
int check_aligned(const void* q, const void* k, const void* v, const void* out) {
  const void* ptrs[4] = {q, k, v, out};
  const char* names[4] = {"q", "k", "v", "out"};
  for (int i = 0; i < 4; ++i)
    if (ptrs[i] && (reinterpret_cast<uintptr_t>(ptrs[i]) & 15))
      return fail(ISA_ERR_ARG, "%s must be 16-byte aligned (device address %p)", names[i], ptrs[i]);
  return ISA_OK;
}

int check_device_io(const void* q, const void* k, const void* v, const void* out, const Plan& p) {
  const int rc = check_io(q, k, v, out, p);
  return rc != ISA_OK ? rc : check_aligned(q, k, v, out);
}

int read_status(void* workspace, cudaStream_t s) {
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "synchronising the stream");
  uint32_t word = 0;
  e = cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (word) {
    cudaMemset(workspace, 0, sizeof(word));
    return fail(ISA_ERR_TIMEOUT, "a kernel wait timed out (error word 0x%x)", word);
  }
  return ISA_OK;
}

// Device buffers of the host-buffer entry points come from a stream-ordered memory pool that
// belongs to this library (one per device, created on first use), not from the device's default
// pool: its release threshold is raised so that repeated calls reuse the memory instead of
// returning it to the driver, and the caller's pools keep whatever settings they had.
int host_pool(cudaMemPool_t* out) {
  static cudaMemPool_t pools[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(ISA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!pools[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool;
    if ((e = cudaMemPoolCreate(&pool, &props)) != cudaSuccess) return cuda_fail(e, "creating the library's memory pool");
    uint64_t thr = UINT64_MAX;
    if ((e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &thr)) != cudaSuccess)
      return cuda_fail(e, "configuring the library's memory pool");
    pools[dev] = pool;
  }
  *out = pools[dev];
  return ISA_OK;
}

// Streams of the host-buffer entry points, one set per device (created on first use): copies in,
// the pass, copies out.
struct HostStreams {
  cudaStream_t in, comp, out;
};
int host_streams(HostStreams* out) {
  static HostStreams streams[64] = {};
  static bool made[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(ISA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!made[dev]) {
    HostStreams hs;
    if ((e = cudaStreamCreateWithFlags(&hs.in, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&hs.comp, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&hs.out, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(e, "creating the library's streams");
    streams[dev] = hs;
    made[dev] = true;
  }
  *out = streams[dev];
  return ISA_OK;
}

// The pass on host buffers (alpha_ns as for isa_forward_ns), synchronous. The (batch, head) slices
// are independent, so the call runs as a pipeline over chunks of slices on three streams: the
// inputs of chunk c + 1 are copied in while chunk c is computed and chunk c - 1 is copied out
// (the two copy directions use separate copy engines), which hides the pass and the output copy
// behind the input copy.
int host_forward(const void* q, const void* k, const void* v, int B, int H, int L_src, int L_ctx, int D, int b,
                 float alpha_s, float alpha_f, float alpha_ns, isa_dtype dt, void* out, int32_t* dbg_sel,
                 int32_t* dbg_route) {
  Plan p;
  int rc = make_plan(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, (int)dt, &p, alpha_ns);
  if (rc != ISA_OK) return rc;
  if ((rc = check_io(q, k, v, out, p)) != ISA_OK) return rc;
  // chunks of cs slices (about 8 chunks; the last may be smaller)
  const int cs = (p.BH + 7) / 8;
  const int nch = (p.BH + cs - 1) / cs;
  Plan pc;  // plan of a full chunk (a chunk is the [1, cs, N, D] call of its slices)
  if ((rc = make_plan(1, cs, L_src, L_ctx, D, b, alpha_s, alpha_f, (int)dt, &pc, alpha_ns)) != ISA_OK) return rc;
  const size_t io = align256((size_t)p.BH * p.N * p.D * p.elem);
  const size_t ws_bytes = workspace_layout(pc, nullptr, nullptr);
  const size_t sel_b = align256(sizeof(int32_t) * (size_t)p.BH * (p.k > 0 ? p.k : 1));
  const size_t route_b = align256(sizeof(int32_t) * (size_t)p.BH * p.n_q);
  const size_t total = 4 * io + ws_bytes + sel_b + route_b;
  HostStreams hs;
  if ((rc = host_streams(&hs)) != ISA_OK) return rc;
  cudaMemPool_t pool;
  if ((rc = host_pool(&pool)) != ISA_OK) return rc;
  cudaEvent_t ev[2 * 8 + 2];
  int n_ev = 0;
  for (; n_ev < 2 * nch + 2; ++n_ev) {
    const cudaError_t e = cudaEventCreateWithFlags(&ev[n_ev], cudaEventDisableTiming);
    if (e != cudaSuccess) {
      for (int i = 0; i < n_ev; ++i) cudaEventDestroy(ev[i]);
      return cuda_fail(e, "creating events");
    }
  }
  cudaEvent_t ev_alloc = ev[2 * nch], ev_end = ev[2 * nch + 1];
  char* dev_buf = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&dev_buf), total, pool, hs.comp);
  if (e != cudaSuccess) {
    for (int i = 0; i < n_ev; ++i) cudaEventDestroy(ev[i]);
    return cuda_fail(e, "allocating device buffers");
  }
  char* dq = dev_buf;
  char* dk = dq + io;
  char* dv = dk + io;
  char* dout = dv + io;
  char* dws = dout + io;
  int32_t* dsel = reinterpret_cast<int32_t*>(dws + ws_bytes);
  int32_t* droute = reinterpret_cast<int32_t*>(dws + ws_bytes + sel_b);
  const size_t slice = (size_t)p.N * p.D * p.elem;
  rc = ISA_OK;
  if ((e = cudaEventRecord(ev_alloc, hs.comp)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(hs.in, ev_alloc, 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(hs.out, ev_alloc, 0)) != cudaSuccess)
    rc = cuda_fail(e, "ordering the streams");
  for (int c = 0; c < nch && rc == ISA_OK; ++c) {
    const int s0 = c * cs, ns = (p.BH - s0) < cs ? (p.BH - s0) : cs;
    const size_t off = (size_t)s0 * slice, nbytes = (size_t)ns * slice;
    Plan pk = pc;
    if (ns != cs && (rc = make_plan(1, ns, L_src, L_ctx, D, b, alpha_s, alpha_f, (int)dt, &pk, alpha_ns)) != ISA_OK)
      break;
    const char* hq = static_cast<const char*>(q) + off;
    const char* hk = static_cast<const char*>(k) + off;
    const char* hv = static_cast<const char*>(v) + off;
    if ((e = cudaMemcpyAsync(dq + off, hq, nbytes, cudaMemcpyHostToDevice, hs.in)) != cudaSuccess ||
        (e = cudaMemcpyAsync(dk + off, hk, nbytes, cudaMemcpyHostToDevice, hs.in)) != cudaSuccess ||
        (e = cudaMemcpyAsync(dv + off, hv, nbytes, cudaMemcpyHostToDevice, hs.in)) != cudaSuccess ||
        (e = cudaEventRecord(ev[2 * c], hs.in)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(hs.comp, ev[2 * c], 0)) != cudaSuccess) {
      rc = cuda_fail(e, "copying inputs to the device");
      break;
    }
    int32_t* csel = dsel + (size_t)s0 * p.k;
    int32_t* croute = droute + (size_t)s0 * p.n_q;
    rc = run_forward(dq + off, dk + off, dv + off, pk, dout + off, dbg_sel ? csel : nullptr,
                     dbg_route ? croute : nullptr, dws, ws_bytes, hs.comp, /*keep_error=*/c > 0);
    if (rc != ISA_OK) break;
    if ((e = cudaEventRecord(ev[2 * c + 1], hs.comp)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(hs.out, ev[2 * c + 1], 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(static_cast<char*>(out) + off, dout + off, nbytes, cudaMemcpyDeviceToHost, hs.out)) !=
            cudaSuccess) {
      rc = cuda_fail(e, "copying the output to the host");
      break;
    }
    if (dbg_sel && p.k > 0 &&
        (e = cudaMemcpyAsync(dbg_sel + (size_t)s0 * p.k, csel, sizeof(int32_t) * (size_t)ns * p.k,
                             cudaMemcpyDeviceToHost, hs.out)) != cudaSuccess) {
      rc = cuda_fail(e, "copying dbg_sel to the host");
      break;
    }
    if (dbg_route && (e = cudaMemcpyAsync(dbg_route + (size_t)s0 * p.n_q, croute,
                                          sizeof(int32_t) * (size_t)ns * p.n_q, cudaMemcpyDeviceToHost, hs.out)) !=
                         cudaSuccess) {
      rc = cuda_fail(e, "copying dbg_route to the host");
      break;
    }
  }
  // whatever happened: the buffers are released only after every copy and kernel that uses them
  if ((e = cudaEventRecord(ev_end, hs.out)) == cudaSuccess) e = cudaStreamWaitEvent(hs.comp, ev_end, 0);
  if (e != cudaSuccess) {
    cudaStreamSynchronize(hs.in);
    cudaStreamSynchronize(hs.out);
  }
  cudaStreamSynchronize(hs.in);
  const int st = read_status(dws, hs.comp);
  if (rc == ISA_OK) rc = st;
  cudaFreeAsync(dev_buf, hs.comp);
  e = cudaStreamSynchronize(hs.comp);
  if (rc == ISA_OK && e != cudaSuccess) rc = cuda_fail(e, "releasing device buffers");
  for (int i = 0; i < n_ev; ++i) cudaEventDestroy(ev[i]);
  return rc;
}

// Variable-length batches: element i of the batch is its own [1, H, N_i, D] call. Checks the
// per-element arguments and returns the plans, the largest workspace and the element sizes.
int varlen_plans(int B, int H, const int32_t* L_src, const int32_t* L_ctx, int D, int b, float alpha_s,
                 float alpha_f, int dt, Plan* plans, size_t* ws_max, size_t* total_elems) {
  if (B <= 0) return fail(ISA_ERR_ARG, "B must be positive (B=%d)", B);
  if (!L_src || !L_ctx) return fail(ISA_ERR_ARG, "the length arrays L_src and L_ctx must not be NULL");
  size_t mx = 0, tot = 0;
  for (int i = 0; i < B; ++i) {
    const int rc = make_plan(1, H, L_src[i], L_ctx[i], D, b, alpha_s, alpha_f, dt, &plans[i]);
    if (rc != ISA_OK) {
      char msg[512];
      snprintf(msg, sizeof(msg), "%s", g_err);
      return fail(rc, "batch element %d: %s", i, msg);
    }
    const size_t ws = workspace_layout(plans[i], nullptr, nullptr);
    if (ws > mx) mx = ws;
    tot += (size_t)H * plans[i].N * D;
  }
  if (ws_max) *ws_max = mx;
  if (total_elems) *total_elems = tot;
  return ISA_OK;
}

constexpr int kMaxVarlenBatch = 4096;

}  // namespace
}  // namespace isa

using namespace isa;

extern "C" {

const char* isa_last_error(void) { return g_err; }

int isa_plan(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, float alpha_f, int32_t* n_q,
             int32_t* k, int32_t* n_flat) {
  Plan p;
  int rc = make_plan(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, ISA_BF16, &p);
  if (rc != ISA_OK) return rc;
  if (n_q) *n_q = p.n_q;
  if (k) *k = p.k;
  if (n_flat) *n_flat = p.n_flat;
  return ISA_OK;
}

size_t isa_workspace_bytes(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, isa_dtype dt) {
  Plan p;
  if (make_plan(B, H, L_src, L_ctx, D, b, alpha_s, 0.0f, (int)dt, &p) != ISA_OK) return 0;
  return workspace_layout(p, nullptr, nullptr);
}

int isa_launch_count(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, float alpha_f, isa_dtype dt) {
  Plan p;
  if (make_plan(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, (int)dt, &p) != ISA_OK) return 0;
  return 3 + (p.k > 0 ? 1 : 0) + (p.dt == ISA_F32 ? 1 : 0);
}

int isa_plan_ns(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, float alpha_f, float alpha_ns,
                int32_t* n_q, int32_t* k, int32_t* n_flat, int32_t* k_ns) {
  Plan p;
  int rc = make_plan(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, ISA_BF16, &p, alpha_ns);
  if (rc != ISA_OK) return rc;
  if (n_q) *n_q = p.n_q;
  if (k) *k = p.k;
  if (n_flat) *n_flat = p.n_flat;
  if (k_ns) *k_ns = p.k_ns;
  return ISA_OK;
}

size_t isa_workspace_bytes_ns(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, float alpha_ns,
                              isa_dtype dt) {
  Plan p;
  if (make_plan(B, H, L_src, L_ctx, D, b, alpha_s, 0.0f, (int)dt, &p, alpha_ns) != ISA_OK) return 0;
  return workspace_layout(p, nullptr, nullptr);
}

int isa_launch_count_ns(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, float alpha_f,
                        float alpha_ns, isa_dtype dt) {
  Plan p;
  if (make_plan(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, (int)dt, &p, alpha_ns) != ISA_OK) return 0;
  return 3 + (p.k > 0 ? 1 : 0) + (p.dt == ISA_F32 ? 1 : 0) + (p.k_ns > 0 && p.n_flat > 0 ? 1 : 0);
}

int isa_forward_ns(const void* q, const void* k, const void* v, int B, int H, int L_src, int L_ctx, int D, int b,
                   float alpha_s, float alpha_f, float alpha_ns, isa_dtype dt, void* out, int32_t* dbg_sel,
                   int32_t* dbg_route, int32_t* dbg_ns, void* workspace, size_t workspace_bytes, void* stream) {
  Plan p;
  int rc = make_plan(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, (int)dt, &p, alpha_ns);
  if (rc != ISA_OK) return rc;
  if ((rc = check_device_io(q, k, v, out, p)) != ISA_OK) return rc;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  rc = run_forward(q, k, v, p, out, dbg_sel, dbg_route, workspace, workspace_bytes, s);
  if (rc != ISA_OK || !dbg_ns || p.k_ns == 0) return rc;
  Work w;
  workspace_layout(p, &w, static_cast<char*>(workspace));
  const cudaError_t e = cudaMemcpyAsync(dbg_ns, w.nsel, sizeof(int32_t) * (size_t)p.BH * p.n_q * p.k_ns,
                                        cudaMemcpyDeviceToDevice, s);
  return e == cudaSuccess ? ISA_OK : cuda_fail(e, "copying dbg_ns");
}

int isa_forward_ex(const void* q, const void* k, const void* v, int B, int H, int L_src, int L_ctx, int D, int b,
                   float alpha_s, float alpha_f, isa_dtype dt, void* out, int32_t* dbg_sel, int32_t* dbg_route,
                   void* workspace, size_t workspace_bytes, void* stream) {
  Plan p;
  int rc = make_plan(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, (int)dt, &p);
  if (rc != ISA_OK) return rc;
  if ((rc = check_device_io(q, k, v, out, p)) != ISA_OK) return rc;
  return run_forward(q, k, v, p, out, dbg_sel, dbg_route, workspace, workspace_bytes,
                     static_cast<cudaStream_t>(stream));
}

int isa_forward(const void* q, const void* k, const void* v, int B, int H, int L_src, int L_ctx, int D, int b,
                float alpha_s, float alpha_f, void* out, int32_t* dbg_sel, int32_t* dbg_route) {
  Plan p;
  int rc = make_plan(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, ISA_BF16, &p);
  if (rc != ISA_OK) return rc;
  if ((rc = check_device_io(q, k, v, out, p)) != ISA_OK) return rc;
  const size_t ws_bytes = workspace_layout(p, nullptr, nullptr);
  void* ws = nullptr;
  cudaStream_t s = 0;
  cudaError_t e = cudaMallocAsync(&ws, ws_bytes, s);
  if (e != cudaSuccess) return cuda_fail(e, "allocating the workspace");
  rc = run_forward(q, k, v, p, out, dbg_sel, dbg_route, ws, ws_bytes, s);
  const int st = read_status(ws, s);
  if (rc == ISA_OK) rc = st;
  cudaFreeAsync(ws, s);
  e = cudaStreamSynchronize(s);
  if (rc == ISA_OK && e != cudaSuccess) rc = cuda_fail(e, "freeing the workspace");
  return rc;
}

int isa_forward_host(const void* q, const void* k, const void* v, int B, int H, int L_src, int L_ctx, int D, int b,
                     float alpha_s, float alpha_f, isa_dtype dt, void* out, int32_t* dbg_sel, int32_t* dbg_route) {
  return host_forward(q, k, v, B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, 0.0f, dt, out, dbg_sel, dbg_route);
}

int isa_forward_host_ns(const void* q, const void* k, const void* v, int B, int H, int L_src, int L_ctx, int D,
                        int b, float alpha_s, float alpha_f, float alpha_ns, isa_dtype dt, void* out,
                        int32_t* dbg_sel, int32_t* dbg_route) {
  return host_forward(q, k, v, B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, alpha_ns, dt, out, dbg_sel, dbg_route);
}

int isa_selftest_wait_timeout(void* workspace, int timeout_ms, void* stream) {
  if (!workspace) return fail(ISA_ERR_WORKSPACE, "workspace is NULL");
  if (timeout_ms <= 0 || timeout_ms > 10000) return fail(ISA_ERR_ARG, "timeout_ms must lie in [1, 10000]");
  cudaError_t e = launch_wait_selftest(static_cast<uint32_t*>(workspace), timeout_ms, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return ISA_OK;
}

int isa_selftest_exp2(const float* x, float* y_poly, float* y_ref, int n, void* stream) {
  if (!x || !y_poly || !y_ref || n < 0) return fail(ISA_ERR_ARG, "x, y_poly and y_ref must not be NULL");
  cudaError_t e = launch_exp2_selftest(x, y_poly, y_ref, n, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "exp2 self-test launch");
  return ISA_OK;
}

int isa_set_stage_events(void* const* events, int n_events) {
  if (!events) {
    g_stage_events_on = false;
    return ISA_OK;
  }
  if (n_events != kStageEvents) return fail(ISA_ERR_ARG, "exactly %d events are needed", kStageEvents);
  for (int i = 0; i < kStageEvents; ++i) {
    if (!events[i]) return fail(ISA_ERR_ARG, "event %d is NULL", i);
    g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
  }
  g_stage_events_on = true;
  return ISA_OK;
}

int isa_device_status(void* workspace, void* stream) {
  if (!workspace) return fail(ISA_ERR_WORKSPACE, "workspace is NULL");
  return read_status(workspace, static_cast<cudaStream_t>(stream));
}

int isa_debug_pooled(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, isa_dtype dt,
                     const void* workspace, float* qc, float* kc, float* vc, float* colscore, float* sharp,
                     void* stream) {
  Plan p;
  int rc = make_plan(B, H, L_src, L_ctx, D, b, alpha_s, 0.0f, (int)dt, &p);
  if (rc != ISA_OK) return rc;
  if (!workspace) return fail(ISA_ERR_WORKSPACE, "workspace is NULL");
  Work w;
  workspace_layout(p, &w, static_cast<char*>(const_cast<void*>(workspace)));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t pooled = sizeof(float) * (size_t)p.BH * p.n_q * p.D;
  struct {
    float* dst;
    const float* src;
    size_t bytes;
  } cp[5] = {{qc, w.qc, pooled},
             {kc, w.kc, pooled},
             {vc, w.vc, pooled},
             {colscore, w.colscore, sizeof(float) * (size_t)p.BH * p.n_ctx},
             {sharp, w.sharp, sizeof(float) * (size_t)p.BH * p.n_q}};
  for (auto& c : cp) {
    if (!c.dst) continue;
    cudaError_t e = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "copying pooled intermediates");
  }
  return ISA_OK;
}

}  // extern "C"

extern "C" {

size_t isa_workspace_bytes_varlen(int B, int H, const int32_t* L_src, const int32_t* L_ctx, int D, int b,
                                  float alpha_s, isa_dtype dt) {
  if (B > kMaxVarlenBatch) {
    fail(ISA_ERR_UNSUPPORTED, "at most %d batch elements", kMaxVarlenBatch);
    return 0;
  }
  std::vector<Plan> plans(B > 0 ? B : 1);
  size_t ws = 0;
  if (varlen_plans(B, H, L_src, L_ctx, D, b, alpha_s, 0.0f, (int)dt, plans.data(), &ws, nullptr) != ISA_OK) return 0;
  return ws;
}

int isa_forward_varlen(const void* q, const void* k, const void* v, int B, int H, const int32_t* L_src,
                       const int32_t* L_ctx, int D, int b, float alpha_s, float alpha_f, isa_dtype dt, void* out,
                       int32_t* dbg_sel, int32_t* dbg_route, void* workspace, size_t workspace_bytes,
                       void* stream) {
  if (B > kMaxVarlenBatch) return fail(ISA_ERR_UNSUPPORTED, "at most %d batch elements", kMaxVarlenBatch);
  std::vector<Plan> plans(B > 0 ? B : 1);
  size_t ws_need = 0, total = 0;
  int rc = varlen_plans(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, (int)dt, plans.data(), &ws_need, &total);
  if (rc != ISA_OK) return rc;
  // the whole packed batch: null, overlap and alignment checks over all elements at once
  {
    const size_t bytes = total * (size_t)plans[0].elem;
    if (!q || !k || !v || !out) return fail(ISA_ERR_ARG, "q, k, v and out must not be NULL");
    if (overlaps(out, q, bytes) || overlaps(out, k, bytes) || overlaps(out, v, bytes))
      return fail(ISA_ERR_ARG, "out must not overlap q, k or v");
    if ((rc = check_aligned(q, k, v, out)) != ISA_OK) return rc;
  }
  if (!workspace) return fail(ISA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", ws_need);
  if (workspace_bytes < ws_need)
    return fail(ISA_ERR_WORKSPACE, "workspace too small: %zu bytes given, %zu needed", workspace_bytes, ws_need);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  size_t off = 0, off_sel = 0, off_route = 0;
  for (int i = 0; i < B; ++i) {
    const Plan& p = plans[i];
    const size_t e = off * p.elem;  // every element starts 16-byte aligned: H * N_i * D * elem, D a multiple of 16
    rc = run_forward(static_cast<const char*>(q) + e, static_cast<const char*>(k) + e,
                     static_cast<const char*>(v) + e, p, static_cast<char*>(out) + e,
                     dbg_sel ? dbg_sel + off_sel : nullptr, dbg_route ? dbg_route + off_route : nullptr, workspace,
                     workspace_bytes, s, /*keep_error=*/i > 0);
    if (rc != ISA_OK) {
      char msg[512];
      snprintf(msg, sizeof(msg), "%s", g_err);
      return fail(rc, "batch element %d: %s", i, msg);
    }
    off += (size_t)H * p.N * p.D;
    off_sel += (size_t)H * p.k;
    off_route += (size_t)H * p.n_q;
  }
  return ISA_OK;
}

}  // extern "C"

extern "C" {

int isa_forward_train(const void* q, const void* k, const void* v, int B, int H, int L_src, int L_ctx, int D, int b,
                      float alpha_s, float alpha_f, isa_dtype dt, void* out, float* lse, void* workspace,
                      size_t workspace_bytes, void* stream) {
  Plan p;
  int rc = make_plan(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, (int)dt, &p);
  if (rc != ISA_OK) return rc;
  if ((rc = check_device_io(q, k, v, out, p)) != ISA_OK) return rc;
  if (!lse) return fail(ISA_ERR_ARG, "lse must not be NULL");
  if (reinterpret_cast<uintptr_t>(lse) & 15) return fail(ISA_ERR_ARG, "lse must be 16-byte aligned");
  const size_t lse_bytes = sizeof(float) * (size_t)p.BH * p.N, io = (size_t)p.BH * p.N * p.D * p.elem;
  if (overlaps2(lse, lse_bytes, q, io) || overlaps2(lse, lse_bytes, k, io) || overlaps2(lse, lse_bytes, v, io) ||
      overlaps2(lse, lse_bytes, out, io) || overlaps2(lse, lse_bytes, workspace, workspace_bytes))
    return fail(ISA_ERR_ARG, "lse must not overlap q, k, v, out or the workspace");
  return run_forward(q, k, v, p, out, nullptr, nullptr, workspace, workspace_bytes, static_cast<cudaStream_t>(stream),
                     false, lse);
}

size_t isa_backward_workspace_bytes(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, isa_dtype dt) {
  Plan p;
  if (make_plan(B, H, L_src, L_ctx, D, b, alpha_s, 0.0f, (int)dt, &p) != ISA_OK) return 0;
  return backward_workspace_bytes(p);
}

int isa_backward(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
                 int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, float alpha_f, isa_dtype dt,
                 void* dq, void* dk, void* dv, void* fwd_workspace, size_t fwd_workspace_bytes, void* bwd_workspace,
                 size_t bwd_workspace_bytes, void* stream) {
  Plan p;
  int rc = make_plan(B, H, L_src, L_ctx, D, b, alpha_s, alpha_f, (int)dt, &p);
  if (rc != ISA_OK) return rc;
  if (!backward_supported(p))
    return fail(ISA_ERR_UNSUPPORTED, "the backward pass needs bfloat16 inputs, D = 128 and lengths that b divides");
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv)
    return fail(ISA_ERR_ARG, "q, k, v, out, lse, dout, dq, dk and dv must not be NULL");
  const void* in[6] = {q, k, v, out, lse, dout};
  void* grads[3] = {dq, dk, dv};
  const size_t io = (size_t)p.BH * p.N * p.D * p.elem;
  for (int i = 0; i < 6; ++i)
    if (reinterpret_cast<uintptr_t>(in[i]) & 15) return fail(ISA_ERR_ARG, "every pointer must be 16-byte aligned");
  for (int g = 0; g < 3; ++g) {
    if (reinterpret_cast<uintptr_t>(grads[g]) & 15) return fail(ISA_ERR_ARG, "every pointer must be 16-byte aligned");
    for (int i = 0; i < 6; ++i)
      if (overlaps2(grads[g], io, in[i], i == 4 ? sizeof(float) * (size_t)p.BH * p.N : io))
        return fail(ISA_ERR_ARG, "dq, dk and dv must not overlap the inputs");
    for (int h = 0; h < g; ++h)
      if (overlaps(grads[g], grads[h], io)) return fail(ISA_ERR_ARG, "dq, dk and dv must not overlap each other");
  }
  const size_t need_f = workspace_layout(p, nullptr, nullptr), need_b = backward_workspace_bytes(p);
  if (!fwd_workspace || fwd_workspace_bytes < need_f)
    return fail(ISA_ERR_WORKSPACE, "the forward workspace (%zu bytes needed) must be the one of the forward call",
                need_f);
  if (!bwd_workspace || bwd_workspace_bytes < need_b)
    return fail(ISA_ERR_WORKSPACE, "backward workspace too small: %zu bytes given, %zu needed", bwd_workspace_bytes,
                need_b);
  if ((reinterpret_cast<uintptr_t>(fwd_workspace) | reinterpret_cast<uintptr_t>(bwd_workspace)) & 255)
    return fail(ISA_ERR_WORKSPACE, "workspaces must be 256-byte aligned");
  Work w;
  workspace_layout(p, &w, static_cast<char*>(fwd_workspace));
  const cudaError_t e = launch_backward(q, k, v, out, lse, dout, dq, dk, dv, p, w, bwd_workspace,
                                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ISA_OK : cuda_fail(e, "backward launch");
}

}  // extern "C"
