// api.cu -- the extern "C" boundary of libattn.so (declared in include/attn.h).
//
// Host-side only: argument validation (before anything is launched), dispatch to the kernel
// families, the device status word read by attn_get_device_status, and a launch counter. Nothing
// here allocates device memory or synchronises, except attn_get_device_status.
#include <math.h>

#include <atomic>
#include <mutex>
#include <string.h>
#include <vector>

#include <cuda_runtime.h>

#include "attn.h"
#include "kernels.h"

namespace attn {
namespace {

std::atomic<uint64_t> g_launches{0};
thread_local const char* g_last_path[3] = {"none", "none", "none"};

constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
int g_dev_arch[kMaxDevices];        // 0 = unknown, else major*10 + minor

}  // namespace

__device__ int g_status_word = 0;

// ---------------------------------------------------------------------------------------------
// Opt-in per-kernel timing: while on, every launch is bracketed by two CUDA events recorded on its
// stream; attn_profile_stop() waits for them and sums the elapsed time per kernel family.
// ---------------------------------------------------------------------------------------------
namespace {
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
};
struct ProfSum {
  const char* name;
  double ms;
  int launches;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof_recs;
std::vector<cudaEvent_t> g_prof_pool;
std::vector<ProfSum> g_prof_sums;

cudaEvent_t prof_event() {
  if (!g_prof_pool.empty()) {
    cudaEvent_t e = g_prof_pool.back();
    g_prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}
}  // namespace

LaunchScope::LaunchScope(const char* name, cudaStream_t st) : name_(name), st_(st), slot_(-1) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on) return;
  ProfRec r{name, prof_event(), prof_event()};
  if (!r.a || !r.b) return;
  cudaEventRecord(r.a, st);
  slot_ = static_cast<int>(g_prof_recs.size());
  g_prof_recs.push_back(r);
}

LaunchScope::~LaunchScope() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (slot_ < 0) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (slot_ < static_cast<int>(g_prof_recs.size())) cudaEventRecord(g_prof_recs[slot_].b, st_);
}

static int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return (dev >= 0 && dev < kMaxDevices) ? dev : -1;
}

namespace {
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name, int version) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, &p, version, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(p);
}
}  // namespace

unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent", 12000);
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId", 12000);
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

bool ContextCache::lookup(int dev, void** out) {
  const unsigned long long id = current_context_id();
  if (id == 0 || dev < 0 || dev >= kMaxCachedDevices || ctx[dev] != id || !ptr[dev]) return false;
  *out = ptr[dev];
  return true;
}

void ContextCache::store(int dev, void* p) {
  if (dev < 0 || dev >= kMaxCachedDevices) return;
  ctx[dev] = current_context_id();  // 0 (never matched) if the context cannot be identified
  ptr[dev] = p;
}

namespace {
ContextCache g_status_cache;
}  // namespace

int* device_status_ptr() {
  const int dev = current_device();
  if (dev < 0) return nullptr;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  void* p = nullptr;
  if (g_status_cache.lookup(dev, &p)) return static_cast<int*>(p);
  if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
  g_status_cache.store(dev, p);
  return static_cast<int*>(p);
}

bool device_is_sm100() {
  const int dev = current_device();
  if (dev < 0) return false;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_dev_arch[dev]) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return false;
    g_dev_arch[dev] = major * 10 + minor;
  }
  return g_dev_arch[dev] == 100;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static attn_status_t check_problem(const Problem& p) {
  if (p.B <= 0 || p.Hq <= 0 || p.Hkv <= 0 || p.Sq <= 0 || p.Sk <= 0 || p.D <= 0) return ATTN_ERR_INVALID_ARG;
  if (p.Hq % p.Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (p.causal != 0 && p.causal != 1) return ATTN_ERR_INVALID_ARG;
  // every index stays inside 32-bit element counts per tensor row set; whole tensors may be larger
  const long long qel = static_cast<long long>(p.B) * p.Sq * p.Hq * p.D;
  const long long kel = static_cast<long long>(p.B) * p.Sk * p.Hkv * p.D;
  if (qel >= (1ll << 40) || kel >= (1ll << 40)) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

template <typename... P>
static attn_status_t check_ptrs(P... ptrs) {
  const void* all[] = {static_cast<const void*>(ptrs)...};
  for (const void* x : all)
    if (!x) return ATTN_ERR_INVALID_ARG;
  for (const void* x : all)
    if (!aligned16(x)) return ATTN_ERR_ALIGNMENT;
  return ATTN_OK;
}

static attn_status_t launch_status(cudaError_t e) { return e == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH; }

attn_status_t check_decode_args(const void* q, const void* k, const void* v, const int* kv_offsets,
                                const int* num_splits, int max_splits, const void* o, const float* lse, int N,
                                int Hq, int Hkv, int D) {
  if (N <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (max_splits < 1 || max_splits > 64) return ATTN_ERR_INVALID_ARG;
  if (N > 65535 || static_cast<long long>(N) * Hq >= (1ll << 31)) return ATTN_ERR_INVALID_ARG;
  attn_status_t s = check_ptrs(q, k, v, kv_offsets, o);
  if (s != ATTN_OK) return s;
  if (num_splits && !aligned16(num_splits)) return ATTN_ERR_ALIGNMENT;
  if (lse && !aligned16(lse)) return ATTN_ERR_ALIGNMENT;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

void set_last_path(int kind, const char* name) {
  if (kind >= 0 && kind < 3) g_last_path[kind] = name;
}

#ifdef ATTN_FAULT_INJECT
int g_fault_family = -1, g_fault_block = -1;
int fault_block_for(int family) { return family == g_fault_family ? g_fault_block : -1; }
#endif

}  // namespace attn

using namespace attn;

extern "C" {

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                       int Sq, int Sk, int D, int causal, float scale, attn_stream_t stream) {
  const Problem p{B, Hq, Hkv, Sq, Sk, D, causal, scale};
  attn_status_t s = check_problem(p);
  if (s != ATTN_OK) return s;
  if ((s = check_ptrs(q, k, v, o, lse)) != ATTN_OK) return s;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!device_is_sm100()) return ATTN_ERR_UNSUPPORTED;
  const cudaError_t e = launch_fwd_sm100(p, q, k, v, o, lse, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) set_last_path(0, "fwd_sm100_tcgen05");
  return launch_status(e);
}

attn_status_t attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, float q_scale,
                           float k_scale, float v_scale, int B, int Hq, int Hkv, int Sq, int Sk, int D, int causal,
                           float scale, attn_stream_t stream) {
  Problem p{B, Hq, Hkv, Sq, Sk, D, causal, scale};
  p.qk_scale = q_scale * k_scale;
  p.v_scale = v_scale;
  attn_status_t s = check_problem(p);
  if (s != ATTN_OK) return s;
  if (!(q_scale > 0.f) || !(k_scale > 0.f) || !(v_scale > 0.f) || !isfinite(p.qk_scale) || !isfinite(v_scale))
    return ATTN_ERR_INVALID_ARG;
  if ((s = check_ptrs(q, k, v, o, lse)) != ATTN_OK) return s;
  if (D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!device_is_sm100()) return ATTN_ERR_UNSUPPORTED;
  const cudaError_t e = launch_fwd_sm100_fp8(p, q, k, v, o, lse, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) set_last_path(0, "fwd_sm100_tcgen05_fp8");
  return launch_status(e);
}

attn_status_t attn_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int Hq,
                           int Hkv, int Sq, int Sk, int D, int causal, float scale, attn_stream_t stream) {
  const Problem p{B, Hq, Hkv, Sq, Sk, D, causal, scale};
  attn_status_t s = check_problem(p);
  if (s != ATTN_OK) return s;
  if ((s = check_ptrs(q, k, v, o, lse)) != ATTN_OK) return s;
  if (D > 256) return ATTN_ERR_UNSUPPORTED;
  if (!device_is_sm100()) return ATTN_ERR_UNSUPPORTED;
  const cudaError_t e = launch_fwd_simt_f32(p, q, k, v, o, lse, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) set_last_path(0, "fwd_simt_f32");
  return launch_status(e);
}

static size_t delta_bytes(int B, int Hq, int Sq) {
  return (static_cast<size_t>(B) * Hq * Sq * sizeof(float) + 255) & ~static_cast<size_t>(255);
}

size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int D) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || Sk <= 0 || D <= 0) return 0;
  return bwd_sm100_workspace_bytes(B, Hq, Hkv, Sq, Sk, D);
}

size_t attn_bwd_f32_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int D) {
  (void)Hkv;
  (void)Sk;
  (void)D;
  if (B <= 0 || Hq <= 0 || Sq <= 0) return 0;
  return delta_bytes(B, Hq, Sq);
}

attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dout, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                       int B, int Hq, int Hkv, int Sq, int Sk, int D, int causal, float scale,
                       attn_stream_t stream) {
  const Problem p{B, Hq, Hkv, Sq, Sk, D, causal, scale};
  attn_status_t s = check_problem(p);
  if (s != ATTN_OK) return s;
  if ((s = check_ptrs(q, k, v, o, lse, dout, dq, dk, dv)) != ATTN_OK) return s;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < attn_bwd_workspace_size(B, Hq, Hkv, Sq, Sk, D)) return ATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_ALIGNMENT;
  if (!device_is_sm100()) return ATTN_ERR_UNSUPPORTED;
  const cudaError_t e = launch_bwd_sm100(p, q, k, v, o, lse, dout, dq, dk, dv, workspace,
                                         static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) set_last_path(1, "bwd_sm100_tcgen05");
  return launch_status(e);
}

attn_status_t attn_bwd_f32(const float* q, const float* k, const float* v, const float* o, const float* lse,
                           const float* dout, float* dq, float* dk, float* dv, void* workspace,
                           size_t workspace_bytes, int B, int Hq, int Hkv, int Sq, int Sk, int D, int causal,
                           float scale, attn_stream_t stream) {
  const Problem p{B, Hq, Hkv, Sq, Sk, D, causal, scale};
  attn_status_t s = check_problem(p);
  if (s != ATTN_OK) return s;
  if ((s = check_ptrs(q, k, v, o, lse, dout, dq, dk, dv)) != ATTN_OK) return s;
  if (D > 256) return ATTN_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < attn_bwd_f32_workspace_size(B, Hq, Hkv, Sq, Sk, D))
    return ATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_ALIGNMENT;
  if (!device_is_sm100()) return ATTN_ERR_UNSUPPORTED;
  const cudaError_t e = launch_bwd_simt_f32(p, q, k, v, o, lse, dout, dq, dk, dv, static_cast<float*>(workspace),
                                            static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) set_last_path(1, "bwd_simt_f32");
  return launch_status(e);
}

static attn_status_t check_varlen(const Problem& p, const int* cu_q, const int* cu_k) {
  if (!cu_q || !cu_k) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_k) & 3u)) return ATTN_ERR_ALIGNMENT;
  if (p.Tq <= 0 || p.Tk <= 0 || p.B > 65535) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(p.Tq) * p.Hq * p.D >= (1ll << 40) || static_cast<long long>(p.Tk) * p.Hkv * p.D >= (1ll << 40))
    return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

attn_status_t attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                              const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                              int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int D, int causal,
                              float scale, attn_stream_t stream) {
  Problem p{B, Hq, Hkv, max_seqlen_q, max_seqlen_k, D, causal, scale};
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.Tq = total_q;
  p.Tk = total_k;
  attn_status_t s = check_problem(p);
  if (s != ATTN_OK) return s;
  if ((s = check_varlen(p, cu_seqlens_q, cu_seqlens_k)) != ATTN_OK) return s;
  if ((s = check_ptrs(q, k, v, o, lse)) != ATTN_OK) return s;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!device_is_sm100()) return ATTN_ERR_UNSUPPORTED;
  const cudaError_t e = launch_fwd_sm100(p, q, k, v, o, lse, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) set_last_path(0, "fwd_sm100_tcgen05_varlen");
  return launch_status(e);
}

size_t attn_bwd_varlen_workspace_size(int B, int Hq, int Hkv, int max_seqlen_q, int max_seqlen_k, int D) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || max_seqlen_q <= 0 || max_seqlen_k <= 0 || D <= 0) return 0;
  return bwd_sm100_workspace_bytes(B, Hq, Hkv, max_seqlen_q, max_seqlen_k, D);
}

attn_status_t attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                              const void* dout, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                              const int* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k, int total_q,
                              int total_k, int Hq, int Hkv, int D, int causal, float scale, void* workspace,
                              size_t workspace_bytes, attn_stream_t stream) {
  Problem p{B, Hq, Hkv, max_seqlen_q, max_seqlen_k, D, causal, scale};
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.Tq = total_q;
  p.Tk = total_k;
  attn_status_t s = check_problem(p);
  if (s != ATTN_OK) return s;
  if ((s = check_varlen(p, cu_seqlens_q, cu_seqlens_k)) != ATTN_OK) return s;
  if ((s = check_ptrs(q, k, v, o, lse, dout, dq, dk, dv)) != ATTN_OK) return s;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < attn_bwd_varlen_workspace_size(B, Hq, Hkv, max_seqlen_q, max_seqlen_k, D))
    return ATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_ALIGNMENT;
  if (!device_is_sm100()) return ATTN_ERR_UNSUPPORTED;
  const cudaError_t e = launch_bwd_sm100(p, q, k, v, o, lse, dout, dq, dk, dv, workspace,
                                         static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) set_last_path(1, "bwd_sm100_tcgen05_varlen");
  return launch_status(e);
}

size_t attn_decode_workspace_size(int N, int Hq, int D, int max_splits) {
  if (N <= 0 || Hq <= 0 || D <= 0 || max_splits <= 0) return 0;
  return decode_workspace_bytes(N, Hq, D, max_splits);
}

int attn_decode_default_splits(int L, int max_splits) {
  if (max_splits <= 0) return 0;
  return decode_default_splits(L < 0 ? 0 : L, max_splits);
}

attn_status_t attn_decode_splitkv(const void* q, const void* k, const void* v, const int* kv_offsets,
                                  const int* num_splits, int max_splits, void* o, float* lse, int N, int Hq,
                                  int Hkv, int D, float scale, void* workspace, size_t workspace_bytes,
                                  attn_stream_t stream) {
  attn_status_t s = check_decode_args(q, k, v, kv_offsets, num_splits, max_splits, o, lse, N, Hq, Hkv, D);
  if (s != ATTN_OK) return s;
  if (!workspace || workspace_bytes < decode_workspace_bytes(N, Hq, D, max_splits)) return ATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_ALIGNMENT;
  if (!device_is_sm100()) return ATTN_ERR_UNSUPPORTED;
  const DecodeProblem p{N, Hq, Hkv, D, max_splits, scale, 1};
  const cudaError_t e = launch_decode(p, q, k, v, kv_offsets, num_splits, o, lse, workspace,
                                      static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) set_last_path(2, "decode_splitkv_mma16816");
  return launch_status(e);
}

static attn_status_t decode_paged_any(const void* q, const void* k_pages, const void* v_pages,
                                      const int* block_table, int max_pages, const int* seq_lens, int page_size,
                                      int num_pages, const int* num_splits, int max_splits, void* o, float* lse,
                                      int N, int q_len, int Hq, int Hkv, int D, float scale, void* workspace,
                                      size_t workspace_bytes, attn_stream_t stream) {
  if (N <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv != 0 || q_len < 1) return ATTN_ERR_INVALID_ARG;
  if (max_splits < 1 || max_splits > 64) return ATTN_ERR_INVALID_ARG;
  if (N > 65535 || static_cast<long long>(N) * q_len * Hq >= (1ll << 31)) return ATTN_ERR_INVALID_ARG;
  if (page_size < 16 || page_size % 16 != 0 || num_pages <= 0 || max_pages <= 0) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(num_pages) * page_size >= (1ll << 31) ||
      static_cast<long long>(max_pages) * page_size >= (1ll << 31) ||
      static_cast<long long>(N) * max_pages >= (1ll << 40))
    return ATTN_ERR_INVALID_ARG;
  attn_status_t s = check_ptrs(q, k_pages, v_pages, block_table, o);
  if (s != ATTN_OK) return s;
  if (!seq_lens) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(seq_lens)) return ATTN_ERR_ALIGNMENT;
  if (num_splits && !aligned16(num_splits)) return ATTN_ERR_ALIGNMENT;
  if (lse && !aligned16(lse)) return ATTN_ERR_ALIGNMENT;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < decode_workspace_bytes(N * q_len, Hq, D, max_splits))
    return ATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_ALIGNMENT;
  if (!device_is_sm100()) return ATTN_ERR_UNSUPPORTED;
  const DecodeProblem p{N, Hq, Hkv, D, max_splits, scale, q_len};
  const cudaError_t e =
      launch_decode_paged(p, q, k_pages, v_pages, block_table, max_pages, seq_lens, page_size, num_pages, num_splits,
                          o, lse, workspace, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess)
    set_last_path(2, q_len == 1 ? "decode_splitkv_paged_mma16816" : "decode_splitkv_paged_qlen_mma16816");
  return launch_status(e);
}

attn_status_t attn_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int* block_table,
                                int max_pages, const int* seq_lens, int page_size, int num_pages,
                                const int* num_splits, int max_splits, void* o, float* lse, int N, int Hq, int Hkv,
                                int D, float scale, void* workspace, size_t workspace_bytes,
                                attn_stream_t stream) {
  return decode_paged_any(q, k_pages, v_pages, block_table, max_pages, seq_lens, page_size, num_pages, num_splits,
                          max_splits, o, lse, N, 1, Hq, Hkv, D, scale, workspace, workspace_bytes, stream);
}

attn_status_t attn_decode_paged_qlen(const void* q, const void* k_pages, const void* v_pages,
                                     const int* block_table, int max_pages, const int* seq_lens, int page_size,
                                     int num_pages, const int* num_splits, int max_splits, void* o, float* lse,
                                     int N, int q_len, int Hq, int Hkv, int D, float scale, void* workspace,
                                     size_t workspace_bytes, attn_stream_t stream) {
  return decode_paged_any(q, k_pages, v_pages, block_table, max_pages, seq_lens, page_size, num_pages, num_splits,
                          max_splits, o, lse, N, q_len, Hq, Hkv, D, scale, workspace, workspace_bytes, stream);
}

attn_status_t attn_decode_splitkv_qlen(const void* q, const void* k, const void* v, const int* kv_offsets,
                                       const int* num_splits, int max_splits, void* o, float* lse, int N,
                                       int q_len, int Hq, int Hkv, int D, float scale, void* workspace,
                                       size_t workspace_bytes, attn_stream_t stream) {
  if (q_len < 1) return ATTN_ERR_INVALID_ARG;
  attn_status_t s = check_decode_args(q, k, v, kv_offsets, num_splits, max_splits, o, lse, N, Hq, Hkv, D);
  if (s != ATTN_OK) return s;
  if (static_cast<long long>(N) * q_len * Hq >= (1ll << 31)) return ATTN_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < decode_workspace_bytes(N * q_len, Hq, D, max_splits))
    return ATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_ALIGNMENT;
  if (!device_is_sm100()) return ATTN_ERR_UNSUPPORTED;
  const DecodeProblem p{N, Hq, Hkv, D, max_splits, scale, q_len};
  const cudaError_t e = launch_decode(p, q, k, v, kv_offsets, num_splits, o, lse, workspace,
                                      static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) set_last_path(2, "decode_splitkv_qlen_mma16816");
  return launch_status(e);
}

attn_status_t attn_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                         int S, int H, int D, attn_stream_t stream) {
  if (B <= 0 || S <= 0 || H <= 0 || D <= 0) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * S * H * D >= (1ll << 40)) return ATTN_ERR_INVALID_ARG;
  attn_status_t s = check_ptrs(o_acc, lse_acc, o_part, lse_part);
  if (s != ATTN_OK) return s;
  if (o_out && !aligned16(o_out)) return ATTN_ERR_ALIGNMENT;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!device_is_sm100()) return ATTN_ERR_UNSUPPORTED;
  return launch_status(launch_merge(o_acc, lse_acc, o_part, lse_part, o_out, B, S, H, D,
                                    static_cast<cudaStream_t>(stream)));
}

#ifdef ATTN_FAULT_INJECT
// Test-only (fault-injection build): see fault_block_for in kernels.h and attn_fault_inject.h.
void attn_fault_inject(int family, int block) {
  attn::g_fault_family = family;
  attn::g_fault_block = block;
}
#endif

const char* attn_status_string(attn_status_t status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported (head dim or device)";
    case ATTN_ERR_ALIGNMENT: return "pointer not aligned";
    case ATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case ATTN_ERR_LAUNCH: return "kernel launch failed";
    case ATTN_ERR_TIMEOUT: return "a bounded on-chip wait timed out";
  }
  return "unknown status";
}

attn_status_t attn_get_device_status(attn_stream_t stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_LAUNCH;
  int value = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&value, g_status_word, sizeof(int)) != cudaSuccess) return ATTN_ERR_LAUNCH;
  if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_LAUNCH;
  return static_cast<attn_status_t>(value);
}

uint64_t attn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

attn_status_t attn_profile_start(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof_recs) {
    g_prof_pool.push_back(r.a);
    g_prof_pool.push_back(r.b);
  }
  g_prof_recs.clear();
  g_prof_sums.clear();
  g_prof_on = true;
  return ATTN_OK;
}

attn_status_t attn_profile_stop(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = false;
  g_prof_sums.clear();
  attn_status_t st = ATTN_OK;
  for (auto& r : g_prof_recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
      st = ATTN_ERR_LAUNCH;
      continue;
    }
    bool found = false;
    for (auto& s : g_prof_sums)
      if (strcmp(s.name, r.name) == 0) {
        s.ms += ms;
        s.launches += 1;
        found = true;
      }
    if (!found) g_prof_sums.push_back(ProfSum{r.name, static_cast<double>(ms), 1});
    g_prof_pool.push_back(r.a);
    g_prof_pool.push_back(r.b);
  }
  g_prof_recs.clear();
  return st;
}

int attn_profile_entries(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  return static_cast<int>(g_prof_sums.size());
}

const char* attn_profile_name(int i) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  return (i >= 0 && i < static_cast<int>(g_prof_sums.size())) ? g_prof_sums[i].name : "";
}

double attn_profile_total_ms(int i) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  return (i >= 0 && i < static_cast<int>(g_prof_sums.size())) ? g_prof_sums[i].ms : 0.0;
}

int attn_profile_launches(int i) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  return (i >= 0 && i < static_cast<int>(g_prof_sums.size())) ? g_prof_sums[i].launches : 0;
}

const char* attn_last_path(int kind) {
  if (kind < 0 || kind > 2) return "none";
  return g_last_path[kind];
}

}  // extern "C"
