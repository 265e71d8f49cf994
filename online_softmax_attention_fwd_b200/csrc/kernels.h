// kernels.h -- internal launcher interface between the C ABI (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "attn.h"

namespace attn {

// A prefill problem. Dense: q [B, Sq, Hq, D], k / v [B, Sk, Hkv, D], lse [B, Hq, Sq]. Packed
// (cu_q != nullptr): B sequences of different lengths, q [Tq, Hq, D], k / v [Tk, Hkv, D], lse
// [Hq, Tq]; sequence b owns rows cu_q[b] .. cu_q[b + 1] - 1 (device arrays), and Sq / Sk are the
// longest sequence's lengths (upper bounds the host passes; the kernels read the real ones).
struct Problem {
  int B, Hq, Hkv, Sq, Sk, D;
  int causal;
  float scale;
  const int* cu_q = nullptr;
  const int* cu_k = nullptr;
  int Tq = 0, Tk = 0;
  // FP8 inputs: the real Q K^T is qk_scale times the product of the codes' values, the real V is
  // v_scale times V's; 1 for bf16.
  float qk_scale = 1.f, v_scale = 1.f;
};

// Brackets one kernel launch: counts it (attn_launch_count) and, while the opt-in profiler is on,
// records CUDA events around it on the launch stream (attn_profile_*). `name` is a static string.
class LaunchScope {
 public:
  LaunchScope(const char* name, cudaStream_t st);
  ~LaunchScope();

 private:
  const char* name_;
  cudaStream_t st_;
  int slot_;
};
// Launch of a kernel that follows another kernel of the same call on the same stream, with
// programmatic dependent launch: its CTAs may be scheduled while the previous kernel's last CTAs
// finish, and it must execute griddep_wait() before it touches anything the previous kernel
// writes (or anything written before that kernel, which the previous kernel waited for).
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Device pointer of the library's status word on the current device (nullptr if unavailable).
int* device_status_ptr();

// Test-only fault injection (built only with ATTN_FAULT_INJECT, into a separate test library):
// the producer warp of CTA 0 of the selected kernel family (0 forward, 1 backward, 2 decode split)
// skips the copy of its load number `block`, so that a consumer's bounded wait runs out and the
// kernel takes its timeout path. -1 = off. Read by the launchers when they build kernel arguments.
#ifdef ATTN_FAULT_INJECT
int fault_block_for(int family);
#endif

// Identity of the CUDA context current on this thread (cuCtxGetId; 0 if there is none or it cannot
// be read). A device address of one of this library's __device__ arrays is valid for one context:
// a context torn down and created again (cudaDeviceReset, a primary context released and retained
// again) loads the module again, possibly at another address.
unsigned long long current_context_id();

// Per-device cache of one symbol's device address, keyed to the context it was looked up in; a
// lookup under another context (or with an unidentifiable one) misses. Callers hold their own lock.
constexpr int kMaxCachedDevices = 64;
struct ContextCache {
  unsigned long long ctx[kMaxCachedDevices] = {};
  void* ptr[kMaxCachedDevices] = {};
  bool lookup(int dev, void** out);
  void store(int dev, void* p);
};

// True if the current device is an sm_100 part (cached per device).
bool device_is_sm100();

// Host-side checks shared by the packed split-KV decode entry points (attn_decode_splitkv and the
// one without a workspace): sizes, split range, null and 16-byte alignment of every pointer, head dim.
attn_status_t check_decode_args(const void* q, const void* k, const void* v, const int* kv_offsets,
                                const int* num_splits, int max_splits, const void* o, const float* lse, int N,
                                int Hq, int Hkv, int D);

// Records the kernel family of a successful call for attn_last_path (kind 0 forward, 1 backward,
// 2 decode), per calling thread.
void set_last_path(int kind, const char* name);

// simt.cu: CUDA-core kernels, any D in [1, 256].
cudaError_t launch_fwd_simt_f32(const Problem& p, const float* q, const float* k, const float* v, float* o,
                                float* lse, cudaStream_t st);
cudaError_t launch_bwd_simt_f32(const Problem& p, const float* q, const float* k, const float* v, const float* o,
                                const float* lse, const float* dout, float* dq, float* dk, float* dv,
                                float* delta, cudaStream_t st);

// decode.cu: split-KV decode, D in {64, 128}.
// q_len query tokens per stream (the newest q_len positions of its cache; 1 for plain decode):
// q and o are [N, q_len, Hq, D], lse [N, Hq, q_len], and the workspace holds
// decode_workspace_bytes(N * q_len, Hq, D, max_splits) bytes.
struct DecodeProblem {
  int N, Hq, Hkv, D, max_splits;
  float scale;
  int q_len;
};
size_t decode_workspace_bytes(int N, int Hq, int D, int max_splits);
int decode_default_splits(int L, int max_splits);
cudaError_t launch_decode(const DecodeProblem& p, const void* q, const void* k, const void* v,
                          const int* kv_offsets, const int* num_splits, void* o, float* lse, void* workspace,
                          cudaStream_t st);
// The same split + combine over a paged cache: key t of stream n is row t % page_size of page
// block_table[n * max_pages + t / page_size] of the pools k_pages / v_pages [num_pages, page_size,
// Hkv, D]; stream n has seq_lens[n] keys. page_size is a multiple of 16.
cudaError_t launch_decode_paged(const DecodeProblem& p, const void* q, const void* k_pages, const void* v_pages,
                                const int* block_table, int max_pages, const int* seq_lens, int page_size,
                                int num_pages, const int* num_splits, void* o, float* lse, void* workspace,
                                cudaStream_t st);

// merge.cu: folds a bf16 partial attention (o_part [B, S, H, D], lse_part [B, H, S]) into an fp32
// running one (o_acc, lse_acc, same layouts) with the monoid, in place; optionally writes the merged
// O rounded to bf16 into o_out. D in {64, 128}.
cudaError_t launch_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                         int S, int H, int D, cudaStream_t st);

// fwd_sm100.cu: tcgen05 / TMA forward, bf16, D in {64, 128}; and the same with e4m3 Q, K, V
// (kind::f8f6f4, bf16 O), D = 128.
cudaError_t launch_fwd_sm100(const Problem& p, const void* q, const void* k, const void* v, void* o, float* lse,
                             cudaStream_t st);
cudaError_t launch_fwd_sm100_fp8(const Problem& p, const void* q, const void* k, const void* v, void* o, float* lse,
                                 cudaStream_t st);

// bwd_sm100.cu: tcgen05 / TMA backward, bf16, D in {64, 128}; workspace = fp32 dQ accumulator
// [B, Hq, Sq_pad, D] + lse2 [B, Hq, Sq_pad] + Delta [B, Hq, Sq_pad], each 256-byte aligned (Sq_pad =
// Sq rounded up to 128).
size_t bwd_sm100_workspace_bytes(int B, int Hq, int Hkv, int Sq, int Sk, int D);
cudaError_t launch_bwd_sm100(const Problem& p, const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                             cudaStream_t st);

}  // namespace attn
