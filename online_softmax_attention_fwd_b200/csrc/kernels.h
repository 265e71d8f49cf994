// kernels.h -- internal launcher interface between the C ABI (api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace attn {

struct Problem {
  int B, Hq, Hkv, Sq, Sk, D;
  int causal;
  float scale;
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

// simt.cu: CUDA-core kernels, any D in [1, 256].
cudaError_t launch_fwd_simt_f32(const Problem& p, const float* q, const float* k, const float* v, float* o,
                                float* lse, cudaStream_t st);
cudaError_t launch_fwd_simt_bf16(const Problem& p, const void* q, const void* k, const void* v, void* o,
                                 float* lse, cudaStream_t st);
cudaError_t launch_bwd_simt_f32(const Problem& p, const float* q, const float* k, const float* v, const float* o,
                                const float* lse, const float* dout, float* dq, float* dk, float* dv,
                                float* delta, cudaStream_t st);
cudaError_t launch_bwd_simt_bf16(const Problem& p, const void* q, const void* k, const void* v, const void* o,
                                 const float* lse, const void* dout, void* dq, void* dk, void* dv, float* delta,
                                 cudaStream_t st);

// decode.cu: split-KV decode, D in {64, 128}.
struct DecodeProblem {
  int N, Hq, Hkv, D, max_splits;
  float scale;
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

// fwd_sm100.cu: tcgen05 / TMA forward, bf16, D in {64, 128}.
cudaError_t launch_fwd_sm100(const Problem& p, const void* q, const void* k, const void* v, void* o, float* lse,
                             cudaStream_t st);

// bwd_sm100.cu: tcgen05 / TMA backward, bf16, D in {64, 128}; workspace = fp32 dQ accumulator
// [B, Sq, Hq, D] + lse2 [B, Hq, Sq] + Delta [B, Hq, Sq], each 256-byte aligned.
size_t bwd_sm100_workspace_bytes(int B, int Hq, int Sq, int D);
cudaError_t launch_bwd_sm100(const Problem& p, const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                             cudaStream_t st);

}  // namespace attn
