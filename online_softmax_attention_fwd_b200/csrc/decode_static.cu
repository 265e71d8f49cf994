// decode_static.cu -- split-KV decode for callers that cannot allocate device memory.
//
// attn_decode_splitkv asks its caller for a workspace buffer that holds the partial (m, l, o)
// triples between the split and combine kernels. Some callers have no way to provide one: a host
// framework that owns every byte of device memory through its own pool and hands plugins no
// workspace, or a latency-bound serving loop where a cudaMalloc (which can synchronise the whole
// device) is not allowed on the hot path. attn_decode_splitkv_static serves them: it runs the very
// same split and combine kernels, but the partial triples live in one fixed array compiled into
// this library (kStaticScratchBytes, 16 MiB), so the call itself allocates nothing.
//
// Rules of use, all stated in include/attn.h:
//  * Every GPU that loads the library holds the 16 MiB array until the process exits.
//  * The first call on a device looks up the array's device address (cudaGetSymbolAddress, once
//    per device, with that device current); make that first call before any stream capture.
//  * Problems whose partial triples need more than 16 MiB are rejected with ATTN_ERR_WORKSPACE
//    before anything is launched.
//  * All calls share the one array, and each call leaves its partial triples there. Nothing needs
//    to start at zero: the split kernel writes every slot the combine kernel then reads. Calls
//    that overlap on the GPU (other streams, other threads) race on the array and give wrong
//    results; serialise them.
#include <mutex>

#include <cuda_runtime.h>

#include "attn.h"
#include "kernels.h"

namespace attn {
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB per device
constexpr int kMaxStaticDevices = 64;

// The scratch itself. Host code must never pass this name to a kernel: on the host it is only a
// stand-in, not a device address. The device address is looked up below.
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_static_mu;
void* g_static_ptr[kMaxStaticDevices];  // device address of g_decode_scratch, per device

// Once per device, with that device current: the device address of the scratch array.
cudaError_t static_scratch_ptr(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxStaticDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return cudaSuccess;
}

bool aligned16_static(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace attn

extern "C" attn_status_t attn_decode_splitkv_static(const void* q, const void* k, const void* v,
                                                    const int* kv_offsets, const int* num_splits,
                                                    int max_splits, void* o, float* lse, int N, int Hq,
                                                    int Hkv, int D, float scale, attn_stream_t stream) {
  using namespace attn;
  if (N <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (max_splits < 1 || max_splits > 64) return ATTN_ERR_INVALID_ARG;
  if (N > 65535 || static_cast<long long>(N) * Hq >= (1ll << 31)) return ATTN_ERR_INVALID_ARG;
  if (!q || !k || !v || !kv_offsets || !o) return ATTN_ERR_INVALID_ARG;
  if (!aligned16_static(q) || !aligned16_static(k) || !aligned16_static(v) || !aligned16_static(kv_offsets) ||
      !aligned16_static(o) || (num_splits && !aligned16_static(num_splits)) || (lse && !aligned16_static(lse)))
    return ATTN_ERR_ALIGNMENT;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (decode_workspace_bytes(N, Hq, D, max_splits) > kStaticScratchBytes) return ATTN_ERR_WORKSPACE;
  int dev = -1, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      major * 10 + minor != 100)
    return ATTN_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (static_scratch_ptr(&scratch) != cudaSuccess) return ATTN_ERR_LAUNCH;
  const DecodeProblem p{N, Hq, Hkv, D, max_splits, scale};
  const cudaError_t e =
      launch_decode(p, q, k, v, kv_offsets, num_splits, o, lse, scratch, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}
