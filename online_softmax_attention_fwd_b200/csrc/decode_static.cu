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
//  * The first call on a device looks up the array's device address (cudaGetSymbolAddress, with
//    that device current) and keeps it for the device's current context; the first call after that
//    context has been torn down and created again (cudaDeviceReset) looks it up again, since the
//    module may then be loaded elsewhere. Make each such first call before any stream capture.
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

// The scratch itself. Host code must never pass this name to a kernel: on the host it is only a
// stand-in, not a device address. The device address is looked up below.
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_static_mu;
ContextCache g_static_cache;  // device address of g_decode_scratch, per device and context

// The device address of the scratch array on the current device: looked up once per device and
// context, with that device current.
cudaError_t static_scratch_ptr(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxCachedDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (g_static_cache.lookup(dev, out)) return cudaSuccess;
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess) return e;
  g_static_cache.store(dev, p);
  *out = p;
  return cudaSuccess;
}

}  // namespace
}  // namespace attn

extern "C" attn_status_t attn_decode_splitkv_static(const void* q, const void* k, const void* v,
                                                    const int* kv_offsets, const int* num_splits,
                                                    int max_splits, void* o, float* lse, int N, int Hq,
                                                    int Hkv, int D, float scale, attn_stream_t stream) {
  using namespace attn;
  // the same argument checks as attn_decode_splitkv; only the scratch differs
  attn_status_t s = check_decode_args(q, k, v, kv_offsets, num_splits, max_splits, o, lse, N, Hq, Hkv, D);
  if (s != ATTN_OK) return s;
  if (decode_workspace_bytes(N, Hq, D, max_splits) > kStaticScratchBytes) return ATTN_ERR_WORKSPACE;
  if (!device_is_sm100()) return ATTN_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (static_scratch_ptr(&scratch) != cudaSuccess) return ATTN_ERR_LAUNCH;
  const DecodeProblem p{N, Hq, Hkv, D, max_splits, scale, 1};
  const cudaError_t e =
      launch_decode(p, q, k, v, kv_offsets, num_splits, o, lse, scratch, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return ATTN_ERR_LAUNCH;
  set_last_path(2, "decode_splitkv_static_mma16816");
  return ATTN_OK;
}
