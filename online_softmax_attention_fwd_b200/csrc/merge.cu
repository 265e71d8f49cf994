// merge.cu -- the online-softmax monoid applied to whole attention results.
//
// Two attentions of the same query rows over disjoint key sets, each given as its normalised
// output O and its log-sum-exp lse, combine into the attention over the union of the keys
// ("Não escreva kernels, derive-os", "Aprofundamento", first paragraph: the online softmax is a
// monoid, so partial results over any partition of the keys merge in any order). With
// M = max(lse_a, lse_b), w_a = e^(lse_a - M), w_b = e^(lse_b - M):
//   lse = M + ln(w_a + w_b),   O = (w_a O_a + w_b O_b) / (w_a + w_b),
// which is the triple merge (m, l, o) with l e^m = e^lse and o = l O. The identity is lse = -inf
// (its O is never read), so a key set that a row cannot see contributes nothing.
//
// attn_merge folds a bf16 partial (O_b, lse_b) -- as attn_fwd writes it -- into an fp32 running
// result (O_acc, lse_acc) in place, and may also write the merged O rounded to bf16. A context-
// parallel ring calls it once per key shard. HBM-bound: one thread per 8 elements of a row, 16-byte
// loads and stores, the row's two weights computed once per row by every thread of it.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace attn {
namespace {

// One row (b, i, h) of O has D elements; DT = D / 8 threads cover it, each 8 elements. lse is
// [B, H, S] (as attn_fwd writes it), O is [B, S, H, D].
template <int D>
__global__ void __launch_bounds__(256) merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc,
                                                    const uint16_t* __restrict__ o_part,
                                                    const float* __restrict__ lse_part, uint16_t* __restrict__ o_out,
                                                    int B, int S, int H) {
  constexpr int DT = D / 8;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rows = static_cast<long long>(B) * S * H;
  if (t >= rows * DT) return;
  const long long row = t / DT;  // (b, i, h), h fastest: the [B, S, H, D] row order
  const int c = static_cast<int>(t % DT) * 8;
  const int h = static_cast<int>(row % H);
  const long long bi = row / H;
  const int i = static_cast<int>(bi % S);
  const long long b = bi / S;
  const long long li = (b * H + h) * S + i;
  const float la = lse_acc[li], lb = lse_part[li];
  const float M = fmaxf(la, lb);
  float wa = 0.f, wb = 0.f;
  if (M != -INFINITY) {
    wa = la == -INFINITY ? 0.f : __expf(la - M);
    wb = lb == -INFINITY ? 0.f : __expf(lb - M);
  }
  const float sum = wa + wb;
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  float* acc = o_acc + row * D + c;
  float x[8];
  if (wa > 0.f) {
    const float4 a0 = *reinterpret_cast<const float4*>(acc), a1 = *reinterpret_cast<const float4*>(acc + 4);
    x[0] = a0.x; x[1] = a0.y; x[2] = a0.z; x[3] = a0.w;
    x[4] = a1.x; x[5] = a1.y; x[6] = a1.z; x[7] = a1.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = 0.f;  // the identity's O is never read
  }
  float y[8];
  if (wb > 0.f) {
    const uint4 p = *reinterpret_cast<const uint4*>(o_part + row * D + c);
    const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      y[2 * e] = bf16_lo(pw[e]);
      y[2 * e + 1] = bf16_hi(pw[e]);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = 0.f;
  }
  float r[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) r[e] = (wa * x[e] + wb * y[e]) * inv;
  *reinterpret_cast<float4*>(acc) = make_float4(r[0], r[1], r[2], r[3]);
  *reinterpret_cast<float4*>(acc + 4) = make_float4(r[4], r[5], r[6], r[7]);
  if (o_out)
    *reinterpret_cast<uint4*>(o_out + row * D + c) =
        make_uint4(pack_bf16(r[0], r[1]), pack_bf16(r[2], r[3]), pack_bf16(r[4], r[5]), pack_bf16(r[6], r[7]));
  // every thread of the row has read lse_acc before any writes it: the row's threads are adjacent
  // lanes of one warp, and the write comes after a warp-wide barrier
  __syncwarp(__activemask());
  if (c == 0) lse_acc[li] = sum > 0.f ? M + __logf(sum) : -INFINITY;
}

template <int D>
cudaError_t launch_merge_d(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out,
                           int B, int S, int H, cudaStream_t st) {
  const long long threads = static_cast<long long>(B) * S * H * (D / 8);
  LaunchScope ls("merge", st);
  merge_kernel<D><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(
      o_acc, lse_acc, static_cast<const uint16_t*>(o_part), lse_part, static_cast<uint16_t*>(o_out), B, S, H);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                         int S, int H, int D, cudaStream_t st) {
  switch (D) {
    case 64: return launch_merge_d<64>(o_acc, lse_acc, o_part, lse_part, o_out, B, S, H, st);
    case 128: return launch_merge_d<128>(o_acc, lse_acc, o_part, lse_part, o_out, B, S, H, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace attn
