// decode.cu -- split-KV decode: partial online-softmax triples per key chunk, then a monoid merge.
//
// One query token per stream attends to all of that stream's cached keys (the decode streams of
// "Não escreva kernels, derive-os", "Aprofundamento", third paragraph). The keys of each
// (stream, kv head) are cut into C contiguous chunks; the split kernel reduces each chunk to a
// triple (m, l, o) -- running max (base-2 units), sum of 2^(s - m), unnormalised sum of
// 2^(s - m) v -- and the combine kernel merges the C triples with the monoid
// (m,l,o) + (m',l',o') = (M, l 2^(m-M) + l' 2^(m'-M), o 2^(m-M) + o' 2^(m'-M)), M = max(m, m'),
// identity (-inf, 0, 0), a weight 2^(-inf - M) taken as 0. The merge is the same one the split
// kernel uses between its four warps, so the result does not depend on how the keys were cut.
//
// The path is HBM-bound (each K/V byte is read once, about 4 flop per byte), so the split kernel is
// CUDA-core code built for bytes in flight: a CTA covers one (chunk, kv head, stream) and all the
// query heads of that kv head's group, so each K/V row is fetched once for GT query heads. Each
// lane scores one key (16-byte vector loads of its K row) and owns D/32 value dimensions (coalesced
// V rows); a block's V loads are issued before its softmax arithmetic so that they overlap it.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace attn {

__host__ __device__ inline int decode_split_rule(int L, int max_splits) {
  int c = (L + 255) / 256;
  c = c < 4 ? 4 : (c > 16 ? 16 : c);
  if (c > max_splits) c = max_splits;
  return c < 1 ? 1 : c;
}

int decode_default_splits(int L, int max_splits) { return decode_split_rule(L, max_splits); }

size_t decode_workspace_bytes(int N, int Hq, int D, int max_splits) {
  const size_t slots = static_cast<size_t>(N) * Hq * max_splits;
  const size_t o_bytes = (slots * D * sizeof(float) + 255) & ~static_cast<size_t>(255);
  const size_t ml_bytes = (slots * 2 * sizeof(float) + 255) & ~static_cast<size_t>(255);
  return o_bytes + ml_bytes;
}

namespace {

__device__ __forceinline__ int stream_splits(const int* num_splits, int n, int L, int max_splits) {
  if (num_splits) {
    const int c = num_splits[n];
    return c < 1 ? 1 : (c > max_splits ? max_splits : c);
  }
  return decode_split_rule(L, max_splits);
}

template <int DPL>
struct VPiece;
template <>
struct VPiece<4> {
  uint32_t w[2];
  __device__ __forceinline__ void load(const uint16_t* p) {
    const uint2 x = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = x.x;
    w[1] = x.y;
  }
  __device__ __forceinline__ void zero() { w[0] = w[1] = 0u; }
  __device__ __forceinline__ float get(int i) const { return (i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]); }
};
template <>
struct VPiece<2> {
  uint32_t w[1];
  __device__ __forceinline__ void load(const uint16_t* p) { w[0] = __ldg(reinterpret_cast<const unsigned*>(p)); }
  __device__ __forceinline__ void zero() { w[0] = 0u; }
  __device__ __forceinline__ float get(int i) const { return (i & 1) ? bf16_hi(w[0]) : bf16_lo(w[0]); }
};

template <int D, int GT>
__global__ void __launch_bounds__(128) decode_split_kernel(const uint16_t* __restrict__ q,
                                                           const uint16_t* __restrict__ k,
                                                           const uint16_t* __restrict__ v,
                                                           const int* __restrict__ offsets,
                                                           const int* __restrict__ num_splits, int max_splits,
                                                           int Hq, int Hkv, float scale_log2,
                                                           float* __restrict__ part_o,
                                                           float* __restrict__ part_ml) {
  constexpr int KV16 = D / 8;  // 16-byte pieces per K row
  constexpr int DPL = D / 32;  // value dimensions per lane
  __shared__ __align__(16) float qs[GT][D];
  __shared__ float red_m[4][GT];
  __shared__ float red_l[4][GT];
  __shared__ __align__(16) float red_o[4][GT][D];

  const int c = blockIdx.x, n = blockIdx.z;
  const int G = Hq / Hkv, npass = G / GT;
  const int g = blockIdx.y / npass;
  const int h0 = g * G + (blockIdx.y % npass) * GT;
  const int start = offsets[n];
  const int L = offsets[n + 1] - start;
  const int C = stream_splits(num_splits, n, L, max_splits);
  if (c >= C) return;  // uniform over the CTA; the combine reads only the first C slots
  const int chunk = (L + C - 1) / C;
  const int k0 = min(L, c * chunk);
  const int k1 = min(L, k0 + chunk);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < GT * D; e += 128) {
    const int t = e / D, d = e - t * D;
    qs[t][d] = __uint_as_float(static_cast<uint32_t>(q[(static_cast<long long>(n) * Hq + h0 + t) * D + d]) << 16) *
               scale_log2;
  }
  __syncthreads();

  float m[GT], ls[GT], acc[GT][DPL];
#pragma unroll
  for (int t = 0; t < GT; ++t) {
    m[t] = -INFINITY;
    ls[t] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[t][e] = 0.f;
  }
  const long long rs = static_cast<long long>(Hkv) * D;
  const uint16_t* kb = k + (static_cast<long long>(start) * Hkv + g) * D;
  const uint16_t* vb = v + (static_cast<long long>(start) * Hkv + g) * D + lane * DPL;

  for (int base = k0 + 32 * warp; base < k1; base += 128) {
    const int j = base + lane;
    const bool valid = j < k1;
    const int nk = min(32, k1 - base);
    uint4 kr[KV16];
    if (valid) {
      const uint4* src = reinterpret_cast<const uint4*>(kb + j * rs);
#pragma unroll
      for (int x = 0; x < KV16; ++x) kr[x] = __ldg(src + x);
    } else {
#pragma unroll
      for (int x = 0; x < KV16; ++x) kr[x] = make_uint4(0u, 0u, 0u, 0u);
    }
    // scores of this lane's key for the GT query heads (base-2 units: q carries scale * log2 e)
    float s[GT];
#pragma unroll
    for (int t = 0; t < GT; ++t) s[t] = 0.f;
#pragma unroll
    for (int x = 0; x < KV16; ++x) {
      const uint32_t w[4] = {kr[x].x, kr[x].y, kr[x].z, kr[x].w};
#pragma unroll
      for (int t = 0; t < GT; ++t) {
        const float4 qa = *reinterpret_cast<const float4*>(&qs[t][8 * x]);
        const float4 qb = *reinterpret_cast<const float4*>(&qs[t][8 * x + 4]);
        float a = s[t];
        a = fmaf(qa.x, bf16_lo(w[0]), a);
        a = fmaf(qa.y, bf16_hi(w[0]), a);
        a = fmaf(qa.z, bf16_lo(w[1]), a);
        a = fmaf(qa.w, bf16_hi(w[1]), a);
        a = fmaf(qb.x, bf16_lo(w[2]), a);
        a = fmaf(qb.y, bf16_hi(w[2]), a);
        a = fmaf(qb.z, bf16_lo(w[3]), a);
        a = fmaf(qb.w, bf16_hi(w[3]), a);
        s[t] = a;
      }
    }
    // V loads go out before the softmax arithmetic so that they overlap it
    VPiece<DPL> vr[32];
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) {
      if (jj < nk)
        vr[jj].load(vb + (base + jj) * rs);
      else
        vr[jj].zero();
    }
    float p[GT];
#pragma unroll
    for (int t = 0; t < GT; ++t) {
      const float st = valid ? s[t] : -INFINITY;
      const float mn = fmaxf(m[t], warp_max(st));  // finite: lane 0's key is valid
      const float alpha = exp2f(m[t] - mn);         // 2^(-inf) = 0 on the first block
      p[t] = valid ? exp2f(st - mn) : 0.f;
      ls[t] = ls[t] * alpha + p[t];
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[t][e] *= alpha;
      m[t] = mn;
    }
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) {
      if (jj < nk) {
#pragma unroll
        for (int t = 0; t < GT; ++t) {
          const float pj = __shfl_sync(0xffffffffu, p[t], jj);
#pragma unroll
          for (int e = 0; e < DPL; ++e) acc[t][e] = fmaf(pj, vr[jj].get(e), acc[t][e]);
        }
      }
    }
  }

  // merge the four warps' triples (a warp that saw no key holds the identity)
#pragma unroll
  for (int t = 0; t < GT; ++t) {
    const float lw = warp_sum(ls[t]);
    if (lane == 0) {
      red_m[warp][t] = m[t];
      red_l[warp][t] = lw;
    }
#pragma unroll
    for (int e = 0; e < DPL; ++e) red_o[warp][t][lane * DPL + e] = acc[t][e];
  }
  __syncthreads();
  for (int e = tid; e < GT * D; e += 128) {
    const int t = e / D, d = e - t * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, red_m[w][t]);
    float Lsum = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = red_m[w][t];
        const float wt = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        Lsum = fmaf(wt, red_l[w][t], Lsum);
        O = fmaf(wt, red_o[w][t][d], O);
      }
    }
    const long long slot = (static_cast<long long>(n) * Hq + h0 + t) * max_splits + c;
    part_o[slot * D + d] = O;
    if (d == 0) {
      part_ml[slot * 2] = M;
      part_ml[slot * 2 + 1] = Lsum;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const float* __restrict__ part_o,
                                                             const float* __restrict__ part_ml,
                                                             const int* __restrict__ offsets,
                                                             const int* __restrict__ num_splits, int max_splits,
                                                             int N, int Hq, uint16_t* __restrict__ o,
                                                             float* __restrict__ lse) {
  constexpr int DPL = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long gw = static_cast<long long>(blockIdx.x) * 4 + warp;
  if (gw >= static_cast<long long>(N) * Hq) return;
  const int n = static_cast<int>(gw / Hq), h = static_cast<int>(gw % Hq);
  const int L = offsets[n + 1] - offsets[n];
  const int C = stream_splits(num_splits, n, L, max_splits);
  const long long slot0 = (static_cast<long long>(n) * Hq + h) * max_splits;
  // lane c holds chunk c and chunk c + 32 (max_splits <= 64)
  float m0 = -INFINITY, l0 = 0.f, m1 = -INFINITY, l1 = 0.f;
  if (lane < C) {
    const float2 ml = *reinterpret_cast<const float2*>(part_ml + (slot0 + lane) * 2);
    m0 = ml.x;
    l0 = ml.y;
  }
  if (lane + 32 < C) {
    const float2 ml = *reinterpret_cast<const float2*>(part_ml + (slot0 + lane + 32) * 2);
    m1 = ml.x;
    l1 = ml.y;
  }
  const float M = warp_max(fmaxf(m0, m1));
  float w0 = 0.f, w1 = 0.f;
  if (M != -INFINITY) {
    w0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - M);
    w1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - M);
  }
  const float Lt = warp_sum(w0 * l0 + w1 * l1);
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  for (int c = 0; c < C; ++c) {
    const float wc = __shfl_sync(0xffffffffu, c < 32 ? w0 : w1, c & 31);
    if (wc != 0.f) {
      const float* src = part_o + (slot0 + c) * D + lane * DPL;
      if constexpr (DPL == 4) {
        const float4 x = *reinterpret_cast<const float4*>(src);
        acc[0] = fmaf(wc, x.x, acc[0]);
        acc[1] = fmaf(wc, x.y, acc[1]);
        acc[2] = fmaf(wc, x.z, acc[2]);
        acc[3] = fmaf(wc, x.w, acc[3]);
      } else {
        const float2 x = *reinterpret_cast<const float2*>(src);
        acc[0] = fmaf(wc, x.x, acc[0]);
        acc[1] = fmaf(wc, x.y, acc[1]);
      }
    }
  }
  const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
  uint16_t* dst = o + (static_cast<long long>(n) * Hq + h) * D + lane * DPL;
  if constexpr (DPL == 4) {
    uint2 w;
    w.x = pack_bf16(acc[0] * inv, acc[1] * inv);
    w.y = pack_bf16(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(dst) = w;
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0 && lse) lse[static_cast<long long>(n) * Hq + h] = Lt > 0.f ? (M + log2f(Lt)) * kLn2 : -INFINITY;
}

template <int D, int GT>
cudaError_t launch_split(const DecodeProblem& p, const void* q, const void* k, const void* v,
                         const int* offsets, const int* num_splits, float* part_o, float* part_ml,
                         cudaStream_t st) {
  const int npass = (p.Hq / p.Hkv) / GT;
  dim3 grid(p.max_splits, p.Hkv * npass, p.N);
  {
    LaunchScope ls("decode_split", st);
    decode_split_kernel<D, GT><<<grid, 128, 0, st>>>(
        static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v),
        offsets, num_splits, p.max_splits, p.Hq, p.Hkv, p.scale * kLog2e, part_o, part_ml);
  }
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_decode_d(const DecodeProblem& p, const void* q, const void* k, const void* v,
                            const int* offsets, const int* num_splits, void* o, float* lse, void* workspace,
                            cudaStream_t st) {
  const size_t slots = static_cast<size_t>(p.N) * p.Hq * p.max_splits;
  float* part_o = static_cast<float*>(workspace);
  float* part_ml = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                            ((slots * D * sizeof(float) + 255) & ~static_cast<size_t>(255)));
  const int G = p.Hq / p.Hkv;
  cudaError_t e;
  bool done = false;
  if constexpr (D == 64) {  // at D = 128 eight heads per CTA would spill registers
    if (G % 8 == 0) {
      e = launch_split<D, 8>(p, q, k, v, offsets, num_splits, part_o, part_ml, st);
      done = true;
    }
  }
  if (done) {
  } else if (G % 4 == 0) {
    e = launch_split<D, 4>(p, q, k, v, offsets, num_splits, part_o, part_ml, st);
  } else if (G % 2 == 0) {
    e = launch_split<D, 2>(p, q, k, v, offsets, num_splits, part_o, part_ml, st);
  } else {
    e = launch_split<D, 1>(p, q, k, v, offsets, num_splits, part_o, part_ml, st);
  }
  if (e != cudaSuccess) return e;
  const long long warps = static_cast<long long>(p.N) * p.Hq;
  {
    LaunchScope ls("decode_combine", st);
    decode_combine_kernel<D><<<static_cast<unsigned>((warps + 3) / 4), 128, 0, st>>>(
        part_o, part_ml, offsets, num_splits, p.max_splits, p.N, p.Hq, static_cast<uint16_t*>(o), lse);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeProblem& p, const void* q, const void* k, const void* v,
                          const int* kv_offsets, const int* num_splits, void* o, float* lse, void* workspace,
                          cudaStream_t st) {
  if (p.D == 128) return launch_decode_d<128>(p, q, k, v, kv_offsets, num_splits, o, lse, workspace, st);
  return launch_decode_d<64>(p, q, k, v, kv_offsets, num_splits, o, lse, workspace, st);
}

}  // namespace attn
