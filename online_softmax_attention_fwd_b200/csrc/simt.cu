// simt.cu -- CUDA-core (FFMA) attention forward and backward.
//
// The fp32 entry points (attn_fwd_f32 / attn_bwd_f32) run these kernels: genuine fp32 arithmetic,
// no TF32, so that results stay within 1e-5 of the fp64 definition.
//
// Forward: one warp per query row. The keys are visited in chunks of 32 (one key per lane for the
// score), and the row's state is the online-softmax triple (m, l, o): running max, running sum of
// exp(x - m) and the unnormalised accumulator, rescaled by exp(m_old - m_new) whenever the max grows
// -- the monoid of "Não escreva kernels, derive-os" ("Aprofundamento", first paragraph) applied one
// chunk at a time.
// Backward: Delta_i = dO_i . O_i; then one warp per query row accumulates
// dQ_i = scale sum_j P_ij (dP_ij - Delta_i) K_j, and one warp per key row accumulates
// dV_j = sum_i P_ij dO_i and dK_j = scale sum_i dS_ij Q_i over every query head of its group
// (P recomputed from lse), so no atomics are needed and the result is deterministic.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace attn {
namespace {

template <typename T>
__device__ __forceinline__ float ldf(const T* p);
template <>
__device__ __forceinline__ float ldf<float>(const float* p) {
  return __ldg(p);
}
template <typename T>
__device__ __forceinline__ void stf(T* p, float x);
template <>
__device__ __forceinline__ void stf<float>(float* p, float x) {
  *p = x;
}

constexpr int kWarps = 4;

template <typename T, int DPL>
__global__ void __launch_bounds__(128) fwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                       const T* __restrict__ v, T* __restrict__ o,
                                                       float* __restrict__ lse, int B, int Hq, int Hkv, int Sq,
                                                       int Sk, int D, int causal, float scale) {
  __shared__ float qs[kWarps][32 * DPL];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kWarps + warp;
  if (row >= static_cast<long long>(B) * Hq * Sq) return;
  const int i = static_cast<int>(row % Sq);
  const int h = static_cast<int>((row / Sq) % Hq);
  const int b = static_cast<int>(row / (static_cast<long long>(Sq) * Hq));
  const int g = h / (Hq / Hkv);
  const T* qrow = q + ((static_cast<long long>(b) * Sq + i) * Hq + h) * D;
#pragma unroll
  for (int t = 0; t < DPL; ++t) {
    const int d = lane + 32 * t;
    qs[warp][d] = d < D ? ldf(qrow + d) : 0.f;
  }
  __syncwarp();
  const long long kstride = static_cast<long long>(Hkv) * D;
  const T* kb = k + (static_cast<long long>(b) * Sk * Hkv + g) * D;
  const T* vb = v + (static_cast<long long>(b) * Sk * Hkv + g) * D;
  const int kend = causal ? min(Sk, i + Sk - Sq + 1) : Sk;  // keys [0, kend) are visible

  float acc[DPL];
#pragma unroll
  for (int t = 0; t < DPL; ++t) acc[t] = 0.f;
  float m = -INFINITY, l = 0.f;
  for (int j0 = 0; j0 < kend; j0 += 32) {
    const int j = j0 + lane;
    float s = -INFINITY;
    if (j < kend) {
      const T* kr = kb + j * kstride;
      float dot = 0.f;
      for (int d = 0; d < D; ++d) dot = fmaf(qs[warp][d], ldf(kr + d), dot);
      s = dot * scale;
    }
    const float mn = fmaxf(m, warp_max(s));  // finite: key j0 is visible
    const float alpha = expf(m - mn);         // m = -inf -> 0
    const float p = (j < kend) ? expf(s - mn) : 0.f;
    l = l * alpha + warp_sum(p);
#pragma unroll
    for (int t = 0; t < DPL; ++t) acc[t] *= alpha;
    const int nk = min(32, kend - j0);
    for (int jj = 0; jj < nk; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const T* vr = vb + (j0 + jj) * kstride;
#pragma unroll
      for (int t = 0; t < DPL; ++t) {
        const int d = lane + 32 * t;
        if (d < D) acc[t] = fmaf(pj, ldf(vr + d), acc[t]);
      }
    }
    m = mn;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  T* orow = o + ((static_cast<long long>(b) * Sq + i) * Hq + h) * D;
#pragma unroll
  for (int t = 0; t < DPL; ++t) {
    const int d = lane + 32 * t;
    if (d < D) stf(orow + d, acc[t] * inv);
  }
  if (lane == 0) lse[(static_cast<long long>(b) * Hq + h) * Sq + i] = l > 0.f ? m + logf(l) : -INFINITY;
}

// Delta[b,h,i] = sum_d dO[b,i,h,d] * O[b,i,h,d]
template <typename T, int DPL>
__global__ void __launch_bounds__(128) bwd_delta_kernel(const T* __restrict__ o, const T* __restrict__ dout,
                                                        float* __restrict__ delta, int B, int Hq, int Sq, int D) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kWarps + warp;
  if (row >= static_cast<long long>(B) * Hq * Sq) return;
  const int i = static_cast<int>(row % Sq);
  const int h = static_cast<int>((row / Sq) % Hq);
  const int b = static_cast<int>(row / (static_cast<long long>(Sq) * Hq));
  const long long base = ((static_cast<long long>(b) * Sq + i) * Hq + h) * D;
  float s = 0.f;
#pragma unroll
  for (int t = 0; t < DPL; ++t) {
    const int d = lane + 32 * t;
    if (d < D) s = fmaf(ldf(o + base + d), ldf(dout + base + d), s);
  }
  s = warp_sum(s);
  if (lane == 0) delta[(static_cast<long long>(b) * Hq + h) * Sq + i] = s;
}

template <typename T, int DPL>
__global__ void __launch_bounds__(128) bwd_dq_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                          const T* __restrict__ v, const T* __restrict__ dout,
                                                          const float* __restrict__ lse,
                                                          const float* __restrict__ delta, T* __restrict__ dq,
                                                          int B, int Hq, int Hkv, int Sq, int Sk, int D, int causal,
                                                          float scale) {
  __shared__ float qs[kWarps][32 * DPL];
  __shared__ float dos[kWarps][32 * DPL];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kWarps + warp;
  if (row >= static_cast<long long>(B) * Hq * Sq) return;
  const int i = static_cast<int>(row % Sq);
  const int h = static_cast<int>((row / Sq) % Hq);
  const int b = static_cast<int>(row / (static_cast<long long>(Sq) * Hq));
  const int g = h / (Hq / Hkv);
  const long long qoff = ((static_cast<long long>(b) * Sq + i) * Hq + h) * D;
#pragma unroll
  for (int t = 0; t < DPL; ++t) {
    const int d = lane + 32 * t;
    qs[warp][d] = d < D ? ldf(q + qoff + d) : 0.f;
    dos[warp][d] = d < D ? ldf(dout + qoff + d) : 0.f;
  }
  __syncwarp();
  const long long li = (static_cast<long long>(b) * Hq + h) * Sq + i;
  const float lse_i = lse[li];
  const float delta_i = delta[li];
  const long long kstride = static_cast<long long>(Hkv) * D;
  const T* kb = k + (static_cast<long long>(b) * Sk * Hkv + g) * D;
  const T* vb = v + (static_cast<long long>(b) * Sk * Hkv + g) * D;
  const int kend = causal ? min(Sk, i + Sk - Sq + 1) : Sk;
  float acc[DPL];
#pragma unroll
  for (int t = 0; t < DPL; ++t) acc[t] = 0.f;
  for (int j0 = 0; j0 < kend; j0 += 32) {
    const int j = j0 + lane;
    float ds = 0.f;
    if (j < kend) {
      const T* kr = kb + j * kstride;
      const T* vr = vb + j * kstride;
      float dot = 0.f, dp = 0.f;
      for (int d = 0; d < D; ++d) {
        dot = fmaf(qs[warp][d], ldf(kr + d), dot);
        dp = fmaf(dos[warp][d], ldf(vr + d), dp);
      }
      const float p = expf(dot * scale - lse_i);
      ds = p * (dp - delta_i);
    }
    const int nk = min(32, kend - j0);
    for (int jj = 0; jj < nk; ++jj) {
      const float dsj = __shfl_sync(0xffffffffu, ds, jj);
      const T* kr = kb + (j0 + jj) * kstride;
#pragma unroll
      for (int t = 0; t < DPL; ++t) {
        const int d = lane + 32 * t;
        if (d < D) acc[t] = fmaf(dsj, ldf(kr + d), acc[t]);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < DPL; ++t) {
    const int d = lane + 32 * t;
    if (d < D) stf(dq + qoff + d, acc[t] * scale);
  }
}

template <typename T, int DPL>
__global__ void __launch_bounds__(128) bwd_dkdv_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                            const T* __restrict__ v, const T* __restrict__ dout,
                                                            const float* __restrict__ lse,
                                                            const float* __restrict__ delta, T* __restrict__ dk,
                                                            T* __restrict__ dv, int B, int Hq, int Hkv, int Sq,
                                                            int Sk, int D, int causal, float scale) {
  __shared__ float ks[kWarps][32 * DPL];
  __shared__ float vs[kWarps][32 * DPL];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kWarps + warp;
  if (row >= static_cast<long long>(B) * Hkv * Sk) return;
  const int j = static_cast<int>(row % Sk);
  const int g = static_cast<int>((row / Sk) % Hkv);
  const int b = static_cast<int>(row / (static_cast<long long>(Sk) * Hkv));
  const int G = Hq / Hkv;
  const long long koff = ((static_cast<long long>(b) * Sk + j) * Hkv + g) * D;
#pragma unroll
  for (int t = 0; t < DPL; ++t) {
    const int d = lane + 32 * t;
    ks[warp][d] = d < D ? ldf(k + koff + d) : 0.f;
    vs[warp][d] = d < D ? ldf(v + koff + d) : 0.f;
  }
  __syncwarp();
  // rows i that see key j: j <= i + Sk - Sq  <=>  i >= j - (Sk - Sq)
  const int istart = causal ? max(0, j - (Sk - Sq)) : 0;
  const long long qstride = static_cast<long long>(Hq) * D;
  float adk[DPL], adv[DPL];
#pragma unroll
  for (int t = 0; t < DPL; ++t) adk[t] = adv[t] = 0.f;
  for (int hh = 0; hh < G; ++hh) {
    const int h = g * G + hh;
    const T* qb = q + (static_cast<long long>(b) * Sq * Hq + h) * D;
    const T* db = dout + (static_cast<long long>(b) * Sq * Hq + h) * D;
    const float* lse_h = lse + (static_cast<long long>(b) * Hq + h) * Sq;
    const float* delta_h = delta + (static_cast<long long>(b) * Hq + h) * Sq;
    for (int i0 = istart; i0 < Sq; i0 += 32) {
      const int i = i0 + lane;
      float p = 0.f, ds = 0.f;
      if (i < Sq) {
        const T* qr = qb + i * qstride;
        const T* dr = db + i * qstride;
        float dot = 0.f, dp = 0.f;
        for (int d = 0; d < D; ++d) {
          dot = fmaf(ldf(qr + d), ks[warp][d], dot);
          dp = fmaf(ldf(dr + d), vs[warp][d], dp);
        }
        p = expf(dot * scale - lse_h[i]);
        ds = p * (dp - delta_h[i]);
      }
      const int ni = min(32, Sq - i0);
      for (int ii = 0; ii < ni; ++ii) {
        const float pi = __shfl_sync(0xffffffffu, p, ii);
        const float dsi = __shfl_sync(0xffffffffu, ds, ii);
        const T* qr = qb + (i0 + ii) * qstride;
        const T* dr = db + (i0 + ii) * qstride;
#pragma unroll
        for (int t = 0; t < DPL; ++t) {
          const int d = lane + 32 * t;
          if (d < D) {
            adv[t] = fmaf(pi, ldf(dr + d), adv[t]);
            adk[t] = fmaf(dsi, ldf(qr + d), adk[t]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < DPL; ++t) {
    const int d = lane + 32 * t;
    if (d < D) {
      stf(dk + koff + d, adk[t] * scale);
      stf(dv + koff + d, adv[t]);
    }
  }
}

inline unsigned blocks_for(long long rows) { return static_cast<unsigned>((rows + kWarps - 1) / kWarps); }

template <typename T, int DPL>
cudaError_t fwd_simt_dpl(const Problem& p, const void* q, const void* k, const void* v, void* o, float* lse,
                         cudaStream_t st) {
  const long long rows = static_cast<long long>(p.B) * p.Hq * p.Sq;
  {
    LaunchScope ls(sizeof(T) == 4 ? "fwd_simt_f32" : "fwd_simt_bf16", st);
    fwd_simt_kernel<T, DPL><<<blocks_for(rows), 128, 0, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), static_cast<T*>(o), lse, p.B,
        p.Hq, p.Hkv, p.Sq, p.Sk, p.D, p.causal, p.scale);
  }
  return cudaGetLastError();
}

template <typename T, int DPL>
cudaError_t bwd_simt_dpl(const Problem& p, const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv, float* delta,
                         cudaStream_t st) {
  const long long qrows = static_cast<long long>(p.B) * p.Hq * p.Sq;
  const long long krows = static_cast<long long>(p.B) * p.Hkv * p.Sk;
  {
    LaunchScope ls("bwd_simt_delta", st);
    bwd_delta_kernel<T, DPL><<<blocks_for(qrows), 128, 0, st>>>(static_cast<const T*>(o),
                                                                 static_cast<const T*>(dout), delta, p.B, p.Hq,
                                                                 p.Sq, p.D);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  {
    LaunchScope ls("bwd_simt_dq", st);
    bwd_dq_simt_kernel<T, DPL><<<blocks_for(qrows), 128, 0, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), static_cast<const T*>(dout),
        lse, delta, static_cast<T*>(dq), p.B, p.Hq, p.Hkv, p.Sq, p.Sk, p.D, p.causal, p.scale);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  {
    LaunchScope ls("bwd_simt_dkdv", st);
    bwd_dkdv_simt_kernel<T, DPL><<<blocks_for(krows), 128, 0, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), static_cast<const T*>(dout),
        lse, delta, static_cast<T*>(dk), static_cast<T*>(dv), p.B, p.Hq, p.Hkv, p.Sq, p.Sk, p.D, p.causal,
        p.scale);
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t fwd_simt_any(const Problem& p, const void* q, const void* k, const void* v, void* o, float* lse,
                         cudaStream_t st) {
  if (p.D <= 32) return fwd_simt_dpl<T, 1>(p, q, k, v, o, lse, st);
  if (p.D <= 64) return fwd_simt_dpl<T, 2>(p, q, k, v, o, lse, st);
  if (p.D <= 128) return fwd_simt_dpl<T, 4>(p, q, k, v, o, lse, st);
  return fwd_simt_dpl<T, 8>(p, q, k, v, o, lse, st);
}

template <typename T>
cudaError_t bwd_simt_any(const Problem& p, const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv, float* delta,
                         cudaStream_t st) {
  if (p.D <= 32) return bwd_simt_dpl<T, 1>(p, q, k, v, o, lse, dout, dq, dk, dv, delta, st);
  if (p.D <= 64) return bwd_simt_dpl<T, 2>(p, q, k, v, o, lse, dout, dq, dk, dv, delta, st);
  if (p.D <= 128) return bwd_simt_dpl<T, 4>(p, q, k, v, o, lse, dout, dq, dk, dv, delta, st);
  return bwd_simt_dpl<T, 8>(p, q, k, v, o, lse, dout, dq, dk, dv, delta, st);
}

}  // namespace

cudaError_t launch_fwd_simt_f32(const Problem& p, const float* q, const float* k, const float* v, float* o,
                                float* lse, cudaStream_t st) {
  return fwd_simt_any<float>(p, q, k, v, o, lse, st);
}
cudaError_t launch_bwd_simt_f32(const Problem& p, const float* q, const float* k, const float* v, const float* o,
                                const float* lse, const float* dout, float* dq, float* dk, float* dv,
                                float* delta, cudaStream_t st) {
  return bwd_simt_any<float>(p, q, k, v, o, lse, dout, dq, dk, dv, delta, st);
}

}  // namespace attn
