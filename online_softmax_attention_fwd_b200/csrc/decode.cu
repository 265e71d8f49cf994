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
// CUDA-core code built to keep many bytes in flight without spending registers on them. A CTA
// covers one (chunk, kv head, stream) and all the query heads of that kv head's group, so each K/V
// row is fetched once for GT query heads. One producer warp streams 32-key K and V blocks of the
// chunk with TMA tile loads (128-byte swizzle) into a 4-stage shared-memory ring; compute warp w
// takes blocks w, w+4, ... and keeps its own online-softmax triples for the GT heads: each lane
// scores one key for all GT heads (its K row read once from shared memory) and owns D/32 value
// dimensions of every head (each V row read once per lane). The four warps' triples are merged
// with the monoid at the end.
// The host does not know the cache's row count T (it lives on the device as kv_offsets[N]), so the
// tensor maps carry a nominal row extent and the kernel issues a 32-row box only when the whole box
// lies below T; the cache's last partial block is fetched in 16-byte pieces with bulk copies. No
// copy ever touches memory past the caller's K and V buffers.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"

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

constexpr int kDecBlk = 32;              // keys per block (one per lane)
constexpr int kDecStages = 4;
// Compute warp w consumes blocks w, w + 4, ... and every stage has a single-arrival "empty" barrier,
// so a stage must always belong to the same warp: the stage count is a multiple of the four compute
// warps (otherwise two warps would share a stage and a parity wait could match the wrong phase).
static_assert(kDecStages % 4 == 0, "decode ring stages must be a multiple of the compute warps");
constexpr int kDecThreads = 160;          // four compute warps + one producer warp
constexpr int kDecMapRows = 0x7fffffff;   // nominal row extent of the K/V tensor maps

template <int D>
struct DecCfg {
  static constexpr int kAtoms = D / 64;
  static constexpr int kAtomBytes = kDecBlk * 128;       // 32 rows x 128 bytes
  static constexpr int kBlkBytes = kAtoms * kAtomBytes;  // 32 key rows x D bf16
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kDecStages * kBlkBytes;
  static constexpr int kOffBar = 2 * kDecStages * kBlkBytes;
  static constexpr int kOffP = kOffBar + 2 * kDecStages * 8 + 16;  // [4 warps][32 keys][4 heads] (p, p)
  static constexpr int kSmemBytes = kOffP + 4 * kDecBlk * 4 * 8 + 1024;
};

__device__ __forceinline__ bool dec_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

// Byte offset of element d of row r in a 128-byte-swizzled block of 64-element column atoms.
template <int D>
__device__ __forceinline__ uint32_t dec_sw(int r, int d) {
  return (d >> 6) * DecCfg<D>::kAtomBytes + sw128_offset(r, (d & 63) >> 3) + (d & 7) * 2;
}

template <int D, int GT>
__global__ void __launch_bounds__(kDecThreads, 3)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                        const uint16_t* __restrict__ v, const int* __restrict__ offsets, int N,
                        const int* __restrict__ num_splits, int max_splits, int Hq, int Hkv, float scale_log2,
                        float* __restrict__ part_o, float* __restrict__ part_ml, int* status) {
  using C = DecCfg<D>;
  constexpr int DPL = D / 32;  // value dimensions per lane
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + kDecStages;
  volatile int* abort = reinterpret_cast<volatile int*>(empty + kDecStages);
  __shared__ __align__(16) float qs[GT][D];
  __shared__ float red_m[4][GT];
  __shared__ float red_l[4][GT];
  // The four compute warps' unnormalised outputs, merged at the end, reuse the K ring (every block
  // has been consumed by then).
  float(*red_o)[GT][D] = reinterpret_cast<float(*)[GT][D]>(sK);

  const int c = blockIdx.x, n = blockIdx.z;
  const int G = Hq / Hkv, npass = G / GT;
  const int g = blockIdx.y / npass;
  const int h0 = g * G + (blockIdx.y % npass) * GT;
  const int start = offsets[n];
  const int L = offsets[n + 1] - start;
  const int C_n = stream_splits(num_splits, n, L, max_splits);
  if (c >= C_n) return;  // uniform over the CTA; the combine reads only the first C_n slots
  const int chunk = (L + C_n - 1) / C_n;
  const int k0 = min(L, c * chunk);
  const int k1 = min(L, k0 + chunk);
  const int nblk = (k1 - k0 + kDecBlk - 1) / kDecBlk;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);  // each block is consumed by exactly one compute warp
    }
    *abort = 0;
    fence_mbar_init();
  }
  for (int e = tid; e < GT * D; e += kDecThreads) {
    const int t = e / D, d = e - t * D;
    qs[t][d] = __uint_as_float(static_cast<uint32_t>(q[(static_cast<long long>(n) * Hq + h0 + t) * D + d]) << 16) *
               scale_log2;
  }
  __syncthreads();

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    const int T = min(offsets[N], kDecMapRows);  // no box may reach past the cache
    const long long rs = static_cast<long long>(Hkv) * D;
    int issued = 0;
    for (int bk = 0; bk < nblk; ++bk) {
      const int s = bk % kDecStages;
      const int row0 = start + k0 + bk * kDecBlk;
      const bool tile = row0 + kDecBlk <= T;
      const int nrows = tile ? kDecBlk : min(kDecBlk, k1 - (k0 + bk * kDecBlk));
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(empty + s, ((bk / kDecStages) & 1) ^ 1, abort, status);
        if (ok) {
          mbar_arrive_expect_tx(full + s, 2u * nrows * D * 2);
          if (tile) {
#pragma unroll
            for (int at = 0; at < C::kAtoms; ++at) {
              tma_load_3d(sK + s * C::kBlkBytes + at * C::kAtomBytes, &tmK, full + s, at * 64, g, row0);
              tma_load_3d(sV + s * C::kBlkBytes + at * C::kAtomBytes, &tmV, full + s, at * 64, g, row0);
            }
          }
        }
      }
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
      if (!tile) {
        // the cache's last rows: 16-byte pieces into the same swizzled places a tile load uses
        for (int idx = lane; idx < nrows * (D / 8); idx += 32) {
          const int r = idx / (D / 8), d = (idx % (D / 8)) * 8;
          bulk_load(sK + s * C::kBlkBytes + dec_sw<D>(r, d), k + (row0 + r) * rs + g * D + d, 16, full + s);
          bulk_load(sV + s * C::kBlkBytes + dec_sw<D>(r, d), v + (row0 + r) * rs + g * D + d, 16, full + s);
        }
      }
      issued = bk + 1;
    }
    // let this CTA's copies land before it can exit (at once on the normal path)
    if (lane == 0)
      for (int bk = max(0, issued - kDecStages); bk < issued; ++bk)
        dec_wait_drain(full + bk % kDecStages, (bk / kDecStages) & 1);
    return;
  }

  // ------------------------------------------------------------------ compute warps
  // Pairs of fp32 values go through the packed f32x2 instructions: the scores accumulate two
  // head-dim products per instruction, the outputs two value dimensions per instruction.
  constexpr int PPL = DPL / 2;  // value-dimension pairs per lane
  float m[GT], ls[GT];
  uint64_t acc2[GT][PPL];
#pragma unroll
  for (int t = 0; t < GT; ++t) {
    m[t] = -INFINITY;
    ls[t] = 0.f;
#pragma unroll
    for (int e = 0; e < PPL; ++e) acc2[t][e] = 0ull;
  }
  const int vd = lane * DPL;  // this lane's value dimensions: vd .. vd + DPL - 1
  // this warp's block probabilities as (p, p) pairs: [32 keys][GT] x 8 bytes
  uint64_t* sp = reinterpret_cast<uint64_t*>(smem + C::kOffP) + warp * kDecBlk * 4;
  for (int bk = warp; bk < nblk; bk += 4) {
    const int s = bk % kDecStages;
    const bool ok = mbar_wait(full + s, (bk / kDecStages) & 1, abort, status);
    if (!__all_sync(0xffffffffu, ok)) break;
    const uint8_t* kb = sK + s * C::kBlkBytes;
    const uint8_t* vb = sV + s * C::kBlkBytes;
    const int nk = min(kDecBlk, k1 - (k0 + bk * kDecBlk));
    const bool valid = lane < nk;
    // scores of this lane's key for the GT heads (base-2 units: q carries scale * log2 e); two
    // independent pair accumulators per head
    uint64_t sc2[GT][2];
#pragma unroll
    for (int t = 0; t < GT; ++t) sc2[t][0] = sc2[t][1] = 0ull;
#pragma unroll
    for (int cc = 0; cc < D / 8; ++cc) {
      const uint4 w = *reinterpret_cast<const uint4*>(kb + dec_sw<D>(lane, cc * 8));
      const uint64_t kp0 = f2_pack(bf16_lo(w.x), bf16_hi(w.x)), kp1 = f2_pack(bf16_lo(w.y), bf16_hi(w.y));
      const uint64_t kp2 = f2_pack(bf16_lo(w.z), bf16_hi(w.z)), kp3 = f2_pack(bf16_lo(w.w), bf16_hi(w.w));
#pragma unroll
      for (int t = 0; t < GT; ++t) {
        const float4 qa = *reinterpret_cast<const float4*>(&qs[t][8 * cc]);
        const float4 qb = *reinterpret_cast<const float4*>(&qs[t][8 * cc + 4]);
        sc2[t][0] = f2_fma(f2_pack(qa.x, qa.y), kp0, sc2[t][0]);
        sc2[t][1] = f2_fma(f2_pack(qa.z, qa.w), kp1, sc2[t][1]);
        sc2[t][0] = f2_fma(f2_pack(qb.x, qb.y), kp2, sc2[t][0]);
        sc2[t][1] = f2_fma(f2_pack(qb.z, qb.w), kp3, sc2[t][1]);
      }
    }
    float p[GT];
#pragma unroll
    for (int t = 0; t < GT; ++t) {
      float a0, a1, b0, b1;
      f2_unpack(sc2[t][0], a0, a1);
      f2_unpack(sc2[t][1], b0, b1);
      const float st = valid ? (a0 + a1) + (b0 + b1) : -INFINITY;
      const float mn = fmaxf(m[t], warp_max(st));  // finite: lane 0's key is valid
      const float alpha = fast_exp2(m[t] - mn);     // 2^(-inf) = 0 on the first block
      p[t] = valid ? fast_exp2(st - mn) : 0.f;
      ls[t] = ls[t] * alpha + p[t];
      const uint64_t al2 = f2_pack(alpha, alpha);
#pragma unroll
      for (int e = 0; e < PPL; ++e) acc2[t][e] = f2_mul(acc2[t][e], al2);
      m[t] = mn;
    }
    // this lane's key probabilities, duplicated into pairs, for the whole warp
#pragma unroll
    for (int t = 0; t < GT; ++t) sp[lane * 4 + t] = f2_pack(p[t], p[t]);
    __syncwarp();
    for (int j = 0; j < nk; ++j) {
      const uint8_t* vr = vb + dec_sw<D>(j, vd);
      uint64_t vp[PPL];
      if constexpr (DPL == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(vr);
        vp[0] = f2_pack(bf16_lo(w.x), bf16_hi(w.x));
        vp[1] = f2_pack(bf16_lo(w.y), bf16_hi(w.y));
      } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(vr);
        vp[0] = f2_pack(bf16_lo(w), bf16_hi(w));
      }
#pragma unroll
      for (int t = 0; t < GT; ++t) {
        const uint64_t pj = sp[j * 4 + t];  // same address in every lane: a broadcast
#pragma unroll
        for (int e = 0; e < PPL; ++e) acc2[t][e] = f2_fma(pj, vp[e], acc2[t][e]);
      }
    }
    __syncwarp();  // sp is rewritten by the next block
    if (lane == 0) mbar_arrive(empty + s);
  }
  float acc[GT][DPL];
#pragma unroll
  for (int t = 0; t < GT; ++t)
#pragma unroll
    for (int e = 0; e < PPL; ++e) f2_unpack(acc2[t][e], acc[t][2 * e], acc[t][2 * e + 1]);

  // merge the four warps' triples (a warp that saw no block holds the identity); red_o overlays the
  // K ring, so every compute warp must be done reading it first
  named_barrier(1, 128);
#pragma unroll
  for (int t = 0; t < GT; ++t) {
    const float lw = warp_sum(ls[t]);
    if (lane == 0) {
      red_m[warp][t] = m[t];
      red_l[warp][t] = lw;
    }
#pragma unroll
    for (int e = 0; e < DPL; ++e) red_o[warp][t][vd + e] = acc[t][e];
  }
  named_barrier(1, 128);  // the four compute warps only
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
        const float wt = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
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
                         const CUtensorMap& mk, const CUtensorMap& mv, const int* offsets, const int* num_splits,
                         float* part_o, float* part_ml, cudaStream_t st) {
  using C = DecCfg<D>;
  const int npass = (p.Hq / p.Hkv) / GT;
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, GT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.max_splits, p.Hkv * npass, p.N);
  {
    LaunchScope ls("decode_split", st);
    decode_split_kernel<D, GT><<<grid, kDecThreads, C::kSmemBytes, st>>>(
        mk, mv, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v),
        offsets, p.N, num_splits, p.max_splits, p.Hq, p.Hkv, p.scale * kLog2e, part_o, part_ml,
        device_status_ptr());
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
  // K and V as 3-D maps (D, Hkv, rows) over the packed caches. The row extent is nominal (the real
  // count is on the device); the kernel never issues a box that reaches past kv_offsets[N].
  CUtensorMap mk, mv;
  if (!make_map_packed_bf16(&mk, k, kDecMapRows, p.Hkv, D, kDecBlk) ||
      !make_map_packed_bf16(&mv, v, kDecMapRows, p.Hkv, D, kDecBlk))
    return cudaErrorInvalidValue;
  const int G = p.Hq / p.Hkv;
  cudaError_t e;
  if (G % 4 == 0)  // at most four query heads per CTA
    e = launch_split<D, 4>(p, q, k, v, mk, mv, offsets, num_splits, part_o, part_ml, st);
  else if (G % 2 == 0)
    e = launch_split<D, 2>(p, q, k, v, mk, mv, offsets, num_splits, part_o, part_ml, st);
  else
    e = launch_split<D, 1>(p, q, k, v, mk, mv, offsets, num_splits, part_o, part_ml, st);
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
