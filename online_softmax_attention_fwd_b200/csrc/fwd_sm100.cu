// fwd_sm100.cu -- attention forward on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The forward is one reduction over key blocks under the online-softmax monoid ("Não escreva
// kernels, derive-os", "Aprofundamento", first paragraph): for a tile of 128 query rows the CTA
// keeps, per row, the triple (m, l, O) -- running max (base-2 units), running sum of 2^(s - m) and
// the unnormalised output -- and folds in one 128-key block at a time:
//   S = Q K^T (tensor cores, fp32 in TMEM), m' = max(m, rowmax S), P = 2^(S - m'),
//   l = l 2^(m - m') + rowsum P, O = O 2^(m - m') + P V (tensor cores, fp32 in TMEM).
// The two contractions are dense, so they run as tcgen05.mma (bf16 operands from shared memory,
// fp32 accumulators in tensor memory); the row statistics run on the CUDA cores, one thread per row.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: read S from TMEM, mask, row max / sum, write P (bf16, swizzled) to SMEM,
//              rescale O in TMEM when a row max grows by more than 2^8, epilogue O / l and lse.
//   warp 4     TMA producer: Q tile once, then K and V blocks into a ring of stages.
//   warp 5     TMEM allocator and MMA issuer (one thread): S_j = Q K_j^T into one of two S buffers,
//              then O += P_{j-1} V_{j-1}, so the next S overlaps the softmax of the current block.
// Lazy rescaling: a row keeps its old max m while the block max stays within m + 8 (base 2); P then
// stays <= 256 and the final O / l and lse = m + log2 l use the same m, so the result is exact.
//
// Shared-memory tiles use the 128-byte swizzle: Q, K and P are K-major (rows of 64 bf16 = 128 B),
// V is read as an MN-major operand (its head dim is contiguous). Every wait is bounded (common.cuh).
#include <math.h>
#include <stdio.h>

#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"

namespace attn {
namespace {

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per block
constexpr int kThreads = 192;
constexpr int kAtomBytes = 128 * 128;  // one 128-row x 128-byte swizzle atom column (16 KB)

template <int D>
struct FwdCfg {
  static constexpr int kAtoms = D / 64;                 // 64-element column atoms per tile row
  static constexpr int kTileBytes = kAtoms * kAtomBytes;  // a 128 x D bf16 tile
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffP = kOffV + kStages * kTileBytes;
  static constexpr int kOffBar = kOffP + 2 * kAtomBytes;  // P is 128 x 128 bf16 = two atoms
  static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 1 + 1 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + slack for 1024-byte alignment
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
};

struct FwdArgs {
  int B, Hq, Hkv, Sq, Sk;
  int causal;
  float scale_log2;  // softmax scale * log2(e)
  int n_qtiles;
  uint16_t* o;
  float* lse;
  int* status;
};

__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity) {
  // Bounded wait that ignores the abort flag: used only to let this thread's own in-flight async
  // work land before the CTA releases its shared and tensor memory.
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sP = smem + C::kOffP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + C::kStages;
  uint64_t* v_full = k_empty + C::kStages;
  uint64_t* v_empty = v_full + C::kStages;
  uint64_t* s_full = v_empty + C::kStages;  // [2]
  uint64_t* s_free = s_full + 2;            // [2]
  uint64_t* p_full = s_free + 2;
  uint64_t* o_done = p_full + 1;
  uint64_t* drain = o_done + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // blockIdx.y walks the query tiles from the last (longest under a causal mask) to the first, and
  // blockIdx.x, which varies fastest in launch order, covers every (batch, head): the longest tiles
  // of all heads start first.
  const int tile = a.n_qtiles - 1 - static_cast<int>(blockIdx.y);
  const int h = static_cast<int>(blockIdx.x) % a.Hq, b = static_cast<int>(blockIdx.x) / a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const int q0 = tile * kBM;
  int kv_end = a.Sk;  // keys [0, kv_end) can be visible to some row of this tile
  if (a.causal) kv_end = min(a.Sk, q0 + kBM + a.Sk - a.Sq);
  const int n_kv = kv_end > 0 ? (kv_end + kBN - 1) / kBN : 0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(s_free + s, 4);
    }
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t kBytes = kBM * D * 2;
      mbar_arrive_expect_tx(q_full, kBytes);
#pragma unroll
      for (int at = 0; at < C::kAtoms; ++at) tma_load_4d(sQ + at * kAtomBytes, &tmQ, q_full, at * 64, h, q0, b);
      int issued_k = 0, issued_v = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % C::kStages;
        const uint32_t ph = (j / C::kStages) & 1;
        if (!mbar_wait(k_empty + s, ph ^ 1, abort, a.status)) break;
        mbar_arrive_expect_tx(k_full + s, kBytes);
#pragma unroll
        for (int at = 0; at < C::kAtoms; ++at)
          tma_load_4d(sK + s * C::kTileBytes + at * kAtomBytes, &tmK, k_full + s, at * 64, g, j * kBN, b);
        issued_k = j + 1;
        if (!mbar_wait(v_empty + s, ph ^ 1, abort, a.status)) break;
        mbar_arrive_expect_tx(v_full + s, kBytes);
#pragma unroll
        for (int at = 0; at < C::kAtoms; ++at)
          tma_load_4d(sV + s * C::kTileBytes + at * kAtomBytes, &tmV, v_full + s, at * 64, g, j * kBN, b);
        issued_v = j + 1;
      }
      // Let every load this thread issued land before the CTA can exit. On the normal path the
      // consumers have already waited for each of them, so these return at once.
      wait_drain(q_full, 0);
      for (int j = max(0, issued_k - C::kStages); j < issued_k; ++j)
        wait_drain(k_full + j % C::kStages, (j / C::kStages) & 1);
      for (int j = max(0, issued_v - C::kStages); j < issued_v; ++j)
        wait_drain(v_full + j % C::kStages, (j / C::kStages) & 1);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, 0, 0);
      constexpr uint32_t kIdescO = idesc_bf16_f32(kBM, D, 0, 1);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
      bool ok = mbar_wait(q_full, 0, abort, a.status);
      for (int j = 0; ok && j <= n_kv; ++j) {
        if (j < n_kv) {
          const int s = j % C::kStages;
          const int sb = j & 1;
          if (!mbar_wait(k_full + s, (j / C::kStages) & 1, abort, a.status)) break;
          if (!mbar_wait(s_free + sb, ((j >> 1) & 1) ^ 1, abort, a.status)) break;
          tc_fence_after();
          const uint32_t dS = tmem + (sb ? C::kColS1 : C::kColS0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kAtomBytes + (kk & 3) * 32;
            umma_ss(dS, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(aK + s * C::kTileBytes + off, 16, 1024),
                    kIdescS, kk > 0);
          }
          umma_commit(s_full + sb);
          umma_commit(k_empty + s);
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int s = jj % C::kStages;
          if (!mbar_wait(p_full, jj & 1, abort, a.status)) break;
          if (!mbar_wait(v_full + s, (jj / C::kStages) & 1, abort, a.status)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint32_t offp = (kk >> 2) * kAtomBytes + (kk & 3) * 32;
            const uint32_t offv = kk * 16 * 128;  // 16 key rows of 128 bytes
            umma_ss(tmem + C::kColO, sdesc_sw128(aP + offp, 16, 1024),
                    sdesc_sw128(aV + s * C::kTileBytes + offv, kAtomBytes, 1024), kIdescO, (jj > 0 || kk > 0));
          }
          umma_commit(v_empty + s);
          umma_commit(o_done);
        }
      }
      // all MMAs issued by this thread complete before the CTA releases TMEM
      umma_commit(drain);
      wait_drain(drain, 0);
    }
  } else {
    // ------------------------------------------------------------------ softmax warpgroup
    const int row = threadIdx.x;  // 0..127 == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const int qrow = q0 + row;
    int row_limit = a.Sk - 1;  // largest visible key index for this row
    if (a.causal) row_limit = min(row_limit, qrow + a.Sk - a.Sq);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // every lane waits; the outcome is made warp-uniform before any warp-collective tcgen05 op
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
      const bool r = mbar_wait(bar, parity, abort, a.status);
      return __all_sync(0xffffffffu, r);
    };
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      if (!wait_warp(s_full + sb, (j >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 16; ++c) tmem_ld16(tmem + lane_addr + (sb ? C::kColS1 : C::kColS0) + c * 16, sr + c * 16);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free + sb);

      const int kbase = j * kBN;
      const bool need_mask = kbase + kBN - 1 > row_limit;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBN; ++c) {
        float x = __uint_as_float(sr[c]) * a.scale_log2;
        if (need_mask && kbase + c > row_limit) x = -INFINITY;
        sr[c] = __float_as_uint(x);
        mx = fmaxf(mx, x);
      }
      // lazy rescale: move the reference max only when the block max exceeds it by more than 8
      float alpha = 1.f;
      if (mx > m + 8.f || (m == -INFINITY && mx != -INFINITY)) {
        alpha = (m == -INFINITY) ? 0.f : exp2f(m - mx);
        m = mx;
      }
      const float m_use = (m == -INFINITY) ? 0.f : m;
      float rs = 0.f;
      uint32_t pk[kBN / 2];
#pragma unroll
      for (int c = 0; c < kBN; c += 2) {
        const float p0 = exp2f(__uint_as_float(sr[c]) - m_use);
        const float p1 = exp2f(__uint_as_float(sr[c + 1]) - m_use);
        rs += p0 + p1;
        pk[c / 2] = pack_bf16(p0, p1);
      }
      l = l * alpha + rs;

      // PV_{j-1} must be complete before O is rescaled and before P's buffer is overwritten.
      if (j >= 1) {
        if (!wait_warp(o_done, (j - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 16) {
            uint32_t orr[16];
            tmem_ld16(tmem + lane_addr + C::kColO + c0, orr);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
            tmem_st16(tmem + lane_addr + C::kColO + c0, orr);
          }
          tmem_wait_st();
        }
      }
      // P row -> shared memory, 128-byte swizzled K-major (two 64-key atoms)
#pragma unroll
      for (int ch = 0; ch < kBN / 8; ++ch) {
        uint4 w = make_uint4(pk[ch * 4 + 0], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
        *reinterpret_cast<uint4*>(sP + (ch >> 3) * kAtomBytes + sw128_offset(row, ch & 7)) = w;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && n_kv > 0) ok = wait_warp(o_done, (n_kv - 1) & 1);
    tc_fence_after();
    // epilogue: O / l -> bf16, lse = (m + log2 l) ln 2
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const bool store = qrow < a.Sq;
    uint16_t* orow = a.o + ((static_cast<long long>(b) * a.Sq + qrow) * a.Hq + h) * D;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 16) {
      uint32_t orr[16];
      if (ok && n_kv > 0) {
        tmem_ld16(tmem + lane_addr + C::kColO + c0, orr);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) orr[e] = 0u;
      }
      if (store) {
        uint4 w0, w1;
        w0.x = pack_bf16(__uint_as_float(orr[0]) * inv, __uint_as_float(orr[1]) * inv);
        w0.y = pack_bf16(__uint_as_float(orr[2]) * inv, __uint_as_float(orr[3]) * inv);
        w0.z = pack_bf16(__uint_as_float(orr[4]) * inv, __uint_as_float(orr[5]) * inv);
        w0.w = pack_bf16(__uint_as_float(orr[6]) * inv, __uint_as_float(orr[7]) * inv);
        w1.x = pack_bf16(__uint_as_float(orr[8]) * inv, __uint_as_float(orr[9]) * inv);
        w1.y = pack_bf16(__uint_as_float(orr[10]) * inv, __uint_as_float(orr[11]) * inv);
        w1.z = pack_bf16(__uint_as_float(orr[12]) * inv, __uint_as_float(orr[13]) * inv);
        w1.w = pack_bf16(__uint_as_float(orr[14]) * inv, __uint_as_float(orr[15]) * inv);
        *reinterpret_cast<uint4*>(orow + c0) = w0;
        *reinterpret_cast<uint4*>(orow + c0 + 8) = w1;
      }
    }
    if (store) a.lse[(static_cast<long long>(b) * a.Hq + h) * a.Sq + qrow] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------------------------
template <int D>
cudaError_t launch_fwd_sm100_d(const Problem& p, const void* q, const void* k, const void* v, void* o, float* lse,
                               cudaStream_t st) {
  using C = FwdCfg<D>;
  CUtensorMap mq, mk, mv;
  if (!make_map_bf16_sw128(&mq, q, p.B, p.Sq, p.Hq, D, kBM) || !make_map_bf16_sw128(&mk, k, p.B, p.Sk, p.Hkv, D, kBN) ||
      !make_map_bf16_sw128(&mv, v, p.B, p.Sk, p.Hkv, D, kBN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(fwd_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  FwdArgs a;
  a.B = p.B;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.Sq = p.Sq;
  a.Sk = p.Sk;
  a.causal = p.causal;
  a.scale_log2 = p.scale * kLog2e;
  a.n_qtiles = (p.Sq + kBM - 1) / kBM;
  a.o = static_cast<uint16_t*>(o);
  a.lse = lse;
  a.status = device_status_ptr();
  dim3 grid(p.Hq * p.B, a.n_qtiles);
  {
    LaunchScope ls("fwd_sm100", st);
    fwd_sm100_kernel<D><<<grid, kThreads, C::kSmemBytes, st>>>(mq, mk, mv, a);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_sm100(const Problem& p, const void* q, const void* k, const void* v, void* o, float* lse,
                             cudaStream_t st) {
  if (p.D == 128) return launch_fwd_sm100_d<128>(p, q, k, v, o, lse, st);
  return launch_fwd_sm100_d<64>(p, q, k, v, o, lse, st);
}

}  // namespace attn
