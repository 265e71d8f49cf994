// bwd_sm100.cu -- attention backward on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The backward of O = softmax(scale Q K^T + mask) V ("Não escreva kernels, derive-os", "Perguntas
// frequentes": the backward comes out of rewrites of the same graph), written from the softmax
// Jacobian: with P recomputed from lse, dP = dO V^T, Delta_i = dO_i . O_i and dS = P (dP - Delta),
//   dV = P^T dO,   dK = scale dS^T Q,   dQ = scale dS K,
// dK and dV summed over the query heads of a key/value head's group.
//
// Three launches on the caller's stream:
//   bwd_prep        Delta_i = dO_i . O_i, lse in base 2, and the fp32 dQ accumulator cleared;
//   bwd_sm100       one CTA per (128-key tile, kv head): loops over the group's query heads x
//                   64-row query tiles, keeps dK and dV for its keys in TMEM, and adds each tile's
//                   dQ into the fp32 accumulator with TMA bulk reduce-add;
//   bwd_dq_convert  dQ = scale * accumulator, rounded to bf16.
//
// The main kernel works on transposed score tiles so that keys sit on the TMEM lanes:
//   S^T = K Q^T and dP^T = V dO^T   (M = 128 keys, N = 64 query rows, K = D),
// then one thread per key computes P^T = 2^(S^T scale log2e - lse2) and dS^T = P^T (dP^T - Delta),
// writes both once to shared memory (bf16, 128-byte swizzle), and three more MMAs use them:
//   dV += P^T dO,  dK += dS^T Q     (M = 128 keys, N = D, K = 64 rows; A K-major, B MN-major)
//   dQ^T = K^T dS^T                 (M = D, N = 64 rows, K = 128 keys; A and B MN-major).
// For D = 64 the dQ^T MMA still runs with M = 128; the upper 64 TMEM lanes hold values that are
// never read.
// TMEM columns: S^T [0,64), dP^T [64,128), dQ^T [128,192), dV [256,256+D), dK [384,384+D).
//
// Warp roles (320 threads): warps 0-3 scores (one key row per thread; at the end the dK/dV
// epilogue), warps 4-7 dQ drain (one TMEM lane per thread: tcgen05.ld -> shared -> per-warp TMA
// reduce-add of 32 columns),
// warp 8 TMA producer (K, V once; Q and dO tiles through a ring), warp 9 TMEM allocator and MMA
// issuer (one elected lane). The MMA issuer puts the next tile's S^T/dP^T ahead of the current tile's gradient MMAs
// so that the tensor cores work while the score warps compute P and dS. Every wait is bounded.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"

namespace attn {
namespace {

constexpr int kBM = 64;    // query rows per iteration
constexpr int kBN = 128;   // keys per CTA
constexpr int kThreads = 320;
constexpr int kKAtom = 128 * 128;  // a 128-row x 128-byte swizzle atom (16 KB)
constexpr int kQAtom = 64 * 128;   // a 64-row x 128-byte swizzle atom (8 KB)

template <int D>
struct BwdCfg {
  static constexpr int kAtoms = D / 64;
  static constexpr int kKVBytes = kAtoms * kKAtom;  // 128 x D bf16
  static constexpr int kQBytes = kAtoms * kQAtom;   // 64 x D bf16
  static constexpr int kStages = (D == 128) ? 2 : 3;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKVBytes;
  static constexpr int kOffQ = kOffV + kKVBytes;
  static constexpr int kOffDO = kOffQ + kStages * kQBytes;
  static constexpr int kOffP = kOffDO + kStages * kQBytes;
  static constexpr int kOffDS = kOffP + kKAtom;           // 128 keys x 64 rows bf16 = one 16 KB atom
  static constexpr int kOffDQ = kOffDS + kKAtom;          // fp32 [64 rows][D] staging for the reduce
  static constexpr int kOffRow = kOffDQ + kBM * D * 4;    // per score warp: 2 x (lse2, Delta) x 64 rows
  static constexpr int kOffBar = kOffRow + 4 * 2 * 2 * kBM * 4;
  static constexpr int kNumBars = 1 + 2 * kStages + 8;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;
  static constexpr uint32_t kColS = 0, kColDP = 64, kColDQ = 128, kColDV = 256, kColDK = 384;
};

struct BwdArgs {
  int B, Hq, Hkv, Sq, Sk;
  int causal;
  float scale;       // softmax scale (dK is multiplied by it here; dQ in the convert kernel)
  float scale_log2;  // scale * log2(e)
  const float* lse2;   // [B, Hq, Sq] lse * log2(e), +inf where a row sees no key
  const float* delta;  // [B, Hq, Sq]
  uint16_t* dk;
  uint16_t* dv;
  int* status;
};

__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                     const __grid_constant__ CUtensorMap tmDQ, const BwdArgs a) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sDO = smem + C::kOffDO;
  uint8_t* sP = smem + C::kOffP;
  uint8_t* sDS = smem + C::kOffDS;
  float* sDQ = reinterpret_cast<float*>(smem + C::kOffDQ);  // per drain warp: [64 rows][32 d] fp32
  float* sRow = reinterpret_cast<float*>(smem + C::kOffRow);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;
  uint64_t* q_empty = q_full + C::kStages;
  uint64_t* s_full = q_empty + C::kStages;
  uint64_t* st_free = s_full + 1;
  uint64_t* p_full = st_free + 1;
  uint64_t* pds_free = p_full + 1;
  uint64_t* dq_full = pds_free + 1;
  uint64_t* dq_free = dq_full + 1;
  uint64_t* all_done = dq_free + 1;
  uint64_t* drain = all_done + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = static_cast<int>(blockIdx.x) % a.Hkv;
  const int b = static_cast<int>(blockIdx.x) / a.Hkv;
  const int kt = blockIdx.y;  // key tile; small indices carry the most work under a causal mask
  const int k0 = kt * kBN;
  const int G = a.Hq / a.Hkv;
  const int n_qt_all = (a.Sq + kBM - 1) / kBM;
  int qt0 = 0;  // first query tile that sees any key of this tile
  if (a.causal) {
    const int qmin = k0 - (a.Sk - a.Sq);  // rows q >= qmin see key k0
    qt0 = qmin <= 0 ? 0 : qmin / kBM;
  }
  const int n_q = qt0 < n_qt_all ? n_qt_all - qt0 : 0;
  const int n_it = G * n_q;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(st_free, 4);
    mbar_init(p_full, 4);
    mbar_init(pds_free, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 4);
    mbar_init(all_done, 1);
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
    tma_prefetch_desc(&tmDQ);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n_it > 0) {
      constexpr uint32_t kKVTx = 2u * kBN * D * 2;
      constexpr uint32_t kQTx = 2u * kBM * D * 2;
      mbar_arrive_expect_tx(kv_full, kKVTx);
#pragma unroll
      for (int at = 0; at < C::kAtoms; ++at) {
        tma_load_4d(sK + at * kKAtom, &tmK, kv_full, at * 64, g, k0, b);
        tma_load_4d(sV + at * kKAtom, &tmV, kv_full, at * 64, g, k0, b);
      }
      int issued = 0;
      for (int j = 0; j < n_it; ++j) {
        const int s = j % C::kStages;
        const int h = g * G + j / n_q;
        const int qt = qt0 + j % n_q;
        if (!mbar_wait(q_empty + s, ((j / C::kStages) & 1) ^ 1, abort, a.status)) break;
        mbar_arrive_expect_tx(q_full + s, kQTx);
#pragma unroll
        for (int at = 0; at < C::kAtoms; ++at) {
          tma_load_4d(sQ + s * C::kQBytes + at * kQAtom, &tmQ, q_full + s, at * 64, h, qt * kBM, b);
          tma_load_4d(sDO + s * C::kQBytes + at * kQAtom, &tmDO, q_full + s, at * 64, h, qt * kBM, b);
        }
        issued = j + 1;
      }
      wait_drain(kv_full, 0);
      for (int j = max(0, issued - C::kStages); j < issued; ++j)
        wait_drain(q_full + j % C::kStages, (j / C::kStages) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    if (n_it > 0) {  // the whole warp runs the loop; one elected lane issues each MMA
      constexpr uint32_t kIdS = idesc_bf16_f32(kBN, kBM, 0, 0);  // S^T, dP^T
      constexpr uint32_t kIdG = idesc_bf16_f32(kBN, D, 0, 1);    // dV, dK
      constexpr uint32_t kIdQ = idesc_bf16_f32(128, kBM, 1, 1);  // dQ^T (M = 128 also for D = 64)
      // base descriptors, built once; each MMA only moves the start address
      const uint64_t kK = sdesc_sw128(smem_u32(sK), 16, 1024);        // K-major operands
      const uint64_t kV = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t kQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t kDO = sdesc_sw128(smem_u32(sDO), 16, 1024);
      const uint64_t kP = sdesc_sw128(smem_u32(sP), 16, 1024);
      const uint64_t kDS = sdesc_sw128(smem_u32(sDS), 16, 1024);
      const uint64_t mQ = sdesc_sw128(smem_u32(sQ), kQAtom, 1024);    // MN-major operands
      const uint64_t mDO = sdesc_sw128(smem_u32(sDO), kQAtom, 1024);
      const uint64_t mK = sdesc_sw128(smem_u32(sK), kKAtom, 1024);
      const uint64_t mDS = sdesc_sw128(smem_u32(sDS), kQAtom, 1024);
      bool ok = __all_sync(0xffffffffu, mbar_wait(kv_full, 0, abort, a.status));
      for (int j = 0; ok && j <= n_it; ++j) {
        if (j < n_it) {
          const int s = j % C::kStages;
          if (!__all_sync(0xffffffffu, mbar_wait(q_full + s, (j / C::kStages) & 1, abort, a.status))) break;
          if (!__all_sync(0xffffffffu, mbar_wait(st_free, (j & 1) ^ 1, abort, a.status))) break;
          tc_fence_after();
          const uint64_t q = sdesc_advance(kQ, s * C::kQBytes), dO = sdesc_advance(kDO, s * C::kQBytes);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t ok_ = (kk >> 2) * kKAtom + (kk & 3) * 32;
            const uint32_t oq = (kk >> 2) * kQAtom + (kk & 3) * 32;
            umma_ss_warp(tmem + C::kColS, sdesc_advance(kK, ok_), sdesc_advance(q, oq), kIdS, kk > 0);
            umma_ss_warp(tmem + C::kColDP, sdesc_advance(kV, ok_), sdesc_advance(dO, oq), kIdS, kk > 0);
          }
          umma_commit_warp(s_full);
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int s = jj % C::kStages;
          if (!__all_sync(0xffffffffu, mbar_wait(p_full, jj & 1, abort, a.status))) break;
          if (!__all_sync(0xffffffffu, mbar_wait(dq_free, (jj & 1) ^ 1, abort, a.status))) break;
          tc_fence_after();
          const uint64_t q = sdesc_advance(mQ, s * C::kQBytes), dO = sdesc_advance(mDO, s * C::kQBytes);
          // dV += P^T dO, dK += dS^T Q: K = 64 query rows in 4 steps of 16
#pragma unroll
          for (int kk = 0; kk < kBM / 16; ++kk) {
            const uint32_t oa = kk * 32;          // 16 rows = 32 bytes along the swizzled K-major row
            const uint32_t ob = kk * 16 * 128;    // 16 rows of 128 bytes in the MN-major operand
            const uint32_t acc = (jj > 0 || kk > 0);
            umma_ss_warp(tmem + C::kColDV, sdesc_advance(kP, oa), sdesc_advance(dO, ob), kIdG, acc);
            umma_ss_warp(tmem + C::kColDK, sdesc_advance(kDS, oa), sdesc_advance(q, ob), kIdG, acc);
          }
          // dQ^T = K^T dS^T: K = 128 keys in 8 steps of 16
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint32_t o = kk * 16 * 128;
            umma_ss_warp(tmem + C::kColDQ, sdesc_advance(mK, o), sdesc_advance(mDS, o), kIdQ, kk > 0);
          }
          umma_commit_warp(q_empty + s);
          umma_commit_warp(pds_free);
          umma_commit_warp(dq_full);
        }
      }
      umma_commit_warp(all_done);
      umma_commit_warp(drain);
      wait_drain(drain, 0);
      __syncwarp();
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------------ score warps (row = key)
    const int t = threadIdx.x;  // TMEM lane == key row in the tile
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const int key = k0 + t;
    bool ok = true;
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
      const bool r = mbar_wait(bar, parity, abort, a.status);
      return __all_sync(0xffffffffu, r);
    };
    // lse2 and Delta of a query tile's 64 rows, staged per warp (no cross-warp barrier): lane l
    // fetches rows l and l + 32 of both; buffer (j & 1) serves tile j.
    float* wrow = sRow + warp * (2 * 2 * kBM);
    auto fetch_rows = [&](int j, float (&v)[4]) {
      const int h = g * G + j / n_q;
      const int qb = (qt0 + j % n_q) * kBM;
      const long long base = (static_cast<long long>(b) * a.Hq + h) * a.Sq;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int q = qb + lane + 32 * u;
        v[u] = q < a.Sq ? a.lse2[base + q] : INFINITY;
        v[2 + u] = q < a.Sq ? a.delta[base + q] : 0.f;
      }
    };
    auto stage_rows = [&](int buf, const float (&v)[4]) {
      float* w = wrow + buf * 2 * kBM;
      w[lane] = v[0];
      w[lane + 32] = v[1];
      w[kBM + lane] = v[2];
      w[kBM + lane + 32] = v[3];
    };
    if (n_it > 0) {
      float v0[4];
      fetch_rows(0, v0);
      stage_rows(0, v0);
    }
    __syncwarp();
    for (int j = 0; j < n_it; ++j) {
      float next[4] = {0.f, 0.f, 0.f, 0.f};
      if (j + 1 < n_it) fetch_rows(j + 1, next);  // in flight during this tile
      const float* rl = wrow + (j & 1) * 2 * kBM;
      const float* rd = rl + kBM;
      const int qt = qt0 + j % n_q;
      if (!wait_warp(s_full, j & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int q0 = qt * kBM;
      // Visible columns of this key's row form one window [cmin, cmax): query rows before the
      // causal limit (q >= key - (Sk - Sq)) and inside Sq; nothing if the key is beyond Sk.
      const int cmin = a.causal ? key - (a.Sk - a.Sq) - q0 : 0;
      const int cmax = key < a.Sk ? min(kBM, a.Sq - q0) : 0;
      uint32_t pk[kBM / 2], dk[kBM / 2];
#pragma unroll
      for (int part = 0; part < kBM / 16; ++part) {  // 16 columns at a time keeps the register count down
        uint32_t sr[16], dp[16];
        tmem_ld16(tmem + lane_addr + C::kColS + part * 16, sr);
        tmem_ld16(tmem + lane_addr + C::kColDP + part * 16, dp);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 16; cc += 2) {
          const int c = part * 16 + cc;
          float p0 = exp2f(fmaf(__uint_as_float(sr[cc]), a.scale_log2, -rl[c]));
          float p1 = exp2f(fmaf(__uint_as_float(sr[cc + 1]), a.scale_log2, -rl[c + 1]));
          p0 = (c >= cmin && c < cmax) ? p0 : 0.f;
          p1 = (c + 1 >= cmin && c + 1 < cmax) ? p1 : 0.f;
          const float d0 = p0 * (__uint_as_float(dp[cc]) - rd[c]);
          const float d1 = p1 * (__uint_as_float(dp[cc + 1]) - rd[c + 1]);
          pk[c / 2] = pack_bf16(p0, p1);
          dk[c / 2] = pack_bf16(d0, d1);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(st_free);
      // the gradient MMAs of the previous tile must be done with P^T and dS^T in shared memory
      if (!wait_warp(pds_free, (j & 1) ^ 1)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int ch = 0; ch < kBM / 8; ++ch) {
        *reinterpret_cast<uint4*>(sP + sw128_offset(t, ch)) =
            make_uint4(pk[ch * 4], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
        *reinterpret_cast<uint4*>(sDS + sw128_offset(t, ch)) =
            make_uint4(dk[ch * 4], dk[ch * 4 + 1], dk[ch * 4 + 2], dk[ch * 4 + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      // the next tile's lse2 / Delta into the other buffer (this warp finished reading it last tile)
      stage_rows((j + 1) & 1, next);
      __syncwarp();
    }
    // dK / dV epilogue: TMEM rows -> bf16 global rows of this key tile
    if (ok && n_it > 0) ok = wait_warp(all_done, 0);
    tc_fence_after();
    const bool store = key < a.Sk;
    const long long row = ((static_cast<long long>(b) * a.Sk + key) * a.Hkv + g) * D;
#pragma unroll 1
    for (int which = 0; which < 2; ++which) {
      const uint32_t col = which == 0 ? C::kColDV : C::kColDK;
      const float mul = which == 0 ? 1.f : a.scale;
      uint16_t* dst = (which == 0 ? a.dv : a.dk) + row;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t r[16];
        if (ok && n_it > 0) {
          tmem_ld16(tmem + lane_addr + col + c0, r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = 0u;
        }
        if (store) {
          uint4 w0, w1;
          w0.x = pack_bf16(__uint_as_float(r[0]) * mul, __uint_as_float(r[1]) * mul);
          w0.y = pack_bf16(__uint_as_float(r[2]) * mul, __uint_as_float(r[3]) * mul);
          w0.z = pack_bf16(__uint_as_float(r[4]) * mul, __uint_as_float(r[5]) * mul);
          w0.w = pack_bf16(__uint_as_float(r[6]) * mul, __uint_as_float(r[7]) * mul);
          w1.x = pack_bf16(__uint_as_float(r[8]) * mul, __uint_as_float(r[9]) * mul);
          w1.y = pack_bf16(__uint_as_float(r[10]) * mul, __uint_as_float(r[11]) * mul);
          w1.z = pack_bf16(__uint_as_float(r[12]) * mul, __uint_as_float(r[13]) * mul);
          w1.w = pack_bf16(__uint_as_float(r[14]) * mul, __uint_as_float(r[15]) * mul);
          *reinterpret_cast<uint4*>(dst + c0) = w0;
          *reinterpret_cast<uint4*>(dst + c0 + 8) = w1;
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ dQ drain (warps 4-7)
    // Warp w drains TMEM lanes 32w..32w+31, i.e. head-dim columns d = 32w + lane of dQ, into its own
    // [64 rows][32] fp32 staging tile, and its lane 0 adds that tile into the accumulator with one
    // TMA bulk reduce: no barrier across warps.
    const int wq = warp - 4;
    const int d = wq * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    float* stage = sDQ + wq * (kBM * 32);
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
      const bool r = mbar_wait(bar, parity, abort, a.status);
      return __all_sync(0xffffffffu, r);
    };
    for (int j = 0; j < n_it; ++j) {
      const int h = g * G + j / n_q;
      const int qt = qt0 + j % n_q;
      if (!wait_warp(dq_full, j & 1)) break;
      tc_fence_after();
      uint32_t r[kBM];
#pragma unroll
      for (int c = 0; c < kBM / 16; ++c) tmem_ld16(tmem + lane_addr + C::kColDQ + c * 16, r + c * 16);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_free);
      if (d < D) {  // at D = 64 warps 6 and 7 hold no dQ column
        if (lane == 0) bulk_wait_read_all();  // this warp's previous reduce has read its staging tile
        __syncwarp();
#pragma unroll
        for (int c = 0; c < kBM; ++c) stage[c * 32 + lane] = __uint_as_float(r[c]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_4d(&tmDQ, stage, wq * 32, h, qt * kBM, b);
          bulk_commit_group();
        }
      }
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Delta = rowsum(dO * O), lse2 = lse * log2(e) (+inf for rows that see no key), dQ accumulator = 0.
// One warp per (b, i, h) row.
template <int D>
__global__ void __launch_bounds__(128) bwd_prep_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
                                                       const float* __restrict__ lse, float* __restrict__ lse2,
                                                       float* __restrict__ delta, float* __restrict__ dq_acc, int B,
                                                       int Hq, int Sq) {
  constexpr int DPL = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * 4 + warp;  // (b, i, h), h fastest
  if (row >= static_cast<long long>(B) * Sq * Hq) return;
  const int h = static_cast<int>(row % Hq);
  const int i = static_cast<int>((row / Hq) % Sq);
  const int b = static_cast<int>(row / (static_cast<long long>(Hq) * Sq));
  const long long base = row * D + lane * DPL;
  float s = 0.f;
  if constexpr (DPL == 4) {
    const uint2 x = *reinterpret_cast<const uint2*>(o + base);
    const uint2 y = *reinterpret_cast<const uint2*>(dout + base);
    s = bf16_lo(x.x) * bf16_lo(y.x) + bf16_hi(x.x) * bf16_hi(y.x) + bf16_lo(x.y) * bf16_lo(y.y) +
        bf16_hi(x.y) * bf16_hi(y.y);
    *reinterpret_cast<float4*>(dq_acc + base) = make_float4(0.f, 0.f, 0.f, 0.f);
  } else {
    const uint32_t x = *reinterpret_cast<const uint32_t*>(o + base);
    const uint32_t y = *reinterpret_cast<const uint32_t*>(dout + base);
    s = bf16_lo(x) * bf16_lo(y) + bf16_hi(x) * bf16_hi(y);
    *reinterpret_cast<float2*>(dq_acc + base) = make_float2(0.f, 0.f);
  }
  s = warp_sum(s);
  if (lane == 0) {
    const long long li = (static_cast<long long>(b) * Hq + h) * Sq + i;
    delta[li] = s;
    const float l = lse[li];
    lse2[li] = (l == -INFINITY) ? INFINITY : l * kLog2e;
  }
}

// dQ = scale * accumulator -> bf16, eight elements per thread.
__global__ void __launch_bounds__(256) bwd_dq_convert_kernel(const float* __restrict__ acc,
                                                             uint16_t* __restrict__ dq, long long n8,
                                                             float scale) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
  const float4 c = reinterpret_cast<const float4*>(acc)[2 * i + 1];
  uint4 w;
  w.x = pack_bf16(a.x * scale, a.y * scale);
  w.y = pack_bf16(a.z * scale, a.w * scale);
  w.z = pack_bf16(c.x * scale, c.y * scale);
  w.w = pack_bf16(c.z * scale, c.w * scale);
  reinterpret_cast<uint4*>(dq)[i] = w;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

template <int D>
cudaError_t launch_bwd_sm100_d(const Problem& p, const void* q, const void* k, const void* v, const void* o,
                               const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                               cudaStream_t st) {
  using C = BwdCfg<D>;
  const size_t rows = static_cast<size_t>(p.B) * p.Hq * p.Sq;
  float* dq_acc = static_cast<float*>(workspace);
  float* lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(rows * D * 4));
  float* delta = reinterpret_cast<float*>(reinterpret_cast<char*>(lse2) + align256(rows * 4));

  CUtensorMap mq, mk, mv, mdo, mdq;
  if (!make_map_bf16_sw128(&mq, q, p.B, p.Sq, p.Hq, D, kBM) || !make_map_bf16_sw128(&mdo, dout, p.B, p.Sq, p.Hq, D, kBM) ||
      !make_map_bf16_sw128(&mk, k, p.B, p.Sk, p.Hkv, D, kBN) || !make_map_bf16_sw128(&mv, v, p.B, p.Sk, p.Hkv, D, kBN) ||
      !make_map_bshd(&mdq, dq_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.B, p.Sq, p.Hq, D, 32, kBM,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;

  {
    LaunchScope ls("bwd_prep", st);
    bwd_prep_kernel<D><<<static_cast<unsigned>((rows + 3) / 4), 128, 0, st>>>(
        static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), lse, lse2, delta, dq_acc, p.B, p.Hq,
        p.Sq);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  e = cudaFuncSetAttribute(bwd_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  BwdArgs a;
  a.B = p.B;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.Sq = p.Sq;
  a.Sk = p.Sk;
  a.causal = p.causal;
  a.scale = p.scale;
  a.scale_log2 = p.scale * kLog2e;
  a.lse2 = lse2;
  a.delta = delta;
  a.dk = static_cast<uint16_t*>(dk);
  a.dv = static_cast<uint16_t*>(dv);
  a.status = device_status_ptr();
  dim3 grid(p.Hkv * p.B, (p.Sk + kBN - 1) / kBN);
  {
    LaunchScope ls("bwd_sm100", st);
    bwd_sm100_kernel<D><<<grid, kThreads, C::kSmemBytes, st>>>(mq, mk, mv, mdo, mdq, a);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  const long long n8 = static_cast<long long>(rows) * D / 8;
  {
    LaunchScope ls("bwd_dq_convert", st);
    bwd_dq_convert_kernel<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, st>>>(
        dq_acc, static_cast<uint16_t*>(dq), n8, p.scale);
  }
  return cudaGetLastError();
}

}  // namespace

size_t bwd_sm100_workspace_bytes(int B, int Hq, int Sq, int D) {
  const size_t rows = static_cast<size_t>(B) * Hq * Sq;
  return align256(rows * D * 4) + 2 * align256(rows * 4);
}

cudaError_t launch_bwd_sm100(const Problem& p, const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                             cudaStream_t st) {
  if (p.D == 128) return launch_bwd_sm100_d<128>(p, q, k, v, o, lse, dout, dq, dk, dv, workspace, st);
  return launch_bwd_sm100_d<64>(p, q, k, v, o, lse, dout, dq, dk, dv, workspace, st);
}

}  // namespace attn
