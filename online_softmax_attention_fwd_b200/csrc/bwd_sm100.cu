// bwd_sm100.cu -- attention backward on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The backward of O = softmax(scale Q K^T + mask) V ("Não escreva kernels, derive-os", "Perguntas
// frequentes": the backward comes out of rewrites of the same graph), written from the softmax
// Jacobian: with P recomputed from lse, dP = dO V^T, Delta_i = dO_i . O_i and dS = P (dP - Delta),
//   dV = P^T dO,   dK = scale dS^T Q,   dQ = scale dS K,
// dK and dV summed over the query heads of a key/value head's group.
//
// Three launches on the caller's stream:
//   bwd_prep        Delta_i = dO_i . O_i, lse in base 2, and the fp32 dQ accumulator cleared, all
//                   padded to a multiple of 128 query rows per (sequence, head) (padding rows:
//                   lse2 = +inf, Delta = 0); packed batches get the longest sequence's padded rows;
//   bwd_sm100       one CTA per (128-key tile, kv head): loops over the group's 64-row query tiles
//                   (from the last one down) x query heads, keeps dK and dV for its keys in TMEM,
//                   and adds each tile's dQ into the fp32 accumulator;
//   bwd_dq_convert  dQ = scale * accumulator, rounded to bf16.
//
// The main kernel works on transposed score tiles so that keys sit on the TMEM lanes:
//   S^T = K Q^T and dP^T = V dO^T            (M = 128 keys, N = 64 query rows, K = D).
// Two query tiles are in flight: tile j lives in TMEM buffer j % 2 (S^T / P^T in 64 columns, dP^T /
// dS^T / dQ^T in 64 more) and is scored by warpgroup j % 2. One thread per key computes
// P^T = 2^(S^T scale log2e - lse2) as soon as S^T is in TMEM (kept in registers and written back as
// bf16 over the first 32 S^T columns), and dS^T = P^T (dP^T - Delta) once dP^T is (written back over
// the first 32 dP^T columns and into the tile's dS^T tile in shared memory, 128-byte swizzle). Then
//   dV += P^T dO,  dK += dS^T Q              (A = P^T / dS^T in TMEM, B = dO / Q MN-major in SMEM)
//   dQ^T = K^T dS^T                          (M = D, N = 64 query rows, K = 128 keys; both in SMEM)
// Issue order for tile j: dV, dK, dQ^T over the dP^T columns (which dK has read), S^T of tile j + 2
// over P^T (which dV has read; it keeps the tensor pipe busy while the drain reads dQ^T), and dP^T of
// tile j + 2 once the drain has read dQ^T. MMAs execute in issue order, which is what makes each
// overwrite in TMEM safe. The drain adds a tile's dQ into the accumulator only once that dP^T is
// complete: its vector reductions use the same L1 data path as the tensor pipe's shared-memory
// operand reads, and slowed the dP^T MMAs when the two ran at the same time. dQ is produced transposed (head
// dim on the TMEM lanes, query rows on the columns), and the fp32 accumulator interleaves groups of
// four query rows, [B, Hq, Sq_pad / 4, D, 4], so that a lane adds four consecutive rows of its
// column with one 16-byte vector reduction and a warp instruction covers 512 contiguous bytes. For
// D = 64 the dQ^T MMA still runs with M = 128; the upper 64 TMEM lanes hold values that are never
// read. TMEM columns: buffer b at [128 b, 128 b + 128), dV [256, 256 + D), dK [384, 384 + D).
//
// Warp roles (448 threads): warps 0-3 / 4-7 score the even / odd tiles (one key row per thread; at
// the end group 0 stores dV and group 1 dK), warps 8-11 dQ drain (one TMEM lane = one head-dim
// column per thread: the whole dQ^T row in one tcgen05.ld, TMEM released at once, then 4-wide fp32
// vector reductions into the interleaved accumulator), warp 12 TMA producer (K, V once; Q and dO
// tiles through a 4-stage ring), warp 13 TMEM allocator and MMA issuer (one elected lane of a
// converged warp). Every wait is bounded.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"

namespace attn {
namespace {

constexpr int kBM = 64;    // query rows per tile (two tiles in flight)
constexpr int kBN = 128;   // keys per CTA
constexpr int kThreads = 448;       // 14 warps
constexpr int kAtom = 128 * 128;    // a 128-row x 128-byte swizzle atom (16 KB)
constexpr int kAtom64 = 64 * 128;   // a 64-row x 128-byte swizzle atom (8 KB)

template <int D>
struct BwdCfg {
  static constexpr int kAtoms = D / 64;
  static constexpr int kKVBytes = kAtoms * kAtom;    // 128 key rows x D bf16 (K, V)
  static constexpr int kQBytes = kAtoms * kAtom64;   // 64 query rows x D bf16 (Q, dO)
  static constexpr int kStages = 4;                  // Q / dO ring: two tiles in flight + two ahead
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKVBytes;
  static constexpr int kOffQ = kOffV + kKVBytes;
  static constexpr int kOffDO = kOffQ + kStages * kQBytes;
  static constexpr int kOffDS = kOffDO + kStages * kQBytes;  // [2 tiles] 128 keys x 64 queries bf16
  static constexpr int kOffBar = kOffDS + 2 * kAtom;
  static constexpr int kNumBars = 1 + 2 * kStages + 6 * 2 + 2;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  // lse2 and Delta of each group's current tile ([2 groups][lse2 64, Delta 64]), read as float4
  static constexpr int kOffRow = (kOffMisc + 64 + 15) & ~15;
  static constexpr int kSmemBytes = kOffRow + 2 * 2 * kBM * 4 + 1024;
  static_assert(kOffRow % 16 == 0, "the lse2 / Delta rows are read with 16-byte loads");
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  // TMEM: tile buffer b holds S^T / P^T at 128 b and dP^T / dS^T / dQ^T at 128 b + 64 (64 columns
  // each); dV at 256, dK at 384
  __host__ __device__ static constexpr uint32_t colS(int b) { return 128u * b; }
  __host__ __device__ static constexpr uint32_t colDP(int b) { return 128u * b + 64u; }
  static constexpr uint32_t kColDV = 256, kColDK = 384;
};

struct BwdArgs {
  int B, Hq, Hkv, Sq, Sk;  // packed batches: the longest sequence's lengths
  int Sq_pad;        // Sq rounded up to a multiple of 128 (row count of lse2, delta, dq_acc per (b, h))
  int causal;
  float scale;       // softmax scale (dK is multiplied by it here; dQ in the convert kernel)
  float scale_log2;  // scale * log2(e)
  const float* lse2;   // [B, Hq, Sq_pad] lse * log2(e); +inf where a row sees no key or is padding
  const float* delta;  // [B, Hq, Sq_pad]; 0 on padding rows
  float* dq_acc;       // fp32, [B, Hq, Sq_pad / 4, D, 4]: element (b, q, h, d) at
                       // (((b Hq + h) Sq_pad / 4 + q / 4) D + d) 4 + q % 4
  uint16_t* dk;
  uint16_t* dv;
  int* status;
  // Packed batches: sequence b owns rows cu_q[b] .. cu_q[b + 1] - 1 of q / dO / dQ ([Tq, Hq, D]) and
  // cu_k[b] .. cu_k[b + 1] - 1 of k / v / dK / dV; null for the dense layout.
  const int* cu_q;
  const int* cu_k;
  int Tq, Tk;
  int fault_block;  // test-only fault-injection build: CTA 0 skips this Q / dO tile (-1: none)
  int n_kt;         // key tiles per sequence (of the longest one in a packed batch)
};

// Rows first .. first + len - 1 of sequence b in a packed tensor of T rows: false (and an empty
// span) when the device offsets fall outside it or exceed the bound the host passed.
__device__ __forceinline__ bool packed_rows(const int* cu, int b, int T, int maxlen, int& first, int& len) {
  const int r0 = cu[b], r1 = cu[b + 1];
  if (r0 < 0 || r1 < r0 || r1 > T || r1 - r0 > maxlen) {
    first = 0;
    len = 0;
    return false;
  }
  first = r0;
  len = r1 - r0;
  return true;
}

// Lengths and first packed rows of sequence b (dense: every sequence has Sq / Sk rows). A packed
// sequence with offsets outside the tensors counts as empty, and the device status records
// ATTN_ERR_INVALID_ARG.
struct BwdSpan {
  int Sq, Sk, q0, k0;
};
template <bool PACKED>
__device__ __forceinline__ BwdSpan bwd_span(const BwdArgs& a, int b) {
  if constexpr (PACKED) {
    BwdSpan s;
    const bool okq = packed_rows(a.cu_q, b, a.Tq, a.Sq, s.q0, s.Sq);
    const bool okk = packed_rows(a.cu_k, b, a.Tk, a.Sk, s.k0, s.Sk);
    if (!okq || !okk) {
      record_status(a.status, kStatusBadArg);
      return BwdSpan{0, 0, 0, 0};
    }
    return s;
  } else {
    return BwdSpan{a.Sq, a.Sk, b * a.Sq, b * a.Sk};
  }
}

__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

// p[0..3] += x[0..3] (fp32 bit patterns) with one vector reduction; p is 16-byte aligned
__device__ __forceinline__ void red_add_v4_f32(float* p, const uint32_t* x) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(__uint_as_float(x[0])),
               "f"(__uint_as_float(x[1])), "f"(__uint_as_float(x[2])), "f"(__uint_as_float(x[3]))
               : "memory");
}

// One CTA per SM. Its 14 warps put four on each of the SM's sub-partitions, and each sub-partition
// has 16 K registers: at most 128 registers per thread, which the compiler derives from these bounds.
template <int D, bool PACKED, bool SEQ_MAJOR>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                     const BwdArgs a) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sDO = smem + C::kOffDO;
  uint8_t* sDS = smem + C::kOffDS;  // [tile buffer] 128 keys x 64 queries, one 128-byte swizzle atom
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;               // [stage]
  uint64_t* q_empty = q_full + C::kStages;   // [stage]
  uint64_t* s_full = q_empty + C::kStages;   // [buffer] S^T of a tile is in TMEM
  uint64_t* dp_full = s_full + 2;            // [buffer] dP^T of a tile is in TMEM
  uint64_t* p_full = dp_full + 2;            // [buffer] P^T and dS^T written (TMEM and shared)
  uint64_t* ds_free = p_full + 2;            // [buffer] the dQ^T MMA has read dS^T in shared memory
  uint64_t* dq_full = ds_free + 2;           // [buffer] dQ^T of a tile is in TMEM
  uint64_t* dq_free = dq_full + 2;           // [buffer] the drain has read dQ^T out of TMEM
  uint64_t* all_done = dq_free + 2;
  uint64_t* drain = all_done + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA -> (sequence b, kv head g, key tile kt); under a causal mask small kt carry the most work.
  // Key tile by key tile over all sequences puts the heaviest CTAs first; sequence by sequence keeps
  // the CTAs that run together on one sequence's Q / dO and dQ rows, for batches whose rows do not
  // fit in L2 together (they would be streamed from DRAM once per wave of key tiles otherwise).
  // Key tile by key tile: grid (B Hkv, key tiles). Sequence by sequence: a 1-D grid, kv head fastest.
  const int bx = static_cast<int>(blockIdx.x);
  const int g = bx % a.Hkv;
  const int b = SEQ_MAJOR ? bx / (a.Hkv * a.n_kt) : bx / a.Hkv;
  const int kt = SEQ_MAJOR ? (bx / a.Hkv) % a.n_kt : static_cast<int>(blockIdx.y);
  const int k0 = kt * kBN;
  const int G = a.Hq / a.Hkv;
  const BwdSpan sp = bwd_span<PACKED>(a, b);
  constexpr bool packed = PACKED;
  // TMA coordinates: dense maps are (D, H, S, B); packed ones (D, H, T, 1) with the sequence's rows
  // starting at its first packed row (rows past its end belong to the next sequence: their lse2 is
  // +inf in the padded per-sequence rows, so their P and dS are 0)
  const int qrow0 = packed ? sp.q0 : 0, krow0 = packed ? sp.k0 : 0, bc = packed ? 0 : b;
  const int n_qt_all = (sp.Sq + kBM - 1) / kBM;  // 64-row query tiles of this sequence
  int qt0 = 0;  // first query tile that sees any key of this tile
  if (a.causal) {
    const int qmin = k0 - (sp.Sk - sp.Sq);  // rows q >= qmin see key k0
    qt0 = qmin <= 0 ? 0 : qmin / kBM;
  }
  const int n_q = (k0 < sp.Sk && qt0 < n_qt_all) ? n_qt_all - qt0 : 0;
  // tiles: query tile (slow, from the last one down) x query head (fast). Every key tile's CTA then
  // visits the query tiles in the same order, the last ones first, so the CTAs running at one time
  // work on nearly the same Q / dO tiles and dQ accumulator rows, which stay in L2 between them.
  const int n_it = G * n_q;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 1);
    }
    for (int bb = 0; bb < 2; ++bb) {
      mbar_init(s_full + bb, 1);
      mbar_init(dp_full + bb, 1);
      mbar_init(p_full + bb, 4);
      mbar_init(ds_free + bb, 1);
      mbar_init(dq_full + bb, 1);
      mbar_init(dq_free + bb, 4);
    }
    mbar_init(all_done, 1);
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == 12 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 12) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n_it > 0) {
      constexpr uint32_t kTxKV = kBN * D * 2, kTxQ = kBM * D * 2;
      mbar_arrive_expect_tx(kv_full, 2 * kTxKV);
#pragma unroll
      for (int at = 0; at < C::kAtoms; ++at) {
        tma_load_4d(sK + at * kAtom, &tmK, kv_full, at * 64, g, krow0 + k0, bc);
        tma_load_4d(sV + at * kAtom, &tmV, kv_full, at * 64, g, krow0 + k0, bc);
      }
      int issued = 0;
      for (int j = 0; j < n_it; ++j) {
        const int s = j % C::kStages;
        const int h = g * G + j % G;
        const int qt = n_qt_all - 1 - j / G;
        if (!mbar_wait(q_empty + s, ((j / C::kStages) & 1) ^ 1, abort, a.status)) break;
#ifdef ATTN_FAULT_INJECT
        if (blockIdx.x == 0 && blockIdx.y == 0 && j == a.fault_block) {  // the MMA warp's wait runs out
          issued = j + 1;
          continue;
        }
#endif
        mbar_arrive_expect_tx(q_full + s, 2 * kTxQ);
#pragma unroll
        for (int at = 0; at < C::kAtoms; ++at) {
          tma_load_4d(sQ + s * C::kQBytes + at * kAtom64, &tmQ, q_full + s, at * 64, h, qrow0 + qt * kBM, bc);
          tma_load_4d(sDO + s * C::kQBytes + at * kAtom64, &tmDO, q_full + s, at * 64, h, qrow0 + qt * kBM, bc);
        }
        issued = j + 1;
      }
      wait_drain(kv_full, 0);
      for (int j = max(0, issued - C::kStages); j < issued; ++j)
        wait_drain(q_full + j % C::kStages, (j / C::kStages) & 1);
    }
  } else if (warp == 13) {
    // ------------------------------------------------------------------ MMA issuer
    if (n_it > 0) {  // the whole warp runs the loop; one elected lane issues each MMA
      constexpr uint32_t kIdS = idesc_bf16_f32(kBN, kBM, 0, 0);  // S^T, dP^T: M 128 keys, N 64 queries
      constexpr uint32_t kIdG = idesc_bf16_f32(kBN, D, 0, 1);    // dV, dK (A in TMEM)
      constexpr uint32_t kIdQ = idesc_bf16_f32(128, kBM, 1, 1);  // dQ^T (M = 128 also for D = 64)
      // base descriptors, built once; each MMA only moves the start address
      const uint64_t kK = sdesc_sw128(smem_u32(sK), 16, 1024);       // K-major operands
      const uint64_t kV = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t kQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t kDO = sdesc_sw128(smem_u32(sDO), 16, 1024);
      const uint64_t mQ = sdesc_sw128(smem_u32(sQ), kAtom64, 1024);  // MN-major operands
      const uint64_t mDO = sdesc_sw128(smem_u32(sDO), kAtom64, 1024);
      const uint64_t mK = sdesc_sw128(smem_u32(sK), kAtom, 1024);
      const uint64_t mDS = sdesc_sw128(smem_u32(sDS), kAtom, 1024);
      auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, a.status)) != 0;
      };
      // S^T = K Q^T (or dP^T = V dO^T) of tile jt into its buffer: K = D in steps of 16; the 128-row
      // A tile and the 64-row B tile have different atom strides
      auto issue_scores = [&](int jt, uint64_t aK, uint64_t bQ, uint32_t col, uint64_t* bar) {
        const uint64_t bq = sdesc_advance(bQ, (jt % C::kStages) * C::kQBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss_warp(tmem + col, sdesc_advance(aK, (kk >> 2) * kAtom + (kk & 3) * 32),
                       sdesc_advance(bq, (kk >> 2) * kAtom64 + (kk & 3) * 32), kIdS, kk > 0);
        umma_commit_warp(bar);
      };
      bool ok = wait(kv_full, 0);
      for (int jt = 0; ok && jt < min(2, n_it); ++jt) {
        if (!wait(q_full + jt % C::kStages, (jt / C::kStages) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_scores(jt, kK, kQ, C::colS(jt & 1), s_full + (jt & 1));
        issue_scores(jt, kV, kDO, C::colDP(jt & 1), dp_full + (jt & 1));
      }
      for (int j = 0; ok && j < n_it; ++j) {
        const int bb = j & 1, s = j % C::kStages;
        // gradients of tile j once its P^T and dS^T are written
        if (!wait(p_full + bb, (j >> 1) & 1)) break;
        tc_fence_after();
        const uint64_t q = sdesc_advance(mQ, s * C::kQBytes), dO = sdesc_advance(mDO, s * C::kQBytes);
        // dV += P^T dO and dK += dS^T Q: K = 64 query rows in 4 steps of 16 (8 TMEM columns each)
#pragma unroll
        for (int kk = 0; kk < kBM / 16; ++kk)
          umma_ts_warp(tmem + C::kColDV, tmem + C::colS(bb) + kk * 8, sdesc_advance(dO, kk * 16 * 128), kIdG,
                       (j > 0 || kk > 0));
#pragma unroll
        for (int kk = 0; kk < kBM / 16; ++kk)
          umma_ts_warp(tmem + C::kColDK, tmem + C::colDP(bb) + kk * 8, sdesc_advance(q, kk * 16 * 128), kIdG,
                       (j > 0 || kk > 0));
        // dQ^T = K^T dS^T over the tile's dP^T / dS^T columns (dK has read dS^T): K = 128 keys in 8 steps
        const uint64_t ds = sdesc_advance(mDS, bb * kAtom);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          umma_ss_warp(tmem + C::colDP(bb), sdesc_advance(mK, kk * 16 * 128), sdesc_advance(ds, kk * 16 * 128), kIdQ,
                       kk > 0);
        umma_commit_warp(q_empty + s);
        umma_commit_warp(ds_free + bb);
        umma_commit_warp(dq_full + bb);
        if (j + 2 < n_it) {
          // S^T of tile j + 2 over P^T of tile j (dV has read it), while the drain reads dQ^T
          if (!wait(q_full + (j + 2) % C::kStages, ((j + 2) / C::kStages) & 1)) break;
          tc_fence_after();
          issue_scores(j + 2, kK, kQ, C::colS(bb), s_full + bb);
          // dP^T of tile j + 2 over dQ^T of tile j, once the drain has read it
          if (!wait(dq_free + bb, (j >> 1) & 1)) break;
          tc_fence_after();
          issue_scores(j + 2, kV, kDO, C::colDP(bb), dp_full + bb);
        }
      }
      umma_commit_warp(all_done);
      umma_commit_warp(drain);
      wait_drain(drain, 0);
      __syncwarp();
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ score warps (row = key)
    // Group gg = warp / 4 scores the tiles j with j % 2 == gg (tile buffer gg); its four warps
    // cover the four TMEM lane quarters, one key row per thread, 64 query columns.
    griddep_wait();  // lse2 and Delta come from bwd_prep
    const int gg = warp >> 2;
    const int t = threadIdx.x & 127;  // TMEM lane == key row in the tile
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_addr + C::colS(gg), tDP = tmem + lane_addr + C::colDP(gg);
    uint8_t* sDSg = sDS + gg * kAtom;
    float* sLse = reinterpret_cast<float*>(smem + C::kOffRow) + gg * 2 * kBM;  // [64]
    float* sDlt = sLse + kBM;                                                  // [64]
    const int key = k0 + t;
    bool ok = true;
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
      const bool r = mbar_wait(bar, parity, abort, a.status);
      return __all_sync(0xffffffffu, r);
    };
    for (int j = gg; j < n_it; j += 2) {
      const int h = g * G + j % G;
      const int q0 = (n_qt_all - 1 - j / G) * kBM;
      const float* lse2 = a.lse2 + (static_cast<long long>(b) * a.Hq + h) * a.Sq_pad + q0;
      const float* dlt = a.delta + (static_cast<long long>(b) * a.Hq + h) * a.Sq_pad + q0;
      // Visible columns of this key's row form one window [cmin, cmax): query rows at or after the
      // causal limit (q >= key - (Sk - Sq)); nothing if the key is beyond Sk. Padding rows carry
      // lse2 = +inf, so their P is 0 without a mask.
      const int cmin = a.causal ? key - (sp.Sk - sp.Sq) - q0 : 0;
      const int cmax = key < sp.Sk ? kBM : 0;
      const bool unmasked = __all_sync(0xffffffffu, cmin <= 0 && cmax == kBM) != 0;
      // this tile's lse2 and Delta into the group's shared rows, once its four warps are done with
      // the last tile's; every warp of the group runs all its tiles (one whose wait failed only
      // passes the barriers), so the named barriers always complete
      named_barrier(1 + gg, 128);
      if (ok) {
        if (t < kBM) sLse[t] = lse2[t];
        else sDlt[t - kBM] = dlt[t - kBM];
      }
      named_barrier(1 + gg, 128);
      if (!ok) continue;
      if (!wait_warp(s_full + gg, (j >> 1) & 1)) {
        ok = false;
        continue;
      }
      tc_fence_after();
      // P^T = 2^(S^T scale log2e - lse2), as bf16 pairs over the first 32 columns (already read):
      // the dV MMA reads them there; this thread keeps its own for dS^T
      uint32_t pk[kBM / 2];
      {
        uint32_t sr[kBM];
        tmem_ld64(tS, sr);
        tmem_wait_ld();
#pragma unroll
        for (int c4 = 0; c4 < kBM; c4 += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(sLse + c4);  // same for every lane
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            const int c = c4 + e;
            float p0 = fast_exp2(fmaf(__uint_as_float(sr[c]), a.scale_log2, -lv[e]));
            float p1 = fast_exp2(fmaf(__uint_as_float(sr[c + 1]), a.scale_log2, -lv[e + 1]));
            if (!unmasked) {
              p0 = (c >= cmin && c < cmax) ? p0 : 0.f;
              p1 = (c + 1 >= cmin && c + 1 < cmax) ? p1 : 0.f;
            }
            pk[c / 2] = pack_bf16(p0, p1);
          }
        }
        tmem_st32(tS, pk);
      }
      if (!wait_warp(dp_full + gg, (j >> 1) & 1)) {
        ok = false;
        continue;
      }
      // the shared dS^T of tile j - 2 must have been consumed by its dQ^T MMA
      if (!wait_warp(ds_free + gg, ((j >> 1) & 1) ^ 1)) {
        ok = false;
        continue;
      }
      tc_fence_after();
      // dS^T = P^T (dP^T - Delta) in two halves of 32 query columns
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t dp[32];
        tmem_ld32(tDP + hf * 32, dp);
        tmem_wait_ld();
        uint32_t dk[16];
#pragma unroll
        for (int c4 = 0; c4 < 32; c4 += 4) {
          const float4 d4 = *reinterpret_cast<const float4*>(sDlt + hf * 32 + c4);
          const float dv4[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            const uint32_t pw = pk[(hf * 32 + c4 + e) / 2];
            const float d0 = bf16_lo(pw) * (__uint_as_float(dp[c4 + e]) - dv4[e]);
            const float d1 = bf16_hi(pw) * (__uint_as_float(dp[c4 + e + 1]) - dv4[e + 1]);
            dk[(c4 + e) / 2] = pack_bf16(d0, d1);
          }
        }
        // dS^T over dP^T columns 16 hf .. 16 hf + 15 (already read), and to shared memory: key row
        // t, query columns 32 hf .. 32 hf + 31 = 16-byte chunks 4 hf .. 4 hf + 3 of the atom
        tmem_st16(tDP + hf * 16, dk);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<uint4*>(sDSg + sw128_offset(t, hf * 4 + u)) =
              make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + gg);
    }
    // dK / dV epilogue: TMEM rows -> bf16 global rows of this key tile (group 0: dV, group 1: dK);
    if (ok && n_it > 0) ok = wait_warp(all_done, 0);
    tc_fence_after();
    const bool store = key < sp.Sk;
    const long long row = ((static_cast<long long>(sp.k0) + key) * a.Hkv + g) * D;
    const uint32_t col = gg == 0 ? C::kColDV : C::kColDK;
    const float mul = gg == 0 ? 1.f : a.scale;
    uint16_t* dst = (gg == 0 ? a.dv : a.dk) + row;
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
  } else {
    // ------------------------------------------------------------------ dQ drain (warps 8-11)
    // Thread e holds TMEM lane e = head-dim column d of dQ^T; for each group of four query rows the
    // warp's 32 lanes add 32 consecutive columns x 4 rows (512 contiguous bytes) into the
    // interleaved accumulator.
    griddep_wait();  // bwd_prep has cleared the accumulator
    const int wq = warp - 8;
    const int d = wq * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
      const bool r = mbar_wait(bar, parity, abort, a.status);
      return __all_sync(0xffffffffu, r);
    };
    for (int j = 0; j < n_it; ++j) {
      const int bb = j & 1;
      const int h = g * G + j % G;
      const int q0 = (n_qt_all - 1 - j / G) * kBM;
      if (!wait_warp(dq_full + bb, (j >> 1) & 1)) break;
      tc_fence_after();
      // the whole dQ^T row of this lane (64 query columns) in one round trip; then its columns may
      // be reused at once
      uint32_t r[kBM];
      tmem_ld64(tmem + lane_addr + C::colDP(bb), r);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_free + bb);
      // the reductions wait until the dP^T MMAs that follow have finished reading shared memory
      if (j + 2 < n_it && !wait_warp(dp_full + bb, ((j + 2) >> 1) & 1)) break;
      if (d < D) {  // at D = 64 warps 10 and 11 hold no dQ column
        // rows q0 + 4i .. q0 + 4i + 3 of column d: 16 contiguous bytes at acc + 4 D i
        float* acc = a.dq_acc + ((static_cast<long long>(b) * a.Hq + h) * a.Sq_pad + q0) * D + 4 * d;
#pragma unroll
        for (int i = 0; i < kBM / 4; ++i) red_add_v4_f32(acc + 4 * D * i, r + 4 * i);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  griddep_launch_dependents();
}

// Delta = rowsum(dO * O), lse2 = lse * log2(e) (+inf for rows that see no key), dQ accumulator = 0;
// rows Sq .. Sq_pad - 1 of each sequence are padding (lse2 = +inf, Delta = 0). A warp takes eight
// consecutive rows i .. i + 7 of one (b, h): D / 8 lanes per row, one 16-byte piece of O and of dO
// each, all eight rows in flight; it then clears those rows' part of the interleaved accumulator,
// two groups of four rows = 8 D contiguous floats.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
                                                       const float* __restrict__ lse, float* __restrict__ lse2,
                                                       float* __restrict__ delta, float* __restrict__ dq_acc, int B,
                                                       int Hq, int Sq, int Sq_pad, const int* __restrict__ cu_q,
                                                       int Tq) {
  // The main kernel may be placed as soon as every block of this grid has started (it waits for
  // this grid's results with griddepcontrol.wait): its set-up and first score MMAs then overlap
  // this kernel's last blocks.
  griddep_launch_dependents();
  constexpr int LPR = D / 8;     // lanes per row
  constexpr int RPW = 32 / LPR;  // rows per warp instruction
  constexpr int U = 8 / RPW;     // instructions for the warp's eight rows
  const int lane = threadIdx.x & 31, sub = lane / LPR, cl = lane % LPR;
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const int chunks_per_bh = Sq_pad / 8;
  const long long n_chunks = static_cast<long long>(B) * Hq * chunks_per_bh;
  for (long long c = gw; c < n_chunks; c += nw) {
    const long long bh = c / chunks_per_bh;
    const int i0 = static_cast<int>(c % chunks_per_bh) * 8;
    const int h = static_cast<int>(bh % Hq);
    const long long b = bh / Hq;
    long long first = b * Sq;  // the sequence's first row in O / dO
    int len = Sq;
    if (cu_q) {
      int f;
      packed_rows(cu_q, static_cast<int>(b), Tq, Sq, f, len);
      first = f;
      // the main kernel reads rows of the sequence's 64-row query tiles only
      if (i0 >= (len + 63) / 64 * 64) continue;
    }
    uint4 x[U], y[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * RPW + sub;
      x[u] = y[u] = make_uint4(0u, 0u, 0u, 0u);
      if (i < len) {
        const long long base = ((first + i) * Hq + h) * D + cl * 8;
        x[u] = *reinterpret_cast<const uint4*>(o + base);
        y[u] = *reinterpret_cast<const uint4*>(dout + base);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t xs[4] = {x[u].x, x[u].y, x[u].z, x[u].w}, ys[4] = {y[u].x, y[u].y, y[u].z, y[u].w};
      float sacc = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc += bf16_lo(xs[e]) * bf16_lo(ys[e]) + bf16_hi(xs[e]) * bf16_hi(ys[e]);
#pragma unroll
      for (int off = LPR / 2; off > 0; off >>= 1) sacc += __shfl_xor_sync(0xffffffffu, sacc, off);
      if (cl == 0) {
        const int i = i0 + u * RPW + sub;
        const long long li = bh * Sq_pad + i;
        delta[li] = sacc;
        float l = -INFINITY;
        if (i < len) l = cu_q ? lse[static_cast<long long>(h) * Tq + first + i] : lse[bh * Sq + i];
        lse2[li] = (l == -INFINITY) ? INFINITY : l * kLog2e;
      }
    }
    // rows i0 .. i0 + 7 of (b, h) in the accumulator [B, Hq, Sq_pad / 4, D, 4]: 8 D floats from
    // (bh Sq_pad / 4 + i0 / 4) D 4 on
    float4* acc = reinterpret_cast<float4*>(dq_acc + (bh * (Sq_pad / 4) + i0 / 4) * D * 4);
#pragma unroll
    for (int e = lane; e < 2 * D; e += 32) acc[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// dQ = scale * accumulator -> bf16. A thread takes four adjacent head-dim columns of one group of
// four query rows (four consecutive float4 of the interleaved accumulator, 64 bytes), transposes
// them and writes four bf16 to each of the four rows that exist; a warp covers 128 columns.
__global__ void __launch_bounds__(256) bwd_dq_convert_kernel(const float* __restrict__ acc,
                                                             uint16_t* __restrict__ dq, int B, int Hq, int Sq,
                                                             int Sq_pad, int D, float scale,
                                                             const int* __restrict__ cu_q, int Tq) {
  griddep_wait();  // the accumulator is complete
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int qd = D / 4, groups = Sq_pad / 4;
  if (i >= static_cast<long long>(B) * Hq * groups * qd) return;
  const int d4 = static_cast<int>(i % qd);
  long long t = i / qd;
  const int g4 = static_cast<int>(t % groups);
  t /= groups;
  const int h = static_cast<int>(t % Hq);
  const long long b = t / Hq;
  long long first = b * Sq;
  int len = Sq;
  if (cu_q) {
    int f;
    packed_rows(cu_q, static_cast<int>(b), Tq, Sq, f, len);
    first = f;
  }
  if (4 * g4 >= len) return;
  const float4* src = reinterpret_cast<const float4*>(acc) + ((b * Hq + h) * groups + g4) * D + 4 * d4;
  const float4 c0 = src[0], c1 = src[1], c2 = src[2], c3 = src[3];  // columns 4 d4 + k, rows 4 g4 .. + 3
  const float r0[4] = {c0.x, c0.y, c0.z, c0.w}, r1[4] = {c1.x, c1.y, c1.z, c1.w};
  const float r2[4] = {c2.x, c2.y, c2.z, c2.w}, r3[4] = {c3.x, c3.y, c3.z, c3.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int q = 4 * g4 + e;
    if (q < len) {
      uint2 w;
      w.x = pack_bf16(r0[e] * scale, r1[e] * scale);
      w.y = pack_bf16(r2[e] * scale, r3[e] * scale);
      *reinterpret_cast<uint2*>(dq + ((first + q) * Hq + h) * D + 4 * d4) = w;
    }
  }
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
int pad128(int s) { return (s + 127) / 128 * 128; }

template <int D, bool PACKED>
cudaError_t launch_bwd_sm100_d(const Problem& p, const void* q, const void* k, const void* v, const void* o,
                               const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                               cudaStream_t st) {
  using C = BwdCfg<D>;
  const int Sq_pad = pad128(p.Sq);
  const size_t rows = static_cast<size_t>(p.B) * p.Hq * Sq_pad;
  float* dq_acc = static_cast<float*>(workspace);
  float* lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(rows * D * 4));
  float* delta = reinterpret_cast<float*>(reinterpret_cast<char*>(lse2) + align256(rows * 4));

  CUtensorMap mq, mk, mv, mdo;
  constexpr bool packed = PACKED;
  const int mB = packed ? 1 : p.B, mSq = packed ? p.Tq : p.Sq, mSk = packed ? p.Tk : p.Sk;
  if (!make_map_bf16_sw128(&mq, q, mB, mSq, p.Hq, D, kBM) || !make_map_bf16_sw128(&mdo, dout, mB, mSq, p.Hq, D, kBM) ||
      !make_map_bf16_sw128(&mk, k, mB, mSk, p.Hkv, D, kBN) || !make_map_bf16_sw128(&mv, v, mB, mSk, p.Hkv, D, kBN))
    return cudaErrorInvalidValue;

  {
    LaunchScope ls("bwd_prep", st);
    // one warp per eight rows (eight warps per block), grid-strided
    const unsigned blocks = static_cast<unsigned>(std::min<size_t>((rows + 63) / 64, 1u << 20));
    bwd_prep_kernel<D><<<blocks, 256, 0, st>>>(
        static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), lse, lse2, delta, dq_acc, p.B, p.Hq,
        p.Sq, Sq_pad, p.cu_q, p.Tq);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  e = cudaFuncSetAttribute(bwd_sm100_kernel<D, PACKED, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_sm100_kernel<D, PACKED, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kSmemBytes);
  if (e != cudaSuccess) return e;
  BwdArgs a;
  a.B = p.B;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.Sq = p.Sq;
  a.Sk = p.Sk;
  a.Sq_pad = Sq_pad;
  a.causal = p.causal;
  a.scale = p.scale;
  a.scale_log2 = p.scale * kLog2e;
  a.lse2 = lse2;
  a.delta = delta;
  a.dq_acc = dq_acc;
  a.dk = static_cast<uint16_t*>(dk);
  a.dv = static_cast<uint16_t*>(dv);
  a.status = device_status_ptr();
  a.cu_q = p.cu_q;
  a.cu_k = p.cu_k;
  a.Tq = p.Tq;
  a.Tk = p.Tk;
#ifdef ATTN_FAULT_INJECT
  a.fault_block = fault_block_for(1);
#else
  a.fault_block = -1;
#endif
  a.n_kt = (p.Sk + kBN - 1) / kBN;
  // Q, dO (bf16) and the dQ accumulator (fp32) of the whole batch: sequence by sequence once they
  // would take more than half of the 126 MB L2
  const double rows_bytes = static_cast<double>(p.B) * p.Hq * D * (4.0 * p.Sq + 4.0 * Sq_pad);
  const bool seq_major = p.B > 1 && rows_bytes > 64.0 * 1024 * 1024;
  {
    LaunchScope ls("bwd_sm100", st);
    e = seq_major ? launch_dependent(bwd_sm100_kernel<D, PACKED, true>,
                                     dim3(static_cast<unsigned>(static_cast<long long>(p.Hkv) * p.B * a.n_kt)),
                                     dim3(kThreads), C::kSmemBytes, st, mq, mk, mv, mdo, a)
                  : launch_dependent(bwd_sm100_kernel<D, PACKED, false>, dim3(p.Hkv * p.B, a.n_kt), dim3(kThreads),
                                     C::kSmemBytes, st, mq, mk, mv, mdo, a);
  }
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  const long long n_conv = static_cast<long long>(p.B) * p.Hq * (Sq_pad / 4) * (D / 4);
  {
    LaunchScope ls("bwd_dq_convert", st);
    e = launch_dependent(bwd_dq_convert_kernel, dim3(static_cast<unsigned>((n_conv + 255) / 256)), dim3(256), 0, st,
                         dq_acc, static_cast<uint16_t*>(dq), p.B, p.Hq, p.Sq, Sq_pad, D, p.scale, p.cu_q, p.Tq);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

size_t bwd_sm100_workspace_bytes(int B, int Hq, int Hkv, int Sq, int Sk, int D) {
  (void)Hkv;
  (void)Sk;
  const size_t rows = static_cast<size_t>(B) * Hq * pad128(Sq);
  return align256(rows * D * 4) + 2 * align256(rows * 4);
}

cudaError_t launch_bwd_sm100(const Problem& p, const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                             cudaStream_t st) {
  const bool packed = p.cu_q != nullptr;
  if (p.D == 128)
    return packed ? launch_bwd_sm100_d<128, true>(p, q, k, v, o, lse, dout, dq, dk, dv, workspace, st)
                  : launch_bwd_sm100_d<128, false>(p, q, k, v, o, lse, dout, dq, dk, dv, workspace, st);
  return packed ? launch_bwd_sm100_d<64, true>(p, q, k, v, o, lse, dout, dq, dk, dv, workspace, st)
                : launch_bwd_sm100_d<64, false>(p, q, k, v, o, lse, dout, dq, dk, dv, workspace, st);
}

}  // namespace attn
