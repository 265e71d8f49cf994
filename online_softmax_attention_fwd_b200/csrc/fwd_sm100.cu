// fwd_sm100.cu -- attention forward on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The forward is one reduction over key blocks under the online-softmax monoid ("Não escreva
// kernels, derive-os", "Aprofundamento", first paragraph): for every query row the CTA keeps the
// triple (m, l, O) -- running max (base-2 units), running sum of 2^(s - m) and the unnormalised
// output -- and folds in one 128-key block at a time:
//   S = Q K^T (tensor cores, fp32 in TMEM), m' = max(m, rowmax S), P = 2^(S - m'),
//   l = l 2^(m - m') + rowsum P, O = O 2^(m - m') + P V (tensor cores, fp32 in TMEM).
// The two contractions are dense, so they run as tcgen05.mma with fp32 accumulators in tensor
// memory; the row statistics run on the CUDA cores, one thread per row.
//
// The grid is persistent (one CTA per SM). A work item is two 128-row query tiles that read the
// same keys, and the CTA streams each 128-key K/V block once for both. When each key/value head
// serves an even number of query heads, the two tiles are the same rows of two query heads of one
// group: under a causal mask both then see the same number of blocks, and items come in 128-row
// steps of length. Otherwise the item folds one head's row tiles: row tile n - 1 - r with row tile
// r, so that under a causal mask a long tile shares its CTA with a short one. Items are sorted
// longest first (under a causal mask the last rows see the most keys) and dealt to the CTAs in
// snake order. Across
// items the K/V ring runs on without a pause. The next item's Q is loaded as soon as the current
// item's last S is complete, and a tile's epilogue overlaps the next item's first S; the first P V
// of an item waits only until that epilogue has read O out of TMEM (barrier o_free).
// Otherwise a CTA works on one item as follows.
// TMEM holds, per tile, S (128 columns) and O (128 columns): 512 in all. The softmax writes P as
// bf16 back over the first 64 columns of its own S, and P V reads it from there (A operand in
// TMEM), so P never goes through shared memory. Every MMA is 128 wide in N, which keeps the tensor
// pipe fed per instruction issued.
//
// Warp roles (320 threads):
//   warps 0-3 / 4-7  softmax of tile 0 / tile 1, one row per thread: S from TMEM in 32-column
//                    chunks (row max, then exp2, row sum and P), lazy O rescale, P to TMEM;
//                    epilogue O / l and lse.
//   warp 8           TMA producer: both Q tiles once, then K and V blocks through two rings.
//   warp 9           TMEM allocator and MMA issuer (one elected lane of a converged warp): for each
//                    tile, O += P V of block j and then at once S = Q K^T of block j + 1, tile 0 and
//                    tile 1 alternating, so the tensor pipe works on one tile while the other tile's
//                    softmax runs. MMAs execute in issue order, so once S of block j is complete,
//                    P V of block j - 1 is too: the softmax may rescale O then without a further wait.
// Lazy rescaling: a row keeps its old max m while the block max stays within m + 8 (base 2); P then
// stays <= 256 and the final O / l and lse = m + log2 l use the same m, so the result is exact.
//
// Shared-memory tiles use the 128-byte swizzle: Q and K are K-major (rows of 64 bf16 = 128 B), V is
// read as an MN-major operand (its head dim is contiguous). Every wait is bounded (common.cuh).
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"

namespace attn {
namespace {

constexpr int kBM = 128;   // query rows per tile (two tiles per CTA)
constexpr int kBN = 128;   // keys per block
constexpr int kThreads = 320;
constexpr int kAtom = 128 * 128;  // 128 rows x 128 bytes (16 KB)
// Packed batches: shared-memory tables for the item list (sequence lengths, sequences by length,
// item counts per rank), for up to kMaxSeqs sequences and kMaxSlots ranks; beyond that every
// (sequence, rank) pair stays an item and the empty ones are skipped.
constexpr int kMaxSeqs = 1024;
constexpr int kMaxSlots = 2048;
constexpr int kTabBytes = (2 * kMaxSeqs + kMaxSlots + 1) * 4;

// F8: e4m3 Q, K, V (one byte per element, D = 128 only) instead of bf16.
template <int D, bool F8 = false>
struct FwdCfg {
  static constexpr int kElt = F8 ? 1 : 2;             // bytes per element
  static constexpr int kAtomElts = 128 / kElt;        // elements per 128-byte swizzle row
  static constexpr int kAtoms = D / kAtomElts;        // column atoms per row
  static constexpr int kTileBytes = kAtoms * kAtom;  // one 128 x D tile (Q, K or V)
  static constexpr int kKStep = 32 / kElt;            // K elements per MMA instruction (32 bytes)
  static constexpr int kKStages = (D == 128) ? 2 : 4;
  static constexpr int kVStages = (D == 128) ? 2 : 4;
  static constexpr int kOffQ = 0;                                      // [2 tiles]
  static constexpr int kOffK = kOffQ + 2 * kTileBytes;                 // [K stages]
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;          // [V stages]
  static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
  static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 2 + 4 + 2 + 2 + 1 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + slack for 1024-byte alignment
  // TMEM: S (and P over its first 64 columns) of tile t at 128 t; O of tile t at 256 + 128 t.
  __host__ __device__ static constexpr uint32_t colS(int t) { return 128u * t; }
  __host__ __device__ static constexpr uint32_t colO(int t) { return 256u + 128u * t; }
};

struct FwdArgs {
  int B, Hq, Hkv, Sq, Sk;  // packed batches: Sq, Sk are the longest sequence's lengths
  int causal;
  float scale_log2;  // softmax scale * log2(e) (FP8: times the Q and K scales)
  float o_scale;     // O multiplier at the end (FP8: the V scale; 1 for bf16)
  // A work item is two 128-row query tiles that read the same K/V blocks. With head_pairs, the two
  // tiles are the same rows of query heads 2 hs and 2 hs + 1 (one key/value group, as the head
  // count ratio is even); otherwise they are row tiles n - 1 - r and r of one head (n row tiles).
  int head_pairs;
  int n_slots;       // items per head set: row tiles (head_pairs) or folded pairs of row tiles
  int n_hsets;       // head sets per batch entry: Hq / 2 (head_pairs) or Hq
  uint16_t* o;
  float* lse;
  int* status;
  // Packed batches of sequences of different lengths: sequence b owns query rows cu_q[b] ..
  // cu_q[b + 1] - 1 of q / o ([Tq, Hq, D]) and key rows cu_k[b] .. cu_k[b + 1] - 1 of k / v, and lse
  // is [Hq, Tq]. Null for the dense [B, S, H, D] layout.
  const int* cu_q;
  const int* cu_k;
  int Tq, Tk;
  int fault_block;  // test-only fault-injection build: CTA 0 skips this K load (-1: none)
  int compact;      // packed batches: deal only the items that exist (tables in shared memory)
};

// Lengths and first packed rows of sequence b (dense: every sequence has Sq / Sk rows). Offsets
// are device data, so they are checked where they are used: a sequence whose rows fall outside the
// packed tensors, or that is longer than the bound the host passed, is not touched (it counts as
// empty) and the device status records ATTN_ERR_INVALID_ARG.
struct SeqSpan {
  int Sq, Sk, q0, k0;
};
template <bool PACKED>
__device__ __forceinline__ SeqSpan seq_span(const FwdArgs& a, int b) {
  if constexpr (PACKED) {
    const int q0 = a.cu_q[b], q1 = a.cu_q[b + 1], k0 = a.cu_k[b], k1 = a.cu_k[b + 1];
    if (q0 < 0 || q1 < q0 || q1 > a.Tq || q1 - q0 > a.Sq || k0 < 0 || k1 < k0 || k1 > a.Tk || k1 - k0 > a.Sk) {
      record_status(a.status, kStatusBadArg);
      return SeqSpan{0, 0, 0, 0};
    }
    return SeqSpan{q1 - q0, k1 - k0, q0, k0};
  } else {
    return SeqSpan{a.Sq, a.Sk, b * a.Sq, b * a.Sk};
  }
}

__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity) {
  // Bounded wait that ignores the abort flag: used only to let this thread's own in-flight async
  // work land before the CTA releases its shared and tensor memory.
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

// Number of 128-key blocks some row of the 128-row tile starting at `qs` can see.
__device__ __forceinline__ int tile_blocks(const SeqSpan& sp, int causal, int qs) {
  if (qs >= sp.Sq) return 0;
  int kv_end = sp.Sk;
  if (causal) kv_end = min(sp.Sk, qs + kBM + sp.Sk - sp.Sq);
  return kv_end > 0 ? (kv_end + kBN - 1) / kBN : 0;
}

// Work item k of CTA c under the snake order (round r = k: CTAs c = 0 .. G-1 left to right on even
// rounds, right to left on odd ones) over items sorted longest first; -1 past the end.
__device__ __forceinline__ int fwd_item_index(int k, int c, int G, int n_items) {
  const int i = k * G + ((k & 1) ? (G - 1 - c) : c);
  return i < n_items ? i : -1;
}

// One CTA per SM. Its 10 warps are dealt to the SM's four sub-partitions (three on some), and each
// sub-partition has 16 K registers: at most 168 registers per thread, which the compiler derives
// from these bounds.
// Instantiated per element type (F8: e4m3), layout (PACKED: cu_seqlens offsets) and item shape (HP:
// head pairs), so that each variant carries only its own index arithmetic.
template <int D, bool F8, bool PACKED, bool HP>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  using C = FwdCfg<D, F8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + C::kKStages;
  uint64_t* v_full = k_empty + C::kKStages;
  uint64_t* v_empty = v_full + C::kVStages;
  uint64_t* s_full = v_empty + C::kVStages;  // [tile]
  uint64_t* p_full = s_full + 2;             // [tile][half]: P of keys 0-63 / 64-127 in TMEM
  uint64_t* o_done = p_full + 4;             // [tile]: every P V of the tile's item is complete
  uint64_t* o_free = o_done + 2;             // [tile]: the epilogue has read O out of TMEM
  uint64_t* q_empty = o_free + 2;            // the item's last S = Q K^T is complete
  uint64_t* drain = q_empty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = a.B * a.n_hsets;
  const int G = static_cast<int>(gridDim.x), cta = static_cast<int>(blockIdx.x);
  // packed item tables (after the barriers and the rest of the per-CTA state)
  int* s_len = reinterpret_cast<int*>(smem + C::kOffMisc + 64);  // [kMaxSeqs] query rows of each sequence
  int* s_order = s_len + kMaxSeqs;                                // [kMaxSeqs] sequences, longest first
  int* s_pref = s_order + kMaxSeqs;                               // [n_slots + 1] items before rank r
  const bool compact = PACKED && a.compact;
  // Item i of head set i % BH, rank r = i / BH (rank 0 the longest under a causal mask). Head
  // pairs: both tiles are row tile n_slots - 1 - r of heads h and h + 1. Otherwise (one head): the
  // item folds the sequence's row tiles, pairing tile n - 1 - r (rows q0, the longer) with tile r
  // (rows q1), so that under a causal mask a long tile shares its CTA with a short one; the middle
  // tile of an odd count runs alone, and ranks past the middle are empty.
  constexpr int dh = HP ? 1 : 0;
  // TMA coordinates: dense tensors are 4-D maps (D, H, S, B); packed ones are (D, H, T, 1), where a
  // sequence's rows start at its first packed row (boxes may run into the next sequence's rows:
  // those keys are masked, their values weighted 0, and those query rows are not stored)
  // With the packed tables, the items are only the (sequence, rank) pairs with rows: rank by rank,
  // and within a rank the sequences longest first, head sets fastest.
  auto item_of = [&](int i, int& b, int& h, int& q0, int& q1, int& n0, int& n1, SeqSpan& sp) {
    int r, hs;
    if (compact) {
      int lo = 0, hi = a.n_slots - 1;  // the last rank whose first item is at or before i
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_pref[mid] <= i) lo = mid;
        else hi = mid - 1;
      }
      r = lo;
      const int w = i - s_pref[r];
      b = s_order[w / a.n_hsets];
      hs = w % a.n_hsets;
    } else {
      const int bh = i % BH;
      r = i / BH;
      b = bh / a.n_hsets;
      hs = bh % a.n_hsets;
    }
    h = hs * (HP ? 2 : 1);
    sp = seq_span<PACKED>(a, b);
    if constexpr (HP) {
      q0 = q1 = (a.n_slots - 1 - r) * kBM;
      n0 = n1 = tile_blocks(sp, a.causal, q0);
    } else {
      const int nt = (sp.Sq + kBM - 1) / kBM, ta = nt - 1 - r;
      q0 = ta * kBM;
      q1 = r * kBM;
      n0 = ta >= r ? tile_blocks(sp, a.causal, q0) : 0;
      n1 = ta > r ? tile_blocks(sp, a.causal, q1) : 0;
    }
  };
  constexpr bool packed = PACKED;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full + t, 1);
      mbar_init(p_full + 2 * t, 4);
      mbar_init(p_full + 2 * t + 1, 4);
      mbar_init(o_done + t, 1);
      mbar_init(o_free + t, 4);
    }
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
  }
  if (compact) {
    // lengths (a sequence with offsets outside the tensors counts as empty), then each sequence's
    // place in the order longest first, and the items of each rank: the sequences long enough to
    // have that rank (a prefix of the order), times the head sets
    for (int b = threadIdx.x; b < a.B; b += kThreads) s_len[b] = seq_span<PACKED>(a, b).Sq;
    __syncthreads();
    for (int b = threadIdx.x; b < a.B; b += kThreads) {
      const int L = s_len[b];
      int rank = 0;
      for (int o = 0; o < a.B; ++o) rank += (s_len[o] > L) || (s_len[o] == L && o < b);
      s_order[rank] = b;
    }
    for (int r = threadIdx.x; r < a.n_slots; r += kThreads) {
      int cnt = 0;
      for (int o = 0; o < a.B; ++o) {
        const int nt = (s_len[o] + kBM - 1) / kBM;  // the sequence's row tiles
        cnt += HP ? (a.n_slots - 1 - r) < nt : 2 * r + 1 <= nt;
      }
      s_pref[r + 1] = cnt * a.n_hsets;
    }
    __syncthreads();
    if (warp == 0) {  // running sum over the ranks, 32 at a time
      int carry = 0;
      if (lane == 0) s_pref[0] = 0;
      for (int base = 1; base <= a.n_slots; base += 32) {
        const int idx = base + lane;
        int v = idx <= a.n_slots ? s_pref[idx] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
        v += carry;
        if (idx <= a.n_slots) s_pref[idx] = v;
        carry = __shfl_sync(0xffffffffu, v, 31);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int n_items = compact ? s_pref[a.n_slots] : BH * a.n_slots;

  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      constexpr uint32_t kTx = kBM * D * C::kElt;
      long long kvb = 0;  // K/V blocks issued so far (ring position)
      int qk = 0;         // items with any block so far
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int i = fwd_item_index(k, cta, G, n_items);
        if (i < 0) break;
        int b, h, q0, q1, n0, n1;
        SeqSpan sp;
        item_of(i, b, h, q0, q1, n0, n1, sp);
        const int nmax = max(n0, n1);
        if (nmax == 0) continue;
        const int g = h / (a.Hq / a.Hkv);
        const int qrow0 = packed ? sp.q0 : 0, krow0 = packed ? sp.k0 : 0, bc = packed ? 0 : b;
        // this item's Q tiles once the previous item's last S has read the buffer
        if (!mbar_wait(q_empty, (qk & 1) ^ 1, abort, a.status)) break;
        mbar_arrive_expect_tx(q_full, (n0 > 0 ? kTx : 0u) + (n1 > 0 ? kTx : 0u));
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if ((t == 0 ? n0 : n1) == 0) continue;
#pragma unroll
          for (int at = 0; at < C::kAtoms; ++at)
            tma_load_4d(sQ + t * C::kTileBytes + at * kAtom, &tmQ, q_full, at * C::kAtomElts, h + t * dh,
                        qrow0 + (t == 0 ? q0 : q1), bc);
        }
        ++qk;
        for (int j = 0; j < nmax; ++j) {
          const long long gj = kvb + j;
          const int sk = static_cast<int>(gj % C::kKStages), sv = static_cast<int>(gj % C::kVStages);
          if (!mbar_wait(k_empty + sk, static_cast<uint32_t>((gj / C::kKStages) & 1) ^ 1, abort, a.status)) {
            ok = false;
            break;
          }
#ifdef ATTN_FAULT_INJECT
          const bool skip = cta == 0 && gj == a.fault_block;  // the MMA warp's wait for it runs out
#else
          constexpr bool skip = false;
#endif
          if (!skip) {
            mbar_arrive_expect_tx(k_full + sk, kTx);
#pragma unroll
            for (int at = 0; at < C::kAtoms; ++at)
              tma_load_4d(sK + sk * C::kTileBytes + at * kAtom, &tmK, k_full + sk, at * C::kAtomElts, g,
                          krow0 + j * kBN, bc);
          }
          if (!mbar_wait(v_empty + sv, static_cast<uint32_t>((gj / C::kVStages) & 1) ^ 1, abort, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(v_full + sv, kTx);
#pragma unroll
          for (int at = 0; at < C::kAtoms; ++at)
            tma_load_4d(sV + sv * C::kTileBytes + at * kAtom, &tmV, v_full + sv, at * C::kAtomElts, g,
                        krow0 + j * kBN, bc);
        }
        kvb += nmax;
      }
      // Let every load this thread issued land before the CTA can exit. On the normal path the
      // consumers have already waited for each of them, so these return at once.
      if (qk > 0) wait_drain(q_full, (qk - 1) & 1);
      for (long long j = max(0ll, kvb - C::kKStages); j < kvb; ++j)
        wait_drain(k_full + j % C::kKStages, static_cast<uint32_t>((j / C::kKStages) & 1));
      for (long long j = max(0ll, kvb - C::kVStages); j < kvb; ++j)
        wait_drain(v_full + j % C::kVStages, static_cast<uint32_t>((j / C::kVStages) & 1));
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    // the whole warp runs the loop; one elected lane issues each MMA
    constexpr uint32_t kIdescS = F8 ? idesc_e4m3_f32(kBM, kBN, 0, 0) : idesc_bf16_f32(kBM, kBN, 0, 0);
    constexpr uint32_t kIdescO = F8 ? idesc_e4m3_f32(kBM, D, 0, 1) : idesc_bf16_f32(kBM, D, 0, 1);
    // base descriptors, built once; each MMA only moves the start address
    const uint64_t dQ0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t dK0 = sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t dV0 = sdesc_sw128(smem_u32(sV), kAtom, 1024);
    // polling waits: the issuer reacts to a completed P or K/V phase without a wake-up delay
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait_spin(bar, parity, abort, a.status)) != 0;
    };
    long long kvb = 0;      // ring position of the item's first K/V block
    long long k_ready = -1, v_ready = -1;  // last K / V block this warp has waited for
    long long sb[2] = {0, 0};  // S blocks of each tile issued in earlier items
    int ct[2] = {0, 0};        // earlier items in which each tile had blocks
    int qk = 0;
    bool ok = true;
    auto wait_k = [&](long long gj) -> bool {
      if (k_ready >= gj) return true;
      k_ready = gj;
      return wait_all(k_full + gj % C::kKStages, static_cast<uint32_t>((gj / C::kKStages) & 1));
    };
    auto wait_v = [&](long long gj) -> bool {
      if (v_ready >= gj) return true;
      v_ready = gj;
      return wait_all(v_full + gj % C::kVStages, static_cast<uint32_t>((gj / C::kVStages) & 1));
    };
    // S_t of ring block gj = Q_t K^T
    auto issue_s = [&](int t, long long gj) {
      tc_fence_after();
      const uint64_t dK = sdesc_advance(dK0, static_cast<uint32_t>(gj % C::kKStages) * C::kTileBytes);
      const uint64_t dQ = sdesc_advance(dQ0, t * C::kTileBytes);
#pragma unroll
      for (int kk = 0; kk < D / C::kKStep; ++kk) {
        const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;  // 32 bytes of K per instruction
        if constexpr (F8)
          umma_ss_warp_f8(tmem + C::colS(t), sdesc_advance(dQ, off), sdesc_advance(dK, off), kIdescS, kk > 0);
        else
          umma_ss_warp(tmem + C::colS(t), sdesc_advance(dQ, off), sdesc_advance(dK, off), kIdescS, kk > 0);
      }
      umma_commit_warp(s_full + t);
    };
    for (int k = 0; ok; ++k) {
      const int i = fwd_item_index(k, cta, G, n_items);
      if (i < 0) break;
      int b, h, q0, q1, n0, n1;
      SeqSpan sp;
      item_of(i, b, h, q0, q1, n0, n1, sp);
      const int nmax = max(n0, n1);
      if (nmax == 0) continue;
      const int nt[2] = {n0, n1};
      if (!wait_all(q_full, qk & 1) || !wait_k(kvb)) break;
      // S of block 0 for both tiles (over P of the previous item, whose P V was issued earlier)
      for (int t = 0; t < 2; ++t)
        if (nt[t] > 0) issue_s(t, kvb);
      umma_commit_warp(k_empty + kvb % C::kKStages);
      if (nmax == 1) umma_commit_warp(q_empty);  // this item's Q has been read by all its S
      // per block j and tile t: O_t += P_t V_j, then at once S_t of block j + 1 (it overwrites P_t in
      // TMEM; the P V that reads P_t was issued just before it and MMAs execute in order). The two
      // tiles' chains are independent, so the tensor pipe alternates between them.
      for (int j = 0; ok && j < nmax; ++j) {
        const long long gj = kvb + j;
        for (int t = 0; t < 2; ++t) {
          if (j < nt[t]) {
            // the first P V of the item overwrites O_t: the previous item's epilogue must have read it
            if (j == 0 && ct[t] > 0 && !wait_all(o_free + t, (ct[t] - 1) & 1)) {
              ok = false;
              break;
            }
            const uint64_t dV = sdesc_advance(dV0, static_cast<uint32_t>(gj % C::kVStages) * C::kTileBytes);
            // P is the A operand in TMEM, 8 columns per instruction (16 bf16 keys, or 32 e4m3 keys);
            // each half of the block's keys goes as soon as the softmax has written its P
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              if ((hf == 0 && !wait_v(gj)) ||
                  !wait_all(p_full + 2 * t + hf, static_cast<uint32_t>((sb[t] + j) & 1))) {
                ok = false;
                break;
              }
              tc_fence_after();
              constexpr int kPerHalf = 64 / C::kKStep;  // instructions per 64 keys
#pragma unroll
              for (int kk = kPerHalf * hf; kk < kPerHalf * hf + kPerHalf; ++kk) {
                if constexpr (F8)
                  umma_ts_warp_f8(tmem + C::colO(t), tmem + C::colS(t) + kk * 8,
                                  sdesc_advance(dV, kk * C::kKStep * 128), kIdescO, (j > 0 || kk > 0));
                else
                  umma_ts_warp(tmem + C::colO(t), tmem + C::colS(t) + kk * 8, sdesc_advance(dV, kk * C::kKStep * 128),
                               kIdescO, (j > 0 || kk > 0));
              }
            }
            if (!ok) break;
            if (j == nt[t] - 1) umma_commit_warp(o_done + t);
          }
          if (j + 1 < nt[t]) {
            if (!wait_k(gj + 1)) {
              ok = false;
              break;
            }
            issue_s(t, gj + 1);
          }
        }
        if (!ok) break;
        if (j + 1 < nmax) umma_commit_warp(k_empty + (gj + 1) % C::kKStages);
        if (j + 2 == nmax) umma_commit_warp(q_empty);  // the item's last S has been issued
        umma_commit_warp(v_empty + gj % C::kVStages);
      }
      if (!ok) break;
      for (int t = 0; t < 2; ++t)
        if (nt[t] > 0) {
          sb[t] += nt[t];
          ++ct[t];
        }
      kvb += nmax;
      ++qk;
    }
    // all MMAs issued by this warp complete before the CTA releases TMEM
    umma_commit_warp(drain);
    wait_drain(drain, 0);
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax warpgroups
    const int t = warp >> 2;               // query tile of this warpgroup
    const int row = threadIdx.x & 127;     // TMEM lane == row in the tile
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_addr + C::colS(t);
    const uint32_t tO = tmem + lane_addr + C::colO(t);
    // every lane waits; the outcome is made warp-uniform before any warp-collective tcgen05 op
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
      const bool r = mbar_wait(bar, parity, abort, a.status);
      return __all_sync(0xffffffffu, r);
    };
    long long sb = 0;  // this tile's S blocks in earlier items
    int ct = 0;        // earlier items in which this tile had blocks
    bool ok = true;
    for (int k = 0;; ++k) {
      const int i = fwd_item_index(k, cta, G, n_items);
      if (i < 0) break;
      int b, h, q0, q1, n0, n1;
      SeqSpan sp;
      item_of(i, b, h, q0, q1, n0, n1, sp);
      const int n_kv = t == 0 ? n0 : n1;
      h += t * dh;
      const int qrow = (t == 0 ? q0 : q1) + row;
      int row_limit = sp.Sk - 1;  // largest visible key index for this row
      if (a.causal) row_limit = min(row_limit, qrow + sp.Sk - sp.Sq);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; ok && j < n_kv; ++j) {
        if (!wait_warp(s_full + t, static_cast<uint32_t>((sb + j) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int kbase = j * kBN;
        // the whole 128-column row of S in registers: one round trip to TMEM
        uint32_t sr[kBN];
  #pragma unroll
        for (int c = 0; c < kBN; c += 64) tmem_ld64(tS + c, sr + c);
        tmem_wait_ld();
        if (kbase + kBN - 1 > row_limit) {  // the block crosses this row's last visible key
  #pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (kbase + c > row_limit) sr[c] = __float_as_uint(-INFINITY);
        }
        float mx8[8];  // eight independent max chains, two new columns per three-input max
  #pragma unroll
        for (int c = 0; c < 8; ++c) mx8[c] = fmaxf(__uint_as_float(sr[c]), __uint_as_float(sr[c + 8]));
  #pragma unroll
        for (int c = 16; c < kBN; c += 16)
  #pragma unroll
          for (int u = 0; u < 8; ++u)
            mx8[u] = fmax3(mx8[u], __uint_as_float(sr[c + u]), __uint_as_float(sr[c + 8 + u]));
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7])) *
                         a.scale_log2;
        // lazy rescale: move the reference max only when the block max exceeds it by more than 8
        float alpha = 1.f;
        if (mx > m + 8.f || (m == -INFINITY && mx != -INFINITY)) {
          alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - mx);
          m = mx;
        }
        const float m_use = (m == -INFINITY) ? 0.f : m;
        // P = 2^(scale s - m) as bf16 pairs over the first 64 columns of S: keys 0-63 first (P columns
        // 0-31), released to the P V MMA at once, then keys 64-127 (ex2 of a masked -inf is 0). FP8:
        // e4m3 quadruples over the first 32 columns (keys 0-63 in columns 0-15). With the lazy
        // rescale P <= 2^8, inside e4m3's range (448).
        const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2), nm2 = f2_pack(-m_use, -m_use);
        uint64_t rs2[4] = {0ull, 0ull, 0ull, 0ull};  // four packed sum chains
  #pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t pk[32];
          float pprev = 0.f, pprev1 = 0.f;
  #pragma unroll
          for (int c = 64 * hf; c < 64 * hf + 64; c += 2) {
            float x0, x1, p0, p1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2, nm2), x0, x1);
            p0 = fast_exp2(x0);
            p1 = fast_exp2(x1);
            rs2[(c >> 1) & 3] = f2_add(rs2[(c >> 1) & 3], f2_pack(p0, p1));
            if constexpr (F8) {
              if (c & 2) pk[(c - 64 * hf) / 4] = pack_e4m3x4(pprev, pprev1, p0, p1);
              pprev = p0;
              pprev1 = p1;
            } else {
              pk[(c - 64 * hf) / 2] = pack_bf16(p0, p1);
            }
          }
          if constexpr (F8) {
            tmem_st16(tS + 16 * hf, pk);
          } else {
            tmem_st32(tS + 32 * hf, pk);
          }
          // S of block j is complete, hence so is P V of block j - 1: O may be rescaled now, before
          // the first P V of block j is released.
          if (hf == 0 && j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
  #pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 16) {
              uint32_t orr[16];
              tmem_ld16(tO + c0, orr);
              tmem_wait_ld();
  #pragma unroll
              for (int e = 0; e < 16; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
              tmem_st16(tO + c0, orr);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full + 2 * t + hf);
        }
        float rsum[8];
  #pragma unroll
        for (int u = 0; u < 4; ++u) f2_unpack(rs2[u], rsum[2 * u], rsum[2 * u + 1]);
        l = l * alpha + (((rsum[0] + rsum[1]) + (rsum[2] + rsum[3])) + ((rsum[4] + rsum[5]) + (rsum[6] + rsum[7])));
      }
      sb += n_kv;
      // epilogue: O / l -> bf16, lse = (m + log2 l) ln 2. O leaves TMEM in two 64-column halves;
      // once both are in registers the next item's first P V may overwrite it.
      const bool have = ok && n_kv > 0;
      if (have) ok = wait_warp(o_done + t, ct & 1);
      tc_fence_after();
      const float inv = l > 0.f ? (F8 ? a.o_scale : 1.f) / l : 0.f;
      const bool store = qrow < sp.Sq;
      uint16_t* orow = a.o + ((static_cast<long long>(sp.q0) + qrow) * a.Hq + h) * D;
      uint32_t orr[D];
      if (have && ok) {
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 64) tmem_ld64(tO + c0, orr + c0);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < D; ++e) orr[e] = 0u;
      }
      if (n_kv > 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free + t);
        ++ct;
      }
      if (store) {
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 16) {
          uint4 w0, w1;
          w0.x = pack_bf16(__uint_as_float(orr[c0 + 0]) * inv, __uint_as_float(orr[c0 + 1]) * inv);
          w0.y = pack_bf16(__uint_as_float(orr[c0 + 2]) * inv, __uint_as_float(orr[c0 + 3]) * inv);
          w0.z = pack_bf16(__uint_as_float(orr[c0 + 4]) * inv, __uint_as_float(orr[c0 + 5]) * inv);
          w0.w = pack_bf16(__uint_as_float(orr[c0 + 6]) * inv, __uint_as_float(orr[c0 + 7]) * inv);
          w1.x = pack_bf16(__uint_as_float(orr[c0 + 8]) * inv, __uint_as_float(orr[c0 + 9]) * inv);
          w1.y = pack_bf16(__uint_as_float(orr[c0 + 10]) * inv, __uint_as_float(orr[c0 + 11]) * inv);
          w1.z = pack_bf16(__uint_as_float(orr[c0 + 12]) * inv, __uint_as_float(orr[c0 + 13]) * inv);
          w1.w = pack_bf16(__uint_as_float(orr[c0 + 14]) * inv, __uint_as_float(orr[c0 + 15]) * inv);
          *reinterpret_cast<uint4*>(orow + c0) = w0;
          *reinterpret_cast<uint4*>(orow + c0 + 8) = w1;
        }
        const long long li = packed ? static_cast<long long>(h) * a.Tq + sp.q0 + qrow
                                    : (static_cast<long long>(b) * a.Hq + h) * a.Sq + qrow;
        a.lse[li] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------------------------
template <int D, bool F8, bool PACKED, bool HP>
cudaError_t launch_fwd_sm100_v(const Problem& p, const void* q, const void* k, const void* v, void* o, float* lse,
                               cudaStream_t st) {
  using C = FwdCfg<D, F8>;
  constexpr int kSmem = C::kSmemBytes + (PACKED ? kTabBytes : 0);
  static_assert(kSmem <= 232448, "shared memory per CTA");
  CUtensorMap mq, mk, mv;
  constexpr bool packed = PACKED;
  // packed batches: one sequence of Tq (Tk) rows as far as the maps are concerned
  const int mB = packed ? 1 : p.B, mSq = packed ? p.Tq : p.Sq, mSk = packed ? p.Tk : p.Sk;
  auto make = [&](CUtensorMap* m, const void* base, int S, int H, int rows) {
    return F8 ? make_map_u8_sw128(m, base, mB, S, H, D, rows) : make_map_bf16_sw128(m, base, mB, S, H, D, rows);
  };
  if (!make(&mq, q, mSq, p.Hq, kBM) || !make(&mk, k, mSk, p.Hkv, kBN) || !make(&mv, v, mSk, p.Hkv, kBN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(fwd_sm100_kernel<D, F8, PACKED, HP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmem);
  if (e != cudaSuccess) return e;
  FwdArgs a;
  a.B = p.B;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.Sq = p.Sq;
  a.Sk = p.Sk;
  a.causal = p.causal;
  a.scale_log2 = p.scale * p.qk_scale * kLog2e;
  a.o_scale = p.v_scale;
  a.head_pairs = HP ? 1 : 0;
  a.n_slots = a.head_pairs ? (p.Sq + kBM - 1) / kBM : (p.Sq + 2 * kBM - 1) / (2 * kBM);
  a.n_hsets = a.head_pairs ? p.Hq / 2 : p.Hq;
  a.o = static_cast<uint16_t*>(o);
  a.lse = lse;
  a.status = device_status_ptr();
  a.cu_q = p.cu_q;
  a.cu_k = p.cu_k;
  a.Tq = p.Tq;
  a.Tk = p.Tk;
#ifdef ATTN_FAULT_INJECT
  a.fault_block = fault_block_for(0);
#else
  a.fault_block = -1;
#endif
  a.compact = packed && p.B <= kMaxSeqs && a.n_slots <= kMaxSlots;
  // a persistent grid: one CTA per SM, each walking its share of the (head, tile pair) items
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long long n_items = static_cast<long long>(a.n_hsets) * p.B * a.n_slots;
  dim3 grid(static_cast<unsigned>(std::min<long long>(n_items, sms)));
  {
    LaunchScope ls(F8 ? "fwd_sm100_fp8" : "fwd_sm100", st);
    fwd_sm100_kernel<D, F8, PACKED, HP><<<grid, kThreads, kSmem, st>>>(mq, mk, mv, a);
  }
  return cudaGetLastError();
}

}  // namespace

// head pairs when each key/value head serves an even number of query heads
template <int D, bool F8, bool PACKED>
cudaError_t launch_fwd_sm100_d(const Problem& p, const void* q, const void* k, const void* v, void* o, float* lse,
                               cudaStream_t st) {
  if ((p.Hq / p.Hkv) % 2 == 0) return launch_fwd_sm100_v<D, F8, PACKED, true>(p, q, k, v, o, lse, st);
  return launch_fwd_sm100_v<D, F8, PACKED, false>(p, q, k, v, o, lse, st);
}

cudaError_t launch_fwd_sm100(const Problem& p, const void* q, const void* k, const void* v, void* o, float* lse,
                             cudaStream_t st) {
  const bool packed = p.cu_q != nullptr;
  if (p.D == 128)
    return packed ? launch_fwd_sm100_d<128, false, true>(p, q, k, v, o, lse, st)
                  : launch_fwd_sm100_d<128, false, false>(p, q, k, v, o, lse, st);
  return packed ? launch_fwd_sm100_d<64, false, true>(p, q, k, v, o, lse, st)
                : launch_fwd_sm100_d<64, false, false>(p, q, k, v, o, lse, st);
}

cudaError_t launch_fwd_sm100_fp8(const Problem& p, const void* q, const void* k, const void* v, void* o, float* lse,
                                 cudaStream_t st) {
  if (p.D != 128 || p.cu_q) return cudaErrorInvalidValue;
  return launch_fwd_sm100_d<128, true, false>(p, q, k, v, o, lse, st);
}

}  // namespace attn
