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
// The path is HBM-bound (each K/V byte is read once, about 4 flop per byte). The split kernel is a
// persistent grid (three CTAs per SM) that walks a static list of work items, one item per
// (chunk, kv head, stream) covering all GT query heads of that kv head's group, so each K/V row is
// fetched once for GT query heads. One producer warp streams the items' 16-key K and V blocks with
// TMA tile loads (128-byte swizzle) into an 8-stage shared-memory ring, without a pause between
// items, and fetches each item's query rows with a bulk copy; compute warp w takes the ring's
// blocks w, w+4, ... (two stages per warp, so one block lands while the other is used). Both
// contractions of a block are warp-level tensor-core products: the GT heads are too few rows for
// tcgen05 (M >= 64) and would waste 16x there, against 4x in m16n8k16. At the end of an item
// warps 1-3 leave their triples in shared memory and warp 0 merges them with its own and writes
// the item's partial triple.
// The host does not know the cache's row count T (it lives on the device as kv_offsets[N]), so the
// tensor maps carry a nominal row extent and the kernel issues a 16-row box only when the whole box
// lies below T; the cache's last partial block is fetched in 16-byte pieces with bulk copies. No
// copy ever touches memory past the caller's K and V buffers.
// A paged cache (pages of a multiple of 16 keys, a block table per stream) runs through the same
// kernels: chunks are then whole 16-key blocks, so a block lies in one page and its box starts at
// the page's pool row. A stream's last block is copied whole too (the box stays inside its page),
// and the consuming warp clears the V rows past the stream's end, since the rest of a page may hold
// anything. A page id outside the pool is not read: its rows count as zeros and the device status
// records ATTN_ERR_INVALID_ARG.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"

namespace attn {

// The built-in split count of a stream of L keys. One query token per stream: chunks of about 256
// keys, 4 to 16 of them. Several tokens per stream: each chunk already carries q_len times the work
// per key and its partial triples q_len times the bytes, so chunks of about 512 keys, 2 to 16 (the
// 48-stream, four-token step took 140 us this way against 169 us with the one-token rule).
__host__ __device__ inline int decode_split_rule(int L, int max_splits, int q_len = 1) {
  int c, lo;
  if (q_len <= 1) {
    c = (L + 255) / 256;
    lo = 4;
  } else {
    c = (L + 511) / 512;
    lo = 2;
  }
  c = c < lo ? lo : (c > 16 ? 16 : c);
  if (c > max_splits) c = max_splits;
  return c < 1 ? 1 : c;
}

int decode_default_splits(int L, int max_splits) { return decode_split_rule(L, max_splits); }

size_t decode_workspace_bytes(int N, int Hq, int D, int max_splits) {
  const size_t slots = static_cast<size_t>(N) * Hq * max_splits;  // N counts (stream, query token) rows
  const size_t o_bytes = (slots * D * sizeof(float) + 255) & ~static_cast<size_t>(255);
  const size_t ml_bytes = (slots * 2 * sizeof(float) + 255) & ~static_cast<size_t>(255);
  return o_bytes + ml_bytes;
}

namespace {

__device__ __forceinline__ int stream_splits(const int* num_splits, int n, int L, int max_splits, int q_len) {
  if (num_splits) {
    const int c = num_splits[n];
    return c < 1 ? 1 : (c > max_splits ? max_splits : c);
  }
  return decode_split_rule(L, max_splits, q_len);
}

// Where the keys of each stream live. Contiguous: stream n owns rows offsets[n] .. offsets[n+1] - 1
// of the packed caches. Paged (block_table != null): key t of stream n is row t % page_size of page
// block_table[n * max_pages + t / page_size] of a pool of num_pages pages, and the stream has
// seq_lens[n] keys (clamped to [0, max_pages * page_size]).
struct DecKV {
  const int* offsets;
  const int* seq_lens;
  const int* block_table;
  int max_pages, page_size, num_pages;
  int page_shift;  // log2(page_size) when it is a power of two, else -1
};

__device__ __forceinline__ void dec_stream(const DecKV& kv, int n, int& start, int& L) {
  if (kv.block_table) {
    start = 0;
    L = min(max(kv.seq_lens[n], 0), kv.max_pages * kv.page_size);
  } else {
    start = kv.offsets[n];
    L = kv.offsets[n + 1] - start;
  }
}

constexpr int kDecBlk = 16;              // keys per block (two lanes per key while scoring)
constexpr int kDecStages = 8;
// Compute warp w consumes blocks w, w + 4, ... and every stage has a single-arrival "empty" barrier,
// so a stage must always belong to the same warp: the stage count is a multiple of the four compute
// warps (otherwise two warps would share a stage and a parity wait could match the wrong phase).
// With eight stages each warp owns two, so its next block is in flight while it computes one.
static_assert(kDecStages % 4 == 0, "decode ring stages must be a multiple of the compute warps");
constexpr int kDecThreads = 160;          // four compute warps + one producer warp
constexpr int kDecMapRows = 0x7fffffff;   // nominal row extent of the K/V tensor maps
// Up to this many streams, every CTA numbers the valid items densely (a prefix sum of the per-stream
// item counts in shared memory), so the static round-robin hands each CTA the same number of items
// to within one; above it, CTAs walk the slot space and skip the slots past a stream's split count.
constexpr int kDecDenseMax = 256;

// The query rows of one item are rows of the m16n8k16 products: row r is query token tq0 + r / GT
// and query head h0 + r % GT. RM is the number of rows the kernel variant carries: 4 (one row per
// lane quad, rows 4-15 zero; one query token per stream, the 48-stream decode) or 16 (two rows per
// lane quad, for several query tokens per stream). The smaller variant fits three CTAs per SM.
template <int RM>
constexpr int dec_ctas_per_sm() {
  return RM == 4 ? 3 : 2;
}

template <int D, int RM>
struct DecCfg {
  static constexpr int kAtoms = D / 64;
  static constexpr int kAtomBytes = kDecBlk * 128;       // 16 rows x 128 bytes
  static constexpr int kBlkBytes = kAtoms * kAtomBytes;  // 16 key rows x D bf16
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kDecStages * kBlkBytes;
  static constexpr int kOffQ = 2 * kDecStages * kBlkBytes;  // [2 items][RM rows][D + 8] bf16
  // Query rows 16 bytes apart beyond their D elements: the compute warps' fragment loads (eight
  // rows, four consecutive words each) then fall on 32 different banks instead of four.
  static constexpr int kQRow = D * 2 + 16;
  static constexpr int kQBuf = RM * kQRow;
  static constexpr int kOffDep = kOffQ + 2 * kQBuf;         // warps 1-3: [3][RM rows][D] fp32
  static constexpr int kOffBar = kOffDep + 3 * RM * D * 4;
  static constexpr int kNumBars = 2 * kDecStages + 4;       // full, empty, q_full[2], q_empty[2]
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;   // abort flag, then the deposits' (m, l)
  static constexpr int kOffBase = kOffMisc + 16 + 2 * 3 * RM * 4;  // dense item numbering, see below
  static constexpr int kSmemBytes = kOffBase + (kDecDenseMax + 1) * 4 + 1024;
  static_assert(kSmemBytes * dec_ctas_per_sm<RM>() <= 232448, "shared memory per SM");
};

// How the query rows of a stream are cut into items: q_len query tokens per stream (the newest
// q_len positions of its cache), GT query heads and TQ query tokens per item, ntp = ceil(q_len / TQ)
// token passes.
struct DecQ {
  int q_len, GT, TQ, ntp;
  int fault_block;  // test-only fault-injection build: CTA 0 skips this ring block's copy (-1: none)
};

// One work item: the key chunk c of stream n for query heads h0 .. h0 + GT - 1 (of kv head g) and
// query tokens tq0 .. tq0 + TQ - 1. L = the stream's length; keys k0 .. k1 - 1 of the stream; nblk
// 16-key blocks, ending at the last key any of the item's tokens can see.
struct DecItem {
  int n, c, g, h0, tq0, start, L, k0, k1, nblk;
};

// The item whose fields are (n, c, gi) -> it; C_n is the stream's split count. Items of one chunk
// are numbered kv head slowest, so the head and token passes that read the same keys are adjacent.
// With `aligned`, chunks are rounded up to whole 16-key blocks (a paged cache: a block must not
// straddle two pages); the last chunks of a stream may then be empty.
__device__ __forceinline__ void dec_item_fill(int n, int c, int gi, int start, int L, int C_n, int Hq, int Hkv,
                                              const DecQ& dq, bool aligned, DecItem& it) {
  const int G = Hq / Hkv, npass = G / dq.GT, per_g = npass * dq.ntp;
  int chunk = (L + C_n - 1) / C_n;
  if (aligned) chunk = (chunk + kDecBlk - 1) / kDecBlk * kDecBlk;
  it.n = n;
  it.c = c;
  it.g = gi / per_g;
  const int r = gi - it.g * per_g;
  it.h0 = it.g * G + (r / dq.ntp) * dq.GT;
  it.tq0 = (r % dq.ntp) * dq.TQ;
  it.start = start;
  it.L = L;
  it.k0 = min(L, c * chunk);
  it.k1 = min(L, it.k0 + chunk);
  // token t sees the stream's keys 0 .. L - q_len + t (the newest q_len positions are its own)
  const int last_tok = min(dq.q_len, it.tq0 + dq.TQ) - 1;
  const int kend = min(it.k1, max(it.k0, L - dq.q_len + last_tok + 1));
  it.nblk = (kend - it.k0 + kDecBlk - 1) / kDecBlk;
}

// Dense item k -> item, with base[n] = NG * (C_0 + ... + C_{n-1}) in shared memory (N + 1 entries):
// stream n holds items base[n] .. base[n + 1] - 1, chunk c = r / NG, head/token group gi = r % NG.
// The groups of one chunk are consecutive items, so neighbouring CTAs read the same cache rows at
// about the same time (a row holds every kv head's keys side by side).
__device__ __forceinline__ void dec_item_dense(int k, int N, int Hq, int Hkv, const DecKV& kv, const DecQ& dq,
                                               const int* base, DecItem& it) {
  int lo = 0, hi = N;  // largest n with base[n] <= k
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (base[mid] <= k) lo = mid; else hi = mid;
  }
  const int NG = Hkv * ((Hq / Hkv) / dq.GT) * dq.ntp;
  const int C_n = (base[lo + 1] - base[lo]) / NG;
  const int r = k - base[lo];
  int start, L;
  dec_stream(kv, lo, start, L);
  dec_item_fill(lo, r / NG, r % NG, start, L, C_n, Hq, Hkv, dq, kv.block_table != nullptr, it);
}

__device__ __forceinline__ bool dec_item(long long idx, int N, int Hq, int Hkv, const DecKV& kv, const DecQ& dq,
                                         const int* num_splits, int max_splits, DecItem& it) {
  const int NG = Hkv * ((Hq / Hkv) / dq.GT) * dq.ntp;
  const long long per_c = static_cast<long long>(N) * NG;
  const int c = static_cast<int>(idx / per_c);
  const int r = static_cast<int>(idx - c * per_c);
  const int n = r / NG, gi = r - (r / NG) * NG;
  int start, L;
  dec_stream(kv, n, start, L);
  const int C_n = stream_splits(num_splits, n, L, max_splits, dq.q_len);
  if (c >= C_n) return false;
  dec_item_fill(n, c, gi, start, L, C_n, Hq, Hkv, dq, kv.block_table != nullptr, it);
  return true;
}

__device__ __forceinline__ bool dec_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

// Byte offset of element d of row r in a 128-byte-swizzled block of 64-element column atoms.
template <int D>
__device__ __forceinline__ uint32_t dec_sw(int r, int d) {
  constexpr int kAtomBytes = kDecBlk * 128;
  return (d >> 6) * kAtomBytes + sw128_offset(r, (d & 63) >> 3) + (d & 7) * 2;
}

template <int D, int RM, bool PAGED>
__global__ void __launch_bounds__(kDecThreads, dec_ctas_per_sm<RM>())
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                        const uint16_t* __restrict__ v, const DecKV kv, const DecQ dq, int N,
                        const int* __restrict__ num_splits, int max_splits, int Hq, int Hkv, float scale_log2,
                        float* __restrict__ part_o, float* __restrict__ part_ml, int* status) {
  using C = DecCfg<D, RM>;
  constexpr int NR = RM == 16 ? 2 : 1;  // rows per lane quad: g and g + 8
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sQ = smem + C::kOffQ;
  float* dep = reinterpret_cast<float*>(smem + C::kOffDep);  // [3][RM][D]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + kDecStages;
  uint64_t* q_full = empty + kDecStages;  // [2]
  uint64_t* q_empty = q_full + 2;         // [2]
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc);
  float* dep_m = reinterpret_cast<float*>(smem + C::kOffMisc + 16);  // [3][RM]
  float* dep_l = dep_m + 3 * RM;                                      // [3][RM]

  const int NG = Hkv * ((Hq / Hkv) / dq.GT) * dq.ntp;
  const long long n_slots = static_cast<long long>(N) * NG * max_splits;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // dense numbering of the valid items (up to kDecDenseMax streams): warp 0 scans the per-stream
  // item counts 32 streams at a time
  int* base = reinterpret_cast<int*>(smem + C::kOffBase);
  const bool dense = N <= kDecDenseMax;
  if (dense && warp == 0) {
    int run = 0;
    for (int n0 = 0; n0 < N; n0 += 32) {
      const int n = n0 + lane;
      int cnt = 0;
      if (n < N) {
        int st0, L;
        dec_stream(kv, n, st0, L);
        cnt = NG * stream_splits(num_splits, n, L, max_splits, dq.q_len);
      }
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (n < N) base[n] = run + incl - cnt;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) base[N] = run;
  }
  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);  // each block is consumed by exactly one compute warp
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(q_full + b, 1);
      mbar_init(q_empty + b, 4);  // every compute warp has read its query fragments
    }
    *abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const long long n_iter = dense ? base[N] : n_slots;  // items (dense) or slots (sparse)
  // item number i of the walk -> item; false for a sparse slot past its stream's split count
  auto next_item = [&](long long i, DecItem& it) -> bool {
    if (dense) {
      dec_item_dense(static_cast<int>(i), N, Hq, Hkv, kv, dq, base, it);
      return true;
    }
    return dec_item(i, N, Hq, Hkv, kv, dq, num_splits, max_splits, it);
  };

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    constexpr bool paged = PAGED;
    const int T = paged ? 0 : min(kv.offsets[N], kDecMapRows);  // no box may reach past the cache
    const long long rs = static_cast<long long>(Hkv) * D;
    const uint32_t qrow_bytes = static_cast<uint32_t>(dq.GT) * D * 2;  // one token's GT heads
    long long gb = 0;  // ring position: blocks issued so far
    int qi = 0;        // items started so far
    bool ok = true;
    for (long long idx = blockIdx.x; ok && idx < n_iter; idx += gridDim.x) {
      DecItem it;
      if (!next_item(idx, it)) continue;
      if (lane == 0) {  // the item's query rows (GT contiguous heads per token) into buffer qi % 2
        ok = mbar_wait(q_empty + (qi & 1), ((qi >> 1) & 1) ^ 1, abort, status);
        if (ok) {
          const int ntok = min(dq.TQ, dq.q_len - it.tq0);
          mbar_arrive_expect_tx(q_full + (qi & 1), ntok * qrow_bytes);
          for (int t = 0; t < ntok; ++t)
            for (int hh = 0; hh < dq.GT; ++hh)
              bulk_load(sQ + (qi & 1) * C::kQBuf + (t * dq.GT + hh) * C::kQRow,
                        q + ((static_cast<long long>(it.n) * dq.q_len + it.tq0 + t) * Hq + it.h0 + hh) * D, D * 2,
                        q_full + (qi & 1));
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      ++qi;
      for (int bk = 0; bk < it.nblk; ++bk) {
        const int s = static_cast<int>(gb % kDecStages);
        const int t0 = it.k0 + bk * kDecBlk;  // the block's first key in the stream
        int row0, nrows;
        bool tile;
        if (paged) {
          // chunks are whole blocks and pages a multiple of 16 keys, so the 16-row box lies inside
          // one page and is always copied whole; the rows of a stream's last block past its end
          // (which may hold anything, NaN included) are cleared in V by the consuming warp, and
          // their scores are masked
          const int pidx = kv.page_shift >= 0 ? t0 >> kv.page_shift : t0 / kv.page_size;
          const int prow = kv.page_shift >= 0 ? t0 & (kv.page_size - 1) : t0 % kv.page_size;
          const int page = kv.block_table[static_cast<long long>(it.n) * kv.max_pages + pidx];
          const bool page_ok = page >= 0 && page < kv.num_pages;
          if (!page_ok && lane == 0) record_status(status, kStatusBadArg);
          row0 = page_ok ? page * kv.page_size + prow : 0;
          tile = page_ok;
          nrows = page_ok ? kDecBlk : 0;  // an invalid page is read as zeros
        } else {
          row0 = it.start + t0;
          tile = row0 + kDecBlk <= T;
          nrows = tile ? kDecBlk : min(kDecBlk, it.k1 - t0);
        }
        if (lane == 0) ok = mbar_wait(empty + s, static_cast<uint32_t>((gb / kDecStages) & 1) ^ 1, abort, status);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (!tile) {
          // Rows past the cache's end stay out of the copy; the tensor-core products read every row
          // of the block (weighted by probability 0), so they must hold finite values: zeros.
          for (int idx2 = lane; idx2 < (kDecBlk - nrows) * (D / 8); idx2 += 32) {
            const int r = nrows + idx2 / (D / 8), d = (idx2 % (D / 8)) * 8;
            *reinterpret_cast<uint4*>(sK + s * C::kBlkBytes + dec_sw<D>(r, d)) = make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(sV + s * C::kBlkBytes + dec_sw<D>(r, d)) = make_uint4(0u, 0u, 0u, 0u);
          }
          __syncwarp();
        }
#ifdef ATTN_FAULT_INJECT
        if (blockIdx.x == 0 && gb == dq.fault_block) {  // a compute warp's wait for it runs out
          ++gb;
          continue;
        }
#endif
        if (lane == 0) {
          mbar_arrive_expect_tx(full + s, 2u * nrows * D * 2);
          if (tile) {
#pragma unroll
            for (int at = 0; at < C::kAtoms; ++at) {
              tma_load_3d(sK + s * C::kBlkBytes + at * C::kAtomBytes, &tmK, full + s, at * 64, it.g, row0);
              tma_load_3d(sV + s * C::kBlkBytes + at * C::kAtomBytes, &tmV, full + s, at * 64, it.g, row0);
            }
          }
        }
        __syncwarp();
        if (!tile) {
          // the cache's last rows: 16-byte pieces into the same swizzled places a tile load uses
          for (int idx2 = lane; idx2 < nrows * (D / 8); idx2 += 32) {
            const int r = idx2 / (D / 8), d = (idx2 % (D / 8)) * 8;
            bulk_load(sK + s * C::kBlkBytes + dec_sw<D>(r, d), k + (row0 + r) * rs + it.g * D + d, 16, full + s);
            bulk_load(sV + s * C::kBlkBytes + dec_sw<D>(r, d), v + (row0 + r) * rs + it.g * D + d, 16, full + s);
          }
        }
        ++gb;
      }
    }
    // let this CTA's copies land before it can exit (at once on the normal path)
    if (lane == 0) {
      for (long long b = max(0ll, gb - kDecStages); b < gb; ++b)
        dec_wait_drain(full + b % kDecStages, static_cast<uint32_t>((b / kDecStages) & 1));
      for (int i = max(0, qi - 2); i < qi; ++i) dec_wait_drain(q_full + (i & 1), (i >> 1) & 1);
    }
    return;
  }

  // ------------------------------------------------------------------ compute warps
  // Lane (g, t) = (lane / 4, lane % 4) holds item row g (and g + 8 when RM = 16): scores of keys 2t,
  // 2t + 1, 8 + 2t, 9 + 2t of a block and output columns 8 j + 2t, 8 j + 2t + 1 of every 8-column
  // tile j. The item's rows (query heads x query tokens) are the rows of the m16n8k16 products
  // (padded to 16 with zeros), so S^T = Q K^T takes K straight from the ring as its column operand
  // and P V takes the probabilities straight from the score accumulators.
  const int gq = lane >> 2, tq = lane & 3;
  constexpr int KS = D / 16;  // 16-wide steps over the head dim
  const int mi = lane >> 3, ri = lane & 7;  // ldmatrix: this lane addresses row ri of matrix mi
  long long gb = 0;  // ring position of the current item's first block
  int qi = 0;
  bool ok = true;    // false once a wait has failed: the warp then only keeps the barrier protocol
  for (long long idx = blockIdx.x; idx < n_iter; idx += gridDim.x) {
    DecItem it;
    if (!next_item(idx, it)) continue;
    // this item's query rows (bf16) in shared memory; each block reads its Q fragments from there
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(q_full + (qi & 1), (qi >> 1) & 1, abort, status)) != 0;
    const int qbuf = qi & 1;
    ++qi;
    const int nrow = dq.GT * min(dq.TQ, dq.q_len - it.tq0);  // valid rows of this item
    bool valid[NR];
    int lim[NR];  // last visible key of the row, relative to the chunk's first key
    const uint32_t* qrow[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const int row = gq + 8 * r;
      valid[r] = row < nrow && row < RM;
      lim[r] = it.L - dq.q_len + it.tq0 + row / dq.GT - it.k0;
      qrow[r] = reinterpret_cast<const uint32_t*>(sQ + qbuf * C::kQBuf + (valid[r] ? row : 0) * C::kQRow);
    }
    float o[D / 8][4];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float mrow[NR], lrow[NR];  // per row: running max (base 2) and this lane's share of the sum
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      mrow[r] = -INFINITY;
      lrow[r] = 0.f;
    }
    for (int bk = (warp - static_cast<int>(gb & 3)) & 3; ok && bk < it.nblk; bk += 4) {
      const long long gbk = gb + bk;
      const int s = static_cast<int>(gbk % kDecStages);
      ok = __all_sync(0xffffffffu, mbar_wait(full + s, static_cast<uint32_t>((gbk / kDecStages) & 1), abort,
                                             status)) != 0;
      if (!ok) break;
      const uint32_t kb = smem_u32(sK + s * C::kBlkBytes);
      const uint32_t vb = smem_u32(sV + s * C::kBlkBytes);
      const int nk = min(kDecBlk, it.k1 - (it.k0 + bk * kDecBlk));  // keys of the chunk in this block
      if (PAGED && nk < kDecBlk) {
        // a paged block copied whole past its stream's end: V rows nk .. 15 to zero (the P V product
        // reads them with probability 0, and 0 times NaN would not be 0)
        for (int idx2 = lane; idx2 < (kDecBlk - nk) * (D / 8); idx2 += 32)
          *reinterpret_cast<uint4*>(sV + s * C::kBlkBytes + dec_sw<D>(nk + idx2 / (D / 8), (idx2 % (D / 8)) * 8)) =
              make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();  // before the stage's next copy, issued once this warp releases it
        __syncwarp();
      }
      // S^T for keys 0-7 (s0) and 8-15 (s1); rows g in s*[0..1], rows g + 8 in s*[2..3]
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        // Q fragments of the lane's rows (zero for padding rows): head dims 16 ks + 2t .. and + 8
        const uint32_t qa = valid[0] ? qrow[0][8 * ks + tq] : 0u, qb = valid[0] ? qrow[0][8 * ks + 4 + tq] : 0u;
        uint32_t qc = 0u, qd = 0u;
        if (NR == 2) {
          qc = valid[NR - 1] ? qrow[NR - 1][8 * ks + tq] : 0u;
          qd = valid[NR - 1] ? qrow[NR - 1][8 * ks + 4 + tq] : 0u;
        }
        uint32_t b00, b01, b10, b11;  // matrices: keys 8 (mi / 2) + ri, head dims 16 ks + 8 (mi % 2) ..
        ldsm_x4(kb + dec_sw<D>(ri + 8 * (mi >> 1), 16 * ks + 8 * (mi & 1)), b00, b01, b10, b11);
        mma_16816(s0, qa, qc, qb, qd, b00, b01);
        mma_16816(s1, qa, qc, qb, qd, b10, b11);
      }
      const int kx[4] = {2 * tq, 2 * tq + 1, 8 + 2 * tq, 9 + 2 * tq};
      float p[NR][4];
      bool rescale = false;
      float alpha[NR];
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        float x[4] = {s0[2 * r], s0[2 * r + 1], s1[2 * r], s1[2 * r + 1]};
        // visible: inside the chunk and at or before the row's causal limit
        const int vis = valid[r] ? min(nk, lim[r] - bk * kDecBlk + 1) : 0;
        float bm = -INFINITY;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          x[e] = kx[e] < vis ? x[e] * scale_log2 : -INFINITY;
          bm = fmaxf(bm, x[e]);
        }
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));  // block max of the row
        // lazy rescale: the reference max moves only when the block max exceeds it by more than 8
        alpha[r] = 1.f;
        if (bm > mrow[r] + 8.f || (mrow[r] == -INFINITY && bm != -INFINITY)) {
          alpha[r] = (mrow[r] == -INFINITY) ? 0.f : fast_exp2(mrow[r] - bm);
          mrow[r] = bm;
        }
        rescale = rescale || alpha[r] != 1.f;
        const float m_use = mrow[r] == -INFINITY ? 0.f : mrow[r];
#pragma unroll
        for (int e = 0; e < 4; ++e) p[r][e] = fast_exp2(x[e] - m_use);  // 2^(-inf) = 0 for hidden keys
      }
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          lrow[r] *= alpha[r];
#pragma unroll
          for (int j = 0; j < D / 8; ++j) {
            o[j][2 * r] *= alpha[r];
            o[j][2 * r + 1] *= alpha[r];
          }
        }
      }
#pragma unroll
      for (int r = 0; r < NR; ++r) lrow[r] += (p[r][0] + p[r][1]) + (p[r][2] + p[r][3]);
      const uint32_t pa0 = pack_bf16(p[0][0], p[0][1]), pa2 = pack_bf16(p[0][2], p[0][3]);
      const uint32_t pa1 = NR == 2 ? pack_bf16(p[NR - 1][0], p[NR - 1][1]) : 0u;
      const uint32_t pa3 = NR == 2 ? pack_bf16(p[NR - 1][2], p[NR - 1][3]) : 0u;
      // O += P V over pairs of 8-column tiles
#pragma unroll
      for (int jp = 0; jp < D / 16; ++jp) {
        uint32_t v0, v1, v2, v3;  // matrices: keys 8 (mi % 2) + ri, head dims 16 jp + 8 (mi / 2) ..
        ldsm_x4_trans(vb + dec_sw<D>(ri + 8 * (mi & 1), 16 * jp + 8 * (mi >> 1)), v0, v1, v2, v3);
        mma_16816(o[2 * jp], pa0, pa1, pa2, pa3, v0, v1);
        mma_16816(o[2 * jp + 1], pa0, pa1, pa2, pa3, v2, v3);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + s);
    }
    gb += it.nblk;
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(q_empty + qbuf);  // done with this item's query rows
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
      lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
    }
    // Merge the four warps' triples (a warp that saw no block of the item holds the identity).
    // Named barrier 1: warps 1-3 have deposited; barrier 2: warp 0 has read the deposits, so they
    // may be overwritten. Every compute warp passes both for every item, also after a failed wait.
    if (warp > 0) {
      if (qi > 1) named_barrier(2, 128);
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        if (!valid[r]) continue;
        const int row = gq + 8 * r;
        float* dw = dep + ((warp - 1) * RM + row) * D;
        if (tq == 0) {
          dep_m[(warp - 1) * RM + row] = mrow[r];
          dep_l[(warp - 1) * RM + row] = lrow[r];
        }
#pragma unroll
        for (int j = 0; j < D / 8; ++j)
          *reinterpret_cast<float2*>(dw + 8 * j + 2 * tq) = make_float2(o[j][2 * r], o[j][2 * r + 1]);
      }
      named_barrier_arrive(1, 128);
    } else {
      named_barrier(1, 128);
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        if (!valid[r]) continue;
        const int row = gq + 8 * r;
        float M = mrow[r];
#pragma unroll
        for (int w = 0; w < 3; ++w) M = fmaxf(M, dep_m[w * RM + row]);
        float e0 = 0.f, ew[3] = {0.f, 0.f, 0.f};
        if (M != -INFINITY) {
          e0 = mrow[r] == -INFINITY ? 0.f : fast_exp2(mrow[r] - M);
#pragma unroll
          for (int w = 0; w < 3; ++w) {
            const float mw = dep_m[w * RM + row];
            ew[w] = mw == -INFINITY ? 0.f : fast_exp2(mw - M);
          }
        }
        float Lsum = e0 * lrow[r];
#pragma unroll
        for (int w = 0; w < 3; ++w) Lsum = fmaf(ew[w], dep_l[w * RM + row], Lsum);
        const int tok = it.tq0 + row / dq.GT, h = it.h0 + row % dq.GT;
        const long long slot = ((static_cast<long long>(it.n) * dq.q_len + tok) * Hq + h) * max_splits + it.c;
        float* dst = part_o + slot * D;
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
          float a0 = e0 * o[j][2 * r], a1 = e0 * o[j][2 * r + 1];
#pragma unroll
          for (int w = 0; w < 3; ++w) {
            const float2 y = *reinterpret_cast<const float2*>(dep + (w * RM + row) * D + 8 * j + 2 * tq);
            a0 = fmaf(ew[w], y.x, a0);
            a1 = fmaf(ew[w], y.y, a1);
          }
          *reinterpret_cast<float2*>(dst + 8 * j + 2 * tq) = make_float2(a0, a1);
        }
        if (tq == 0) {
          part_ml[slot * 2] = M;
          part_ml[slot * 2 + 1] = Lsum;
        }
      }
      named_barrier_arrive(2, 128);
    }
  }
  if (warp > 0 && qi > 0) named_barrier(2, 128);  // pairs with warp 0's arrival for the last item
  griddep_launch_dependents();
}

// Merge of the partial triples of one output row (stream n, query token t, query head h): one warp.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const float* __restrict__ part_o,
                                                             const float* __restrict__ part_ml,
                                                             const DecKV kv,
                                                             const int* __restrict__ num_splits, int max_splits,
                                                             int N, int q_len, int Hq, uint16_t* __restrict__ o,
                                                             float* __restrict__ lse) {
  constexpr int DPL = D / 32;
  griddep_wait();  // the split kernel's partial triples
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long gw = static_cast<long long>(blockIdx.x) * 4 + warp;  // (n, t, h), h fastest
  if (gw >= static_cast<long long>(N) * q_len * Hq) return;
  const int h = static_cast<int>(gw % Hq);
  const long long nt = gw / Hq;
  const int n = static_cast<int>(nt / q_len), tok = static_cast<int>(nt % q_len);
  int st0, L;
  dec_stream(kv, n, st0, L);
  const int C = stream_splits(num_splits, n, L, max_splits, q_len);
  const long long slot0 = gw * max_splits;
  // The first 16 partial rows are loaded before anything else, so their loads and those of the
  // (m, l) pairs are in flight together; lane c holds the pair of chunk c and c + 32 (max_splits
  // <= 64).
  constexpr int kFirst = 16;
  float x[kFirst][DPL];
#pragma unroll
  for (int c = 0; c < kFirst; ++c) {
    const float* src = part_o + (slot0 + c) * D + lane * DPL;
    if constexpr (DPL == 4) {
      const float4 y = c < C ? *reinterpret_cast<const float4*>(src) : make_float4(0.f, 0.f, 0.f, 0.f);
      x[c][0] = y.x;
      x[c][1] = y.y;
      x[c][2] = y.z;
      x[c][3] = y.w;
    } else {
      const float2 y = c < C ? *reinterpret_cast<const float2*>(src) : make_float2(0.f, 0.f);
      x[c][0] = y.x;
      x[c][1] = y.y;
    }
  }
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
#pragma unroll
  for (int c = 0; c < kFirst; ++c) {
    const float wc = __shfl_sync(0xffffffffu, w0, c);  // 0 for c >= C
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = fmaf(wc, x[c][e], acc[e]);
  }
  // any further partials, four per round
  for (int c0 = kFirst; c0 < C; c0 += 4) {
    float y4[4][DPL], wv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + u;
      wv[u] = __shfl_sync(0xffffffffu, c < 32 ? w0 : w1, c & 31);
      const float* src = part_o + (slot0 + c) * D + lane * DPL;
#pragma unroll
      for (int e = 0; e < DPL; ++e) y4[u][e] = c < C ? src[e] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(wv[u], y4[u][e], acc[e]);
  }
  const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
  uint16_t* dst = o + gw * D + lane * DPL;  // o [N, q_len, Hq, D]: row (n, t, h) is row gw
  if constexpr (DPL == 4) {
    uint2 w;
    w.x = pack_bf16(acc[0] * inv, acc[1] * inv);
    w.y = pack_bf16(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(dst) = w;
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16(acc[0] * inv, acc[1] * inv);
  }
  // lse [N, Hq, q_len]
  if (lane == 0 && lse)
    lse[(static_cast<long long>(n) * Hq + h) * q_len + tok] = Lt > 0.f ? (M + log2f(Lt)) * kLn2 : -INFINITY;
}

template <int D, int RM, bool PAGED>
cudaError_t launch_split(const DecodeProblem& p, const DecQ& dq, const void* q, const void* k, const void* v,
                         const CUtensorMap& mk, const CUtensorMap& mv, const DecKV& kv, const int* num_splits,
                         float* part_o, float* part_ml, cudaStream_t st) {
  using C = DecCfg<D, RM>;
  const int NG = p.Hkv * ((p.Hq / p.Hkv) / dq.GT) * dq.ntp;
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, RM, PAGED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  // a persistent grid: as many CTAs as fit on the SMs, capped by the number of item slots
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long long n_slots = static_cast<long long>(p.N) * NG * p.max_splits;
  const unsigned grid = static_cast<unsigned>(
      std::min<long long>(n_slots, static_cast<long long>(sms) * dec_ctas_per_sm<RM>()));
  {
    LaunchScope ls("decode_split", st);
    decode_split_kernel<D, RM, PAGED><<<grid, kDecThreads, C::kSmemBytes, st>>>(
        mk, mv, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v),
        kv, dq, p.N, num_splits, p.max_splits, p.Hq, p.Hkv, p.scale * kLog2e, part_o, part_ml,
        device_status_ptr());
  }
  return cudaGetLastError();
}

// Rows of an item: GT query heads (4, 2 or 1, a divisor of the group size) x TQ query tokens. One
// token per stream keeps to the 4-row variant; more tokens fill up to 16 rows.
DecQ decode_rows(int G, int q_len, int& rm) {
  DecQ dq;
  dq.q_len = q_len;
  dq.GT = (G % 4 == 0) ? 4 : ((G % 2 == 0) ? 2 : 1);
  if (q_len * dq.GT <= 4) {
    rm = 4;
    dq.TQ = q_len;
  } else {
    rm = 16;
    dq.TQ = std::min(q_len, 16 / dq.GT);
  }
  dq.ntp = (q_len + dq.TQ - 1) / dq.TQ;
#ifdef ATTN_FAULT_INJECT
  dq.fault_block = fault_block_for(2);
#else
  dq.fault_block = -1;
#endif
  return dq;
}

template <int D>
cudaError_t launch_decode_d(const DecodeProblem& p, const void* q, const void* k, const void* v, const DecKV& kv,
                            long long map_rows, const int* num_splits, void* o, float* lse, void* workspace,
                            cudaStream_t st) {
  const size_t slots = static_cast<size_t>(p.N) * p.q_len * p.Hq * p.max_splits;
  float* part_o = static_cast<float*>(workspace);
  float* part_ml = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                            ((slots * D * sizeof(float) + 255) & ~static_cast<size_t>(255)));
  // K and V as 3-D maps (D, Hkv, rows) over the packed caches or the page pool. For packed caches
  // the row extent is nominal (the real count is on the device) and the kernel never issues a box
  // that reaches past kv_offsets[N]; a pool's extent is its real row count.
  CUtensorMap mk, mv;
  if (!make_map_packed_bf16(&mk, k, map_rows, p.Hkv, D, kDecBlk) ||
      !make_map_packed_bf16(&mv, v, map_rows, p.Hkv, D, kDecBlk))
    return cudaErrorInvalidValue;
  int rm = 4;
  const DecQ dq = decode_rows(p.Hq / p.Hkv, p.q_len, rm);
  // one instantiation per cache layout (packed / paged) and row variant
  cudaError_t e;
  if (kv.block_table)
    e = rm == 4 ? launch_split<D, 4, true>(p, dq, q, k, v, mk, mv, kv, num_splits, part_o, part_ml, st)
                : launch_split<D, 16, true>(p, dq, q, k, v, mk, mv, kv, num_splits, part_o, part_ml, st);
  else
    e = rm == 4 ? launch_split<D, 4, false>(p, dq, q, k, v, mk, mv, kv, num_splits, part_o, part_ml, st)
                : launch_split<D, 16, false>(p, dq, q, k, v, mk, mv, kv, num_splits, part_o, part_ml, st);
  if (e != cudaSuccess) return e;
  const long long warps = static_cast<long long>(p.N) * p.q_len * p.Hq;
  {
    LaunchScope ls("decode_combine", st);
    const cudaError_t e2 =
        launch_dependent(decode_combine_kernel<D>, dim3(static_cast<unsigned>((warps + 3) / 4)), dim3(128), 0, st,
                         part_o, part_ml, kv, num_splits, p.max_splits, p.N, p.q_len, p.Hq,
                         static_cast<uint16_t*>(o), lse);
    if (e2 != cudaSuccess) return e2;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeProblem& p, const void* q, const void* k, const void* v,
                          const int* kv_offsets, const int* num_splits, void* o, float* lse, void* workspace,
                          cudaStream_t st) {
  const DecKV kv{kv_offsets, nullptr, nullptr, 0, 0, 0, -1};
  if (p.D == 128) return launch_decode_d<128>(p, q, k, v, kv, kDecMapRows, num_splits, o, lse, workspace, st);
  return launch_decode_d<64>(p, q, k, v, kv, kDecMapRows, num_splits, o, lse, workspace, st);
}

cudaError_t launch_decode_paged(const DecodeProblem& p, const void* q, const void* k_pages, const void* v_pages,
                                const int* block_table, int max_pages, const int* seq_lens, int page_size,
                                int num_pages, const int* num_splits, void* o, float* lse, void* workspace,
                                cudaStream_t st) {
  int shift = -1;
  for (int b = 4; b < 31; ++b)
    if (page_size == (1 << b)) shift = b;
  const DecKV kv{nullptr, seq_lens, block_table, max_pages, page_size, num_pages, shift};
  const long long rows = static_cast<long long>(num_pages) * page_size;
  if (p.D == 128) return launch_decode_d<128>(p, q, k_pages, v_pages, kv, rows, num_splits, o, lse, workspace, st);
  return launch_decode_d<64>(p, q, k_pages, v_pages, kv, rows, num_splits, o, lse, workspace, st);
}

}  // namespace attn
