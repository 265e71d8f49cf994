/*
 * attn.h -- C ABI of libattn.so: online-softmax attention on NVIDIA B200 (sm_100a).
 *
 * What is computed. Scaled-dot-product attention written as one reduction over the keys under the
 * online-softmax monoid (running max m, running sum l, rescaled accumulator o, with an associative
 * merge): the form that "Não escreva kernels, derive-os" (ceviu.com.br, section "Aprofundamento",
 * first paragraph) says flash attention falls out of once the online softmax is seen as a monoid.
 * The backward is the gradient of the same expression (same page, "Perguntas frequentes",
 * "O que o Tang propõe de diferente?"); causal forward passes are named on the aibriefing page
 * "Tang Project Derives GPU Kernels via IR ..." ("Details"); the decode streams (16 to 48) and the
 * 44k-token prefill are in the third paragraph of "Aprofundamento".
 *
 *   x_ij  = scale * sum_d Q[b,i,h,d] * K[b,j,g,d],  g = h / (Hq/Hkv)     (grouped-query heads)
 *   causal: key j is visible to query i iff j <= i + (Sk - Sq)           (bottom-right aligned)
 *   O[b,i,h,:] = sum_j softmax_j(x_i.) V[b,j,g,:],  lse[b,h,i] = ln sum_j exp(x_ij)  (natural log)
 *   A query row that sees no key gets O = 0 and lse = -inf.
 *
 * Layouts (row-major, contiguous, no padding):
 *   Q, O, dO, dQ : [B, Sq, Hq, D]      K, V, dK, dV : [B, Sk, Hkv, D]      lse : [B, Hq, Sq] fp32
 *   decode: q, o : [N, Hq, D]   k, v : [T, Hkv, D] packed by stream   kv_offsets : [N+1] int32
 * bf16 tensors are passed as void* to 16-bit storage (bfloat16 bit patterns); fp32 as float*.
 *
 * Conventions shared by every call:
 *   - Every tensor pointer is a DEVICE pointer owned by the caller. The library never allocates,
 *     never frees and never synchronises (attn_get_device_status is the one call that waits).
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream) in
 *     stream order. Results are valid once that stream's prior work has completed.
 *   - Arguments are validated on the host BEFORE anything is launched; on error nothing is
 *     enqueued and an attn_status_t error code is returned. Checks: null pointers, B/H/S/D <= 0,
 *     Hq % Hkv != 0, unsupported D, pointers not 16-byte aligned, workspace too small, device not
 *     sm_100. Launch failures (cudaGetLastError after the launch) return ATTN_ERR_LAUNCH.
 *   - Kernels that wait on on-chip barriers bound every wait; if a bound is hit the kernel records
 *     ATTN_ERR_TIMEOUT in a device status word and exits (read it with attn_get_device_status).
 *   - `scale` is used exactly as given (no default inside the ABI).
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, Hq % Hkv != 0, bad causal flag */
  ATTN_ERR_UNSUPPORTED = 2,   /* head dim not supported by this entry point, or GPU not sm_100  */
  ATTN_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned                                */
  ATTN_ERR_WORKSPACE = 4,     /* workspace pointer null or workspace_bytes too small             */
  ATTN_ERR_LAUNCH = 5,        /* a CUDA launch failed                                            */
  ATTN_ERR_TIMEOUT = 6        /* a kernel's bounded on-chip wait ran out (device status only)    */
} attn_status_t;

/* A cudaStream_t, passed as an opaque pointer so that this header needs no CUDA include. */
typedef void* attn_stream_t;

/* ------------------------------------------------------------------------------------------ *
 * Forward.  ("Não escreva kernels, derive-os", "Aprofundamento", first paragraph: attention as
 * one comprehension reduced under the online-softmax monoid.)
 *
 * attn_fwd: bf16 Q, K, V -> bf16 O and fp32 lse, fp32 accumulation on the tensor cores.
 *   q [B,Sq,Hq,D] bf16, k/v [B,Sk,Hkv,D] bf16 (inputs, read only); o [B,Sq,Hq,D] bf16 and
 *   lse [B,Hq,Sq] fp32 (outputs, fully overwritten; lse is required). D must be 64 or 128
 *   (else ATTN_ERR_UNSUPPORTED). causal is 0 or 1.
 * attn_fwd_f32: the same with fp32 tensors everywhere and genuine fp32 arithmetic (no TF32),
 *   any D in [1, 256].
 * ------------------------------------------------------------------------------------------ */
attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                       int B, int Hq, int Hkv, int Sq, int Sk, int D, int causal, float scale,
                       attn_stream_t stream);

/* attn_fwd_fp8: FP8 (e4m3) inputs with per-tensor scales (the FP8 checkpoint that the third
 *   paragraph of "Aprofundamento" credits with a far shorter time to first token). q [B,Sq,Hq,D],
 *   k / v [B,Sk,Hkv,D] hold E4M3 codes (one byte each: sign, 4 exponent bits with bias 7, 3 mantissa
 *   bits; S.1111.111 is NaN); the real inputs are q_scale * q, k_scale * k, v_scale * v (scales > 0,
 *   finite). Scores and P V run on the tensor cores as kind::f8f6f4 with fp32 accumulation; P is
 *   rounded to e4m3 before P V (its largest value is 2^8 under the kernel's lazy rescale, within
 *   e4m3's range), so O is accurate to e4m3's precision, not bf16's. o [B,Sq,Hq,D] bf16, lse
 *   [B,Hq,Sq] fp32 as for attn_fwd. D must be 128 (else ATTN_ERR_UNSUPPORTED). */
attn_status_t attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                           float q_scale, float k_scale, float v_scale,
                           int B, int Hq, int Hkv, int Sq, int Sk, int D, int causal, float scale,
                           attn_stream_t stream);

attn_status_t attn_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                           int B, int Hq, int Hkv, int Sq, int Sk, int D, int causal, float scale,
                           attn_stream_t stream);

/* ------------------------------------------------------------------------------------------ *
 * Backward.  (Same page, "Perguntas frequentes", "O que o Tang propõe de diferente?": the backward
 * comes out of rewrites of the forward graph; the third paragraph of "Aprofundamento" notes a fused
 * bf16 backward that misses an fp32 tolerance, so the bf16 path is held to bf16 tolerances.)
 *
 * With P = softmax rows recomputed from (Q, K, lse), dP = dO V^T, Delta_i = sum_d dO_i O_i and
 * dS = P * (dP - Delta):  dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO, with dK and dV summed
 * over the Hq/Hkv query heads that share a key/value head. Only O is differentiated (not lse).
 *
 * attn_bwd: bf16 q, k, v, o, dout and fp32 lse (as written by attn_fwd) -> bf16 dq, dk, dv (fully
 *   overwritten). D must be 64 or 128. `workspace` is caller-owned device scratch of at least
 *   attn_bwd_workspace_size(...) bytes, 256-byte aligned; its contents on entry do not matter and
 *   it must not be used by other work on other streams while the call runs.
 * attn_bwd_f32: fp32 everywhere, genuine fp32 arithmetic, any D in [1, 256]; its workspace size
 *   is attn_bwd_f32_workspace_size(...).
 * ------------------------------------------------------------------------------------------ */
size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int D);

attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o,
                       const float* lse, const void* dout, void* dq, void* dk, void* dv,
                       void* workspace, size_t workspace_bytes,
                       int B, int Hq, int Hkv, int Sq, int Sk, int D, int causal, float scale,
                       attn_stream_t stream);

size_t attn_bwd_f32_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int D);

attn_status_t attn_bwd_f32(const float* q, const float* k, const float* v, const float* o,
                           const float* lse, const float* dout, float* dq, float* dk, float* dv,
                           void* workspace, size_t workspace_bytes,
                           int B, int Hq, int Hkv, int Sq, int Sk, int D, int causal, float scale,
                           attn_stream_t stream);

/* ------------------------------------------------------------------------------------------ *
 * Packed variable-length prefill.  (The multi-stream prefill behind the 44k-token time to first
 * token of "Não escreva kernels, derive-os", "Aprofundamento", third paragraph: a serving engine
 * prefills several prompts of different lengths at once, packed back to back without padding.)
 *
 * Sequence b (0 <= b < B) owns query rows cu_seqlens_q[b] .. cu_seqlens_q[b+1] - 1 of q / o / dout /
 * dq and key/value rows cu_seqlens_k[b] .. cu_seqlens_k[b+1] - 1 of k / v / dk / dv, and attends only
 * to its own keys, with the same definition as attn_fwd / attn_bwd per sequence (causal: bottom-right
 * aligned within the sequence). A sequence with no key gives its rows O = 0, lse = -inf and zero
 * gradients.
 *   q, o, dout, dq [total_q, Hq, D] bf16; k, v, dk, dv [total_k, Hkv, D] bf16; lse [Hq, total_q] fp32.
 *   cu_seqlens_q / cu_seqlens_k: [B+1] int32 DEVICE arrays (4-byte aligned), non-decreasing, first
 *   entry 0, last entry total_q / total_k. max_seqlen_q / max_seqlen_k: upper bounds of the sequence
 *   lengths (they size the grids and the backward's workspace). The offsets live on the device and
 *   are checked there: a sequence whose rows fall outside [0, total) or exceed the max_seqlen bound
 *   is not read or written (its outputs are left as they were) and the device status records
 *   ATTN_ERR_INVALID_ARG (attn_get_device_status).
 *   Tiles of one sequence may read rows of the next one in the packed tensors (their keys are masked,
 *   their values weighted by 0, their query rows not stored), so those rows must hold finite values.
 *   D is 64 or 128. The backward's workspace: attn_bwd_varlen_workspace_size(B, Hq, Hkv,
 *   max_seqlen_q, max_seqlen_k, D) bytes, 256-byte aligned (fp32 dQ accumulator and per-row
 *   statistics, max_seqlen_q rows per sequence and head).
 * ------------------------------------------------------------------------------------------ */
attn_status_t attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                              const int* cu_seqlens_q, const int* cu_seqlens_k, int B,
                              int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                              int Hq, int Hkv, int D, int causal, float scale, attn_stream_t stream);

size_t attn_bwd_varlen_workspace_size(int B, int Hq, int Hkv, int max_seqlen_q, int max_seqlen_k, int D);

attn_status_t attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                              const float* lse, const void* dout, void* dq, void* dk, void* dv,
                              const int* cu_seqlens_q, const int* cu_seqlens_k, int B,
                              int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                              int Hq, int Hkv, int D, int causal, float scale,
                              void* workspace, size_t workspace_bytes, attn_stream_t stream);

/* ------------------------------------------------------------------------------------------ *
 * Split-KV decode.  (Decode streams of "Não escreva kernels, derive-os", "Aprofundamento", third
 * paragraph; the aibriefing page, "Details", ties its 48-stream accuracy to split granularity.)
 *
 * Stream n has one query token q[n,:,:] and the L_n = kv_offsets[n+1] - kv_offsets[n] keys and
 * values k/v[kv_offsets[n] : kv_offsets[n+1], :, :]; it attends to all of them (no mask). The keys
 * of each (stream, kv head) are cut into C_n contiguous chunks of ceil(L_n / C_n) keys; each chunk
 * yields a partial (m, l, o) triple in `workspace`, and a combine kernel merges the C_n triples with
 * the monoid (m,l,o)+(m',l',o') = (M, l e^{m-M} + l' e^{m'-M}, o e^{m-M} + o' e^{m'-M}).
 *
 *   q [N,Hq,D] bf16; k, v [T,Hkv,D] bf16 with T = kv_offsets[N]; kv_offsets [N+1] int32 DEVICE
 *   array, non-decreasing, kv_offsets[0] = 0 (not checked on the host: it lives on the device).
 *   num_splits: [N] int32 DEVICE array of per-stream chunk counts, or NULL for the built-in rule
 *   C(L) = min(max_splits, clamp(ceil(L/256), 4, 16)) (see attn_decode_default_splits); values
 *   outside [1, max_splits] are clamped on the device. max_splits in [1, 64].
 *   o [N,Hq,D] bf16 (output); lse [N,Hq] fp32 (output, may be NULL). A stream with L_n = 0 gets
 *   O = 0 and lse = -inf. D must be 64 or 128.
 *   workspace: caller-owned device scratch of at least attn_decode_workspace_size(N,Hq,D,max_splits)
 *   bytes, 256-byte aligned (partial triples, fp32).
 * ------------------------------------------------------------------------------------------ */
size_t attn_decode_workspace_size(int N, int Hq, int D, int max_splits);

attn_status_t attn_decode_splitkv(const void* q, const void* k, const void* v,
                                  const int* kv_offsets, const int* num_splits, int max_splits,
                                  void* o, float* lse, int N, int Hq, int Hkv, int D, float scale,
                                  void* workspace, size_t workspace_bytes, attn_stream_t stream);

/* Split-KV decode that allocates nothing (the pages have no counterpart: this entry point exists
 * for callers of this library that cannot hand it a workspace -- a host framework that owns all
 * device memory through its own pool and gives plugins no scratch, or a latency-bound serving loop
 * that may not call cudaMalloc, which can synchronise the device, on its hot path).
 * Same arguments, kernels and results as attn_decode_splitkv, minus the workspace: the partial
 * (m, l, o) triples live in a 16 MiB array compiled into the library, which every GPU that loads the
 * library holds until the process exits. Problems needing more than 16 MiB of partial triples
 * (attn_decode_workspace_size(N, Hq, D, max_splits) > 16777216) return ATTN_ERR_WORKSPACE before
 * anything is launched; e.g. 48 streams x 32 heads x 16 splits at D = 128 need 12.8 MB and fit.
 * The first call on each device looks up the array's device address (with that device current)
 * and keeps it for that device's current CUDA context; after the context has been torn down and
 * created again (cudaDeviceReset), the next call looks it up again, since the library's module may
 * then sit elsewhere. Make each such first call before any stream capture. All calls share the array and
 * leave their partial triples in it; nothing has to start at zero. Calls that overlap on the GPU
 * (other streams or threads) race on the array and give wrong results: serialise them. */
attn_status_t attn_decode_splitkv_static(const void* q, const void* k, const void* v,
                                         const int* kv_offsets, const int* num_splits, int max_splits,
                                         void* o, float* lse, int N, int Hq, int Hkv, int D,
                                         float scale, attn_stream_t stream);

/* Host helper: the built-in split count for a stream of L keys (the rule named above). */
int attn_decode_default_splits(int L, int max_splits);

/* Split-KV decode over a paged key/value cache (the pages have no counterpart: a serving engine
 * keeps its decode streams' caches in fixed-size pages of one pool, and this entry point reads
 * them in place, with the same split + combine and the same monoid as attn_decode_splitkv).
 *
 *   k_pages, v_pages [num_pages, page_size, Hkv, D] bf16: the pools. Key t of stream n is row
 *   t % page_size of page block_table[n * max_pages + t / page_size].
 *   block_table [N, max_pages] int32 DEVICE array of page ids; seq_lens [N] int32 DEVICE array of
 *   stream lengths (L_n is clamped to [0, max_pages * page_size]). Only the entries for pages that
 *   hold keys of a stream are read. A page id outside [0, num_pages) is not read: its keys count as
 *   zeros and the device status records ATTN_ERR_INVALID_ARG (read it with attn_get_device_status).
 *   page_size: a multiple of 16, at least 16; num_pages * page_size < 2^31.
 *   Rows of a stream's last page past its length may hold anything (also NaN): they are not read.
 *   Chunks are whole 16-key blocks (ceil(L_n / C_n) rounded up to 16), so for the same split count
 *   the partial triples can differ from attn_decode_splitkv's by rounding only.
 *   q, o, lse, num_splits, max_splits, scale, workspace: as for attn_decode_splitkv (the same
 *   workspace size, attn_decode_workspace_size(N, Hq, D, max_splits)). D is 64 or 128. */
attn_status_t attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                                const int* block_table, int max_pages, const int* seq_lens, int page_size,
                                int num_pages, const int* num_splits, int max_splits, void* o, float* lse,
                                int N, int Hq, int Hkv, int D, float scale, void* workspace,
                                size_t workspace_bytes, attn_stream_t stream);

/* ------------------------------------------------------------------------------------------ *
 * Decode with several query tokens per stream (speculative or chunked decode steps). The decode
 * steps of "Não escreva kernels, derive-os" ("Aprofundamento", third paragraph) serve 16 to 48
 * streams; a step that verifies draft tokens, or feeds a short chunk of a prompt, brings q_len new
 * tokens per stream instead of one. Their keys and values are already the newest q_len rows of the
 * stream's cache, so token t (0-based) sits at position L_n - q_len + t and attends to keys
 * 0 .. L_n - q_len + t: the causal mask among the new tokens, aligned to the newest position
 * (bottom-right, as in attn_fwd with Sq = q_len, Sk = L_n). A token that sees no key (L_n < q_len)
 * gets O = 0 and lse = -inf. Same split + combine and the same monoid as attn_decode_splitkv; with
 * q_len = 1 the result is that of attn_decode_splitkv.
 *
 *   q, o [N, q_len, Hq, D] bf16 (row (n, t, h) of o is the output of token t of stream n, head h);
 *   lse [N, Hq, q_len] fp32 (may be NULL); q_len >= 1, N * q_len * Hq < 2^31.
 *   k, v, kv_offsets, num_splits, max_splits, scale: as for attn_decode_splitkv (one split count per
 *   stream, shared by its tokens), except that with num_splits NULL and q_len > 1 the built-in rule
 *   cuts about 512 keys per chunk: C(L) = min(max_splits, clamp(ceil(L/512), 2, 16)) (each chunk
 *   carries q_len times the work; results differ from other split counts by rounding only).
 *   workspace: at least attn_decode_workspace_size(N * q_len, Hq, D, max_splits) bytes, 256-byte
 *   aligned.
 * attn_decode_paged_qlen: the same over a paged cache (arguments as attn_decode_paged).
 * ------------------------------------------------------------------------------------------ */
attn_status_t attn_decode_splitkv_qlen(const void* q, const void* k, const void* v,
                                       const int* kv_offsets, const int* num_splits, int max_splits,
                                       void* o, float* lse, int N, int q_len, int Hq, int Hkv, int D,
                                       float scale, void* workspace, size_t workspace_bytes,
                                       attn_stream_t stream);

attn_status_t attn_decode_paged_qlen(const void* q, const void* k_pages, const void* v_pages,
                                     const int* block_table, int max_pages, const int* seq_lens,
                                     int page_size, int num_pages, const int* num_splits, int max_splits,
                                     void* o, float* lse, int N, int q_len, int Hq, int Hkv, int D,
                                     float scale, void* workspace, size_t workspace_bytes,
                                     attn_stream_t stream);

/* ------------------------------------------------------------------------------------------ *
 * Merge of partial attentions.  ("Não escreva kernels, derive-os", "Aprofundamento", first
 * paragraph: the online softmax is a monoid, so attention over a union of key sets is the merge of
 * the attentions over each set, in any order.) A context-parallel forward across GPUs computes, on
 * each rank, the attention of its query rows against one key/value shard after another and folds
 * each partial result in with this call.
 *
 * With M = max(lse_acc, lse_part), w_a = e^(lse_acc - M), w_b = e^(lse_part - M):
 *   lse_acc <- M + ln(w_a + w_b),   o_acc <- (w_a o_acc + w_b o_part) / (w_a + w_b),
 * row by row; lse = -inf is the identity (its O is not read; a row that is -inf in both stays
 * O = 0, lse = -inf).
 *   o_acc [B, S, H, D] fp32 and lse_acc [B, H, S] fp32: the running result, read and written in
 *   place (start it with lse_acc = -inf; o_acc may then hold anything).
 *   o_part [B, S, H, D] bf16 and lse_part [B, H, S] fp32: a partial result as attn_fwd writes it.
 *   o_out [B, S, H, D] bf16: if not NULL, also receives the merged O rounded to bf16.
 *   D is 64 or 128; all pointers 16-byte aligned.
 * ------------------------------------------------------------------------------------------ */
attn_status_t attn_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                         void* o_out, int B, int S, int H, int D, attn_stream_t stream);

/* ------------------------------------------------------------------------------------------ *
 * Status and introspection.
 * ------------------------------------------------------------------------------------------ */

/* Human-readable name of a status code (static string, never NULL). */
const char* attn_status_string(attn_status_t status);

/* Waits for `stream`, then reads and clears the library's device status word on the current
 * device: ATTN_OK, ATTN_ERR_TIMEOUT if a kernel gave up a bounded wait since the last read, or
 * ATTN_ERR_INVALID_ARG if attn_decode_paged met a page id outside its pool. */
attn_status_t attn_get_device_status(attn_stream_t stream);

/* Number of CUDA kernels this library has launched in this process (all devices, all calls). */
uint64_t attn_launch_count(void);

/* Opt-in per-kernel timing (for benchmarks). Between attn_profile_start() and attn_profile_stop()
 * every kernel this library launches is bracketed by two CUDA events recorded on its launch stream
 * (events are created on first use and reused; no device memory is allocated). attn_profile_stop()
 * waits for the recorded events and sums the elapsed time per kernel family; the sums are then read
 * with attn_profile_entries / _name / _total_ms / _launches (index 0 .. entries-1). Not for use
 * while a stream is being captured into a CUDA graph. */
attn_status_t attn_profile_start(void);
attn_status_t attn_profile_stop(void);
int attn_profile_entries(void);
const char* attn_profile_name(int i);
double attn_profile_total_ms(int i);
int attn_profile_launches(int i);

/* Name of the kernel family the last successful call of each kind dispatched to on this thread,
 * e.g. "fwd_sm100_tcgen05" (static string). kind: 0 = forward, 1 = backward, 2 = decode. */
const char* attn_last_path(int kind);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* ATTN_H_ */
