/*
 * attn_fault_inject.h -- test-only entry point of libattn_faultinject.so.
 *
 * libattn_faultinject.so is the library built a second time with ATTN_FAULT_INJECT, for the tests
 * of the kernels' timeout path only; the shipped libattn.so does not export this symbol. In that
 * build every bounded on-chip wait gives up after 20 ms instead of 2 s, and the call below makes
 * the producer warp of CTA 0 of one kernel family skip one copy, so that a consumer's wait for it
 * runs out. The kernel then records ATTN_ERR_TIMEOUT in the device status word, lets its own copies
 * and tensor-core operations land, frees its tensor memory and returns; nothing traps, spins
 * unbounded or touches memory out of bounds, and the context stays usable.
 *
 *   family: 0 = attn_fwd's kernel (skips K block number `block` of CTA 0's ring),
 *           1 = attn_bwd's main kernel (skips Q/dO tile number `block` of CTA 0),
 *           2 = the split-KV decode's split kernel (skips ring block number `block` of CTA 0);
 *           -1 (or a negative block) switches injection off.
 * The setting is process-wide host state, read when each later call builds its kernel arguments.
 */
#ifndef ATTN_FAULT_INJECT_H_
#define ATTN_FAULT_INJECT_H_

#ifdef __cplusplus
extern "C" {
#endif

void attn_fault_inject(int family, int block);

#ifdef __cplusplus
}
#endif

#endif  /* ATTN_FAULT_INJECT_H_ */
