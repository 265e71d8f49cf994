"""Online-softmax attention for NVIDIA B200 (sm_100a): a C-ABI library (libattn.so) and its binding.

Scaled-dot-product attention computed as one reduction under the online-softmax monoid, the form
"Não escreva kernels, derive-os" ("Aprofundamento", first paragraph) derives flash attention from:

* ``fwd`` -- bf16 prefill forward (tcgen05 tensor cores, TMA, TMEM), GQA, causal, lse output;
* ``bwd`` -- bf16 backward to dQ, dK, dV;
* ``decode`` -- split-KV decode over packed varlen caches, partial (m, l, o) triples merged by the
  monoid in a combine kernel; ``decode_paged`` -- the same over a paged cache (block table);
* ``fwd_f32`` / ``bwd_f32`` -- genuine fp32 CUDA-core versions;
* ``fwd_fp8`` -- e4m3 inputs with per-tensor scales (kind::f8f6f4 tensor cores);
* ``fwd_varlen`` / ``bwd_varlen`` -- packed sequences of different lengths (cu_seqlens);
* ``merge`` -- the monoid merge of partial (O, lse) results; ``ring`` -- a context-parallel ring
  forward across ranks built on it.

The C entry points are declared in ``include/attn.h``; this package only marshals torch tensors to
them (see ``_binding.py``). ``workloads`` draws the seeded synthetic inputs.
"""
from ._binding import (  # noqa: F401
    AttnError,
    LIB_PATH,
    SIGNATURES,
    bwd,
    bwd_f32,
    bwd_varlen,
    bwd_workspace_size,
    decode,
    decode_paged,
    decode_workspace_size,
    default_splits,
    device_status,
    fwd,
    fwd_f32,
    fwd_fp8,
    fwd_varlen,
    last_path,
    launch_count,
    lib,
    merge,
    profile_start,
    profile_stop,
    status_string,
)
