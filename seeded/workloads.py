"""The five synthetic workloads, as plain numbers (no arithmetic of the method).

Each entry gives the model's execution configuration (loop range, pass count,
mHC settings, shapes) plus the batch/sequence and seed of the run.  The CUDA
library and the oracle each turn these numbers into their own config struct.
"""

from __future__ import annotations

import copy

_TINY = dict(
    n_prelude=4, n_block=4, n_loops=2, n_coda=4, group=4, full_slot=3,
    hidden=256, ffn=768, vocab=1024, n_q=4, n_kv=2, head_dim=64,
    n_lin=4, lin_dim=64, lin_chunk=64, n_streams=2, sinkhorn_iters=20,
    rope_base=1.0e4, norm_eps=1.0e-6, dtype=0, io_mode=0,
)

_LOOP9B = dict(
    n_prelude=4, n_block=24, n_loops=2, n_coda=4, group=4, full_slot=3,
    hidden=4096, ffn=12288, vocab=248320, n_q=32, n_kv=8, head_dim=128,
    n_lin=32, lin_dim=128, lin_chunk=64, n_streams=2, sinkhorn_iters=20,
    rope_base=1.0e4, norm_eps=1.0e-6, dtype=1, io_mode=0,
)

_GROUP9B = dict(_LOOP9B, n_prelude=0, n_block=4, n_coda=0, vocab=0, io_mode=1)

WORKLOADS = {
    # tiny looped decoder, fp32: 12 stored layers, 16 executions
    "tiny_fp32": dict(model=_TINY, batch=1, seq=128, seed=0),
    # one 4-layer group at 9B width run twice, hidden in -> hidden out, bf16
    "group9b_s4096": dict(model=_GROUP9B, batch=1, seq=4096, seed=1),
    # the 9B-shaped looped decoder, prefill 4 x 8192
    "loop9b_prefill_b4_s8192": dict(model=_LOOP9B, batch=4, seq=8192, seed=2),
    # the 9B-shaped looped decoder, 64 sequences decoding after 32,768 tokens
    "loop9b_decode_b64_ctx32768": dict(model=_LOOP9B, batch=64, seq=32768, seed=3, decode_steps=128),
    # the 9B-shaped looped decoder, one 262,144-token prefill
    "loop9b_prefill_b1_s262144": dict(model=_LOOP9B, batch=1, seq=262144, seed=4),
    # small probes for kernel captures (9B kernel shapes, a few GB on the device)
    "probe_decode_b64_ctx4096": dict(model=dict(_GROUP9B, vocab=4096, io_mode=0), batch=64, seq=4096, seed=3,
                                     decode_steps=16),
}


def model_config(name: str, **override) -> dict:
    """The model fields of a workload, with overrides (e.g. a smaller max_ctx)."""
    m = copy.deepcopy(WORKLOADS[name]["model"])
    m.update(override)
    return m
