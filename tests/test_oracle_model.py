"""Whole-model pins for the oracle: identities the looped method must satisfy.

* looped == unrolled: running the shared block twice equals a plain model
  whose block weights (and mHC parameters) are duplicated;
* causality: a prefix's logits do not depend on later tokens;
* cache bookkeeping: prefill(S) then decode steps equals prefill(S + k);
* each pass keeps its own KV cache and linear-attention state.
"""

import numpy as np
import pytest

import oracle
import seeded
from seeded import workloads as W

W_PER_LAYER = 10


def tiny(**kw):
    base = dict(W.model_config("tiny_fp32"), max_batch=2, max_ctx=40)
    base.update(kw)
    return oracle.make_config(**base)


def _unrolled_weights(looped: oracle.Model, c: oracle.Config):
    """Weights of an unrolled model: prelude, block, block again, coda."""
    w = [looped.weight(i) for i in range(looped.num_weights())]
    n_phys = c.n_prelude + c.n_block + c.n_coda
    layer = lambda p: w[2 + W_PER_LAYER * p: 2 + W_PER_LAYER * (p + 1)]
    sites = w[2 + W_PER_LAYER * n_phys:]
    order = list(range(c.n_prelude)) + [c.n_prelude + j for j in range(c.n_block)] * c.n_loops + \
        [c.n_prelude + c.n_block + j for j in range(c.n_coda)]
    out = w[:2]
    for p in order:
        out += layer(p)
    return out + sites * c.n_loops


def test_looped_equals_unrolled_bit_exact():
    c = tiny()
    m = oracle.Model(c, seed=0)
    cu = tiny(n_block=c.n_block * c.n_loops, n_loops=1)
    mu = oracle.Model(cu, seed=0, weights=_unrolled_weights(m, c))
    tok = seeded.tokens(0, 2, 24, c.vocab)
    a = m.prefill(tok, all_positions=True)
    b = mu.prefill(tok, all_positions=True)
    np.testing.assert_array_equal(a, b)
    # same per-execution caches too
    for slot in range(4):
        ka, va = m.kv(slot, 2, 24)
        kb, vb = mu.kv(slot, 2, 24)
        np.testing.assert_array_equal(ka, kb)
        np.testing.assert_array_equal(va, vb)
    for slot in range(12):
        np.testing.assert_array_equal(m.state(slot, 2), mu.state(slot, 2))
    # and one decode step later
    nxt = seeded.tokens(0, 2, 1, c.vocab, stream=seeded.S_DECODE_TOKENS)
    np.testing.assert_array_equal(m.decode_step(nxt), mu.decode_step(nxt))


def test_loop_count_matters():
    c1 = tiny(n_loops=1)
    c2 = tiny()
    tok = seeded.tokens(0, 1, 16, c2.vocab)
    a = oracle.Model(c1, seed=0).prefill(tok)
    b = oracle.Model(c2, seed=0).prefill(tok)
    assert np.abs(a - b).max() > 1e-3


def test_causal_prefix():
    c = tiny()
    m = oracle.Model(c, seed=0)
    tok = seeded.tokens(1, 2, 30, c.vocab)
    full = m.prefill(tok, all_positions=True)
    pre = m.prefill(tok[:, :11], all_positions=True)
    np.testing.assert_array_equal(full[:, :11], pre)
    np.testing.assert_array_equal(m.prefill(tok[:, :11])[:, None, :], full[:, 10:11])


def test_prefill_then_decode_equals_longer_prefill():
    c = tiny()
    m = oracle.Model(c, seed=0)
    tok = seeded.tokens(2, 2, 20, c.vocab)
    ref = m.prefill(tok, all_positions=True)
    ref_states = [m.state(s, 2) for s in range(12)]
    ref_kv = [m.kv(s, 2, 20) for s in range(4)]
    m.prefill(tok[:, :15])
    assert m.seq_len(0) == 15 and m.seq_len(1) == 15
    for t in range(15, 20):
        got = m.decode_step(tok[:, t])
        np.testing.assert_array_equal(got, ref[:, t])
    assert m.seq_len(0) == 20
    for s in range(12):
        np.testing.assert_array_equal(m.state(s, 2), ref_states[s])
    for s in range(4):
        k, v = m.kv(s, 2, 20)
        np.testing.assert_array_equal(k, ref_kv[s][0])
        np.testing.assert_array_equal(v, ref_kv[s][1])


def test_passes_keep_separate_caches():
    c = tiny()
    m = oracle.Model(c, seed=0)
    m.prefill(seeded.tokens(3, 1, 12, c.vocab))
    t = oracle.schedule(c)
    # layer 7 (full attention) runs in both passes: its two executions own
    # different KV slots, and pass 2 sees different inputs, so the caches differ
    e1, e2 = [e for e in range(len(t)) if t[e, 0] == 7]
    k1, _ = m.kv(int(t[e1, 3]), 1, 12)
    k2, _ = m.kv(int(t[e2, 3]), 1, 12)
    assert t[e1, 3] != t[e2, 3] and np.abs(k1 - k2).max() > 1e-3
    e1, e2 = [e for e in range(len(t)) if t[e, 0] == 5]
    assert t[e1, 3] != t[e2, 3]
    assert np.abs(m.state(int(t[e1, 3]), 1) - m.state(int(t[e2, 3]), 1)).max() > 1e-4


def test_prefill_resets_sequences():
    c = tiny()
    m = oracle.Model(c, seed=0)
    tok = seeded.tokens(4, 1, 10, c.vocab)
    a = m.prefill(tok)
    m.decode_step(np.array([5]))
    b = m.prefill(tok)
    np.testing.assert_array_equal(a, b)


def test_bf16_mode_rounds_weights_and_stays_close():
    cb = tiny(dtype=1)
    cf = tiny()
    mb, mf = oracle.Model(cb, seed=0), oracle.Model(cf, seed=0)
    w = mb.weight(2 + 1)  # layer 0 W_q
    np.testing.assert_array_equal(w, seeded.to_bf16_f32(w))
    np.testing.assert_array_equal(w, seeded.weights(0, seeded.layer_stream(0, seeded.K_WQ), w.size, True))
    tok = seeded.tokens(5, 1, 16, cf.vocab)
    a, b = mf.prefill(tok), mb.prefill(tok)
    cos = float((a * b).sum() / np.linalg.norm(a) / np.linalg.norm(b))
    assert cos > 0.99


def test_hidden_mode_group():
    c = oracle.make_config(**W.model_config("group9b_s4096", hidden=64, ffn=96, n_q=4, n_kv=2, head_dim=16,
                                             n_lin=4, lin_dim=16), max_batch=1, max_ctx=16)
    m = oracle.Model(c, seed=1)
    h = seeded.hidden(1, 1, 9, 64)
    out = m.prefill(hidden=h)
    assert out.shape == (1, 9, 64) and np.isfinite(out).all()
    # with zero projections everywhere the block is the identity on each stream,
    # so the collapsed output is s_0 + s_1 = 2 h
    ws = [m.weight(i) for i in range(m.num_weights())]
    zero = [np.zeros_like(x) if (i >= 2 and (i - 2) % 10 in (5, 9)) else x for i, x in enumerate(ws)]
    mz = oracle.Model(c, seed=1, weights=zero)
    np.testing.assert_allclose(mz.prefill(hidden=h), 2 * h, rtol=1e-6, atol=1e-6)
