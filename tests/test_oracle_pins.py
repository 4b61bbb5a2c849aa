"""Pins for the CPU oracle: checks against facts the pages state and against
mathematics that does not depend on the oracle's own code (closed forms,
invariants, special cases, brute force on tiny inputs)."""

import json
import math
import os

import numpy as np
import pytest

import oracle
import seeded
from seeded import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------- generator

def test_splitmix64_published_vector():
    g = load("splitmix64.json")
    assert seeded.splitmix64_sequence(g["state"], 5) == g["outputs"]


def test_counter_stream_is_splitmix64_from_key():
    # u64(seed, stream, j) is the SplitMix64 sequence started at key(seed, stream).
    key = seeded.stream_key(5, 1234)
    seq = seeded.splitmix64_sequence(key, 8)
    assert [int(x) for x in seeded.u64(5, 1234, 0, 8)] == seq
    assert [oracle.rng_u64(5, 1234, j) for j in range(8)] == seq


def test_oracle_generator_matches_seeded_module():
    for stream in (1, 1001, 100011):
        ref = seeded.u64(2, stream, 1000, 64)
        got = [oracle.rng_u64(2, stream, 1000 + j) for j in range(64)]
        assert [int(x) for x in ref] == got
        zn = seeded.normal(2, stream, 999, 33)
        got_n = np.array([oracle.rng_normal(2, stream, 999 + j) for j in range(33)])
        np.testing.assert_allclose(got_n, zn, rtol=0, atol=1e-13)


def test_normal_moments_and_tokens():
    z = seeded.normal(0, 77, 0, 200000)
    assert abs(z.mean()) < 0.01 and abs(z.var() - 1) < 0.01
    assert abs((z**4).mean() - 3) < 0.05  # Gaussian kurtosis
    t = seeded.tokens(3, 4, 1000, 248320)
    assert t.min() >= 0 and t.max() < 248320 and t.dtype == np.int32


def test_bf16_rounding_ties_to_even():
    x = np.array([1.0 + 2**-8, 1.0 + 3 * 2**-8, 1.0 + 2**-9, -2.5], dtype=np.float32)
    np.testing.assert_array_equal(seeded.to_bf16_f32(x), np.array([1.0, 1.0 + 4 * 2**-8, 1.0, -2.5], np.float32))


# --------------------------------------------------------------------------- exp and Sinkhorn

def test_exp_spec_accuracy():
    xs = np.concatenate([np.linspace(-87, 0, 20001), np.linspace(-5, 5, 2001)]).astype(np.float32)
    got = np.array([oracle.exp_spec(float(x)) for x in xs], dtype=np.float32)
    ref = np.exp(xs.astype(np.float64))
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    assert np.max(np.abs(got - ref) / ulp) <= 2.0
    assert oracle.exp_spec(0.0) == 1.0
    assert np.all(np.diff(got[:20001]) >= 0)  # monotone on the sweep
    assert oracle.exp_spec(-105.0) == 0.0 and oracle.exp_spec(89.0) == math.inf


def _cross_delta(l):
    return l[..., 0, 0] + l[..., 1, 1] - l[..., 0, 1] - l[..., 1, 0]


def test_sinkhorn_2x2_closed_form():
    # The 2x2 limit is [[a, 1-a], [1-a, a]] with a = sigmoid(Delta / 2): row and
    # column scaling keep the cross ratio P00 P11 / (P01 P10) = exp(Delta).
    rng = np.random.default_rng(0)
    l = rng.normal(0, 2.0, size=(4000, 2, 2))
    d = _cross_delta(l)
    a = 1 / (1 + np.exp(-d / 2))
    limit = np.stack([np.stack([a, 1 - a], -1), np.stack([1 - a, a], -1)], -2)
    near = np.abs(d) <= 10  # tanh(10/4)^4000 < 1e-23: iterated to the limit
    P = oracle.sinkhorn_f64(l[near], iters=2000)
    np.testing.assert_allclose(P, limit[near], atol=1e-12)
    # after 20 iterations the error is bounded by the contraction tanh(|Delta|/4)^40
    P20 = oracle.sinkhorn_f64(l, iters=20)
    bound = np.tanh(np.abs(d) / 4) ** 40
    err = np.abs(P20 - limit).max(axis=(1, 2))
    assert np.all(err <= 2 * bound + 1e-14)


def test_sinkhorn_doubly_stochastic_and_special_cases():
    rng = np.random.default_rng(1)
    l = rng.normal(0, 0.45, size=(20000, 2, 2))
    P = oracle.sinkhorn_f32(l.astype(np.float32), 20).astype(np.float64)
    # ends on a column normalisation: columns sum to 1 to rounding
    assert np.abs(P.sum(axis=1) - 1).max() < 4 * 2**-24
    # rows reach 1e-6 where the cross ratio is moderate
    ok = np.abs(_cross_delta(l)) <= 3.5
    assert np.abs(P.sum(axis=2) - 1)[ok].max() < 1e-6
    # constant logits: 1/n after one iteration; n = 1 gives 1
    for n in (1, 2, 3, 4):
        c = np.full((1, n, n), 0.7)
        np.testing.assert_allclose(oracle.sinkhorn_f64(c, 1), np.full((1, n, n), 1.0 / n), atol=1e-15)
    # zero iterations: exp(l - max l)
    P0 = oracle.sinkhorn_f64(l[:5], 0)
    np.testing.assert_allclose(P0, np.exp(l[:5] - l[:5].max(axis=(1, 2), keepdims=True)), rtol=1e-15)


def test_sinkhorn_3x3_is_diagonal_scaling():
    # the limit is diag(u) exp(l) diag(v): every 2x2 cross ratio of exp(l) is kept
    rng = np.random.default_rng(2)
    l = rng.normal(0, 1.0, size=(50, 3, 3))
    P = oracle.sinkhorn_f64(l, 2000)
    np.testing.assert_allclose(P.sum(axis=1), 1, atol=1e-12)
    np.testing.assert_allclose(P.sum(axis=2), 1, atol=1e-12)
    for (i, j, k, m) in [(0, 1, 0, 1), (0, 2, 1, 2), (1, 2, 0, 2)]:
        lhs = np.log(P[:, i, k] * P[:, j, m] / (P[:, i, m] * P[:, j, k]))
        rhs = l[:, i, k] + l[:, j, m] - l[:, i, m] - l[:, j, k]
        np.testing.assert_allclose(lhs, rhs, atol=1e-9)


def test_sinkhorn_f32_tracks_f64():
    rng = np.random.default_rng(3)
    l = rng.normal(0, 1.81, size=(5000, 2, 2))
    a = oracle.sinkhorn_f32(l.astype(np.float32), 20)
    b = oracle.sinkhorn_f64(l.astype(np.float32).astype(np.float64), 20)
    assert np.abs(a - b).max() < 2e-6


# --------------------------------------------------------------------------- schedule

def _cfg(name, **kw):
    return oracle.make_config(**W.model_config(name, **kw), max_batch=1, max_ctx=8)


def test_schedule_matches_page_facts():
    f = load("page_facts.json")
    t = oracle.schedule(_cfg("loop9b_prefill_b4_s8192"))
    assert len(t) == f["executions_per_forward"]["value"] == sum(f["executions_per_forward"]["terms"])
    phys = list(t[:, 0])
    pre = f["prelude_layers"]["value"]
    b0, b1 = f["block_layers"]["value"]
    c0, c1 = f["coda_layers"]["value"]
    blk = list(range(b0, b1 + 1))
    assert phys == pre + blk + blk + list(range(c0, c1 + 1))
    assert len(set(phys)) == f["n_physical_layers"]["value"]
    # B(B(h)): pass index 0 for the first block run, 1 for the second
    assert list(t[4:28, 1]) == [0] * 24 and list(t[28:52, 1]) == [1] * 24
    assert list(t[:, 4]) == [0] * 4 + [1] * 48 + [2] * 4
    pat = f["group_pattern"]["value"]
    kinds = ["full" if k == oracle.FULL else "linear" for k in t[:, 2]]
    assert all(kinds[e] == pat[phys[e] % 4] for e in range(56))
    assert kinds[4:28] == kinds[28:52]  # both passes see the same pattern
    assert (len(blk) // 4) == f["block_groups"]["value"] and b0 % 4 == 0
    full = t[t[:, 2] == oracle.FULL]
    lin = t[t[:, 2] == oracle.LINEAR]
    assert len(full) == 14 and len(lin) == 42
    # every execution owns its own cache slot: the two passes never share one
    assert sorted(full[:, 3]) == list(range(14)) and sorted(lin[:, 3]) == list(range(42))


def test_schedule_other_workloads_and_rejections():
    t = oracle.schedule(_cfg("tiny_fp32"))
    assert len(t) == 16 and (t[:, 2] == oracle.FULL).sum() == 4
    t = oracle.schedule(_cfg("group9b_s4096"))
    assert len(t) == 8 and (t[:, 2] == oracle.FULL).sum() == 2 and list(t[:, 0]) == [0, 1, 2, 3] * 2
    # a block that does not start or end on a group boundary is rejected
    with pytest.raises(ValueError):
        oracle.schedule(_cfg("tiny_fp32", n_block=5))
    with pytest.raises(ValueError):
        oracle.schedule(_cfg("tiny_fp32", n_prelude=2))
    # more passes: K x 24 executions in the block
    t = oracle.schedule(_cfg("loop9b_prefill_b4_s8192", n_loops=3))
    assert len(t) == 4 + 3 * 24 + 4


# --------------------------------------------------------------------------- small operators

def test_rmsnorm_hand_case():
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    y = oracle.rmsnorm(x, np.array([1.0, 1.0, 2.0, 0.5]), 0.0)
    r = math.sqrt((1 + 4 + 9 + 16) / 4)
    np.testing.assert_allclose(y, [[1 / r, 2 / r, 6 / r, 2 / r]], rtol=1e-15)


def _gla_quadratic(q, k, v, g):
    T = len(q)
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        for s in range(t + 1):
            o[t] += np.prod(g[s + 1:t + 1]) * (q[t] @ k[s]) * v[s]
    return o


def _gla_chunked(q, k, v, g, C):
    T, dk = q.shape
    S = np.zeros((dk, v.shape[1]))
    o = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        b = np.cumsum(np.log(g[c0:c1]))
        qc, kc, vc = q[c0:c1], k[c0:c1], v[c0:c1]
        D = np.tril(np.exp(b[:, None] - b[None, :]))
        o[c0:c1] = ((qc @ kc.T) * D) @ vc + (qc * np.exp(b)[:, None]) @ S
        S = np.exp(b[-1]) * S + (kc * np.exp(b[-1] - b)[:, None]).T @ vc
    return o, S


def test_gla_recurrent_equals_quadratic_and_chunked():
    rng = np.random.default_rng(4)
    T, dk, dv = 13, 6, 5
    q, k = rng.normal(size=(T, dk)), rng.normal(size=(T, dk))
    v = rng.normal(size=(T, dv))
    g = rng.uniform(0.3, 1.0, size=T)
    o, S = oracle.gla_recurrent(q, k, v, g)
    np.testing.assert_allclose(o, _gla_quadratic(q, k, v, g), atol=1e-12)
    for C in (1, 3, 4, T):
        oc, Sc = _gla_chunked(q, k, v, g, C)
        np.testing.assert_allclose(o, oc, atol=1e-12)
        np.testing.assert_allclose(S, Sc, atol=1e-12)
    # g = 1: plain causal linear attention sum_{s<=t} (q_t . k_s) v_s
    o1, _ = oracle.gla_recurrent(q, k, v, np.ones(T))
    np.testing.assert_allclose(o1, np.tril(q @ k.T) @ v, atol=1e-12)
    # keys orthogonal to every query: zero output
    qz = np.zeros((T, dk)); qz[:, 0] = 1.0
    kz = rng.normal(size=(T, dk)); kz[:, 0] = 0.0
    oz, _ = oracle.gla_recurrent(qz, kz, v, g)
    assert np.abs(oz).max() == 0.0
    # a carried-in state decays by the product of gates
    S0 = rng.normal(size=(dk, dv))
    oS, _ = oracle.gla_recurrent(q, np.zeros((T, dk)), v, g, state=S0)
    np.testing.assert_allclose(oS, np.cumprod(g)[:, None] * (q @ S0), atol=1e-12)


def _attention_online(q, k, v, q0, block):
    d = q.shape[1]
    out = np.zeros((len(q), v.shape[1]))
    for i in range(len(q)):
        last = q0 + i
        m, l, acc = -np.inf, 0.0, np.zeros(v.shape[1])
        for j0 in range(0, last + 1, block):
            j1 = min(last + 1, j0 + block)
            s = k[j0:j1] @ q[i] / math.sqrt(d)
            mn = max(m, s.max())
            p = np.exp(s - mn)
            acc = acc * math.exp(m - mn) + p @ v[j0:j1]
            l = l * math.exp(m - mn) + p.sum()
            m = mn
        out[i] = acc / l
    return out


def test_attention_naive_equals_online_softmax():
    rng = np.random.default_rng(5)
    Tk, d = 37, 8
    k, v = rng.normal(size=(Tk, d)) * 2, rng.normal(size=(Tk, d))
    q = rng.normal(size=(10, d)) * 2
    o = oracle.attention_naive(q, k, v, q0=27)
    np.testing.assert_allclose(o, _attention_online(q, k, v, 27, 5), atol=1e-12)
    # one key: the output is that value; zero queries: prefix means of V
    np.testing.assert_allclose(oracle.attention_naive(q[:1], k[:1], v[:1], 0), v[:1], atol=1e-15)
    o0 = oracle.attention_naive(np.zeros((Tk, d)), k, v, 0)
    np.testing.assert_allclose(o0, np.cumsum(v, axis=0) / np.arange(1, Tk + 1)[:, None], atol=1e-12)


def test_rope_properties():
    rng = np.random.default_rng(6)
    d, base = 16, 1e4
    x = rng.normal(size=(5, 2, d))
    pos = np.array([0, 1, 7, 1000, 262143])
    y = oracle.rope(x, pos, base)
    np.testing.assert_array_equal(y[0], x[0])  # position 0 is the identity
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    # as complex numbers z_i = x_i + i x_{i+d/2} rotated by e^{i pos base^(-2i/d)}
    th = pos[:, None] * base ** (-2.0 * np.arange(d // 2) / d)
    z = (x[..., : d // 2] + 1j * x[..., d // 2:]) * np.exp(1j * th)[:, None, :]
    np.testing.assert_allclose(y, np.concatenate([z.real, z.imag], -1), atol=1e-12)
    # q . k depends only on the position difference
    q, k = rng.normal(size=(1, 1, d)), rng.normal(size=(1, 1, d))
    dots = [float((oracle.rope(q, np.array([p + 5]), base) * oracle.rope(k, np.array([p]), base)).sum())
            for p in (0, 10, 12345)]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-9)


# --------------------------------------------------------------------------- mHC site

def test_mhc_write_reduces_to_residual_add():
    rng = np.random.default_rng(7)
    s = rng.normal(size=(2, 9))
    y = rng.normal(size=9)
    coef = np.array([1.0, 0.0, 1.0, 0.0, 1.0, 0.0, 0.0, 1.0])  # pre, post, res = identity
    out = oracle.mhc_write(s, coef, y)
    np.testing.assert_array_equal(out[0], s[0] + y)
    np.testing.assert_array_equal(out[1], s[1])


def test_mhc_write_conserves_stream_sum():
    rng = np.random.default_rng(8)
    s = rng.normal(size=(2, 11))
    y = rng.normal(size=11)
    l = rng.normal(0, 3, size=(1, 2, 2))
    res = oracle.sinkhorn_f64(l, 20)[0]  # columns sum to 1
    post = np.array([0.3, 1.7])
    out = oracle.mhc_write(s, np.concatenate([[0.5, 0.5], post, res.ravel()]), y)
    np.testing.assert_allclose(out.sum(0) - s.sum(0), post.sum() * y, atol=1e-12)
    # mixing index order: stream i gets sum_j res[i, j] s_j
    np.testing.assert_allclose(out[0], res[0, 0] * s[0] + res[0, 1] * s[1] + post[0] * y, atol=1e-14)


def test_mhc_site_coefficients():
    rng = np.random.default_rng(9)
    n, H = 2, 6
    s = rng.normal(size=(n, H))
    gm = rng.uniform(0.5, 1.5, size=n * H)
    gain = rng.uniform(0.5, 1.5, size=H)
    u = s.ravel() / math.sqrt((s**2).mean() + 1e-6) * gm
    # zero projection: H_pre = 1/2, H_post = 1, H_res = 1/2 everywhere
    coef, xh = oracle.mhc_site(s, gm, np.zeros((8, n * H)), gain)
    np.testing.assert_allclose(coef, [0.5, 0.5, 1, 1, 0.5, 0.5, 0.5, 0.5], atol=1e-15)
    x = 0.5 * (s[0] + s[1])
    np.testing.assert_allclose(xh, x / math.sqrt((x**2).mean() + 1e-6) * gain, rtol=1e-13)
    # one-hot rows of Phi pick single normalised stream entries, in the order
    # pre0, pre1, post0, post1, res00, res01, res10, res11
    phi = np.zeros((8, n * H))
    picks = [3, 8, 1, 10, 0, 0, 0, 0]
    for c in range(4):
        phi[c, picks[c]] = 1.0
    phi[4, 2] = 1.0  # res00 logit = u[2], other res logits 0
    coef, _ = oracle.mhc_site(s, gm, phi, gain)
    sig = lambda t: 1 / (1 + math.exp(-t))
    np.testing.assert_allclose(coef[:4], [sig(u[3]), sig(u[8]), 2 * sig(u[1]), 2 * sig(u[10])], rtol=1e-13)
    np.testing.assert_allclose(coef[4:].reshape(1, 2, 2),
                               oracle.sinkhorn_f64(np.array([[[u[2], 0.0], [0.0, 0.0]]]), 20), rtol=1e-13)


# --------------------------------------------------------------------------- the model's sublayers
#
# The model calls these same oracle functions with its own weights and cache
# slots, so each hand-computed case below pins the in-model arithmetic.

# Values of the logistic function sigma(x) = 1 / (1 + e^-x), to double precision.
SIG_1 = 0.7310585786300049
SIG_2 = 0.8807970779778823


def _sub_cfg(**kw):
    base = dict(n_prelude=0, n_block=4, n_loops=1, n_coda=0, group=4, full_slot=3, hidden=2, ffn=2, vocab=8,
                n_q=1, n_kv=1, head_dim=2, n_lin=1, lin_dim=2, lin_chunk=64, n_streams=2, sinkhorn_iters=20,
                rope_base=10000.0, norm_eps=1e-6, dtype=0, io_mode=0, max_batch=1, max_ctx=8)
    base.update(kw)
    return oracle.make_config(**base)


def test_ffn_sublayer_hand_case():
    # SwiGLU, y = W_down (silu(x W_gate) * (x W_up)), on x = (1, 2):
    #   gate = (1, 2), up = (2, 1), silu(z) = z sigma(z)
    #   a = (1 sigma(1) 2, 2 sigma(2) 1) = (2 sigma(1), 2 sigma(2))
    #   W_down = [[1, 10], [100, 1000]] -> y = (a0 + 10 a1, 100 a0 + 1000 a1)
    # Swapping gate and up (or applying silu to up) gives a = (2 sigma(2), 2 sigma(1));
    # a transposed W_down gives y0 = a0 + 100 a1.
    cfg = _sub_cfg(hidden=2, ffn=2)
    a0, a1 = 2 * SIG_1, 2 * SIG_2
    y = oracle.ffn_sublayer(cfg, np.eye(2), np.array([[0.0, 1.0], [1.0, 0.0]]),
                            np.array([[1.0, 10.0], [100.0, 1000.0]]), np.array([[1.0, 2.0]]))
    np.testing.assert_allclose(y, [[a0 + 10 * a1, 100 * a0 + 1000 * a1]], rtol=1e-14)


def test_attention_sublayer_gqa_head_map():
    # 8 query heads over 2 kv heads (group 4, as in the 9B shape), head_dim 2,
    # hidden 4.  W_q = W_k = 0 makes every score 0, so each head averages the
    # values of its kv head over the causal prefix; W_v = I gives kv head 0 the
    # values (x0, x1) and kv head 1 the values (x2, x3).  W_o reads head 1's
    # output into y0, y1, head 4's first component into y2 and head 7's second
    # into y3.  With kv head = q head / 4, heads 1 -> kv 0 and heads 4, 7 -> kv 1;
    # the map q head % 2 would send head 1 to kv 1 and head 4 to kv 0.
    cfg = _sub_cfg(hidden=4, n_q=8, n_kv=2, head_dim=2, max_ctx=4)
    wo = np.zeros((4, 16))
    wo[0, 2], wo[1, 3], wo[2, 8], wo[3, 15] = 1, 1, 1, 1
    w = (np.zeros((16, 4)), np.zeros((4, 4)), np.eye(4), wo)
    x = np.array([[[1.0, 2.0, 3.0, 4.0], [5.0, 6.0, 7.0, 8.0]]])
    y, kc, vc = oracle.attention_sublayer(cfg, *w, x, [0])
    # t = 0: the one value; t = 1: the mean of two
    np.testing.assert_allclose(y[0], [[1, 2, 3, 4], [3, 4, 5, 6]], atol=1e-14)
    np.testing.assert_array_equal(vc[0, :, :2], [[[1, 2], [5, 6]], [[3, 4], [7, 8]]])
    assert not kc.any()
    # one more token continuing at position 2 against the cache: mean of three
    y2, kc, vc = oracle.attention_sublayer(cfg, *w, np.array([[[9.0, 10.0, 11.0, 12.0]]]), [2], kc, vc)
    np.testing.assert_allclose(y2[0], [[5, 6, 7, 8]], atol=1e-14)
    np.testing.assert_array_equal(vc[0, :, 2], [[9, 10], [11, 12]])


def test_attention_sublayer_scale_and_rope():
    # One head, head_dim 2, hidden 4.  Token 0: x = (0, 0, 1, 0); token 1:
    # x = (c, 1, 0, 0) with c = sqrt(2) ln 3.  W_q takes x0 into q's first
    # component, W_k takes x1 into k's first, W_v maps x -> (x2, x1):
    #   q(1) = (c, 0), k(0) = (0, 0), k(1) = (1, 0), v(0) = (1, 0), v(1) = (0, 1).
    # RoPE rotates q(1) and k(1) by the same angle (both at position 1), which
    # leaves q(1) . k(1) = c; k(0) = 0.  With the scale 1/sqrt(2) the scores of
    # query 1 are (0, ln 3), so its weights are (1/4, 3/4) and o(1) = (1/4, 3/4).
    # Without the scale the weights would be (1 + 3^sqrt2)^-1 (1, 3^sqrt2).
    cfg = _sub_cfg(hidden=4, n_q=1, n_kv=1, head_dim=2, max_ctx=2)
    c = math.sqrt(2.0) * math.log(3.0)
    wq = np.array([[1.0, 0, 0, 0], [0, 0, 0, 0]])
    wk = np.array([[0, 1.0, 0, 0], [0, 0, 0, 0]])
    wv = np.array([[0, 0, 1.0, 0], [0, 1.0, 0, 0]])
    wo = np.array([[1.0, 0], [0, 1.0], [0, 0], [0, 0]])
    x = np.array([[[0, 0, 1.0, 0], [c, 1.0, 0, 0]]])
    y, kc, _ = oracle.attention_sublayer(cfg, wq, wk, wv, wo, x, [0])
    np.testing.assert_allclose(y[0], [[1, 0, 0, 0], [0.25, 0.75, 0, 0]], atol=1e-13)
    # the cached key of position 1 is k(1) rotated by 1 radian (frequency base^0 = 1)
    np.testing.assert_allclose(kc[0, 0, 1], [math.cos(1.0), math.sin(1.0)], atol=1e-7)


# eps = 2^-20 and entries scaled by 2^-10 make every L2 norm exact:
# |u|^2 = 3 eps gives sqrt(|u|^2 + eps) = 2^-9, |u|^2 = 8 eps gives 3 * 2^-10.
_EPS = 2.0**-20
_U = 2.0**-10


def test_gla_sublayer_hand_case():
    # One head, d = 2, hidden 7: x = (q0, q1, k0, k1, v0, v1, z) with identity
    # projections and the gate z.  q and k are L2-normalised with eps inside
    # the square root, g = sigmoid(z), S_t = g_t S_{t-1} + k_t v_t^T, o_t = q_t S_t.
    #   token 0: q = (sqrt3 u, 0) -> q^ = (sqrt3/2, 0); k = (sqrt8 u, 0) -> k^ = (kap, 0),
    #            kap = sqrt8/3; v = (1, 2); z = 0 -> g = 1/2 (S_0 = 0 anyway)
    #            S_0 = [[kap, 2 kap], [0, 0]], o_0 = (sqrt3/2)(kap, 2 kap) = (sqrt6/3, 2 sqrt6/3)
    #   token 1: q = (u, sqrt2 u) -> q^ = (1/2, sqrt2/2); k = (0, sqrt8 u) -> k^ = (0, kap);
    #            v = (3, 5); z = ln 3 -> g = 3/4
    #            S_1 = (3/4) S_0 + [[0, 0], [3 kap, 5 kap]] = [[sqrt2/2, sqrt2], [2 sqrt2, 10 sqrt2/3]]
    #            o_1 = (1/2)(sqrt2/2, sqrt2) + (sqrt2/2)(2 sqrt2, 10 sqrt2/3) = (2 + sqrt2/4, 10/3 + sqrt2/2)
    # eps outside the root, a log-sigmoid gate, or the gate applied after the
    # outer product each change these values.
    cfg = _sub_cfg(hidden=7, n_lin=1, lin_dim=2, norm_eps=_EPS)
    r2, r3, r6, r8 = math.sqrt(2), math.sqrt(3), math.sqrt(6), math.sqrt(8)
    x = np.array([[[r3 * _U, 0, r8 * _U, 0, 1, 2, 0], [_U, r2 * _U, 0, r8 * _U, 3, 5, math.log(3.0)]]])
    eye = np.eye(7)
    wo = np.zeros((7, 2))
    wo[0, 0], wo[1, 1] = 1, 1
    y, st = oracle.gla_sublayer(cfg, eye[0:2], eye[2:4], eye[4:6], eye[6:7], wo, x)
    np.testing.assert_allclose(y[0, :, :2], [[r6 / 3, 2 * r6 / 3], [2 + r2 / 4, 10 / 3 + r2 / 2]], rtol=1e-13)
    assert not y[0, :, 2:].any()
    np.testing.assert_allclose(st[0, 0], [[r2 / 2, r2], [2 * r2, 10 * r2 / 3]], rtol=1e-13)


def test_gla_sublayer_equals_recurrence_on_normalised_inputs():
    # A random case: the sublayer equals the pinned token-by-token recurrence
    # run on q, k divided by sqrt(|.|^2 + eps) and g = 1 / (1 + e^-z).
    rng = np.random.default_rng(11)
    H, nh, d, S = 12, 2, 4, 9
    cfg = _sub_cfg(hidden=H, n_lin=nh, lin_dim=d, norm_eps=1e-3)
    wq, wk, wv = (rng.normal(size=(nh * d, H)).astype(np.float32) for _ in range(3))
    wg = rng.normal(size=(nh, H)).astype(np.float32)
    wo = rng.normal(size=(H, nh * d)).astype(np.float32)
    x = rng.normal(size=(1, S, H))
    s0 = rng.normal(size=(1, nh, d, d))
    y, st = oracle.gla_sublayer(cfg, wq, wk, wv, wg, wo, x, state=s0)
    q = (x[0] @ wq.T.astype(np.float64)).reshape(S, nh, d)
    k = (x[0] @ wk.T.astype(np.float64)).reshape(S, nh, d)
    v = (x[0] @ wv.T.astype(np.float64)).reshape(S, nh, d)
    z = x[0] @ wg.T.astype(np.float64)
    eps = float(np.float32(1e-3))
    o = np.zeros((S, nh, d))
    for h in range(nh):
        qn = q[:, h] / np.sqrt((q[:, h] ** 2).sum(-1, keepdims=True) + eps)
        kn = k[:, h] / np.sqrt((k[:, h] ** 2).sum(-1, keepdims=True) + eps)
        o[:, h], sh = oracle.gla_recurrent(qn, kn, v[:, h], 1 / (1 + np.exp(-z[:, h])), state=s0[0, h])
        np.testing.assert_allclose(st[0, h], sh, atol=1e-12)
    np.testing.assert_allclose(y[0], o.reshape(S, nh * d) @ wo.T.astype(np.float64), atol=1e-11)
