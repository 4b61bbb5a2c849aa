"""GPU parity of the tiny fp32 looped decoder (12 stored layers, 16
executions, hidden 256) against the oracle, through the C ABI."""

import numpy as np
import pytest

import oracle
import seeded
from seeded import workloads as W
from metrics import TOL_F32, rel_err

torch = pytest.importorskip("torch")
import looped_weight_shared_b200 as L  # noqa: E402

pytestmark = pytest.mark.gpu

W_PER_LAYER = 10


def cfg(**kw):
    m = dict(W.model_config("tiny_fp32"), max_batch=2, max_ctx=160)
    m.update(kw)
    return m


@pytest.fixture(scope="module")
def pair():
    m = cfg()
    g = L.loop_model_create(L.make_config(**m), seed=0)
    o = oracle.Model(oracle.make_config(**m), seed=0)
    yield m, g, o
    L.loop_model_destroy(g)


def gpu_prefill(g, tok, vocab, all_positions=True):
    B, S = tok.shape
    out = torch.empty((B, S, vocab) if all_positions else (B, vocab), device="cuda")
    L.loop_prefill(g, tokens=torch.from_numpy(tok).cuda(), out=out,
                   flags=L.LOOP_ALL_POSITIONS if all_positions else 0)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_device_weights_follow_the_generator(pair):
    m, g, o = pair
    for idx in (0, 2 + 1, 2 + W_PER_LAYER * 3 + 9, 2 + W_PER_LAYER * 12 + 1, 2 + W_PER_LAYER * 5 + 7):
        ref = o.weight(idx)
        out = torch.empty(ref.size, device="cuda")
        L.loop_weight_read(g, idx, out)
        got = out.cpu().numpy()
        bad = np.count_nonzero(got != ref)
        assert bad <= max(1, ref.size // 10**6), (idx, bad)


def test_tiny_prefill_matches_oracle(pair):
    m, g, o = pair
    tok = seeded.tokens(0, 1, 128, m["vocab"])
    ref = o.prefill(tok, all_positions=True)
    got = gpu_prefill(g, tok, m["vocab"])
    assert rel_err(got, ref) < TOL_F32
    last = gpu_prefill(g, tok, m["vocab"], all_positions=False)
    assert rel_err(last, ref[:, -1]) < TOL_F32
    assert L.loop_seq_len(g, 0) == 128 == o.seq_len(0)


def test_tiny_caches_match_oracle(pair):
    m, g, o = pair
    tok = seeded.tokens(5, 2, 37, m["vocab"])
    o.prefill(tok)
    gpu_prefill(g, tok, m["vocab"], all_positions=False)
    for slot in range(4):
        kv = torch.empty((2, 2, m["n_kv"], 37, m["head_dim"]), device="cuda")
        L.loop_cache_read(g, L.LOOP_KIND_FULL, slot, 2, 37, kv)
        k, v = o.kv(slot, 2, 37)
        torch.cuda.synchronize()
        assert rel_err(kv[0].cpu().numpy(), k) < TOL_F32
        assert rel_err(kv[1].cpu().numpy(), v) < TOL_F32
    for slot in range(12):
        st = torch.empty((2, m["n_lin"], m["lin_dim"], m["lin_dim"]), device="cuda")
        L.loop_cache_read(g, L.LOOP_KIND_LINEAR, slot, 2, 0, st)
        torch.cuda.synchronize()
        assert rel_err(st.cpu().numpy(), o.state(slot, 2)) < TOL_F32


def test_tiny_decode_matches_oracle(pair):
    m, g, o = pair
    tok = seeded.tokens(7, 2, 24, m["vocab"])
    nxt = seeded.tokens(7, 2, 6, m["vocab"], stream=seeded.S_DECODE_TOKENS)
    o.prefill(tok)
    gpu_prefill(g, tok, m["vocab"], all_positions=False)
    for t in range(6):
        ref = o.decode_step(nxt[:, t])
        out = torch.empty((2, m["vocab"]), device="cuda")
        L.loop_decode_step(g, torch.from_numpy(np.ascontiguousarray(nxt[:, t])).cuda(), out)
        torch.cuda.synchronize()
        assert rel_err(out.cpu().numpy(), ref) < TOL_F32
        assert L.loop_seq_len(g, 0) == o.seq_len(0) == 25 + t
        assert L.loop_seq_len(g, 1) == o.seq_len(1)


def test_decode_equals_longer_prefill_on_gpu(pair):
    m, g, o = pair
    tok = seeded.tokens(9, 1, 40, m["vocab"])
    full = gpu_prefill(g, tok, m["vocab"])
    gpu_prefill(g, tok[:, :35], m["vocab"], all_positions=False)
    for t in range(35, 40):
        out = torch.empty((1, m["vocab"]), device="cuda")
        L.loop_decode_step(g, torch.from_numpy(np.ascontiguousarray(tok[:, t])).cuda(), out)
        torch.cuda.synchronize()
        assert rel_err(out.cpu().numpy(), full[:, t]) < TOL_F32


def test_looped_equals_unrolled_on_gpu(pair):
    m, g, o = pair
    ws = [o.weight(i) for i in range(o.num_weights())]
    n_phys = 12
    layer = lambda p: ws[2 + W_PER_LAYER * p: 2 + W_PER_LAYER * (p + 1)]
    sites = ws[2 + W_PER_LAYER * n_phys:]
    unrolled = ws[:2]
    for p in list(range(4)) + list(range(4, 8)) * 2 + list(range(8, 12)):
        unrolled += layer(p)
    unrolled += sites * 2
    mu = cfg(n_block=8, n_loops=1)
    gl = L.loop_model_create(L.make_config(**m), host_weights=ws)
    gu = L.loop_model_create(L.make_config(**mu), host_weights=unrolled)
    try:
        tok = seeded.tokens(11, 2, 50, m["vocab"])
        a = gpu_prefill(gl, tok, m["vocab"])
        b = gpu_prefill(gu, tok, m["vocab"])
        np.testing.assert_array_equal(a, b)
        # caller weights equal the device generator's values: same logits
        c = gpu_prefill(g, tok, m["vocab"])
        assert rel_err(a, c) < 1e-6
    finally:
        L.loop_model_destroy(gl)
        L.loop_model_destroy(gu)


def test_range_errors(pair):
    m, g, o = pair
    tok = torch.zeros((1, 161), dtype=torch.int32, device="cuda")
    out = torch.empty((1, m["vocab"]), device="cuda")
    with pytest.raises(L.LoopError) as e:
        L.loop_prefill(g, tokens=tok, out=out)
    assert e.value.code == L.LOOP_ERANGE
    with pytest.raises(L.LoopError) as e:
        L.loop_prefill(g, tokens=torch.zeros((3, 4), dtype=torch.int32, device="cuda"),
                       out=torch.empty((3, m["vocab"]), device="cuda"))
    assert e.value.code == L.LOOP_ERANGE
    L.loop_prefill(g, tokens=torch.zeros((1, 160), dtype=torch.int32, device="cuda"), out=out)
    with pytest.raises(L.LoopError) as e:
        L.loop_decode_step(g, torch.zeros(1, dtype=torch.int32, device="cuda"), out)
    assert e.value.code == L.LOOP_ERANGE
    assert L.loop_seq_len(g, 0) == 160
    assert L.loop_device_status() == 0


def test_mhc_sinkhorn_bit_exact():
    rng = np.random.default_rng(0)
    for n, scale, count in ((2, 0.45, 50000), (2, 1.81, 50000), (2, 30.0, 2000), (3, 1.0, 3000), (4, 2.0, 2000),
                            (8, 1.0, 500), (1, 1.0, 10)):
        x = rng.normal(0, scale, size=(count, n, n)).astype(np.float32)
        ref = oracle.sinkhorn_f32(x, 20)
        xd = torch.from_numpy(x).cuda()
        out = torch.empty_like(xd)
        L.mhc_sinkhorn(xd, out, iters=20)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(out.cpu().numpy(), ref)
    # zero iterations and a single iteration
    x = rng.normal(0, 1, size=(100, 2, 2)).astype(np.float32)
    for it in (0, 1):
        out = torch.empty((100, 2, 2), device="cuda")
        L.mhc_sinkhorn(torch.from_numpy(x).cuda(), out, iters=it)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(out.cpu().numpy(), oracle.sinkhorn_f32(x, it))


def test_hidden_mode_matches_oracle():
    m = dict(W.model_config("group9b_s4096", hidden=128, ffn=256, n_q=4, n_kv=2, head_dim=32, n_lin=4,
                            lin_dim=32, dtype=0), max_batch=2, max_ctx=64)
    g = L.loop_model_create(L.make_config(**m), seed=1)
    try:
        o = oracle.Model(oracle.make_config(**m), seed=1)
        h = seeded.hidden(1, 2, 33, 128)
        ref = o.prefill(hidden=h)
        out = torch.empty((2, 33, 128), device="cuda")
        L.loop_prefill(g, hidden=torch.from_numpy(h).cuda(), out=out)
        torch.cuda.synchronize()
        assert rel_err(out.cpu().numpy(), ref) < TOL_F32
    finally:
        L.loop_model_destroy(g)


@pytest.mark.parametrize("n_loops", [1, 3])
def test_loop_count_matches_oracle(n_loops):
    """Loop counts other than the pages' two, B^K(h) with K = 1 and 3: one
    weight set reused K times and K sets of per-pass caches, against the
    oracle through prefill, decode and the last linear-attention state."""
    m = cfg(n_loops=n_loops)
    g = L.loop_model_create(L.make_config(**m), seed=0)
    try:
        o = oracle.Model(oracle.make_config(**m), seed=0)
        tok = seeded.tokens(12, 2, 40, m["vocab"])
        assert rel_err(gpu_prefill(g, tok, m["vocab"]), o.prefill(tok, all_positions=True)) < TOL_F32
        nxt = seeded.tokens(12, 2, 2, m["vocab"], stream=seeded.S_DECODE_TOKENS)
        for t in range(2):
            r = o.decode_step(nxt[:, t])
            d = torch.empty((2, m["vocab"]), device="cuda")
            L.loop_decode_step(g, torch.from_numpy(np.ascontiguousarray(nxt[:, t])).cuda(), d)
            torch.cuda.synchronize()
            assert rel_err(d.cpu().numpy(), r) < TOL_F32
        # prelude, K passes of the block and coda each hold one group: 3 linear executions per group
        last = 3 * (2 + n_loops) - 1
        st = torch.empty((2, m["n_lin"], m["lin_dim"], m["lin_dim"]), device="cuda")
        L.loop_cache_read(g, L.LOOP_KIND_LINEAR, last, 2, 0, st)
        torch.cuda.synchronize()
        assert rel_err(st.cpu().numpy(), o.state(last, 2)) < TOL_F32
        assert L.loop_device_status() == 0
    finally:
        L.loop_model_destroy(g)


@pytest.mark.parametrize("k", [1, 6])
def test_extend_equals_decode_steps(k):
    """loop_extend appends k tokens per sequence in one pass; the oracle
    appends them one decode step at a time: every appended position's logits,
    the lengths and a following decode step agree."""
    m = cfg()
    g = L.loop_model_create(L.make_config(**m), seed=0)
    try:
        o = oracle.Model(oracle.make_config(**m), seed=0)
        B, S = 2, 30
        tok = seeded.tokens(13, B, S, m["vocab"])
        o.prefill(tok)
        gpu_prefill(g, tok, m["vocab"], all_positions=False)
        ext = seeded.tokens(13, B, k + 1, m["vocab"], stream=seeded.S_DECODE_TOKENS)
        ref = np.stack([o.decode_step(ext[:, t]) for t in range(k)], axis=1)
        out = torch.empty((B, k, m["vocab"]), device="cuda")
        L.loop_extend(g, torch.from_numpy(np.ascontiguousarray(ext[:, :k])).cuda(), out, flags=L.LOOP_ALL_POSITIONS)
        torch.cuda.synchronize()
        assert rel_err(out.cpu().numpy(), ref) < TOL_F32
        assert L.loop_seq_len(g, 0) == S + k and L.loop_seq_len(g, 1) == S + k
        r = o.decode_step(ext[:, k])
        d = torch.empty((B, m["vocab"]), device="cuda")
        L.loop_decode_step(g, torch.from_numpy(np.ascontiguousarray(ext[:, k])).cuda(), d)
        torch.cuda.synchronize()
        assert rel_err(d.cpu().numpy(), r) < TOL_F32
        with pytest.raises(L.LoopError) as e:  # past max_ctx
            L.loop_extend(g, torch.zeros((B, 160), dtype=torch.int32, device="cuda"),
                          torch.empty((B, m["vocab"]), device="cuda"))
        assert e.value.code == L.LOOP_ERANGE
        assert L.loop_device_status() == 0
    finally:
        L.loop_model_destroy(g)


def _oracle_decode(os_, toks):
    return np.concatenate([o.decode_step(np.array([t], dtype=np.int32)) for o, t in zip(os_, toks)], axis=0)


def test_ragged_prefill_and_mixed_length_decode():
    """Continuous batching: sequences of lengths 30, 7 and 19 prefilled into
    slots 0-2, a decode step over all three at their own lengths, then slot 1
    refilled with a new 12-token sequence while 0 and 2 keep their caches.
    Each sequence is checked against its own single-sequence oracle."""
    m = cfg(max_batch=3)
    g = L.loop_model_create(L.make_config(**m), seed=0)
    try:
        lens = [30, 7, 19]
        seqs = [seeded.tokens(20 + i, 1, n, m["vocab"])[0] for i, n in enumerate(lens)]
        os_ = [oracle.Model(oracle.make_config(**m), seed=0) for _ in lens]
        ref = np.concatenate([o.prefill(s[None, :]) for o, s in zip(os_, seqs)], axis=0)
        out = torch.empty((3, m["vocab"]), device="cuda")
        L.loop_prefill_ragged(g, torch.from_numpy(np.concatenate(seqs)).cuda(), lens, out)
        torch.cuda.synchronize()
        assert rel_err(out.cpu().numpy(), ref) < TOL_F32
        assert [L.loop_seq_len(g, b) for b in range(3)] == lens
        nxt = seeded.tokens(30, 2, 3, m["vocab"], stream=seeded.S_DECODE_TOKENS)
        d = torch.empty((3, m["vocab"]), device="cuda")
        L.loop_decode_step(g, torch.from_numpy(np.ascontiguousarray(nxt[0])).cuda(), d)
        torch.cuda.synchronize()
        assert rel_err(d.cpu().numpy(), _oracle_decode(os_, nxt[0])) < TOL_F32
        # slot 1 takes a new request; slots 0 and 2 keep decoding
        new = seeded.tokens(31, 1, 12, m["vocab"])
        os_[1] = oracle.Model(oracle.make_config(**m), seed=0)
        r1 = os_[1].prefill(new)
        o1 = torch.empty((1, m["vocab"]), device="cuda")
        L.loop_prefill_ragged(g, torch.from_numpy(new[0]).cuda(), [12], o1, b0=1)
        torch.cuda.synchronize()
        assert rel_err(o1.cpu().numpy(), r1) < TOL_F32
        assert [L.loop_seq_len(g, b) for b in range(3)] == [31, 12, 20]
        L.loop_decode_step(g, torch.from_numpy(np.ascontiguousarray(nxt[1])).cuda(), d)
        torch.cuda.synchronize()
        assert rel_err(d.cpu().numpy(), _oracle_decode(os_, nxt[1])) < TOL_F32
        with pytest.raises(L.LoopError) as e:
            L.loop_prefill_ragged(g, torch.from_numpy(new[0]).cuda(), [12], o1, b0=3)
        assert e.value.code == L.LOOP_ERANGE
        assert L.loop_device_status() == 0
    finally:
        L.loop_model_destroy(g)
