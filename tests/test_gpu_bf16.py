"""GPU parity of the bf16 path against the oracle in its bf16 mode
(tolerance: max-abs relative error 2e-2 and cosine >= 0.999)."""

import numpy as np
import pytest

import oracle
import seeded
from seeded import workloads as W
from metrics import COS_BF16, TOL_BF16, cosine, rel_err

torch = pytest.importorskip("torch")
import looped_weight_shared_b200 as L  # noqa: E402

pytestmark = pytest.mark.gpu


def check(got, ref):
    e, c = rel_err(got, ref), cosine(got, ref)
    assert e < TOL_BF16 and c > COS_BF16, (e, c)
    return e, c


def test_tiny_bf16_prefill_and_decode():
    m = dict(W.model_config("tiny_fp32", dtype=1), max_batch=3, max_ctx=200)
    g = L.loop_model_create(L.make_config(**m), seed=0)
    try:
        o = oracle.Model(oracle.make_config(**m), seed=0)
        tok = seeded.tokens(3, 3, 150, m["vocab"])
        ref = o.prefill(tok, all_positions=True)
        out = torch.empty((3, 150, m["vocab"]), device="cuda")
        L.loop_prefill(g, tokens=torch.from_numpy(tok).cuda(), out=out, flags=L.LOOP_ALL_POSITIONS)
        torch.cuda.synchronize()
        check(out.cpu().numpy(), ref)
        nxt = seeded.tokens(3, 3, 3, m["vocab"], stream=seeded.S_DECODE_TOKENS)
        for t in range(3):
            r = o.decode_step(nxt[:, t])
            d = torch.empty((3, m["vocab"]), device="cuda")
            L.loop_decode_step(g, torch.from_numpy(np.ascontiguousarray(nxt[:, t])).cuda(), d)
            torch.cuda.synchronize()
            check(d.cpu().numpy(), r)
        assert L.loop_device_status() == 0
    finally:
        L.loop_model_destroy(g)


@pytest.mark.parametrize("S", [160])
def test_group9b_bf16_matches_oracle(S):
    """One 4-layer group at the 9B width (3 GLA + 1 full attention, hidden
    4096, FFN 12288) run twice with shared weights, hidden in -> hidden out."""
    m = dict(W.model_config("group9b_s4096"), max_batch=1, max_ctx=S)
    g = L.loop_model_create(L.make_config(**m), seed=1)
    try:
        o = oracle.Model(oracle.make_config(**m), seed=1)
        h = seeded.hidden(1, 1, S, m["hidden"])
        ref = o.prefill(hidden=h)
        out = torch.empty((1, S, m["hidden"]), device="cuda")
        L.loop_prefill(g, hidden=torch.from_numpy(h).cuda(), out=out)
        torch.cuda.synchronize()
        check(out.cpu().numpy(), ref)
        # the states and caches of both passes
        for slot in range(6):
            st = torch.empty((1, 32, 128, 128), device="cuda")
            L.loop_cache_read(g, L.LOOP_KIND_LINEAR, slot, 1, 0, st)
            torch.cuda.synchronize()
            check(st.cpu().numpy(), o.state(slot, 1))
        for slot in range(2):
            kv = torch.empty((2, 1, 8, S, 128), device="cuda")
            L.loop_cache_read(g, L.LOOP_KIND_FULL, slot, 1, S, kv)
            k, v = o.kv(slot, 1, S)
            torch.cuda.synchronize()
            check(kv[0].cpu().numpy(), k)
            check(kv[1].cpu().numpy(), v)
        assert L.loop_device_status() == 0
    finally:
        L.loop_model_destroy(g)


def test_group9b_extend_matches_oracle():
    """loop_extend at the 9B width: 6 new tokens on each of 2 sequences, all
    positions, against the oracle's decode steps.  At hidden 4096 an append
    runs the prefill kernels: the packed flash tile (4 query heads x 6 rows),
    the chunked GLA continuing each state, and the next mHC site's partial
    projections formed in the mHC-write epilogue."""
    w = W.WORKLOADS["probe_decode_b64_ctx4096"]
    B, S, k = 2, 40, 6
    m = dict(w["model"], max_batch=B, max_ctx=S + k)
    g = L.loop_model_create(L.make_config(**m), seed=9)
    try:
        o = oracle.Model(oracle.make_config(**m), seed=9)
        tok = seeded.tokens(9, B, S, m["vocab"])
        ext = seeded.tokens(9, B, k, m["vocab"], stream=seeded.S_DECODE_TOKENS)
        o.prefill(tok)
        out = torch.empty((B, m["vocab"]), device="cuda")
        L.loop_prefill(g, tokens=torch.from_numpy(tok).cuda(), out=out)
        got = torch.empty((B, k, m["vocab"]), device="cuda")
        L.loop_extend(g, torch.from_numpy(ext).cuda(), got, flags=L.LOOP_ALL_POSITIONS)
        torch.cuda.synchronize()
        ref = np.stack([o.decode_step(ext[:, t]) for t in range(k)], axis=1)
        check(got.cpu().numpy(), ref)
        assert [L.loop_seq_len(g, b) for b in range(B)] == [S + k] * B
        assert L.loop_device_status() == 0
    finally:
        L.loop_model_destroy(g)


MID = dict(hidden=512, ffn=512, vocab=2048, n_q=4, n_kv=2, head_dim=128, n_lin=4, lin_dim=128, dtype=1)


@pytest.mark.parametrize("B,S", [(2, 700), (1, 64), (3, 129), (2, 1)])
def test_mid_bf16_all_positions(B, S):
    """head_dim 128 (the flash-attention and fused-epilogue shapes) with a
    narrow model so the oracle stays fast: several ragged query blocks."""
    m = dict(W.model_config("tiny_fp32", **MID), max_batch=B, max_ctx=S)
    g = L.loop_model_create(L.make_config(**m), seed=5)
    try:
        o = oracle.Model(oracle.make_config(**m), seed=5)
        tok = seeded.tokens(5, B, S, m["vocab"])
        ref = o.prefill(tok, all_positions=True)
        out = torch.empty((B, S, m["vocab"]), device="cuda")
        L.loop_prefill(g, tokens=torch.from_numpy(tok).cuda(), out=out, flags=L.LOOP_ALL_POSITIONS)
        torch.cuda.synchronize()
        check(out.cpu().numpy(), ref)
        for slot in range(4):
            kv = torch.empty((2, B, 2, S, 128), device="cuda")
            L.loop_cache_read(g, L.LOOP_KIND_FULL, slot, B, S, kv)
            k, v = o.kv(slot, B, S)
            torch.cuda.synchronize()
            check(kv[0].cpu().numpy(), k)
            check(kv[1].cpu().numpy(), v)
        assert L.loop_device_status() == 0
    finally:
        L.loop_model_destroy(g)


MID4 = dict(MID, n_q=8, n_kv=2)  # GQA group 4 at head_dim 128: the decode-attention kernel's shape


def test_mid_bf16_decode_matches_oracle():
    """Prefill then decode steps on the tensor-core decode path (split-K
    weight-streaming GEMM, chunked decode attention, GLA step)."""
    B, S, steps = 3, 300, 4
    m = dict(W.model_config("tiny_fp32", **MID4), max_batch=B, max_ctx=S + steps)
    g = L.loop_model_create(L.make_config(**m), seed=6)
    try:
        o = oracle.Model(oracle.make_config(**m), seed=6)
        tok = seeded.tokens(6, B, S, m["vocab"])
        nxt = seeded.tokens(6, B, steps, m["vocab"], stream=seeded.S_DECODE_TOKENS)
        ref = o.prefill(tok)
        out = torch.empty((B, m["vocab"]), device="cuda")
        L.loop_prefill(g, tokens=torch.from_numpy(tok).cuda(), out=out)
        torch.cuda.synchronize()
        check(out.cpu().numpy(), ref)
        for t in range(steps):
            r = o.decode_step(nxt[:, t])
            L.loop_decode_step(g, torch.from_numpy(np.ascontiguousarray(nxt[:, t])).cuda(), out)
            torch.cuda.synchronize()
            check(out.cpu().numpy(), r)
            assert L.loop_seq_len(g, 2) == o.seq_len(2) == S + t + 1
        for slot in range(12):
            st = torch.empty((B, 4, 128, 128), device="cuda")
            L.loop_cache_read(g, L.LOOP_KIND_LINEAR, slot, B, 0, st)
            torch.cuda.synchronize()
            check(st.cpu().numpy(), o.state(slot, B))
        kv = torch.empty((2, B, 2, S + steps, 128), device="cuda")
        L.loop_cache_read(g, L.LOOP_KIND_FULL, 3, B, S + steps, kv)
        k, v = o.kv(3, B, S + steps)
        torch.cuda.synchronize()
        check(kv[0].cpu().numpy(), k)
        check(kv[1].cpu().numpy(), v)
        assert L.loop_device_status() == 0
    finally:
        L.loop_model_destroy(g)


def test_group9b_decode_matches_oracle():
    """Decode at the 9B width (hidden 4096, FFN 12288, GQA 32/8 x 128, 32 GLA
    heads): the decode-only kernels (one-launch mHC site, weight-streaming
    GEMM, decode attention, GLA step) against the oracle, on a 4-layer group
    run twice with a 4096-token vocabulary."""
    w = W.WORKLOADS["probe_decode_b64_ctx4096"]
    B, S, steps = 2, 32, 2
    m = dict(w["model"], max_batch=B, max_ctx=S + steps)
    g = L.loop_model_create(L.make_config(**m), seed=7)
    try:
        o = oracle.Model(oracle.make_config(**m), seed=7)
        tok = seeded.tokens(7, B, S, m["vocab"])
        nxt = seeded.tokens(7, B, steps, m["vocab"], stream=seeded.S_DECODE_TOKENS)
        ref = o.prefill(tok)
        out = torch.empty((B, m["vocab"]), device="cuda")
        L.loop_prefill(g, tokens=torch.from_numpy(tok).cuda(), out=out)
        torch.cuda.synchronize()
        check(out.cpu().numpy(), ref)
        for t in range(steps):
            r = o.decode_step(nxt[:, t])
            L.loop_decode_step(g, torch.from_numpy(np.ascontiguousarray(nxt[:, t])).cuda(), out)
            torch.cuda.synchronize()
            check(out.cpu().numpy(), r)
        for slot in (0, 5):
            st = torch.empty((B, 32, 128, 128), device="cuda")
            L.loop_cache_read(g, L.LOOP_KIND_LINEAR, slot, B, 0, st)
            torch.cuda.synchronize()
            check(st.cpu().numpy(), o.state(slot, B))
        assert L.loop_device_status() == 0
    finally:
        L.loop_model_destroy(g)


def test_mid_bf16_extend_matches_decode_steps():
    """loop_extend on the bf16 tensor-core path: 130 appended tokens span a
    full 128-token GLA tile plus a ragged one (the chunked kernel resuming from
    a non-zero state) and attention with keys before the new positions."""
    B, S, k = 2, 70, 130
    m = dict(W.model_config("tiny_fp32", **MID), max_batch=B, max_ctx=S + k + 1)
    g = L.loop_model_create(L.make_config(**m), seed=8)
    try:
        o = oracle.Model(oracle.make_config(**m), seed=8)
        tok = seeded.tokens(8, B, S, m["vocab"])
        o.prefill(tok)
        L.loop_prefill(g, tokens=torch.from_numpy(tok).cuda(), out=torch.empty((B, m["vocab"]), device="cuda"))
        ext = seeded.tokens(8, B, k + 1, m["vocab"], stream=seeded.S_DECODE_TOKENS)
        ref = np.stack([o.decode_step(ext[:, t]) for t in range(k)], axis=1)
        out = torch.empty((B, k, m["vocab"]), device="cuda")
        L.loop_extend(g, torch.from_numpy(np.ascontiguousarray(ext[:, :k])).cuda(), out, flags=L.LOOP_ALL_POSITIONS)
        torch.cuda.synchronize()
        check(out.cpu().numpy(), ref)
        r = o.decode_step(ext[:, k])
        d = torch.empty((B, m["vocab"]), device="cuda")
        L.loop_decode_step(g, torch.from_numpy(np.ascontiguousarray(ext[:, k])).cuda(), d)
        torch.cuda.synchronize()
        check(d.cpu().numpy(), r)
        for slot in (0, 5):
            st = torch.empty((B, 4, 128, 128), device="cuda")
            L.loop_cache_read(g, L.LOOP_KIND_LINEAR, slot, B, 0, st)
            torch.cuda.synchronize()
            check(st.cpu().numpy(), o.state(slot, B))
        assert L.loop_device_status() == 0
    finally:
        L.loop_model_destroy(g)


def test_mid_bf16_mixed_length_decode():
    """Decode over sequences of different lengths on the bf16 tensor-core
    path (decode attention with per-sequence key counts across several
    1024-key chunks, the GLA step, the decode GEMM): ragged prefill of 1500,
    77 and 1030 tokens, then two decode steps, each sequence against its own
    oracle."""
    lens = [1500, 77, 1030]
    m = dict(W.model_config("tiny_fp32", **MID4), max_batch=3, max_ctx=1510)
    g = L.loop_model_create(L.make_config(**m), seed=9)
    try:
        seqs = [seeded.tokens(40 + i, 1, n, m["vocab"])[0] for i, n in enumerate(lens)]
        os_ = [oracle.Model(oracle.make_config(**m), seed=9) for _ in lens]
        ref = np.concatenate([o.prefill(s[None, :]) for o, s in zip(os_, seqs)], axis=0)
        out = torch.empty((3, m["vocab"]), device="cuda")
        L.loop_prefill_ragged(g, torch.from_numpy(np.concatenate(seqs)).cuda(), lens, out)
        torch.cuda.synchronize()
        check(out.cpu().numpy(), ref)
        nxt = seeded.tokens(50, 2, 3, m["vocab"], stream=seeded.S_DECODE_TOKENS)
        d = torch.empty((3, m["vocab"]), device="cuda")
        for t in range(2):
            L.loop_decode_step(g, torch.from_numpy(np.ascontiguousarray(nxt[t])).cuda(), d)
            torch.cuda.synchronize()
            r = np.concatenate([o.decode_step(np.array([x], dtype=np.int32)) for o, x in zip(os_, nxt[t])], axis=0)
            check(d.cpu().numpy(), r)
        assert L.loop_device_status() == 0
    finally:
        L.loop_model_destroy(g)


@pytest.mark.parametrize("k", [8, 32, 33])
def test_mid_bf16_extend_after_ragged_prefill(k):
    """loop_extend of k tokens on sequences of different lengths: the
    tensor-core flash kernel with a different start position per sequence
    (keys before the new positions, the causal block among them), each
    sequence against its own oracle's decode steps.  With 4 query heads per kv
    head, k <= 32 runs the packed tile (the group's heads share one 128-row
    tile; k = 32 fills it) and k = 33 the unpacked one."""
    lens = [1100, 77, 530]
    m = dict(W.model_config("tiny_fp32", **MID4), max_batch=3, max_ctx=1100 + k)
    g = L.loop_model_create(L.make_config(**m), seed=12)
    try:
        seqs = [seeded.tokens(70 + i, 1, n, m["vocab"])[0] for i, n in enumerate(lens)]
        os_ = [oracle.Model(oracle.make_config(**m), seed=12) for _ in lens]
        for o, s in zip(os_, seqs):
            o.prefill(s[None, :])
        out = torch.empty((3, m["vocab"]), device="cuda")
        L.loop_prefill_ragged(g, torch.from_numpy(np.concatenate(seqs)).cuda(), lens, out)
        ext = seeded.tokens(71, 3, k, m["vocab"], stream=seeded.S_DECODE_TOKENS)
        got = torch.empty((3, k, m["vocab"]), device="cuda")
        L.loop_extend(g, torch.from_numpy(ext).cuda(), got, flags=L.LOOP_ALL_POSITIONS)
        torch.cuda.synchronize()
        ref = np.stack([np.concatenate([o.decode_step(ext[i, t:t + 1]) for t in range(k)]) for i, o in enumerate(os_)])
        check(got.cpu().numpy(), ref)
        assert [L.loop_seq_len(g, i) for i in range(3)] == [n + k for n in lens]
        assert L.loop_device_status() == 0
    finally:
        L.loop_model_destroy(g)


def test_mid_bf16_paged_kv_pool_shared_by_sequences():
    """A KV page pool smaller than max_batch x max_ctx, shared by sequences of
    different lengths: ragged prefills that release and take pages (so a
    sequence's pages end up scattered over the pool), decode steps that cross
    64-position page boundaries, a re-prefill of one sequence, and a prefill
    that would need more pages than are free (LOOP_ERANGE, nothing changed).
    Every sequence against its own oracle (a dense cache)."""
    m = dict(W.model_config("tiny_fp32", **MID4), max_batch=4, max_ctx=600, kv_pages=20)
    V = m["vocab"]
    g = L.loop_model_create(L.make_config(**m), seed=13)
    try:
        om = dict(m, max_batch=1)
        os_ = [oracle.Model(oracle.make_config(**om), seed=13) for _ in range(3)]
        lens = [126, 200, 63]  # 2 + 4 + 1 pages
        seqs = [seeded.tokens(80 + b, 1, n, V)[0] for b, n in enumerate(lens)]
        ref = np.concatenate([o.prefill(s[None, :]) for o, s in zip(os_, seqs)])
        out = torch.empty((3, V), device="cuda")
        L.loop_prefill_ragged(g, torch.from_numpy(np.concatenate(seqs)).cuda(), lens, out)
        torch.cuda.synchronize()
        check(out.cpu().numpy(), ref)

        def decode(step):
            tok = seeded.tokens(90 + step, 1, 3, V, stream=seeded.S_DECODE_TOKENS)[0]
            d = torch.empty((3, V), device="cuda")
            L.loop_decode_step(g, torch.from_numpy(tok).cuda(), d)
            torch.cuda.synchronize()
            r = np.concatenate([o.decode_step(np.array([t], dtype=np.int32)) for o, t in zip(os_, tok)])
            check(d.cpu().numpy(), r)

        for step in range(3):  # sequence 0 crosses 128, sequence 2 crosses 64
            decode(step)
        # sequence 1 again, longer: its 4 pages go back, 8 are taken (some of them freed ones)
        s1 = seeded.tokens(85, 1, 450, V)[0]
        r1 = os_[1].prefill(s1[None, :])
        o1 = torch.empty((1, V), device="cuda")
        L.loop_prefill_ragged(g, torch.from_numpy(s1).cuda(), [450], o1, b0=1)
        torch.cuda.synchronize()
        check(o1.cpu().numpy(), r1)
        for step in range(3, 5):
            decode(step)
        # 3 + 8 + 2 pages held, 7 free: a 500-token sequence (8 pages) does not fit
        with pytest.raises(L.LoopError) as err:
            L.loop_prefill_ragged(g, torch.from_numpy(seeded.tokens(86, 1, 500, V)[0]).cuda(), [500],
                                  torch.empty((1, V), device="cuda"), b0=3)
        assert err.value.code == L.LOOP_ERANGE
        decode(5)
        # the paged cache read back in position order
        kv = torch.empty((2, 1, 2, lens[0] + 6, 128), device="cuda")
        L.loop_cache_read(g, L.LOOP_KIND_FULL, 1, 1, lens[0] + 6, kv)
        torch.cuda.synchronize()
        k_ref, v_ref = os_[0].kv(1, 1, lens[0] + 6)
        check(kv[0].cpu().numpy(), k_ref)
        check(kv[1].cpu().numpy(), v_ref)
        assert L.loop_device_status() == 0
    finally:
        L.loop_model_destroy(g)
