"""Pins for the CPU oracle, checked against what the method and mathematics fix.

None of these compare the oracle with itself: each check uses a hand-worked
fixture, a closed form, an invariant, or an independent brute force written here
with numpy / Python sorting. Method: "Hierarchical Global Attention (HGA)"
(arXiv 2606.30709) abstract, and the HISA article's keep-beginning-and-end rule.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def to_bf16_bits(x) -> np.ndarray:
    """float64 values that are exactly bfloat16 -> bits (asserts exactness)."""
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float32)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(oracle.bf16_to_f64(bits), x), "not exactly representable in bfloat16"
    return bits


def rne_bf16_numpy(x: np.ndarray) -> np.ndarray:
    """Independent double -> bfloat16 rounding (frexp + round-half-even), normals only."""
    m, e = np.frexp(np.abs(x))
    r = np.ldexp(np.rint(m * 256.0), e - 8)
    return np.copysign(r, x)


def dense_attention(q, K, V, scale):
    """Brute-force softmax attention in float64 (numpy)."""
    z = (q @ K.T) * scale
    z = z - z.max(axis=1, keepdims=True)
    w = np.exp(z)
    return (w @ V) / w.sum(axis=1, keepdims=True)


def rand_bf16(rng, shape, scale=1.0):
    return (torch.from_numpy(rng.standard_normal(shape) * scale).to(torch.bfloat16)
            .view(torch.int16).numpy().view(np.uint16))


# ------------------------------------------------------------------ bfloat16


def test_bf16_rne_matches_torch_on_float32_values():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),  # bfloat16 subnormals
        np.array([1 + 2**-8, 1 + 3 * 2**-8, -(1 + 2**-8), 3.4e38, 1e-45, 0.0, -0.0, 2**-126,
                  255.5, 256.5, -0.0078125], dtype=np.float32),
    ])
    ours = np.array([oracle.bf16_rne(float(v)) for v in x], dtype=np.uint16)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_rne_rounds_double_directly():
    # 1 + 2^-8 is a tie (rounds to even: 1.0); anything above it must round up to
    # 1 + 2^-7. A float32 detour would lose the 2^-40 and round down.
    assert oracle.bf16_rne(1 + 2**-8) == 0x3F80
    assert oracle.bf16_rne(1 + 2**-8 + 2**-40) == 0x3F81
    assert oracle.bf16_rne(-(1 + 2**-8 + 2**-40)) == 0xBF81
    assert oracle.bf16_rne(1 + 3 * 2**-8) == 0x3F82  # tie between 0x3F81 and 0x3F82 -> even
    assert oracle.bf16_rne(float("inf")) == 0x7F80
    assert oracle.bf16_rne(2.0**128) == 0x7F80


# ----------------------------------------------------------------- summaries


def test_summaries_brute_force_means():
    rng = np.random.default_rng(2)
    L, d, C, g = 200, 16, 32, 8  # 6 full chunks and a 8-token tail
    K = rand_bf16(rng, (L, d))
    cs, gs, cf, gf = oracle.summaries(K, C, g, with_f64=True)
    Kf = oracle.bf16_to_f64(K)
    nf = L // C
    assert cs.shape == (nf, d) and gs.shape == (nf, C // g, d)
    want_c = Kf[: nf * C].reshape(nf, C, d).mean(axis=1)
    want_g = Kf[: nf * C].reshape(nf, C // g, g, d).mean(axis=2)
    np.testing.assert_allclose(cf, want_c, rtol=0, atol=1e-15)
    np.testing.assert_allclose(gf, want_g, rtol=0, atol=1e-15)
    assert np.array_equal(oracle.bf16_to_f64(cs), rne_bf16_numpy(want_c))
    assert np.array_equal(oracle.bf16_to_f64(gs), rne_bf16_numpy(want_g))


def test_summary_linearity():
    # The chunk mean is the mean of its group means, and the head-summed score of a
    # chunk summary is the mean over its tokens of the head-summed q.K_t.
    rng = np.random.default_rng(3)
    L, d, C, g, R = 256, 32, 64, 16, 4
    K = rand_bf16(rng, (L, d))
    q = rand_bf16(rng, (R, d))
    _, _, cf, gf = oracle.summaries(K, C, g, with_f64=True)
    np.testing.assert_allclose(cf, gf.mean(axis=1), rtol=0, atol=1e-14)
    qs = oracle.bf16_to_f64(q).sum(axis=0)
    per_token = oracle.bf16_to_f64(K) @ qs
    np.testing.assert_allclose(cf @ qs, per_token.reshape(L // C, C).mean(axis=1), rtol=1e-12, atol=1e-12)


def test_constant_chunks_give_exact_summaries():
    L, d, C, g = 96, 8, 32, 16
    vals = np.array([0.5, -1.25, 3.0])
    Kf = np.repeat(vals, C)[:, None] * np.ones((1, d))
    cs, gs = oracle.summaries(to_bf16_bits(Kf), C, g)
    assert np.array_equal(oracle.bf16_to_f64(cs), vals[:, None] * np.ones((1, d)))
    assert np.array_equal(oracle.bf16_to_f64(gs), vals[:, None, None] * np.ones((1, C // g, d)))


# ------------------------------------------------------------------- routing


def brute_route(q_f64, cs_f64, gs_f64, L, C, g, k, G):
    """Two-level routing by direct enumeration and Python sorting."""
    nf = L // C
    if nf <= 2:
        return list(range(L))
    qq = q_f64 if q_f64.ndim == 3 else q_f64[None]
    head_sums = [[sum(qq[p, i, e] for i in range(qq.shape[1])) for e in range(qq.shape[2])]
                 for p in range(qq.shape[0])]

    def score(s):
        return max(sum(hs[e] * s[e] for e in range(len(s))) for hs in head_sums)

    cands = sorted(range(1, nf - 1), key=lambda c: (-score(cs_f64[c]), c))
    kept = sorted(cands[:k])
    toks = list(range(C))
    for c in kept:
        gpc = C // g
        order = sorted(range(gpc), key=lambda j: (-score(gs_f64[c, j]), j))
        for j in sorted(order[:G]):
            toks += list(range(c * C + j * g, c * C + (j + 1) * g))
    toks += list(range((nf - 1) * C, L))
    return toks


@pytest.mark.parametrize("seed", range(12))
def test_route_matches_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    C = int(rng.choice([16, 32, 64]))
    g = int(rng.choice([x for x in (4, 8, 16) if C % x == 0]))
    L = int(rng.integers(1, 14 * C))
    d = int(rng.choice([8, 16]))
    R = int(rng.integers(1, 5))
    k = int(rng.integers(1, 8))
    G = int(rng.integers(1, C // g + 1))
    K = rand_bf16(rng, (L, d))
    q = rand_bf16(rng, (R, d))
    cs, gs = oracle.summaries(K, C, g)
    got = oracle.route(q, cs, gs, L, C, g, k, G)
    want = brute_route(oracle.bf16_to_f64(q), oracle.bf16_to_f64(cs), oracle.bf16_to_f64(gs), L, C, g, k, G)
    assert got.tolist() == want
    assert len(got) == oracle.max_routed(L, C, g, k, G)


def test_route_ties_go_to_lower_index():
    # Every chunk and group summary identical: all scores tie, so the lowest
    # candidate chunks and the lowest groups are kept.
    L, d, C, g, k, G = 10 * 16, 8, 16, 4, 3, 2
    K = to_bf16_bits(np.ones((L, d)))
    q = to_bf16_bits(np.ones((2, d)))
    cs, gs = oracle.summaries(K, C, g)
    got = oracle.route(q, cs, gs, L, C, g, k, G).tolist()
    want = list(range(16))
    for c in (1, 2, 3):
        want += list(range(c * 16, c * 16 + 8))
    want += list(range(9 * 16, L))
    assert got == want


def load_hand_fixture():
    cases, attends, params = [], [], {}
    K = V = None
    for line in open(os.path.join(GOLDEN, "route_hand.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        tag, *rest = line.split()
        kv = dict(x.split("=") for x in rest if "=" in x)
        if tag == "params":
            params = {a: int(b) for a, b in kv.items()}
        elif tag in ("K", "V"):
            rows = np.array([[float(x) for x in r.split(",")] for r in rest])
            if tag == "K":
                K = rows
            else:
                V = rows
        elif tag == "route":
            cases.append(([float(x) for x in kv["q"].split(",")], [int(x) for x in kv["tokens"].split(",")]))
        elif tag == "attend":
            attends.append(([float(x) for x in kv["q"].split(",")], float(kv["scale"]),
                            [float(x) for x in kv["out"].split(",")]))
    return params, K, V, cases, attends


def test_route_hand_worked_fixture():
    p, K, V, cases, attends = load_hand_fixture()
    Kb, Vb = to_bf16_bits(K), to_bf16_bits(V)
    cs, gs = oracle.summaries(Kb, p["C"], p["g"])
    assert oracle.bf16_to_f64(cs).tolist() == [[0, 0], [2, 0], [1, 1.5], [2, 2]]
    for qv, want in cases:
        got = oracle.route(to_bf16_bits([qv]), cs, gs, p["L"], p["C"], p["g"], p["k"], p["G"])
        assert got.tolist() == want, (qv, got)
    for qv, scale, want in attends:
        qb = to_bf16_bits([qv])
        tok = oracle.route(qb, cs, gs, p["L"], p["C"], p["g"], p["k"], p["G"])
        out = oracle.attend(qb, Kb, Vb, tok, scale=scale)
        np.testing.assert_allclose(out[0], want, rtol=0, atol=1e-14)


def test_routed_fraction_closed_form():
    rows = [list(map(int, l.split())) for l in open(os.path.join(GOLDEN, "routed_fraction.txt"))
            if l.strip() and not l.startswith("#")]
    w = synth.DECODE_64K
    for L, nf, r, S in rows:
        assert L // w.chunk == nf and min(w.top_chunks, nf - 2) == r
        s = synth.sequence(w, 0, L, [L - 1])
        cs, gs = oracle.summaries(s.k[0], w.chunk, w.group)
        tok = oracle.route(s.q[0, : w.n_q_heads // w.n_kv_heads], cs, gs, L, w.chunk, w.group,
                           w.top_chunks, w.top_groups)
        assert len(tok) == S
        assert len(np.unique(tok)) == S and np.all(np.diff(tok) > 0)
        assert tok[:128].tolist() == list(range(128))
        assert tok[-128:].tolist() == list(range((nf - 1) * 128, L))
    # the abstract's sparsity at 64K: roughly three percent
    assert 0.025 < rows[-1][3] / rows[-1][0] < 0.04


def test_tiny_workload_selects_all_planted_chunks():
    w = synth.TINY_DECODE_4K
    inp = synth.decode_inputs(w)
    R = w.n_q_heads // w.n_kv_heads
    cs, gs = oracle.summaries(inp.k[0, 0], w.chunk, w.group)
    _, kept = oracle.route(inp.q[0, :R], cs, gs, w.ctx_len, w.chunk, w.group, w.top_chunks, w.top_groups,
                           return_chunks=True)
    assert len(inp.planted[0]) == 4
    assert set(inp.planted[0].tolist()) <= set(kept.tolist())


def test_gqa_with_identical_heads_routes_like_one_head():
    rng = np.random.default_rng(5)
    L, d, C, g = 40 * 16, 16, 32, 8
    K = rand_bf16(rng, (L, d))
    V = rand_bf16(rng, (L, d))
    q1 = rand_bf16(rng, (1, d))
    q8 = np.repeat(q1, 8, axis=0)
    cs, gs = oracle.summaries(K, C, g)
    t1 = oracle.route(q1, cs, gs, L, C, g, 5, 2)
    t8 = oracle.route(q8, cs, gs, L, C, g, 5, 2)
    assert t1.tolist() == t8.tolist()
    o1 = oracle.attend(q1, K, V, t1)
    o8 = oracle.attend(q8, K, V, t8)
    np.testing.assert_array_equal(o8, np.repeat(o1, 8, axis=0))


# ----------------------------------------------------------------- attention


@pytest.mark.parametrize("d", [16, 64])
def test_full_coverage_equals_dense_causal_attention(d):
    # Routing that keeps every chunk and every group must give dense attention
    # over the whole causal window [0, L): "exact attention over the retrieved set".
    rng = np.random.default_rng(6 + d)
    C, g, R = 32, 8, 4
    for L in (5, 70, 96, 97, 500):
        K = rand_bf16(rng, (L, d))
        V = rand_bf16(rng, (L, d))
        q = rand_bf16(rng, (R, d), scale=2.0)
        cs, gs = oracle.summaries(K, C, g)
        tok = oracle.route(q, cs, gs, L, C, g, k=L, G=C // g)
        assert tok.tolist() == list(range(L))
        out, lse = oracle.attend(q, K, V, tok, with_lse=True)
        qf, Kf, Vf = (oracle.bf16_to_f64(x) for x in (q, K, V))
        want = dense_attention(qf, Kf, Vf, 1 / math.sqrt(d))
        np.testing.assert_allclose(out, want, rtol=0, atol=1e-12)
        z = qf @ Kf.T / math.sqrt(d)
        m = z.max(axis=1)
        np.testing.assert_allclose(lse, m + np.log(np.exp(z - m[:, None]).sum(axis=1)), rtol=0, atol=1e-12)


def test_single_token_returns_its_value_row():
    rng = np.random.default_rng(7)
    K = rand_bf16(rng, (50, 32))
    V = rand_bf16(rng, (50, 32))
    q = rand_bf16(rng, (3, 32), scale=10.0)
    out = oracle.attend(q, K, V, [17])
    assert np.array_equal(out, np.repeat(oracle.bf16_to_f64(V[17])[None], 3, axis=0))


def test_equal_logits_give_mean_of_values():
    rng = np.random.default_rng(8)
    K = rand_bf16(rng, (64, 16))
    V = rand_bf16(rng, (64, 16))
    q = np.zeros((2, 16), dtype=np.uint16)
    tok = [3, 9, 10, 40, 63]
    out = oracle.attend(q, K, V, tok)
    np.testing.assert_allclose(out[0], oracle.bf16_to_f64(V[tok]).mean(axis=0), rtol=0, atol=1e-15)


def test_attention_is_invariant_to_token_order():
    rng = np.random.default_rng(9)
    K = rand_bf16(rng, (300, 64))
    V = rand_bf16(rng, (300, 64))
    q = rand_bf16(rng, (4, 64))
    tok = rng.choice(300, size=77, replace=False)
    a = oracle.attend(q, K, V, np.sort(tok))
    b = oracle.attend(q, K, V, tok)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


def test_empty_token_set():
    K = np.zeros((4, 8), dtype=np.uint16)
    out, lse = oracle.attend(np.zeros((2, 8), dtype=np.uint16), K, K, [], with_lse=True)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


# ------------------------------------------------------------------- prefill


def test_prefill_block_routing_takes_max_over_queries():
    rng = np.random.default_rng(10)
    L, d, C, g, R, nq = 30 * 32, 16, 32, 8, 2, 5
    K = rand_bf16(rng, (L, d))
    q = rand_bf16(rng, (nq, R, d))
    cs, gs = oracle.summaries(K, C, g)
    got = oracle.route(q, cs, gs, L, C, g, 6, 2)
    qf, csf, gsf = oracle.bf16_to_f64(q), oracle.bf16_to_f64(cs), oracle.bf16_to_f64(gs)
    want = brute_route(qf, csf, gsf, L, C, g, 6, 2)
    assert got.tolist() == want
    # the block decision differs from any single query's in general; the max rule
    # must see all queries: dropping the last query changes the scores used
    sc_all = oracle.chunk_scores(q, cs)
    np.testing.assert_allclose(sc_all, (qf.sum(axis=1) @ csf.T).max(axis=0), rtol=1e-13, atol=1e-12)


def test_prefill_full_coverage_is_dense_causal():
    # With full coverage the cache part is every cache token, so query p of a block
    # starting at P attends exactly to [0, P+p]: dense causal attention.
    rng = np.random.default_rng(11)
    L0, nq, d, C, g, R = 8 * 32, 16, 16, 32, 8, 2
    K = rand_bf16(rng, (L0 + nq, d))
    V = rand_bf16(rng, (L0 + nq, d))
    q = rand_bf16(rng, (nq, R, d))
    cs, gs = oracle.summaries(K[:L0], C, g)
    tok = oracle.route(q, cs, gs, L0, C, g, k=100, G=C // g)
    assert tok.tolist() == list(range(L0))
    out = oracle.prefill_block(q, K, V, tok, P=L0)
    qf, Kf, Vf = (oracle.bf16_to_f64(x) for x in (q, K, V))
    for p in range(nq):
        want = dense_attention(qf[p], Kf[: L0 + p + 1], Vf[: L0 + p + 1], 1 / math.sqrt(d))
        np.testing.assert_allclose(out[p], want, rtol=0, atol=1e-12)


# ------------------------------------------------- block-then-token routing


def brute_hisa(q_f64, cs_f64, K_f64, L, C, m, k_tok):
    """Block-then-token routing by direct enumeration and Python sorting."""
    nf = L // C
    hs = q_f64.sum(axis=0)

    def score(v):
        return float(sum(hs[e] * v[e] for e in range(len(v))))

    if nf <= 2:
        cand = list(range(L))
    else:
        blocks = sorted(range(1, nf - 1), key=lambda c: (-score(cs_f64[c]), c))
        kept = sorted(blocks[:m])
        cand = list(range(C)) + [c * C + t for c in kept for t in range(C)] + list(range((nf - 1) * C, L))
    order = sorted(cand, key=lambda t: (-score(K_f64[t]), t))
    return sorted(order[:k_tok])


@pytest.mark.parametrize("seed", range(10))
def test_hisa_route_matches_brute_force(seed):
    rng = np.random.default_rng(300 + seed)
    C = int(rng.choice([8, 16, 32]))
    L = int(rng.integers(1, 12 * C))
    d = int(rng.choice([8, 16]))
    R = int(rng.integers(1, 5))
    m = int(rng.integers(1, 6))
    k_tok = int(rng.integers(1, 4 * C))
    K = rand_bf16(rng, (L, d))
    q = rand_bf16(rng, (R, d))
    cs, _ = oracle.summaries(K, C, 4)
    got, scored = oracle.hisa_route(q, cs, K, L, C, m, k_tok, return_scored=True)
    want = brute_hisa(oracle.bf16_to_f64(q), oracle.bf16_to_f64(cs), oracle.bf16_to_f64(K), L, C, m, k_tok)
    assert got.tolist() == want
    nf = L // C
    n_cand = oracle.hisa_candidates(L, C, m)
    assert len(got) == min(k_tok, n_cand)
    # the work the article's cost model counts: block summaries scored + candidate tokens scored
    assert scored == (nf - 2 if nf > 2 else 0) + n_cand


def test_hisa_full_coverage_keeps_every_token():
    rng = np.random.default_rng(7)
    L, C, d = 10 * 16 + 5, 16, 8
    K = rand_bf16(rng, (L, d))
    q = rand_bf16(rng, (3, d))
    cs, _ = oracle.summaries(K, C, 4)
    assert oracle.hisa_route(q, cs, K, L, C, 100, 10 * L).tolist() == list(range(L))


def test_hisa_ties_go_to_lower_position():
    # identical keys: every block and token score ties, so the lowest blocks and
    # then the lowest positions are kept
    L, C, d, m, k_tok = 8 * 16, 16, 8, 2, 20
    K = to_bf16_bits(np.ones((L, d)))
    q = to_bf16_bits(np.ones((2, d)))
    cs, _ = oracle.summaries(K, C, 4)
    assert oracle.hisa_route(q, cs, K, L, C, m, k_tok).tolist() == list(range(20))


def test_hisa_keeps_the_highest_scoring_candidates():
    # one key per candidate block made clearly highest along q: the token step must
    # keep exactly those (and the rest of the kept set scores no higher than them)
    rng = np.random.default_rng(11)
    L, C, d = 12 * 16, 16, 16
    Kf = rng.standard_normal((L, d)) * 0.1
    qf = np.zeros((1, d))
    qf[0, 0] = 1.0
    hot = [3, 70, 150, 190]  # first block, two middle blocks, the last block
    for t in hot:
        Kf[t, 0] = 4.0
    K = (torch.from_numpy(Kf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    q = to_bf16_bits(qf)
    cs, _ = oracle.summaries(K, C, 4)
    got = oracle.hisa_route(q, cs, K, L, C, 3, len(hot)).tolist()
    assert got == hot


def test_hisa_cost_matches_the_articles_model():
    # Summed over the queries of a long prefill, the scored vectors per query,
    # (L/C - 2) summaries + (m + 2) C tokens (+ the tail), total about
    # N^2 / (2C) + N (m + 2) C: the article's O(L^2/B + L m B) with B = C.
    C, m, N = 128, 32, 65536
    total = 0
    for L in range(1, N + 1):
        nf = L // C
        total += (nf - 2 if nf > 2 else 0) + oracle.hisa_candidates(L, C, m)
    model = N * N / (2 * C) + N * (m + 2) * C
    assert abs(total / model - 1.0) < 0.02
