"""Parity helpers shared by the GPU tests: compare the CUDA path with the oracle.

Tolerances (stated once, used everywhere):
  - summaries: within 1 bfloat16 ulp of the oracle's double-precision mean
    (the GPU accumulates in fp32 before the single bf16 rounding);
  - routed index sets: bit-exact, except at a selection boundary where the
    oracle's k-th and (k+1)-th scores are within 1e-3 relative: there any set
    whose members all score >= s_(k+1) - tol and whose non-members all score
    <= s_k + tol passes (tol = 1e-3 * max(|s_k|, 1e-6));
  - attention outputs: |gpu - oracle| <= 2e-3 + 1e-2 * |oracle| elementwise, the
    oracle run in double precision over the token set the GPU chose;
  - log-sum-exp: |gpu - oracle| <= 1e-3 + 1e-3 * |oracle|.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

ATOL, RTOL = 2e-3, 1e-2
LSE_ATOL, LSE_RTOL = 1e-3, 1e-3
TIE_REL = 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    """bfloat16 CUDA/CPU tensor -> numpy uint16 bit patterns."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def assert_summaries_close(gpu_bits: np.ndarray, ref_bits: np.ndarray, what: str) -> None:
    g = oracle.bf16_to_f64(gpu_bits)
    r = oracle.bf16_to_f64(ref_bits)
    mag = np.maximum(np.abs(g), np.abs(r))
    ulp = np.where(mag > 0, np.exp2(np.floor(np.log2(np.where(mag > 0, mag, 1.0))) - 7), 2.0**-133)
    bad = np.abs(g - r) > ulp
    assert not bad.any(), f"{what}: {bad.sum()} values differ by more than 1 bf16 ulp"
    exact = np.mean(gpu_bits == ref_bits)
    assert exact > 0.99, f"{what}: only {exact:.4f} bit-exact"


def _check_selection(scores: dict, chosen: set, n_keep: int, what: str) -> None:
    """Near-tie rule on one selection: scores {id: double score}, chosen ids."""
    assert len(chosen) == n_keep, f"{what}: kept {len(chosen)} != {n_keep}"
    if n_keep == len(scores):
        assert chosen == set(scores), what
        return
    order = sorted(scores, key=lambda i: (-scores[i], i))
    s_k, s_k1 = scores[order[n_keep - 1]], scores[order[n_keep]]
    if chosen == set(order[:n_keep]):
        return
    tol = TIE_REL * max(abs(s_k), 1e-6)
    lo = min(scores[i] for i in chosen)
    hi = max(scores[i] for i in scores if i not in chosen)
    assert lo >= s_k1 - tol and hi <= s_k + tol, (
        f"{what}: selection differs from the oracle beyond the near-tie rule "
        f"(s_k={s_k}, s_k+1={s_k1}, min kept={lo}, max dropped={hi})")


def check_route(tokens: np.ndarray, q_heads: np.ndarray, cs: np.ndarray, gs: np.ndarray, L: int,
                C: int, g: int, k: int, G: int, what: str = "route") -> bool:
    """Check a routed token list against the oracle's routing on the same summaries.

    q_heads [R][d] (or [n_q][R][d] for a prefill block), cs [nf][d], gs [nf][C/g][d]
    (bfloat16 bits). Returns True when the list equals the oracle's exactly.
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    want = oracle.route(q_heads, cs, gs, L, C, g, k, G)
    if tokens.shape == want.shape and np.array_equal(tokens, want):
        return True
    nf = L // C
    assert nf > 2, f"{what}: dense case must match exactly"
    assert np.all(np.diff(tokens) > 0), f"{what}: not ascending"
    assert tokens.size == want.size, f"{what}: size {tokens.size} != {want.size}"
    assert np.array_equal(tokens[:C], np.arange(C)), f"{what}: sink chunk"
    tail = np.arange((nf - 1) * C, L)
    assert np.array_equal(tokens[-tail.size:], tail), f"{what}: local chunk"
    mid = tokens[C:tokens.size - tail.size]
    chunks = sorted(set((mid // C).tolist()))
    cscore = oracle.chunk_scores(q_heads, cs)
    _check_selection({c: cscore[c] for c in range(1, nf - 1)}, set(chunks), min(k, nf - 2), what + " chunks")
    gpc = C // g
    for c in chunks:
        in_c = mid[(mid // C) == c]
        groups = sorted(set(((in_c - c * C) // g).tolist()))
        for j in groups:
            assert np.array_equal(in_c[(in_c - c * C) // g == j], np.arange(c * C + j * g, c * C + (j + 1) * g)), \
                f"{what}: group {c}/{j} incomplete"
        gscore = oracle.group_scores(q_heads, gs[c])
        _check_selection({j: gscore[j] for j in range(gpc)}, set(groups), min(G, gpc), f"{what} groups of {c}")
    return False


def assert_attention_close(gpu: np.ndarray, ref: np.ndarray, what: str) -> None:
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - ref)
    lim = ATOL + RTOL * np.abs(ref)
    bad = err > lim
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside 2e-3 abs + 1e-2 rel; "
                           f"max err {err.max():.3g}")


def assert_lse_close(gpu: np.ndarray, ref: np.ndarray, what: str) -> None:
    gpu = np.asarray(gpu, dtype=np.float64)
    both_inf = np.isneginf(gpu) & np.isneginf(ref)
    with np.errstate(invalid="ignore"):  # -inf - -inf where both are empty
        err = np.where(both_inf, 0.0, np.abs(gpu - ref))
    assert (err <= LSE_ATOL + LSE_RTOL * np.where(both_inf, 0.0, np.abs(ref))).all(), f"{what}: lse max err {err.max()}"


def scale_for(d: int) -> float:
    return 1.0 / math.sqrt(d)


def check_hisa_route(tokens: np.ndarray, q_heads: np.ndarray, cs: np.ndarray, K: np.ndarray, L: int, C: int,
                     m: int, k_tok: int, what: str = "hisa route") -> bool:
    """Check a block-then-token list against oracle.hisa_route on the same summaries and keys.

    Returns True when it equals the oracle's list. Otherwise it must have the oracle's length, be
    ascending inside [0, L), come from allowed blocks (first, last + tail, or a middle block scoring
    within the near-tie rule of the block boundary) and, when its visible blocks are the oracle's,
    be a top-k_tok of the oracle's candidates under the near-tie rule.
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    want = oracle.hisa_route(q_heads, cs, K, L, C, m, k_tok)
    if tokens.shape == want.shape and np.array_equal(tokens, want):
        return True
    assert tokens.size == want.size, f"{what}: size {tokens.size} != {want.size}"
    assert np.all(np.diff(tokens) > 0) and tokens.min() >= 0 and tokens.max() < L, f"{what}: not a valid list"
    nf = L // C
    tau = oracle.token_scores(q_heads, np.ascontiguousarray(K[:L]))
    if nf <= 2:
        cands = list(range(L))
    else:
        cscore = oracle.chunk_scores(q_heads, cs[:nf])
        r = min(m, nf - 2)
        order = sorted(range(1, nf - 1), key=lambda c: (-cscore[c], c))
        kept = set(order[:r])
        visible = {int(t) // C for t in tokens if C <= t < (nf - 1) * C}
        if r < nf - 2:
            s_r, s_r1 = cscore[order[r - 1]], cscore[order[r]]
            tol = TIE_REL * max(abs(s_r), 1e-6)
            for c in visible:
                assert cscore[c] >= s_r1 - tol, f"{what}: block {c} is not among the top blocks"
        if not visible <= kept:
            return False  # a near-tie block swap: the token step ran on other candidates
        cands = list(range(C)) + [c * C + t for c in sorted(kept) for t in range(C)] + list(range((nf - 1) * C, L))
    _check_selection({t: tau[t] for t in cands}, set(tokens.tolist()), tokens.size, what + " tokens")
    return False
