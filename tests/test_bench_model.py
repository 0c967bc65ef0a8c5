"""The benchmark's algorithmic byte and flop counts (the numerators of its
roofline fractions) against a count taken from what the oracle actually routes:
summary rows scored, routed or kept tokens, and, for prefill, the (query, key)
pairs. CPU only."""
import numpy as np
import pytest

import bench
import oracle
import synth


def routed_bytes_by_count(w, inp, L):
    """Bytes one decode query reads and writes, counted from the oracle's routing of every KV head."""
    C, g, d, hkv, hq = w.chunk, w.group, w.head_dim, w.n_kv_heads, w.n_q_heads
    R = hq // hkv
    nf = L // C
    total = 0
    for h in range(hkv):
        K = np.ascontiguousarray(inp.k[0, h, :L])
        cs, gs = oracle.summaries(K, C, g)
        toks, kept = oracle.route(inp.q[0, h * R:(h + 1) * R], cs, gs, L, C, g, w.top_chunks, w.top_groups,
                                  return_chunks=True)
        n_cand = max(nf - 2, 0)
        routed_chunks = [c for c in kept if 0 < c < nf - 1]
        total += n_cand * d * 2                                  # candidate chunk summaries
        if w.top_groups < C // g:
            total += len(routed_chunks) * (C // g) * d * 2       # group summaries of routed chunks
        total += toks.size * d * 2 * 2                           # K and V of every routed token
    return total + hq * d * 2 + hq * d * 4 + hq * 4              # q in, out and lse


@pytest.mark.parametrize("L", [4096, 16384, 65536])
def test_decode_bytes_match_the_oracles_routing(L):
    w = synth.with_len(synth.DECODE_64K, L)
    inp = synth.decode_inputs(w, lengths=[L])
    assert bench.decode_bytes(L) == routed_bytes_by_count(w, inp, L)


def test_decode_bytes_at_64k_is_the_stated_figure():
    assert bench.decode_bytes(65536) == 5_527_680


@pytest.mark.parametrize("L,k_tok", [(16384, 2048), (65536, 2048), (65536, 8192), (300, 100)])
def test_hisa_bytes_match_the_oracles_scoring(L, k_tok):
    w = synth.with_len(synth.DECODE_64K, max(L, 384))
    inp = synth.decode_inputs(w, lengths=[L], max_len=max(L, 384))
    C, d, hkv, hq = w.chunk, w.head_dim, w.n_kv_heads, w.n_q_heads
    R = hq // hkv
    total = reread = logit_bytes = 0
    for h in range(hkv):
        K = np.ascontiguousarray(inp.k[0, h, :L])
        cs, _ = oracle.summaries(K, C, w.group)
        toks, scored = oracle.hisa_route(inp.q[0, h * R:(h + 1) * R], cs, K, L, C, w.top_chunks, k_tok,
                                         return_scored=True)
        n_cand = oracle.hisa_candidates(L, C, w.top_chunks)
        n_blocks = scored - n_cand                                   # block summaries scored
        token_rows = n_cand if n_cand > k_tok else 0                 # K rows the token step reads
        kept_rows = toks.size if token_rows else 2 * toks.size       # V (K too when no token step ran)
        total += (n_blocks + token_rows + kept_rows) * d * 2
        reread += toks.size * d * 2 if token_rows else 0             # kept K read again by the attention
        # or: 8 fp32 logits written per candidate, read back for the kept tokens
        logit_bytes += (n_cand + toks.size) * 8 * 4 if token_rows else 0
    total += hq * d * 2 + hq * d * 4 + hq * 4
    assert bench.hisa_bytes(L, k_tok) == total
    assert bench.hisa_bytes(L, k_tok, reread=True) == total + reread
    assert bench.hisa_bytes(L, k_tok, logits=True) == total + logit_bytes


def test_prefill_flops_count_every_query_key_pair():
    # a small prefill: 4 blocks of 64 queries on a 1536-token cache, routing from the oracle
    w = synth.Workload("pf_small", 1, 32, 4, 128, 1536, 128, 16, 4, 2, -1, 71, n_new=256, block=64)
    inp = synth.prefill_inputs(w)
    L0, T, blk = inp.cache_len, w.n_new, w.block
    R = w.n_q_heads // w.n_kv_heads
    pairs = 0
    routed_total = 0
    for b in range(T // blk):
        for h in range(w.n_kv_heads):
            K = np.ascontiguousarray(inp.k[0, h, :L0])
            cs, gs = oracle.summaries(K, w.chunk, w.group)
            qb = inp.q[b * blk:(b + 1) * blk, h * R:(h + 1) * R]
            toks = oracle.route(qb, cs, gs, L0, w.chunk, w.group, w.top_chunks, w.top_groups)
            routed_total += toks.size
            for i in range(blk):
                pairs += R * (toks.size + i + 1)   # routed cache keys + own causal prefix
    assert bench.prefill_flops(routed_total, (T // blk) * w.n_kv_heads, w) == 4 * w.head_dim * pairs
