"""GPU parity of block-then-token routed decode (hga_decode_hisa: top chunks by
summary, then the top tokens inside them, then exact attention) against the
CPU oracle, through the C ABI. Lists are checked with the near-tie rule of
tests/parity.py; attention against the oracle's attention over the GPU list."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_attention_close, assert_lse_close, check_hisa_route

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hga():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import hierarchical_routed_sparse_build_b200 as m
    m.hga_set_launch_option(m.HGA_OPT_CTAS_PER_HEAD, 0)
    return m


@pytest.fixture(params=[True, False], ids=["logits_workspace", "k_reread"])
def logits(request):
    """hga_decode_hisa_ws (per-head logits kept from the token step) or hga_decode_hisa (K read again)."""
    return request.param


def run_hisa(hga, w, inp, m, k_tok, units=None, page_table=None, k_pool=None, v_pool=None, logits=True):
    from hierarchical_routed_sparse_build_b200.runtime import RoutedCache
    if page_table is None:
        c = RoutedCache(inp.k, inp.v, inp.seq_lens, chunk=w.chunk, group=w.group, top_chunks=m,
                        top_groups=w.top_groups, n_q_heads=w.n_q_heads)
    else:
        c = RoutedCache(k_pool, v_pool, inp.seq_lens, chunk=w.chunk, group=w.group, top_chunks=m,
                        top_groups=w.top_groups, n_q_heads=w.n_q_heads, page_table=page_table)
    c.build_summaries()
    out, lse, idx, n_idx = c.decode_hisa(c.q_tensor(inp.q), k_tok, want_idx=True, logits_workspace=logits)
    st, b = hga.hga_get_device_error()
    assert st == 0, b
    R = w.n_q_heads // w.n_kv_heads
    idx_h, n_h, out_h, lse_h = idx.cpu().numpy(), n_idx.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()
    units = units or [(b_, h) for b_ in range(len(inp.seq_lens)) for h in range(w.n_kv_heads)]
    exact = 0
    for (b_, h) in units:
        L = int(inp.seq_lens[b_])
        K = np.ascontiguousarray(inp.k[b_, h, :L])
        V = np.ascontiguousarray(inp.v[b_, h, :L])
        qh = np.ascontiguousarray(inp.q[b_, h * R:(h + 1) * R])
        cs, _ = oracle.summaries(K, w.chunk, w.group)
        toks = idx_h[b_, h, :n_h[b_, h]]
        exact += check_hisa_route(toks, qh, cs, K, L, w.chunk, m, k_tok, f"hisa b{b_} h{h}")
        ref, rl = oracle.attend(qh, K, V, toks.astype(np.int64), with_lse=True)
        sl = slice(h * R, (h + 1) * R)
        assert_attention_close(out_h[b_, sl], ref, f"hisa attn b{b_} h{h}")
        assert_lse_close(lse_h[b_, sl], rl, f"hisa lse b{b_} h{h}")
    return exact, len(units)


def test_hisa_decode_16k(hga, logits):
    w = synth.DECODE_16K
    inp = synth.decode_inputs(w)
    exact, n = run_hisa(hga, w, inp, m=16, k_tok=1024, logits=logits)
    assert exact >= n - 1


@pytest.mark.parametrize("ctas", [1, 3, 8])
def test_hisa_cluster_sizes(hga, ctas, logits):
    w = synth.with_len(synth.DECODE_64K, 12000)
    inp = synth.decode_inputs(w, lengths=[12000, 9999], max_len=12032)
    hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, ctas)
    try:
        exact, n = run_hisa(hga, w, inp, m=8, k_tok=700, logits=logits)
    finally:
        hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, 0)
    assert exact >= n - 1


def test_hisa_edge_lengths(hga, logits):
    # empty, dense (< 3 chunks), candidates fewer than the tokens to keep, ragged tails
    w = synth.Workload("hisa_edge", 1, 32, 4, 128, 0, 128, 16, 4, 2, -1, 31)
    lens = [0, 1, 200, 383, 384, 700, 1000, 2049, 5000]
    inp = synth.decode_inputs(w, lengths=lens, max_len=5120)
    run_hisa(hga, w, inp, m=4, k_tok=300, logits=logits)


@pytest.mark.parametrize("hq,hkv,d", [(8, 1, 64), (12, 4, 64), (6, 2, 128)])
def test_hisa_head_shapes(hga, hq, hkv, d, logits):
    w = synth.Workload(f"hisa{hq}x{hkv}x{d}", 1, hq, hkv, d, 4000, 64, 16, 6, 2, -1, 37)
    inp = synth.decode_inputs(w, lengths=[4000, 3333], max_len=4032)
    run_hisa(hga, w, inp, m=6, k_tok=256, logits=logits)


def test_hisa_paged(hga, logits):
    w = synth.Workload("hisa_paged", 1, 32, 4, 128, 9000, 128, 16, 8, 2, -1, 41)
    lens = np.array([9000, 4100, 6400], dtype=np.int32)
    inp = synth.decode_inputs(w, lengths=list(lens), max_len=9088)
    per = 9088 // 128
    table = np.random.default_rng(3).permutation(3 * per).astype(np.int32).reshape(3, per)
    kpool = np.zeros((3 * per, 4, 128, 128), dtype=np.uint16)
    vpool = np.zeros_like(kpool)
    for b in range(3):
        kpool[table[b]] = inp.k[b].reshape(4, per, 128, 128).transpose(1, 0, 2, 3)
        vpool[table[b]] = inp.v[b].reshape(4, per, 128, 128).transpose(1, 0, 2, 3)
    exact, n = run_hisa(hga, w, inp, m=8, k_tok=1024, page_table=table, k_pool=kpool, v_pool=vpool, logits=logits)
    assert exact >= n - 1


def test_hisa_full_coverage_is_dense_attention(hga):
    w = synth.Workload("hisa_full", 1, 32, 4, 128, 2000, 64, 16, 1000, 4, -1, 43)
    inp = synth.decode_inputs(w, lengths=[2000, 1337], max_len=2048)
    from hierarchical_routed_sparse_build_b200.runtime import RoutedCache
    c = RoutedCache(inp.k, inp.v, inp.seq_lens, chunk=64, group=16, top_chunks=1000, top_groups=4, n_q_heads=32)
    c.build_summaries()
    out, _, idx, n_idx = c.decode_hisa(c.q_tensor(inp.q), 4096, want_idx=True)
    for b, L in enumerate(inp.seq_lens):
        for h in range(4):
            assert n_idx[b, h].item() == L
            assert np.array_equal(idx[b, h, :L].cpu().numpy(), np.arange(L))
            ref = oracle.attend(inp.q[b, h * 8:(h + 1) * 8], inp.k[b, h, :L], inp.v[b, h, :L], np.arange(L))
            assert_attention_close(out[b, h * 8:(h + 1) * 8].cpu().numpy(), ref, f"dense b{b} h{h}")


def test_hisa_decode_64k_sampled(hga, logits):
    w = synth.DECODE_64K
    inp = synth.decode_inputs(w, lengths=[w.ctx_len] * 2)
    exact, n = run_hisa(hga, w, inp, m=32, k_tok=2048, units=[(0, 0), (0, 3), (1, 1)], logits=logits)
    assert exact >= n - 1


@pytest.mark.parametrize("ctas", [0, 3])
def test_hisa_ties_take_lower_positions(hga, ctas, logits):
    # every key equal: all chunk summaries and all token scores tie, so the kept
    # set is the first k_tok candidates by position (the select's refinement path)
    w = synth.Workload("hisa_ties", 1, 32, 4, 128, 9000, 128, 16, 8, 2, -1, 47)
    inp = synth.decode_inputs(w, lengths=[9000, 6100], max_len=9088)
    inp.k[:] = inp.k[:, :, :1, :]
    hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, ctas)
    try:
        from hierarchical_routed_sparse_build_b200.runtime import RoutedCache
        c = RoutedCache(inp.k, inp.v, inp.seq_lens, chunk=128, group=16, top_chunks=8, top_groups=2, n_q_heads=32)
        c.build_summaries()
        out, _, idx, n_idx = c.decode_hisa(c.q_tensor(inp.q), 700, want_idx=True, logits_workspace=logits)
        assert hga.hga_get_device_error()[0] == 0
    finally:
        hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, 0)
    for b, L in enumerate(inp.seq_lens):
        assert oracle.hisa_candidates(int(L), 128, 8) > 700
        for h in range(4):
            K = inp.k[b, h, :L]
            cs, _ = oracle.summaries(K, 128, 16)
            ref = oracle.hisa_route(inp.q[b, h * 8:(h + 1) * 8], cs, K, int(L), 128, 8, 700)
            assert np.array_equal(ref, np.arange(700))  # chunks 1..8 win their ties
            assert n_idx[b, h].item() == 700
            assert np.array_equal(idx[b, h, :700].cpu().numpy(), ref), f"ties b{b} h{h}"


def test_hisa_many_blocks(hga, logits):
    # 64 kept chunks of 126 at 16K: 8448 candidate tokens in shared memory
    w = synth.DECODE_16K
    inp = synth.decode_inputs(w, lengths=[w.ctx_len] * 2)
    exact, n = run_hisa(hga, w, inp, m=64, k_tok=3000, units=[(0, 0), (0, 2), (1, 3)], logits=logits)
    assert exact >= n - 1
