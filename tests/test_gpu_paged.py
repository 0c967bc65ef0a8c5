"""GPU parity of batched decode on a paged K/V pool (16 ragged sequences of
4K-64K tokens, page = chunk = 128 tokens, shuffled page table) against the
oracle, which sees each sequence gathered back to contiguous memory. Every
(sequence, KV head) is checked: routed lists under the near-tie rule, hga_attend
on the oracle's lists, and the fused decode on the lists it chose."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_attention_close, assert_lse_close, assert_summaries_close, bits, check_route

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import hierarchical_routed_sparse_build_b200 as hga
    from hierarchical_routed_sparse_build_b200.runtime import RoutedCache
    hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, 0)
    w = synth.BATCHED_PAGED
    inp = synth.paged_inputs(w)
    c = RoutedCache(inp.k_pool, inp.v_pool, inp.seq_lens, chunk=w.chunk, group=w.group,
                    top_chunks=w.top_chunks, top_groups=w.top_groups, n_q_heads=w.n_q_heads,
                    page_table=inp.page_table)
    c.build_summaries()
    return hga, w, inp, c


def test_paged_lengths_and_table(setup):
    _, w, inp, _ = setup
    assert len(inp.seq_lens) == 16
    assert inp.seq_lens.min() >= 4096 and inp.seq_lens.max() <= 65536
    used = inp.page_table[inp.page_table >= 0]
    assert len(np.unique(used)) == used.size == inp.k_pool.shape[0]


@pytest.mark.parametrize("kernel", [2, 3], ids=["fused", "balanced"])
def test_paged_decode_matches_oracle(setup, kernel):
    hga, w, inp, c = setup
    q = c.q_tensor(inp.q)
    hga.hga_set_launch_option(hga.HGA_OPT_DECODE_KERNEL, kernel)
    try:
        out, lse, idx, n_idx = c.decode(q, want_idx=True)
    finally:
        hga.hga_set_launch_option(hga.HGA_OPT_DECODE_KERNEL, 0)
    st, b = hga.hga_get_device_error()
    assert st == 0, b
    cs_gpu, gs_gpu = bits(c.chunk_sum), bits(c.group_sum)
    idx_h, n_h = idx.cpu().numpy(), n_idx.cpu().numpy()
    out_h, lse_h = out.cpu().numpy(), lse.cpu().numpy()
    R = w.n_q_heads // w.n_kv_heads
    exact = total = 0
    o_idx = torch.zeros_like(idx)
    o_n = torch.zeros_like(n_idx)
    refs = {}
    for bi, L in enumerate(inp.seq_lens):
        L = int(L)
        K, V = inp.contiguous(bi)
        pages = inp.page_table[bi, : L // w.chunk]
        for h in range(w.n_kv_heads):
            qh = inp.q[bi, h * R:(h + 1) * R]
            cs, gs = oracle.summaries(K[h], w.chunk, w.group)
            assert_summaries_close(cs_gpu[pages, h], cs, f"chunk sums b{bi} h{h}")
            assert_summaries_close(gs_gpu[pages, h], gs, f"group sums b{bi} h{h}")
            tok = oracle.route(qh, cs, gs, L, w.chunk, w.group, w.top_chunks, w.top_groups)
            same = check_route(idx_h[bi, h, :n_h[bi, h]], qh, cs, gs, L, w.chunk, w.group, w.top_chunks,
                               w.top_groups, f"route b{bi} h{h}")
            exact += same
            total += 1
            o_idx[bi, h, :tok.size] = torch.from_numpy(tok).cuda()
            o_n[bi, h] = tok.size
            ref, rl = oracle.attend(qh, K[h], V[h], tok, with_lse=True)
            # the fused decode's output against the oracle's attention over the
            # list the decode chose (the oracle's own list when they agree)
            toks_d = idx_h[bi, h, :n_h[bi, h]].astype(np.int64)
            ref_d, rl_d = (ref, rl) if same else oracle.attend(qh, K[h], V[h], toks_d, with_lse=True)
            refs[(bi, h)] = (ref, rl, ref_d, rl_d)
    assert exact >= total - 2
    out_a, lse_a = c.attend(q, o_idx, o_n)
    st, b = hga.hga_get_device_error()
    assert st == 0, b
    out_a, lse_a = out_a.cpu().numpy(), lse_a.cpu().numpy()
    for (bi, h), (ref, rl, ref_d, rl_d) in refs.items():
        sl = slice(h * R, (h + 1) * R)
        assert_attention_close(out_a[bi, sl], ref, f"attend b{bi} h{h}")
        assert_lse_close(lse_a[bi, sl], rl, f"attend lse b{bi} h{h}")
        assert_attention_close(out_h[bi, sl], ref_d, f"decode b{bi} h{h}")
        assert_lse_close(lse_h[bi, sl], rl_d, f"decode lse b{bi} h{h}")


def test_bad_page_is_reported(setup):
    hga, w, inp, c = setup
    saved = c.page_table[3, 5].item()
    c.page_table[3, 5] = 10 ** 6
    try:
        c.decode(c.q_tensor(inp.q))
        st, b = hga.hga_get_device_error()
        assert st == 4 and (b & 2)
    finally:
        c.page_table[3, 5] = saved
    assert hga.hga_get_device_error() == (0, 0)
