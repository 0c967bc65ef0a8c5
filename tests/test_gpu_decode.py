"""GPU parity of the decode path (summaries, routing, attention, fused decode)
against the CPU oracle, through the C ABI. Every oracle input comes from the
seeded generator; nothing the GPU computes is fed to the oracle. Tolerances are
stated in tests/parity.py."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import (assert_attention_close, assert_lse_close, assert_summaries_close, bits, check_route,
                    scale_for)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hga():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import hierarchical_routed_sparse_build_b200 as m
    m.hga_set_launch_option(m.HGA_OPT_CTAS_PER_HEAD, 0)
    return m


@pytest.fixture(params=[2, 3], ids=["fused", "balanced"])
def decode_path(hga, request):
    """Run a test with the fused one-kernel decode and with the route + balanced
    attention pair (RoutedCache.decode calls hga_decode_ws)."""
    hga.hga_set_launch_option(hga.HGA_OPT_DECODE_KERNEL, request.param)
    yield request.param
    hga.hga_set_launch_option(hga.HGA_OPT_DECODE_KERNEL, 0)


def cache_for(hga, w, k, v, lens, page_table=None):
    from hierarchical_routed_sparse_build_b200.runtime import RoutedCache
    c = RoutedCache(k, v, lens, chunk=w.chunk, group=w.group, top_chunks=w.top_chunks,
                    top_groups=w.top_groups, n_q_heads=w.n_q_heads, page_table=page_table)
    c.build_summaries()
    return c


def no_device_error(hga):
    st, b = hga.hga_get_device_error()
    assert st == 0, f"device error bits {b}"


def oracle_unit(w, inp_k, inp_v, q, b, h, L):
    """Oracle summaries, routing and attention for (sequence b, KV head h)."""
    R = w.n_q_heads // w.n_kv_heads
    K = np.ascontiguousarray(inp_k[b, h, :L]) if inp_k.ndim == 4 else inp_k
    V = np.ascontiguousarray(inp_v[b, h, :L]) if inp_v.ndim == 4 else inp_v
    qh = np.ascontiguousarray(q[b, h * R:(h + 1) * R])
    cs, gs = oracle.summaries(K, w.chunk, w.group)
    tok = oracle.route(qh, cs, gs, L, w.chunk, w.group, w.top_chunks, w.top_groups)
    out, lse = oracle.attend(qh, K, V, tok, with_lse=True)
    return dict(K=K, V=V, q=qh, cs=cs, gs=gs, tok=tok, out=out, lse=lse)


def run_and_check(hga, w, inp, units=None, check_summaries=True):
    """Build, route, attend (on oracle-chosen lists) and decode; compare each with the oracle."""
    c = cache_for(hga, w, inp.k, inp.v, inp.seq_lens)
    q = c.q_tensor(inp.q)
    idx, n_idx = c.route(q)
    out_d, lse_d, idx_d, n_idx_d = c.decode(q, want_idx=True)
    no_device_error(hga)
    R = w.n_q_heads // w.n_kv_heads
    B = len(inp.seq_lens)
    units = units or [(b, h) for b in range(B) for h in range(w.n_kv_heads)]
    idx_h, n_h = idx.cpu().numpy(), n_idx.cpu().numpy()
    idx_dh, n_dh = idx_d.cpu().numpy(), n_idx_d.cpu().numpy()
    assert np.array_equal(n_dh, n_h)
    out_h, lse_h = out_d.cpu().numpy(), lse_d.cpu().numpy()
    cs_gpu, gs_gpu = bits(c.chunk_sum), bits(c.group_sum)
    # attention on the oracle's own token lists
    o_idx = torch.zeros_like(idx)
    o_n = torch.zeros_like(n_idx)
    refs = {}
    for (b, h) in units:
        L = int(inp.seq_lens[b])
        ref = oracle_unit(w, inp.k, inp.v, inp.q, b, h, L)
        refs[(b, h)] = ref
        o_idx[b, h, :ref["tok"].size] = torch.from_numpy(ref["tok"]).to(o_idx.device)
        o_n[b, h] = ref["tok"].size
    out_a, lse_a = c.attend(q, o_idx, o_n)
    no_device_error(hga)
    out_a, lse_a = out_a.cpu().numpy(), lse_a.cpu().numpy()
    exact = 0
    for (b, h), ref in refs.items():
        L = int(inp.seq_lens[b])
        nf = L // w.chunk
        if check_summaries and nf > 0:
            assert_summaries_close(cs_gpu[b, h, :nf], ref["cs"], f"chunk sums b{b} h{h}")
            assert_summaries_close(gs_gpu[b, h, :nf], ref["gs"], f"group sums b{b} h{h}")
        toks = idx_h[b, h, :n_h[b, h]]
        same = check_route(toks, ref["q"], ref["cs"], ref["gs"], L, w.chunk, w.group, w.top_chunks,
                           w.top_groups, f"route b{b} h{h}")
        exact += same
        sl = slice(h * R, (h + 1) * R)
        assert_attention_close(out_a[b, sl], ref["out"], f"attend b{b} h{h}")
        assert_lse_close(lse_a[b, sl], ref["lse"], f"attend lse b{b} h{h}")
        # the fused decode routes on its own (fp32 scores summed in another order
        # than hga_route): its list must pass the same check, and its attention
        # must match the oracle's attention over that list
        toks_d = idx_dh[b, h, :n_dh[b, h]]
        if not np.array_equal(toks_d, toks):
            check_route(toks_d, ref["q"], ref["cs"], ref["gs"], L, w.chunk, w.group, w.top_chunks, w.top_groups,
                        f"decode route b{b} h{h}")
        ref_d, lse_ref_d = (ref["out"], ref["lse"]) if np.array_equal(toks_d, ref["tok"]) else \
            oracle.attend(ref["q"], ref["K"], ref["V"], toks_d.astype(np.int64), with_lse=True)
        assert_attention_close(out_h[b, sl], ref_d, f"decode b{b} h{h}")
        assert_lse_close(lse_h[b, sl], lse_ref_d, f"decode lse b{b} h{h}")
    return exact, len(refs)


def test_tiny_decode_4k(hga, decode_path):
    w = synth.TINY_DECODE_4K
    inp = synth.decode_inputs(w)
    exact, n = run_and_check(hga, w, inp)
    assert exact == n


def test_decode_16k(hga, decode_path):
    w = synth.DECODE_16K
    exact, n = run_and_check(hga, w, synth.decode_inputs(w))
    assert exact >= n - 1


def test_decode_64k(hga, decode_path):
    w = synth.DECODE_64K
    exact, n = run_and_check(hga, w, synth.decode_inputs(w))
    assert exact >= n - 1


@pytest.mark.parametrize("L", [4096, 8192, 32768])
def test_decode_sweep_lengths(hga, decode_path, L):
    w = synth.with_len(synth.DECODE_64K, L)
    exact, n = run_and_check(hga, w, synth.decode_inputs(w))
    assert exact >= n - 1


def test_ragged_batch_edge_lengths(hga, decode_path):
    # dense cases (fewer than 3 full chunks), exact chunk multiples, ragged tails,
    # a single token, and an empty sequence, in one batch
    w = synth.Workload("edge", 1, 32, 4, 128, 0, 128, 16, 4, 2, -1, 7)
    lens = [0, 1, 15, 16, 17, 255, 383, 384, 385, 1000, 1024, 2049, 5000]
    inp = synth.decode_inputs(w, lengths=lens, max_len=5120)
    run_and_check(hga, w, inp)
    c = cache_for(hga, w, inp.k, inp.v, inp.seq_lens)
    out, lse = c.decode(c.q_tensor(inp.q))
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))


@pytest.mark.parametrize("hq,hkv,d", [(4, 4, 128), (12, 4, 64), (6, 2, 128), (8, 1, 64)])
def test_head_shapes(hga, decode_path, hq, hkv, d):
    w = synth.Workload(f"heads{hq}x{hkv}x{d}", 1, hq, hkv, d, 3000, 64, 16, 6, 2, -1, 11)
    inp = synth.decode_inputs(w, lengths=[3000, 2500], max_len=3000)
    run_and_check(hga, w, inp)


def test_full_coverage_is_dense_attention(hga, decode_path):
    # top_chunks >= candidates and top_groups = C/g: every token is routed, so the
    # output must be dense attention over the whole context.
    w = synth.Workload("full", 1, 32, 4, 128, 2000, 64, 16, 1000, 4, -1, 13)
    inp = synth.decode_inputs(w, lengths=[2000, 1337], max_len=2000)
    c = cache_for(hga, w, inp.k, inp.v, inp.seq_lens)
    out, _, idx, n_idx = c.decode(c.q_tensor(inp.q), want_idx=True)
    no_device_error(hga)
    for b, L in enumerate(inp.seq_lens):
        for h in range(4):
            assert n_idx[b, h].item() == L
            assert np.array_equal(idx[b, h, :L].cpu().numpy(), np.arange(L))
            ref = oracle.attend(inp.q[b, h * 8:(h + 1) * 8], inp.k[b, h, :L], inp.v[b, h, :L], np.arange(L))
            assert_attention_close(out[b, h * 8:(h + 1) * 8].cpu().numpy(), ref, f"dense b{b} h{h}")


@pytest.mark.parametrize("kernel", [1, 2, 3])
@pytest.mark.parametrize("ctas", [1, 2, 3, 8, 16])
def test_cluster_sizes_agree(hga, ctas, kernel):
    w = synth.with_len(synth.DECODE_64K, 16384)
    inp = synth.decode_inputs(w)
    hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, ctas)
    hga.hga_set_launch_option(hga.HGA_OPT_DECODE_KERNEL, kernel)
    try:
        exact, n = run_and_check(hga, w, inp, check_summaries=False)
    finally:
        hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, 0)
        hga.hga_set_launch_option(hga.HGA_OPT_DECODE_KERNEL, 0)
    assert exact >= n - 1


def test_one_cta_per_head_ragged_and_paged(hga):
    # one CTA per (sequence, KV head), the automatic choice above 148 units, on
    # ragged lengths (dense units included), then the same sequences in shuffled
    # pages: the paged decode must equal the contiguous one bit for bit
    w = synth.Workload("onecta", 1, 32, 4, 128, 0, 128, 16, 6, 2, -1, 61)
    lens = [0, 1, 200, 383, 384, 385, 700, 1024, 2049, 3000, 4095, 4096]
    inp = synth.decode_inputs(w, lengths=lens, max_len=4096)
    hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, 1)
    try:
        exact, n = run_and_check(hga, w, inp, check_summaries=False)
        assert exact >= n - 1
        B, per = len(lens), 4096 // 128
        table = np.random.default_rng(13).permutation(B * per).astype(np.int32).reshape(B, per)
        kpool = np.zeros((B * per, 4, 128, 128), dtype=np.uint16)
        vpool = np.zeros_like(kpool)
        for b in range(B):
            kpool[table[b]] = inp.k[b].reshape(4, per, 128, 128).transpose(1, 0, 2, 3)
            vpool[table[b]] = inp.v[b].reshape(4, per, 128, 128).transpose(1, 0, 2, 3)
        c = cache_for(hga, w, kpool, vpool, inp.seq_lens, page_table=table)
        out_p, lse_p, idx_p, n_p = c.decode(c.q_tensor(inp.q), want_idx=True)
        no_device_error(hga)
        c2 = cache_for(hga, w, inp.k, inp.v, inp.seq_lens)
        out_c, lse_c, idx_c, n_c = c2.decode(c2.q_tensor(inp.q), want_idx=True)
        no_device_error(hga)
        assert torch.equal(n_p, n_c) and torch.equal(idx_p, idx_c)
        assert torch.equal(out_p, out_c) and torch.equal(lse_p, lse_c)
    finally:
        hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, 0)


@pytest.mark.parametrize("group,chunk,top_groups", [(8, 128, 4), (32, 128, 2), (16, 64, 4), (16, 256, 3)])
def test_group_sizes(hga, decode_path, group, chunk, top_groups):
    # g = 8 runs the phase-by-phase kernel (a 16-token tile spans two groups);
    # g = 32 and chunk 256 run the fused kernel with two tiles per group and 16
    # groups per chunk; top_groups = C/g (all groups) runs its whole-chunk path
    w = synth.Workload(f"g{group}c{chunk}", 1, 32, 4, 128, 6000, chunk, group, 5, top_groups, -1, 23)
    inp = synth.decode_inputs(w, lengths=[6000, 4099, 777], max_len=6016)
    exact, n = run_and_check(hga, w, inp)
    assert exact >= n - 1
    w_all = synth.Workload(f"g{group}c{chunk}all", 1, 32, 4, 128, 6000, chunk, group, 5, chunk // group, -1, 29)
    inp = synth.decode_inputs(w_all, lengths=[6000, 2222], max_len=6016)
    run_and_check(hga, w_all, inp)


def test_attend_arbitrary_token_order_and_ragged_list(hga):
    # hga_attend takes any token list: unsorted, with a ragged last tile
    w = synth.Workload("anyorder", 1, 32, 4, 128, 3000, 128, 16, 4, 2, -1, 17)
    inp = synth.decode_inputs(w, lengths=[3000])
    c = cache_for(hga, w, inp.k, inp.v, inp.seq_lens)
    rng = np.random.default_rng(3)
    idx = torch.zeros((1, 4, 64), dtype=torch.int32, device="cuda")
    n = torch.zeros((1, 4), dtype=torch.int32, device="cuda")
    lists = {}
    for h in range(4):
        t = rng.choice(3000, size=37 + 5 * h, replace=False).astype(np.int32)
        lists[h] = t
        idx[0, h, :t.size] = torch.from_numpy(t).cuda()
        n[0, h] = t.size
    out, lse = c.attend(c.q_tensor(inp.q), idx, n)
    no_device_error(hga)
    for h in range(4):
        ref, rl = oracle.attend(inp.q[0, h * 8:(h + 1) * 8], inp.k[0, h], inp.v[0, h], lists[h], with_lse=True)
        assert_attention_close(out[0, h * 8:(h + 1) * 8].cpu().numpy(), ref, f"attend h{h}")
        assert_lse_close(lse[0, h * 8:(h + 1) * 8].cpu().numpy(), rl, f"lse h{h}")


def test_device_errors_are_reported_not_faulted(hga, decode_path):
    w = synth.Workload("err", 1, 8, 1, 128, 1024, 128, 16, 2, 2, -1, 19)
    inp = synth.decode_inputs(w, lengths=[1024, 512])
    c = cache_for(hga, w, inp.k, inp.v, inp.seq_lens)
    no_device_error(hga)
    q = c.q_tensor(inp.q)
    # a sequence length beyond max_len: the kernel treats it as empty and reports
    c.seq_lens[1] = 5000
    out, lse = c.decode(q)
    st, b = hga.hga_get_device_error()
    assert st == 4 and (b & 1)
    assert torch.all(out[1] == 0)
    assert hga.hga_get_device_error() == (0, 0)  # the word was cleared
    c.seq_lens[1] = 512
    # token indices outside the sequence in hga_attend
    idx = torch.tensor([[[0, 5, 4000, -3]], [[1, 2, 3, 4]]], dtype=torch.int32, device="cuda")
    n = torch.tensor([[4], [4]], dtype=torch.int32, device="cuda")
    c.attend(q, idx, n)
    st, b = hga.hga_get_device_error()
    assert st == 4 and (b & 4)
    # n_idx above the stride
    n[0, 0] = 99
    c.attend(q, idx, n)
    st, b = hga.hga_get_device_error()
    assert st == 4 and (b & 4)
    assert hga.hga_get_device_error() == (0, 0)
