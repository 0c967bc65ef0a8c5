"""GPU checks of the chunk select at its edges, and of the decode at the launch
configuration the benchmark times, against the CPU oracle through the C ABI.

Ties: with every key equal, every chunk and group summary is the same bf16
vector, so every chunk score and every group score is bit-identical on the GPU
(the same dot products in the same order for every row) and in the oracle. The
tie rule (higher score first, then lower chunk / group index) then fixes the
routed list exactly: chunks 1..k, groups 0..G-1. With 638 candidate chunks all
in one histogram bucket, the select of the fused decode and of the balanced
pair's route kernel cannot rank the boundary bucket in its 512-key
shared-memory area and takes its fallback scan over all keys; the
phase-by-phase kernel (hga_route) ranks them in its larger area. All must give
the oracle's list bit for bit, at one and at eight CTAs per (sequence, KV
head).

Benchmark configuration: 64K-token sequences decoded with one CTA per
(sequence, KV head), the shape the automatic choice takes for a batch of 64;
every routed list and every output is checked.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_attention_close, assert_lse_close, check_route

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hga():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import hierarchical_routed_sparse_build_b200 as m
    m.hga_set_launch_option(m.HGA_OPT_CTAS_PER_HEAD, 0)
    m.hga_set_launch_option(m.HGA_OPT_DECODE_KERNEL, 0)
    return m


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def no_device_error(hga):
    st, b = hga.hga_get_device_error()
    assert st == 0, f"device error bits {b}"


@pytest.fixture(scope="module")
def tied_cache(hga):
    """Two sequences (40997 and 33000 tokens) whose keys are all one vector."""
    from hierarchical_routed_sparse_build_b200.runtime import RoutedCache
    rng = np.random.default_rng(4242)
    B, hq, hkv, d, C, g, k, G = 2, 32, 4, 128, 64, 16, 32, 2
    lens = [40997, 33000]  # 640 and 515 full chunks: 638 and 513 candidates, both above 512
    Lmax = max(lens)
    key = to_bf16_bits(rng.standard_normal(d))
    K = np.broadcast_to(key, (B, hkv, Lmax, d)).copy()
    V = to_bf16_bits(rng.standard_normal((B, hkv, Lmax, d)))
    q = to_bf16_bits(rng.standard_normal((B, hq, d)))
    c = RoutedCache(K, V, lens, chunk=C, group=g, top_chunks=k, top_groups=G, n_q_heads=hq)
    c.build_summaries()
    no_device_error(hga)
    want = {}
    R = hq // hkv
    for b, L in enumerate(lens):
        for h in range(hkv):
            qh = np.ascontiguousarray(q[b, h * R:(h + 1) * R])
            cs, gs = oracle.summaries(np.ascontiguousarray(K[b, h, :L]), C, g)
            tok = oracle.route(qh, cs, gs, L, C, g, k, G)
            nf = L // C
            # the tie rule written out: sink, chunks 1..k with groups 0..G-1, local chunk + tail
            expect = list(range(C)) + [c_ * C + t for c_ in range(1, k + 1) for t in range(G * g)] + \
                list(range((nf - 1) * C, L))
            assert tok.tolist() == expect
            ref, rl = oracle.attend(qh, np.ascontiguousarray(K[b, h, :L]), np.ascontiguousarray(V[b, h, :L]), tok,
                                    with_lse=True)
            want[(b, h)] = (tok, ref, rl)
    return dict(c=c, q=c.q_tensor(q), lens=lens, want=want, R=R)


@pytest.mark.parametrize("kernel", [1, 2, 3], ids=["phase_by_phase", "fused", "balanced"])
@pytest.mark.parametrize("ctas", [1, 8])
def test_all_tied_scores_keep_the_lowest_ids(hga, tied_cache, ctas, kernel):
    c, q, R = tied_cache["c"], tied_cache["q"], tied_cache["R"]
    hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, ctas)
    hga.hga_set_launch_option(hga.HGA_OPT_DECODE_KERNEL, kernel)
    try:
        idx_r, n_r = c.route(q)
        out, lse, idx_d, n_d = c.decode(q, want_idx=True)
        no_device_error(hga)
    finally:
        hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, 0)
        hga.hga_set_launch_option(hga.HGA_OPT_DECODE_KERNEL, 0)
    idx_r, n_r, idx_d, n_d = idx_r.cpu().numpy(), n_r.cpu().numpy(), idx_d.cpu().numpy(), n_d.cpu().numpy()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for (b, h), (tok, ref, rl) in tied_cache["want"].items():
        assert np.array_equal(idx_r[b, h, :n_r[b, h]], tok), f"hga_route b{b} h{h}: not the lowest ids"
        assert np.array_equal(idx_d[b, h, :n_d[b, h]], tok), f"hga_decode b{b} h{h}: not the lowest ids"
        sl = slice(h * R, (h + 1) * R)
        assert_attention_close(out[b, sl], ref, f"tied decode b{b} h{h}")
        assert_lse_close(lse[b, sl], rl, f"tied decode lse b{b} h{h}")


@pytest.mark.parametrize("kernel", [2, 3], ids=["fused", "balanced"])
def test_decode_64k_at_the_benchmark_launch_shape(hga, kernel):
    """16 sequences of 65536 tokens (8 drawn, each repeated in separate memory, as
    the benchmark builds its batch), one CTA per (sequence, KV head) in the fused
    kernel (and in the route kernel of the balanced pair)."""
    from hierarchical_routed_sparse_build_b200.runtime import RoutedCache
    w = synth.DECODE_64K
    B = 16
    inp = synth.decode_inputs(w, lengths=[w.ctx_len] * B, replicas_of=8)
    c = RoutedCache(inp.k, inp.v, inp.seq_lens, chunk=w.chunk, group=w.group, top_chunks=w.top_chunks,
                    top_groups=w.top_groups, n_q_heads=w.n_q_heads)
    c.build_summaries()
    q = c.q_tensor(inp.q)
    hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, 1)
    hga.hga_set_launch_option(hga.HGA_OPT_DECODE_KERNEL, kernel)
    try:
        out, lse, idx, n_idx = c.decode(q, want_idx=True)
        no_device_error(hga)
    finally:
        hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, 0)
        hga.hga_set_launch_option(hga.HGA_OPT_DECODE_KERNEL, 0)
    idx, n_idx, out, lse = idx.cpu().numpy(), n_idx.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()
    R = w.n_q_heads // w.n_kv_heads
    L = w.ctx_len
    exact = total = 0
    summaries = {}
    for b in range(B):
        for h in range(w.n_kv_heads):
            src = b % 8
            K, V = np.ascontiguousarray(inp.k[src, h]), np.ascontiguousarray(inp.v[src, h])
            if (src, h) not in summaries:
                summaries[(src, h)] = oracle.summaries(K, w.chunk, w.group)
            cs, gs = summaries[(src, h)]
            qh = np.ascontiguousarray(inp.q[b, h * R:(h + 1) * R])
            toks = idx[b, h, :n_idx[b, h]].astype(np.int64)
            exact += check_route(toks, qh, cs, gs, L, w.chunk, w.group, w.top_chunks, w.top_groups,
                                 f"route b{b} h{h}")
            total += 1
            ref, rl = oracle.attend(qh, K, V, toks, with_lse=True)
            sl = slice(h * R, (h + 1) * R)
            assert_attention_close(out[b, sl], ref, f"decode b{b} h{h}")
            assert_lse_close(lse[b, sl], rl, f"decode lse b{b} h{h}")
    assert exact >= total - 2
    # the repeated sequences (same values, other memory) route identically; the
    # fused kernel then gives the same bits (the balanced pair cuts their tiles
    # into other slices, so its merges may round differently)
    assert np.array_equal(idx[:8], idx[8:])
    if kernel == 2:
        assert np.array_equal(out[:8], out[8:]) and np.array_equal(lse[:8], lse[8:])
