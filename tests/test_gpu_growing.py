"""Growing-history chunked prefill (every block routes over all tokens before
it, earlier blocks of the same call included), incremental summaries
(hga_append) and a decode loop captured in a CUDA graph, against the CPU
oracle. The oracle sees, for block b at P_b = cache_len + 64 b, the summaries of
K[:P_b] and the routing rule over [0, P_b); for the decode loop, the cache at
every step's length. Tolerances are those of tests/parity.py."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_attention_close, assert_lse_close, bits, check_route

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hga():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import hierarchical_routed_sparse_build_b200 as m
    m.hga_set_launch_option(m.HGA_OPT_CTAS_PER_HEAD, 0)
    return m


def dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def run_growing(hga, w, L0, T, blocks, attn_pairs):
    """Route and attend a growing-history prefill; check routing of `blocks` (all heads) and attention of
    `attn_pairs` (block, head) against the oracle. Returns (exact route count, checked count, out)."""
    inp = synth.prefill_inputs(w, cache_len=L0, n_new=T)
    hq, hkv, d, C, g = w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.group
    R, nb = hq // hkv, T // 64
    K, V, Q = inp.k[0], inp.v[0], inp.q
    k, v, q = dev_bf16(inp.k), dev_bf16(inp.v), dev_bf16(inp.q)
    lens = torch.tensor([L0 + T], dtype=torch.int32, device="cuda")
    kv = hga.make_kv(k, v, lens, n_kv_heads=hkv, head_dim=d, max_len=k.shape[2], batch=1)
    p = hga.make_params(C, g, w.top_chunks, w.top_groups)
    nc = k.shape[2] // C
    cs = torch.zeros((1, hkv, nc, d), dtype=torch.bfloat16, device="cuda")
    gs = torch.zeros((1, hkv, nc, C // g, d), dtype=torch.bfloat16, device="cuda")
    hga.hga_build_summaries(kv, p, cs, gs)
    ws_bytes = hga.hga_prefill_growing_workspace_size(kv, hq, T, 64, L0, p)
    stride = ws_bytes // (4 * nb * hkv) - 1
    idx = torch.zeros((nb, hkv, stride), dtype=torch.int32, device="cuda")
    n_idx = torch.zeros((nb, hkv), dtype=torch.int32, device="cuda")
    hga.hga_route_blocks_growing(q, hq, T, 64, kv, L0, cs, gs, p, idx, stride, n_idx)
    out = torch.full((T, hq, d), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros(ws_bytes // 4, dtype=torch.int32, device="cuda")
    hga.hga_prefill_growing(q, hq, T, 64, kv, L0, cs, gs, p, out, ws, ws_bytes)
    st, bits_ = hga.hga_get_device_error()
    assert st == 0, bits_
    idx_h, n_h, out_h = idx.cpu().numpy(), n_idx.cpu().numpy(), out.cpu().numpy()
    exact = checked = 0
    for b in blocks:
        P = L0 + 64 * b
        for h in range(hkv):
            qb = np.ascontiguousarray(Q[64 * b:64 * b + 64, h * R:(h + 1) * R])
            csb, gsb = oracle.summaries(np.ascontiguousarray(K[h, :P]), C, g)
            toks = idx_h[b, h, :n_h[b, h]]
            exact += check_route(toks, qb, csb, gsb, P, C, g, w.top_chunks, w.top_groups, f"growing b{b} h{h}")
            checked += 1
            assert toks.size == 0 or toks.max() < P
    for (b, h) in attn_pairs:
        P = L0 + 64 * b
        qb = np.ascontiguousarray(Q[64 * b:64 * b + 64, h * R:(h + 1) * R])
        toks = idx_h[b, h, :n_h[b, h]].astype(np.int64)
        ref = oracle.prefill_block(qb, np.ascontiguousarray(K[h]), np.ascontiguousarray(V[h]), toks, P)
        assert_attention_close(out_h[64 * b:64 * b + 64, h * R:(h + 1) * R], ref, f"growing attn b{b} h{h}")
    return exact, checked, out_h


def small(hq, hkv, L0, T, k=8, G=2):
    return synth.Workload(f"growing_{hq}_{hkv}_{L0}", 1, hq, hkv, 128, L0, 128, 16, k, G, -1, 211,
                          n_new=T, block=64)


def test_growing_prefill_small(hga):
    L0, T = 3000, 256
    w = small(32, 4, L0, T)
    pairs = [(b, h) for b in range(T // 64) for h in range(4)]
    exact, n, _ = run_growing(hga, w, L0, T, range(T // 64), pairs)
    assert exact >= n - 1


def test_growing_prefill_ragged_history(hga):
    # histories that are not multiples of 16 or of the chunk: segments of the
    # routed list straddle the cache / own-token boundary
    L0, T = 5077, 192
    w = small(16, 2, L0, T)
    pairs = [(b, h) for b in range(T // 64) for h in range(2)]
    run_growing(hga, w, L0, T, range(T // 64), pairs)


def test_growing_first_block_equals_plain_prefill(hga):
    # block 0 has no earlier new tokens: both readings coincide for it
    L0, T = 3000, 128
    w = small(32, 4, L0, T)
    _, _, out_g = run_growing(hga, w, L0, T, [0], [])
    inp = synth.prefill_inputs(w, cache_len=L0, n_new=T)
    k, v, q = dev_bf16(inp.k), dev_bf16(inp.v), dev_bf16(inp.q)
    lens = torch.tensor([L0 + T], dtype=torch.int32, device="cuda")
    kv = hga.make_kv(k, v, lens, n_kv_heads=4, head_dim=128, max_len=k.shape[2], batch=1)
    p = hga.make_params(128, 16, 8, 2)
    nc = k.shape[2] // 128
    cs = torch.zeros((1, 4, nc, 128), dtype=torch.bfloat16, device="cuda")
    gs = torch.zeros((1, 4, nc, 8, 128), dtype=torch.bfloat16, device="cuda")
    hga.hga_build_summaries(kv, p, cs, gs)
    wsb = hga.hga_prefill_workspace_size(kv, 32, T, 64, L0, p)
    ws = torch.zeros(wsb // 4, dtype=torch.int32, device="cuda")
    out = torch.zeros((T, 32, 128), dtype=torch.float32, device="cuda")
    hga.hga_prefill(q, 32, T, 64, kv, L0, cs, gs, p, out, ws, wsb)
    assert np.array_equal(out.cpu().numpy()[:64], out_g[:64])


def test_growing_prefill_full_size(hga):
    # 2048 new tokens on a 63488-token cache, every block routing over its whole history
    w = synth.PREFILL_64K
    exact, n, _ = run_growing(hga, w, 63488, 2048, [0, 1, 15, 31], [(1, 0), (31, 3)])
    assert exact >= n - 1


def to_pages(K, page, n_pages):
    """[Hkv][L][d] -> n_pages pages [n_pages][Hkv][page][d] in sequence order (zero padded)."""
    hkv, L, d = K.shape
    kk = np.pad(K, ((0, 0), (0, n_pages * page - L), (0, 0))).reshape(hkv, n_pages, page, d)
    return kk.transpose(1, 0, 2, 3)


@pytest.mark.parametrize("paged", [False, True], ids=["contiguous", "paged"])
def test_append_decode_loop_in_cuda_graph(hga, paged):
    from hierarchical_routed_sparse_build_b200.runtime import RoutedCache
    L0 = np.array([3000, 4090], dtype=np.int32)  # the second crosses a chunk boundary at 4096
    N, max_len = 40, 4224
    w = synth.Workload("append", 2, 32, 4, 128, int(L0.max()) + N, 128, 16, 8, 2, -1, 223)
    full = synth.decode_inputs(w, lengths=list(L0 + N), max_len=max_len)
    B, hkv, d, R = 2, 4, 128, 8
    rng = np.random.default_rng(5)
    q_steps = to_bf16_bits(rng.standard_normal((N, B, 32, d)))
    kn = np.stack([np.stack([full.k[b, :, L0[b] + i] for b in range(B)]) for i in range(N)])  # [N][B][Hkv][d]
    vn = np.stack([np.stack([full.v[b, :, L0[b] + i] for b in range(B)]) for i in range(N)])
    k0, v0 = full.k.copy(), full.v.copy()
    for b in range(B):  # the cache holds only the first L0[b] tokens; the loop appends the rest
        k0[b, :, L0[b]:] = 0
        v0[b, :, L0[b]:] = 0
    if paged:
        page, per = 128, max_len // 128
        perm = np.random.default_rng(9).permutation(B * per).astype(np.int32)
        table = perm.reshape(B, per)
        kpool = np.zeros((B * per, hkv, page, d), dtype=np.uint16)
        vpool = np.zeros_like(kpool)
        for b in range(B):
            kpool[table[b]] = to_pages(k0[b], page, per)
            vpool[table[b]] = to_pages(v0[b], page, per)
        c = RoutedCache(kpool, vpool, L0, chunk=128, group=16, top_chunks=8, top_groups=2, n_q_heads=32,
                        page_table=table)
    else:
        c = RoutedCache(k0, v0, L0, chunk=128, group=16, top_chunks=8, top_groups=2, n_q_heads=32)
    c.build_summaries()
    kn_d, vn_d, q_d = dev_bf16(kn), dev_bf16(vn), dev_bf16(q_steps)
    kbuf, vbuf, qbuf = kn_d[0].clone(), vn_d[0].clone(), q_d[0].clone()
    out, lse = c.out_buffers()
    idx, n_idx = c.idx_buffers()
    c.decode(qbuf, out, lse, idx, n_idx)  # sets launch attributes before capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        c.append(kbuf, vbuf)
        c.decode(qbuf, out, lse, idx, n_idx)
    checks = {0, 5, 6, N - 1}
    for i in range(N):
        kbuf.copy_(kn_d[i])
        vbuf.copy_(vn_d[i])
        qbuf.copy_(q_d[i])
        graph.replay()
        if i not in checks:
            continue
        torch.cuda.synchronize()
        st, bits_ = hga.hga_get_device_error()
        assert st == 0, bits_
        idx_h, n_h, out_h, lse_h = idx.cpu().numpy(), n_idx.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()
        for b in range(B):
            L = int(L0[b]) + i + 1
            for h in range(hkv):
                K = np.ascontiguousarray(full.k[b, h, :L])
                Vh = np.ascontiguousarray(full.v[b, h, :L])
                qh = np.ascontiguousarray(q_steps[i, b, h * R:(h + 1) * R])
                cs, gs = oracle.summaries(K, 128, 16)
                toks = idx_h[b, h, :n_h[b, h]]
                check_route(toks, qh, cs, gs, L, 128, 16, 8, 2, f"step {i} b{b} h{h}")
                ref, rl = oracle.attend(qh, K, Vh, toks.astype(np.int64), with_lse=True)
                assert_attention_close(out_h[b, h * R:(h + 1) * R], ref, f"step {i} b{b} h{h}")
                assert_lse_close(lse_h[b, h * R:(h + 1) * R], rl, f"step {i} lse b{b} h{h}")
    assert np.array_equal(c.seq_lens.cpu().numpy(), L0 + N)
    # summaries kept by the appends equal a rebuild from the final cache, bit for bit
    cs_inc, gs_inc = bits(c.chunk_sum).copy(), bits(c.group_sum).copy()
    c.build_summaries()
    assert np.array_equal(bits(c.chunk_sum), cs_inc) and np.array_equal(bits(c.group_sum), gs_inc)
    del graph
