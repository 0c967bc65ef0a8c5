"""GPU parity of chunked prefill: block-shared routing (hga_route_blocks) and
the tcgen05 attention (hga_prefill_attend, hga_prefill) against the CPU oracle.
Routing is compared with the oracle's routing of the raw keys (its own
summaries); attention is driven with the oracle's routed lists."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_attention_close, check_route

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hga():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import hierarchical_routed_sparse_build_b200 as m
    return m


def dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


class Prefill:
    """Device buffers of one prefill problem (batch 1, contiguous cache)."""

    def __init__(self, hga, w, cache_len, n_new):
        self.hga, self.w = hga, w
        self.inp = synth.prefill_inputs(w, cache_len=cache_len, n_new=n_new)
        self.L0, self.T = cache_len, n_new
        self.k, self.v = dev_bf16(self.inp.k), dev_bf16(self.inp.v)
        self.q = dev_bf16(self.inp.q)
        self.max_len = self.inp.k.shape[2]
        self.lens = torch.tensor([cache_len], dtype=torch.int32, device="cuda")
        self.kv = hga.make_kv(self.k, self.v, self.lens, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                              max_len=self.max_len, batch=1)
        self.p = hga.make_params(w.chunk, w.group, w.top_chunks, w.top_groups)
        nc = self.max_len // w.chunk
        self.cs = torch.zeros((1, w.n_kv_heads, nc, w.head_dim), dtype=torch.bfloat16, device="cuda")
        self.gs = torch.zeros((1, w.n_kv_heads, nc, w.chunk // w.group, w.head_dim), dtype=torch.bfloat16,
                              device="cuda")
        hga.hga_build_summaries(self.kv, self.p, self.cs, self.gs)
        self.nb = n_new // w.block
        self.stride = oracle.max_routed(cache_len, w.chunk, w.group, w.top_chunks, w.top_groups)
        self.R = w.n_q_heads // w.n_kv_heads

    def route(self):
        idx = torch.full((self.nb, self.w.n_kv_heads, self.stride), -1, dtype=torch.int32, device="cuda")
        n = torch.zeros((self.nb, self.w.n_kv_heads), dtype=torch.int32, device="cuda")
        self.hga.hga_route_blocks(self.q, self.w.n_q_heads, self.T, self.w.block, self.kv, self.L0, self.cs,
                                  self.gs, self.p, idx, self.stride, n)
        return idx, n

    def q_block(self, b, h):
        return np.ascontiguousarray(self.inp.q[b * 64:(b + 1) * 64, h * self.R:(h + 1) * self.R])

    def oracle_route(self, b, h):
        cs, gs = oracle.summaries(self.inp.k[0, h, :self.L0], self.w.chunk, self.w.group)
        tok = oracle.route(self.q_block(b, h), cs, gs, self.L0, self.w.chunk, self.w.group, self.w.top_chunks,
                           self.w.top_groups)
        return tok, cs, gs

    def oracle_attend(self, b, h, tok):
        return oracle.prefill_block(self.q_block(b, h), self.inp.k[0, h], self.inp.v[0, h], tok,
                                    P=self.L0 + 64 * b)


def no_err(hga):
    st, bits = hga.hga_get_device_error()
    assert st == 0, bits


def run_case(hga, w, L0, T, units=None, attn_units=None):
    pf = Prefill(hga, w, L0, T)
    idx, n = pf.route()
    no_err(hga)
    idx_h, n_h = idx.cpu().numpy(), n.cpu().numpy()
    units = units or [(b, h) for b in range(pf.nb) for h in range(w.n_kv_heads)]
    o_idx = torch.zeros_like(idx)
    o_n = torch.zeros_like(n)
    toks = {}
    exact = 0
    cache = {}
    for (b, h) in units:
        if h not in cache:
            cache[h] = oracle.summaries(pf.inp.k[0, h, :L0], w.chunk, w.group)
        cs, gs = cache[h]
        tok = oracle.route(pf.q_block(b, h), cs, gs, L0, w.chunk, w.group, w.top_chunks, w.top_groups)
        exact += check_route(idx_h[b, h, :n_h[b, h]], pf.q_block(b, h), cs, gs, L0, w.chunk, w.group,
                             w.top_chunks, w.top_groups, f"block route b{b} h{h}")
        toks[(b, h)] = tok
        o_idx[b, h, :tok.size] = torch.from_numpy(tok).cuda()
        o_n[b, h] = tok.size
    # attention on the oracle's lists, and the fused call
    out = torch.zeros((T, w.n_q_heads, 128), dtype=torch.float32, device="cuda")
    hga.hga_prefill_attend(pf.q, w.n_q_heads, T, w.block, pf.kv, L0, o_idx, pf.stride, o_n, pf.p, out)
    no_err(hga)
    ws_bytes = hga.hga_prefill_workspace_size(pf.kv, w.n_q_heads, T, w.block, L0, pf.p)
    ws = torch.zeros(ws_bytes // 4, dtype=torch.int32, device="cuda")
    out2 = torch.zeros_like(out)
    hga.hga_prefill(pf.q, w.n_q_heads, T, w.block, pf.kv, L0, pf.cs, pf.gs, pf.p, out2, ws, ws_bytes)
    no_err(hga)
    out_h, out2_h = out.cpu().numpy(), out2.cpu().numpy()
    for (b, h) in (attn_units or units):
        ref = pf.oracle_attend(b, h, toks[(b, h)])  # [64][R][d]
        got = out_h[b * 64:(b + 1) * 64, h * pf.R:(h + 1) * pf.R]
        assert_attention_close(got, ref, f"prefill attend b{b} h{h}")
        # hga_prefill routes with the same kernel as hga_route_blocks (same inputs,
        # deterministic), so its attention is checked against the oracle's
        # attention over the list the GPU chose, wherever that differs from the
        # oracle's own list under the near-tie rule
        gpu_tok = idx_h[b, h, :n_h[b, h]].astype(np.int64)
        ref_fused = ref if np.array_equal(gpu_tok, toks[(b, h)]) else pf.oracle_attend(b, h, gpu_tok)
        assert_attention_close(out2_h[b * 64:(b + 1) * 64, h * pf.R:(h + 1) * pf.R], ref_fused,
                               f"prefill fused b{b} h{h}")
    return exact, len(units)


def small(hq, hkv, L0, T, k=8, G=2):
    return synth.Workload(f"prefill_small_{hq}_{hkv}", 1, hq, hkv, 128, L0, 128, 16, k, G, -1, 101,
                          n_new=T, block=64)


def test_prefill_small_aligned(hga):
    w = small(32, 4, 4096, 256)
    exact, n = run_case(hga, w, 4096, 256)
    assert exact >= n - 1


def test_prefill_small_ragged_cache(hga):
    # cache length not a multiple of the chunk or of 16: the local chunk carries a
    # tail and the block's own tokens start at an unaligned position
    w = small(16, 2, 5000 + 77, 192)
    run_case(hga, w, 5077, 192)


@pytest.mark.parametrize("hq,hkv", [(8, 4), (16, 4), (8, 1)])
def test_prefill_head_groups(hga, hq, hkv):
    w = small(hq, hkv, 3000, 128)
    run_case(hga, w, 3000, 128)


def test_prefill_dense_short_cache(hga):
    # fewer than three full chunks in the cache: every cache token is attended
    w = small(8, 2, 300, 128)
    run_case(hga, w, 300, 128)


def test_prefill_full_size(hga):
    # 2048 new tokens on a 63488-token cache: every block's routing is checked,
    # attention sampled on a few (block, head) pairs
    w = synth.PREFILL_64K
    units = [(b, h) for b in range(32) for h in range(4)]
    exact, n = run_case(hga, w, 63488, 2048, units=units, attn_units=[(0, 0), (13, 1), (31, 3)])
    assert exact >= n - 2


@pytest.mark.parametrize("fail_tile", [0, 3])
def test_prefill_wait_expiry_is_reported_and_clean(hga, fail_tile):
    # The test hook makes every CTA treat its wait for key tile `fail_tile` as
    # expired after that wait has really completed (no MMA is outstanding), so
    # the kernel takes its timeout exit: no output row written, the timeout
    # reported. The next call, with the hook off, must be clean and correct.
    w = small(32, 4, 4096, 128)
    pf = Prefill(hga, w, 4096, 128)
    idx, n = pf.route()
    no_err(hga)
    out = torch.full((128, 32, 128), 7.0, dtype=torch.float32, device="cuda")
    hga.hga_set_launch_option(hga.HGA_OPT_TEST_EXPIRE_PREFILL_WAIT, fail_tile + 1)
    try:
        hga.hga_prefill_attend(pf.q, 32, 128, 64, pf.kv, 4096, idx, pf.stride, n, pf.p, out)
    finally:
        hga.hga_set_launch_option(hga.HGA_OPT_TEST_EXPIRE_PREFILL_WAIT, 0)
    st, bits = hga.hga_get_device_error()
    assert st == 5 and bits == 8, (st, bits)  # HGA_ERR_TIMEOUT, timeout bit only
    assert torch.all(out == 7.0), "a CTA that took the timeout exit wrote output"
    assert hga.hga_get_device_error() == (0, 0)
    hga.hga_prefill_attend(pf.q, 32, 128, 64, pf.kv, 4096, idx, pf.stride, n, pf.p, out)
    no_err(hga)
    out_h, idx_h, n_h = out.cpu().numpy(), idx.cpu().numpy(), n.cpu().numpy()
    for b in range(2):
        for h in range(4):
            ref = pf.oracle_attend(b, h, idx_h[b, h, :n_h[b, h]].astype(np.int64))
            assert_attention_close(out_h[b * 64:(b + 1) * 64, h * 8:(h + 1) * 8], ref, f"after expiry b{b} h{h}")


@pytest.mark.parametrize("L0,T,step", [(63488, 2048, 3), (5077, 192, 1)])
def test_prefill_attend_on_gpu_lists(hga, L0, T, step):
    # The attention kernel on the lists the GPU routed, against the oracle's
    # attention over the same list: every (block, KV head) of the ragged case,
    # every third one at full size (43 of 128, spread over all blocks and heads).
    w = synth.PREFILL_64K if L0 == 63488 else small(16, 2, L0, T)
    pf = Prefill(hga, w, L0, T)
    idx, n = pf.route()
    no_err(hga)
    idx_h, n_h = idx.cpu().numpy(), n.cpu().numpy()
    out = torch.full((T, w.n_q_heads, 128), 7.0, dtype=torch.float32, device="cuda")
    hga.hga_prefill_attend(pf.q, w.n_q_heads, T, w.block, pf.kv, L0, idx, pf.stride, n, pf.p, out)
    no_err(hga)
    out_h = out.cpu().numpy()
    units = [(b, h) for b in range(pf.nb) for h in range(w.n_kv_heads)][::step]
    for (b, h) in units:
        ref = pf.oracle_attend(b, h, idx_h[b, h, :n_h[b, h]].astype(np.int64))
        assert_attention_close(out_h[b * 64:(b + 1) * 64, h * pf.R:(h + 1) * pf.R], ref, f"b{b} h{h}")
