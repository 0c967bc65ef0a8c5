"""hga_prefill_noalloc: the prefill entry point for callers that cannot allocate
device memory (for instance a plugin whose host framework owns all device
allocations, or a serving loop that must not call cudaMalloc). It takes no
workspace; its routed lists live in a fixed 2 MiB array inside the library.

Checked through the C ABI against hga_prefill (the same computation with a
caller-provided workspace), on two different problems called back to back, so
that the second call runs on an area that still holds the first call's lists.
This file is collected last; it also passes when run alone.
"""
import numpy as np
import pytest
import torch

import synth
from parity import assert_attention_close

pytestmark = pytest.mark.gpu


def dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def problem(hga, cache_len, n_new, hq, hkv, seed):
    w = synth.Workload(f"noalloc_{cache_len}", 1, hq, hkv, 128, cache_len, 128, 16, 8, 2, -1, seed,
                       n_new=n_new, block=64)
    inp = synth.prefill_inputs(w, cache_len=cache_len, n_new=n_new)
    k, v, q = dev_bf16(inp.k), dev_bf16(inp.v), dev_bf16(inp.q)
    lens = torch.tensor([cache_len], dtype=torch.int32, device="cuda")
    kv = hga.make_kv(k, v, lens, n_kv_heads=hkv, head_dim=128, max_len=k.shape[2], batch=1)
    p = hga.make_params(w.chunk, w.group, w.top_chunks, w.top_groups)
    nc = k.shape[2] // w.chunk
    cs = torch.zeros((1, hkv, nc, 128), dtype=torch.bfloat16, device="cuda")
    gs = torch.zeros((1, hkv, nc, w.chunk // w.group, 128), dtype=torch.bfloat16, device="cuda")
    hga.hga_build_summaries(kv, p, cs, gs)
    return dict(w=w, k=k, v=v, q=q, lens=lens, kv=kv, p=p, cs=cs, gs=gs, L0=cache_len, T=n_new, hq=hq)


def with_workspace(hga, pr):
    out = torch.zeros((pr["T"], pr["hq"], 128), dtype=torch.float32, device="cuda")
    nbytes = hga.hga_prefill_workspace_size(pr["kv"], pr["hq"], pr["T"], 64, pr["L0"], pr["p"])
    ws = torch.zeros(nbytes // 4, dtype=torch.int32, device="cuda")
    hga.hga_prefill(pr["q"], pr["hq"], pr["T"], 64, pr["kv"], pr["L0"], pr["cs"], pr["gs"], pr["p"], out, ws,
                    nbytes)
    return out


def without_allocation(hga, pr):
    out = torch.full((pr["T"], pr["hq"], 128), float("nan"), dtype=torch.float32, device="cuda")
    hga.hga_prefill_noalloc(pr["q"], pr["hq"], pr["T"], 64, pr["kv"], pr["L0"], pr["cs"], pr["gs"], pr["p"], out)
    return out


def test_prefill_noalloc_matches_prefill_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import hierarchical_routed_sparse_build_b200 as hga

    first = problem(hga, 4096, 256, 32, 4, 301)
    second = problem(hga, 5077, 192, 16, 2, 302)  # different sizes: different list layout in the area
    ref1 = with_workspace(hga, first)
    ref2 = with_workspace(hga, second)
    got1 = without_allocation(hga, first)
    got2 = without_allocation(hga, second)
    st, bits = hga.hga_get_device_error()
    assert st == 0, bits
    for got, ref, what in ((got1, ref1, "first call"), (got2, ref2, "second call")):
        g, r = got.cpu().numpy(), ref.cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all(), what
        assert_attention_close(g, r, what)


def test_prefill_noalloc_rejects_problems_beyond_its_area():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import hierarchical_routed_sparse_build_b200 as hga

    # 8192 queries in blocks of 64 on a 63488-token cache, 8 KV heads:
    # 128 blocks x 8 heads x 2305 x 4 bytes = 9.4 MB > 2 MiB
    hq, hkv, L0, T = 16, 8, 63488, 8192
    k = torch.zeros((1, hkv, L0 + T, 128), dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([L0], dtype=torch.int32, device="cuda")
    kv = hga.make_kv(k, k, lens, n_kv_heads=hkv, head_dim=128, max_len=L0 + T, batch=1)
    p = hga.make_params(128, 16, 32, 4)
    q = torch.zeros((T, hq, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((T, hq, 128), dtype=torch.float32, device="cuda")
    cs = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(hga.HgaError) as e:
        hga.hga_prefill_noalloc(q, hq, T, 64, kv, L0, cs, cs, p, out)
    assert e.value.status == 2  # HGA_ERR_UNSUPPORTED
