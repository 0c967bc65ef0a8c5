"""hga_prefill_noalloc: the prefill entry point for callers that cannot allocate
device memory (for instance a plugin whose host framework owns all device
allocations, or a serving loop that must not call cudaMalloc). It takes no
workspace; its routed lists live in a fixed 2 MiB array inside the library.

Checked through the C ABI against hga_prefill (the same two kernels with a
caller-provided workspace): the outputs must be bit-identical, on two different
problems called back to back (the second call runs on an area that still holds
the first call's lists) and on a problem whose lists fill the array exactly.
One sampled (block, head) pair is also checked against the CPU oracle. This
file is collected last; it also passes when run alone.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_attention_close

pytestmark = pytest.mark.gpu


def dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def problem(hga, cache_len, n_new, hq, hkv, seed, top_chunks=8, top_groups=2):
    w = synth.Workload(f"noalloc_{cache_len}", 1, hq, hkv, 128, cache_len, 128, 16, top_chunks, top_groups, -1,
                       seed, n_new=n_new, block=64)
    inp = synth.prefill_inputs(w, cache_len=cache_len, n_new=n_new)
    k, v, q = dev_bf16(inp.k), dev_bf16(inp.v), dev_bf16(inp.q)
    lens = torch.tensor([cache_len], dtype=torch.int32, device="cuda")
    kv = hga.make_kv(k, v, lens, n_kv_heads=hkv, head_dim=128, max_len=k.shape[2], batch=1)
    p = hga.make_params(w.chunk, w.group, w.top_chunks, w.top_groups)
    nc = k.shape[2] // w.chunk
    cs = torch.zeros((1, hkv, nc, 128), dtype=torch.bfloat16, device="cuda")
    gs = torch.zeros((1, hkv, nc, w.chunk // w.group, 128), dtype=torch.bfloat16, device="cuda")
    hga.hga_build_summaries(kv, p, cs, gs)
    return dict(w=w, inp=inp, k=k, v=v, q=q, lens=lens, kv=kv, p=p, cs=cs, gs=gs, L0=cache_len, T=n_new, hq=hq,
                hkv=hkv)


def with_workspace(hga, pr):
    out = torch.zeros((pr["T"], pr["hq"], 128), dtype=torch.float32, device="cuda")
    nbytes = hga.hga_prefill_workspace_size(pr["kv"], pr["hq"], pr["T"], 64, pr["L0"], pr["p"])
    ws = torch.zeros(nbytes // 4, dtype=torch.int32, device="cuda")
    hga.hga_prefill(pr["q"], pr["hq"], pr["T"], 64, pr["kv"], pr["L0"], pr["cs"], pr["gs"], pr["p"], out, ws,
                    nbytes)
    return out, ws


def without_allocation(hga, pr):
    out = torch.full((pr["T"], pr["hq"], 128), float("nan"), dtype=torch.float32, device="cuda")
    hga.hga_prefill_noalloc(pr["q"], pr["hq"], pr["T"], 64, pr["kv"], pr["L0"], pr["cs"], pr["gs"], pr["p"], out)
    return out


def no_device_error(hga):
    st, bits = hga.hga_get_device_error()
    assert st == 0, bits


def test_prefill_noalloc_matches_prefill_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import hierarchical_routed_sparse_build_b200 as hga

    first = problem(hga, 4096, 256, 32, 4, 301)
    second = problem(hga, 5077, 192, 16, 2, 302)  # different sizes: different list layout in the area
    ref1, ws1 = with_workspace(hga, first)
    ref2, _ = with_workspace(hga, second)
    got1 = without_allocation(hga, first)
    got2 = without_allocation(hga, second)
    no_device_error(hga)
    # the same two kernels on the same inputs: bit-identical results
    assert torch.equal(got1, ref1), "first call differs from hga_prefill"
    assert torch.equal(got2, ref2), "second call differs from hga_prefill"

    # one sampled (block, KV head) pair of the first problem against the oracle,
    # over the routed list that hga_prefill left in its workspace
    pr, b, h = first, 2, 1
    nb, stride = pr["T"] // 64, hga.hga_prefill_workspace_size(pr["kv"], 32, pr["T"], 64, pr["L0"], pr["p"]) \
        // (4 * (pr["T"] // 64) * pr["hkv"]) - 1
    ws = ws1.cpu().numpy()
    n_idx = ws[nb * pr["hkv"] * stride:].reshape(nb, pr["hkv"])
    tok = ws[:nb * pr["hkv"] * stride].reshape(nb, pr["hkv"], stride)[b, h, :n_idx[b, h]].astype(np.int64)
    R = 8
    qb = np.ascontiguousarray(pr["inp"].q[b * 64:(b + 1) * 64, h * R:(h + 1) * R])
    ref = oracle.prefill_block(qb, pr["inp"].k[0, h], pr["inp"].v[0, h], tok, P=pr["L0"] + 64 * b)
    assert_attention_close(got1.cpu().numpy()[b * 64:(b + 1) * 64, h * R:(h + 1) * R], ref, "no-alloc vs oracle")


def test_prefill_noalloc_at_its_limit():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import hierarchical_routed_sparse_build_b200 as hga

    # cache 1663 = 11 * 128 + 255: 12 full chunks, 10 routed (top 10) x 4 groups x 16
    # + sink 128 + local chunk and tail 255 = 1023 routed tokens per list; 4096
    # queries = 64 blocks x 8 KV heads = 512 lists of 1023 + 1 counts: exactly 2 MiB
    pr = problem(hga, 1663, 4096, 16, 8, 303, top_chunks=10, top_groups=4)
    assert hga.hga_prefill_workspace_size(pr["kv"], 16, 4096, 64, 1663, pr["p"]) == 2 << 20
    ref, _ = with_workspace(hga, pr)
    got = without_allocation(hga, pr)
    no_device_error(hga)
    assert torch.equal(got, ref), "a problem that fills the array exactly differs from hga_prefill"
    # one block more is over the limit: refused before anything is enqueued
    T = 4160
    k = torch.zeros((1, 8, 1663 + T, 128), dtype=torch.bfloat16, device="cuda")
    kv = hga.make_kv(k, k, pr["lens"], n_kv_heads=8, head_dim=128, max_len=1663 + T, batch=1)
    q = torch.zeros((T, 16, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.full((T, 16, 128), 3.0, dtype=torch.float32, device="cuda")
    assert hga.hga_prefill_workspace_size(kv, 16, T, 64, 1663, pr["p"]) == (2 << 20) + 8 * 1024 * 4
    with pytest.raises(hga.HgaError) as e:
        hga.hga_prefill_noalloc(q, 16, T, 64, kv, 1663, pr["cs"], pr["gs"], pr["p"], out)
    assert e.value.status == 2  # HGA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)


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
