"""Host-resident K/V (the pages' placement: the whole cache in host memory, only
the routed rows moved to the GPU): the same kernels read K/V through the host
link from pinned, mapped host memory, with the summaries in device memory.
Checked against the CPU oracle (routed lists under the near-tie rule of
tests/parity.py, attention over the list the GPU chose), and against the
device-resident cache, which must give the same results bit for bit (same
kernels, same data)."""
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


def pinned_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()


def test_host_resident_decode_equals_device_resident(hga):
    from hierarchical_routed_sparse_build_b200.runtime import RoutedCache
    w = synth.Workload("host_kv", 3, 32, 4, 128, 9000, 128, 16, 16, 4, -1, 227)
    inp = synth.decode_inputs(w, lengths=[9000, 6001, 8192], max_len=9088)
    dev = RoutedCache(inp.k, inp.v, inp.seq_lens, chunk=128, group=16, top_chunks=16, top_groups=4, n_q_heads=32)
    dev.build_summaries()
    q = dev.q_tensor(inp.q)
    out_d, lse_d, idx_d, n_d = dev.decode(q, want_idx=True)

    kh, vh = pinned_bf16(inp.k), pinned_bf16(inp.v)
    kdev, vdev = hga.hga_host_kv_pointer(kh), hga.hga_host_kv_pointer(vh)
    lens = torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda")
    kv = hga.make_kv(kdev, vdev, lens, n_kv_heads=4, head_dim=128, max_len=9088, batch=3)
    p = hga.make_params(128, 16, 16, 4)
    cs = torch.zeros_like(dev.chunk_sum)
    gs = torch.zeros_like(dev.group_sum)
    hga.hga_build_summaries(kv, p, cs, gs)
    out_h, lse_h = torch.empty_like(out_d), torch.empty_like(lse_d)
    idx_h, n_h = torch.full_like(idx_d, -1), torch.zeros_like(n_d)
    hga.hga_decode(q, 32, kv, cs, gs, p, out_h, lse_h, idx_h, idx_d.shape[2], n_h)
    st, b = hga.hga_get_device_error()
    assert st == 0, b
    assert np.array_equal(bits(cs), bits(dev.chunk_sum)) and np.array_equal(bits(gs), bits(dev.group_sum))
    assert torch.equal(n_h, n_d) and torch.equal(idx_h, idx_d)
    assert torch.equal(out_h, out_d) and torch.equal(lse_h, lse_d)

    # the host-resident results against the oracle, every (sequence, KV head)
    idx_c, n_c = idx_h.cpu().numpy(), n_h.cpu().numpy()
    out_c, lse_c = out_h.cpu().numpy(), lse_h.cpu().numpy()
    R = 8
    exact = 0
    for b, L in enumerate(inp.seq_lens):
        L = int(L)
        for h in range(4):
            K, V = np.ascontiguousarray(inp.k[b, h, :L]), np.ascontiguousarray(inp.v[b, h, :L])
            qh = np.ascontiguousarray(inp.q[b, h * R:(h + 1) * R])
            cs_o, gs_o = oracle.summaries(K, 128, 16)
            toks = idx_c[b, h, :n_c[b, h]].astype(np.int64)
            exact += check_route(toks, qh, cs_o, gs_o, L, 128, 16, 16, 4, f"host route b{b} h{h}")
            ref, rl = oracle.attend(qh, K, V, toks, with_lse=True)
            assert_attention_close(out_c[b, h * R:(h + 1) * R], ref, f"host decode b{b} h{h}")
            assert_lse_close(lse_c[b, h * R:(h + 1) * R], rl, f"host decode lse b{b} h{h}")
    assert exact >= 11


def test_host_kv_pointer_rejects_unmapped_memory(hga):
    with pytest.raises(hga.HgaError):
        hga.hga_host_kv_pointer(torch.zeros(4096, dtype=torch.bfloat16))  # pageable host memory
    with pytest.raises(hga.HgaError):
        hga.hga_host_kv_pointer(torch.zeros(4096, dtype=torch.bfloat16, device="cuda"))  # device memory
