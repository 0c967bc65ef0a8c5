"""C ABI checks that need no GPU: the library loads, exports every call that
include/hga.h declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import oracle
import hierarchical_routed_sparse_build_b200 as hga

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hga.h")

INVALID, UNSUPPORTED = 1, 2
FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails before any launch


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hga_[a-z_]+)\s*\(", text)))


def test_header_declarations_are_all_exported():
    names = declared_functions()
    assert len(names) >= 9
    lib = ctypes.CDLL(hga.library_path())
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(hga.EXPORTED)


def test_status_strings():
    for s in range(6):
        assert hga.hga_status_string(s)
    assert hga.hga_status_string(99) == "unknown status"


def kv_desc(**over):
    d = dict(k=FAKE, v=FAKE, seq_lens=FAKE, n_kv_heads=4, head_dim=128, max_len=65536, batch=2)
    d.update(over)
    return hga.make_kv(d.pop("k"), d.pop("v"), d.pop("seq_lens"), **d)


def params(**over):
    d = dict(chunk=128, group=16, top_chunks=32, top_groups=4, scale=0.0)
    d.update(over)
    return hga.make_params(**d)


def raw_decode(kv, p, q=FAKE, hq=32, out=FAKE, idx=None, stride=0, n_idx=None):
    return hga._lib.hga_decode(q, hq, ctypes.byref(kv), FAKE, FAKE, ctypes.byref(p), out, None, idx, stride,
                               n_idx, None)


@pytest.mark.parametrize("kv_over,p_over,hq,want", [
    (dict(k=0), {}, 32, INVALID),                      # null K
    (dict(seq_lens=0), {}, 32, INVALID),               # null lengths
    (dict(head_dim=96), {}, 32, UNSUPPORTED),          # head dim
    (dict(batch=0), {}, 32, INVALID),
    (dict(k=FAKE + 8), {}, 32, INVALID),               # misaligned
    ({}, dict(group=24), 32, INVALID),                 # g does not divide C
    ({}, dict(top_groups=9), 32, INVALID),             # G > C/g
    ({}, dict(top_chunks=0), 32, INVALID),
    ({}, dict(chunk=256, group=4), 32, UNSUPPORTED),   # C/g > 32
    ({}, dict(scale=-1.0), 32, INVALID),
    ({}, {}, 30, INVALID),                             # Hq % Hkv != 0
    ({}, {}, 48, UNSUPPORTED),                         # 12 query heads per KV head
    (dict(max_len=4096 * 128 + 128), {}, 32, UNSUPPORTED),  # more than 4096 chunks
    (dict(page_table=FAKE, page_size=64, max_pages=1024, num_pages=8), {}, 32, UNSUPPORTED),  # page != chunk
    (dict(page_table=FAKE, page_size=128, max_pages=4, num_pages=8), {}, 32, INVALID),  # table too short
])
def test_decode_rejects_bad_arguments_on_host(kv_over, p_over, hq, want):
    assert raw_decode(kv_desc(**kv_over), params(**p_over), hq=hq) == want


def test_decode_output_and_index_arguments():
    kv, p = kv_desc(), params()
    assert raw_decode(kv, p, out=0) == INVALID
    assert raw_decode(kv, p, q=0) == INVALID
    assert raw_decode(kv, p, idx=FAKE, stride=4096, n_idx=None) == INVALID  # idx without n_idx
    assert raw_decode(kv, p, idx=FAKE, stride=100, n_idx=FAKE) == INVALID   # stride below the bound


def test_route_and_attend_validation():
    kv, p = kv_desc(), params()
    L = hga._lib
    assert L.hga_route(FAKE, 32, ctypes.byref(kv), FAKE, FAKE, ctypes.byref(p), FAKE, 10, FAKE, None) == INVALID
    assert L.hga_route(FAKE, 32, ctypes.byref(kv), None, FAKE, ctypes.byref(p), FAKE, 4096, FAKE, None) == INVALID
    assert L.hga_attend(FAKE, 32, ctypes.byref(kv), None, 16, FAKE, ctypes.byref(p), FAKE, None, None) == INVALID
    assert L.hga_attend(FAKE, 32, ctypes.byref(kv_desc(v=0)), FAKE, 16, FAKE, ctypes.byref(p), FAKE, None,
                        None) == INVALID
    assert L.hga_build_summaries(ctypes.byref(kv), ctypes.byref(p), None, FAKE, None) == INVALID
    assert L.hga_build_summaries(None, ctypes.byref(p), FAKE, FAKE, None) == INVALID


@pytest.mark.parametrize("max_len,C,g,k,G", [
    (65536, 128, 16, 32, 4), (16384, 128, 16, 16, 4), (4096, 64, 16, 8, 2), (100, 64, 16, 8, 2),
    (65536 + 77, 128, 16, 32, 4), (1000, 16, 4, 100, 4), (383, 128, 16, 2, 1), (384, 128, 16, 2, 1),
])
def test_max_routed_tokens_bounds_every_length(max_len, C, g, k, G):
    kv = kv_desc(max_len=max_len, head_dim=64)
    n = hga.hga_max_routed_tokens(kv, params(chunk=C, group=g, top_chunks=k, top_groups=G))
    want = max(oracle.max_routed(L, C, g, k, G) for L in range(1, max_len + 1))
    assert n == want


def test_summary_bytes():
    kv = kv_desc()
    cb, gb = hga.hga_summary_bytes(kv, params())
    assert cb == 2 * 4 * 512 * 128 * 2 and gb == cb * 8
    kvp = kv_desc(page_table=FAKE, page_size=128, max_pages=512, num_pages=1000)
    cb, gb = hga.hga_summary_bytes(kvp, params())
    assert cb == 1000 * 4 * 128 * 2 and gb == cb * 8


def test_launch_option_validation():
    with pytest.raises(hga.HgaError):
        hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, 17)
    with pytest.raises(hga.HgaError):
        hga.hga_set_launch_option(7, 1)
    with pytest.raises(hga.HgaError):
        hga.hga_set_launch_option(3, 1)  # no option 3: the prefill attention has one kernel
    with pytest.raises(hga.HgaError):
        hga.hga_set_launch_option(hga.HGA_OPT_TEST_EXPIRE_PREFILL_WAIT, -1)
    hga.hga_set_launch_option(hga.HGA_OPT_TEST_EXPIRE_PREFILL_WAIT, 0)
    hga.hga_set_launch_option(hga.HGA_OPT_CTAS_PER_HEAD, 0)


def raw_hisa(kv, p, top_tokens=2048, q=FAKE, cs=FAKE, out=FAKE, idx=None, stride=0, n_idx=None, hq=32):
    return hga._lib.hga_decode_hisa(q, hq, ctypes.byref(kv), cs, ctypes.byref(p), top_tokens, out, None, idx,
                                    stride, n_idx, None)


def test_hisa_rejects_bad_arguments_on_host():
    kv, p = kv_desc(), params()
    assert raw_hisa(kv, p, top_tokens=0) == INVALID
    assert raw_hisa(kv, p, q=0) == INVALID
    assert raw_hisa(kv, p, cs=0) == INVALID
    assert raw_hisa(kv, p, cs=FAKE + 8) == INVALID
    assert raw_hisa(kv, p, out=0) == INVALID
    assert raw_hisa(kv, p, idx=FAKE, stride=4096, n_idx=None) == INVALID      # idx without n_idx
    assert raw_hisa(kv, p, idx=FAKE, stride=100, n_idx=FAKE) == INVALID       # stride below the bound
    assert raw_hisa(kv, params(chunk=24, group=8, top_groups=2)) == UNSUPPORTED  # 16-token batches span chunks
    assert raw_hisa(kv, p, hq=48) == UNSUPPORTED                              # 12 query heads per KV head
    assert raw_hisa(kv_desc(head_dim=96), p) == UNSUPPORTED


@pytest.mark.parametrize("max_len,C,m,k_tok", [
    (65536, 128, 32, 2048), (16384, 128, 64, 3000), (4096, 64, 8, 700), (300, 64, 4, 100),
    (65536 + 77, 128, 32, 100000), (9088, 128, 8, 1024), (383, 128, 2, 5000), (384, 128, 2, 5000),
])
def test_max_hisa_tokens_bounds_every_length(max_len, C, m, k_tok):
    kv = kv_desc(max_len=max_len, head_dim=64)
    n = hga._lib.hga_max_hisa_tokens(ctypes.byref(kv), ctypes.byref(params(chunk=C, group=16, top_chunks=m,
                                                                           top_groups=2)), k_tok)
    want = max(min(k_tok, oracle.hisa_candidates(L, C, m)) for L in range(1, max_len + 1))
    assert n == want


def test_append_rejects_bad_arguments_on_host():
    kv, p = kv_desc(), params()
    L = hga._lib
    other_lens = FAKE + 0x100  # not the descriptor's seq_lens
    assert L.hga_append(ctypes.byref(kv), other_lens, FAKE, FAKE, ctypes.byref(p), FAKE, FAKE, None) == INVALID
    assert L.hga_append(ctypes.byref(kv), FAKE, FAKE + 8, FAKE, ctypes.byref(p), FAKE, FAKE, None) == INVALID
    assert L.hga_append(ctypes.byref(kv), FAKE, FAKE, FAKE, ctypes.byref(p), None, FAKE, None) == INVALID
    assert L.hga_append(ctypes.byref(kv_desc(v=0)), FAKE, FAKE, FAKE, ctypes.byref(p), FAKE, FAKE, None) == INVALID


def raw_prefill(kv, p, n_queries=2048, block=64, cache_len=63488, hq=32, out=FAKE, ws=FAKE, ws_bytes=1 << 30):
    return hga._lib.hga_prefill(FAKE, hq, n_queries, block, ctypes.byref(kv), cache_len, FAKE, FAKE,
                                ctypes.byref(p), out, ws, ws_bytes, None)


def test_prefill_rejects_bad_arguments_on_host():
    kv1, p = kv_desc(batch=1), params()
    assert raw_prefill(kv1, p, cache_len=65536 - 2047) == INVALID           # past max_len
    assert raw_prefill(kv1, p, n_queries=0) == INVALID
    assert raw_prefill(kv1, p, cache_len=-1) == INVALID
    assert raw_prefill(kv1, p, out=0) == INVALID
    assert raw_prefill(kv1, p, ws=0) == INVALID
    assert raw_prefill(kv1, p, ws_bytes=16) == INVALID                      # workspace too small
    assert raw_prefill(kv_desc(batch=2), p) == UNSUPPORTED                 # one sequence per call
    assert raw_prefill(kv1, p, block=32) == UNSUPPORTED
    assert raw_prefill(kv1, p, n_queries=2000) == UNSUPPORTED               # not a multiple of the block
    assert raw_prefill(kv_desc(batch=1, head_dim=64), p) == UNSUPPORTED


def test_prefill_workspace_holds_the_lists():
    kv1, p = kv_desc(batch=1), params()
    need = hga._lib.hga_prefill_workspace_size(ctypes.byref(kv1), 32, 2048, 64, 63488, ctypes.byref(p))
    stride = oracle.max_routed(63488, 128, 16, 32, 4)
    assert need >= 32 * 4 * (stride + 1) * 4


def test_hisa_rejects_candidate_sets_beyond_shared_memory():
    # 64K context, top 510 chunks: (510 + 3) * 128 candidate keys of 8 bytes do not fit one CTA
    kv, p = kv_desc(), params(top_chunks=510)
    assert raw_hisa(kv, p) == UNSUPPORTED


@pytest.mark.parametrize("cache_len,n_queries,C,g,k,G", [
    (63488, 2048, 128, 16, 32, 4), (1000, 512, 128, 16, 4, 2), (0, 256, 128, 16, 8, 4),
    (4000, 1024, 64, 16, 8, 2), (383, 128, 128, 16, 2, 1),
])
def test_prefill_workspace_sizes_hold_the_longest_list(cache_len, n_queries, C, g, k, G):
    kv1 = kv_desc(batch=1, max_len=cache_len + n_queries)
    p = params(chunk=C, group=g, top_chunks=k, top_groups=G)
    units = (n_queries // 64) * 4
    plain = hga._lib.hga_prefill_workspace_size(ctypes.byref(kv1), 32, n_queries, 64, cache_len, ctypes.byref(p))
    assert plain == units * (oracle.max_routed(cache_len, C, g, k, G) + 1) * 4
    grow = hga._lib.hga_prefill_growing_workspace_size(ctypes.byref(kv1), 32, n_queries, 64, cache_len,
                                                       ctypes.byref(p))
    longest = max(oracle.max_routed(cache_len + 64 * b, C, g, k, G) for b in range(n_queries // 64))
    assert grow == units * (longest + 1) * 4


def test_hisa_kept_list_is_bounded_by_the_candidates():
    # a top_tokens above every length's candidate count keeps every candidate; the
    # kept list (and the shared memory it takes) is bounded by the candidates
    kv, p = kv_desc(), params()
    assert hga._lib.hga_max_hisa_tokens(ctypes.byref(kv), ctypes.byref(p), 10_000_000) == \
        max(oracle.hisa_candidates(L, 128, 32) for L in range(65536 - 256, 65537))


def raw_decode_ws(kv, p, ws=FAKE, nbytes=1 << 30, hq=32):
    return hga._lib.hga_decode_ws(FAKE, hq, ctypes.byref(kv), FAKE, FAKE, ctypes.byref(p), FAKE, None, None, 0,
                                  None, ws, nbytes, None)


def test_decode_workspace_size_and_validation():
    kv, p = kv_desc(batch=64), params()
    n = hga.hga_decode_workspace_size(kv, 32, p)
    units, sms = 64 * 4, 148  # no device here: the library assumes a B200's 148 SMs
    # routed tile lists (32 chunks x 4 groups x one 16-token tile each), one partial
    # softmax state per (CTA of a 2-per-SM grid + unit), one merge count per unit
    floor = units * 32 * 4 * 4 + (2 * sms + units) * 8 * 130 * 4 + units * 4
    assert floor <= n <= floor + 3 * 256
    # groups that are not whole 16-token tiles run the one-kernel decode: no real workspace
    assert hga.hga_decode_workspace_size(kv, 32, params(group=8)) == 256
    assert hga._lib.hga_decode_workspace_size(ctypes.byref(kv_desc(head_dim=96)), 32, ctypes.byref(p)) == 0
    assert raw_decode_ws(kv, p, ws=0) == INVALID                     # no workspace
    assert raw_decode_ws(kv, p, ws=FAKE + 16) == INVALID             # not 256-byte aligned
    assert raw_decode_ws(kv, p, nbytes=n - 1) == INVALID             # too small
    assert raw_decode_ws(kv_desc(head_dim=96), p) == UNSUPPORTED     # the decode's own checks still apply


def raw_hisa_ws(kv, p, ws=FAKE, nbytes=1 << 30, hq=32, top_tokens=2048):
    return hga._lib.hga_decode_hisa_ws(FAKE, hq, ctypes.byref(kv), FAKE, ctypes.byref(p), top_tokens, FAKE, None,
                                       None, 0, None, ws, nbytes, None)


def test_hisa_logits_workspace_size_and_validation():
    kv, p = kv_desc(batch=64), params()
    n = hga.hga_decode_hisa_workspace_size(kv, p)
    # 32 bytes (8 fp32 logits) per candidate of the longest context, per (sequence, KV head):
    # (top_chunks + 3) chunks of candidates, the bound of the token keys
    nf = kv.max_len // p.chunk
    assert n == 64 * 4 * (min(p.top_chunks, nf - 2) + 3) * p.chunk * 32
    assert n >= 64 * 4 * 32 * max(oracle.hisa_candidates(L, p.chunk, p.top_chunks)
                                  for L in range(kv.max_len - 2 * p.chunk, kv.max_len + 1))
    assert hga._lib.hga_decode_hisa_workspace_size(ctypes.byref(kv_desc(head_dim=96)), ctypes.byref(p)) == 0
    assert raw_hisa_ws(kv, p, ws=0) == INVALID                   # no workspace
    assert raw_hisa_ws(kv, p, ws=FAKE + 16) == INVALID           # not 256-byte aligned
    assert raw_hisa_ws(kv, p, nbytes=n - 1) == INVALID           # too small
    assert raw_hisa_ws(kv, p, top_tokens=0) == INVALID           # the block-then-token checks still apply
    assert raw_hisa_ws(kv, p, hq=48) == UNSUPPORTED
