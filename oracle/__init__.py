"""CPU oracle for Hierarchical Global Attention routed attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package. The library under ``hierarchical_routed_sparse_build_b200``
never does: the two share no code, and the oracle takes the same seeded inputs
(bfloat16 bit patterns as ``numpy.uint16``) from ``synth``.

The arithmetic is in ``hga_oracle.c`` (plain C, double precision); this module
compiles it with gcc and wraps each function for numpy arrays. Each wrapper names
the step of the method it states: chunk/group summaries, head-summed routing
scores, chunk top-k with sink and local chunks kept, group top-G, exact softmax
attention over the routed set, the block-shared routing of chunked prefill, and
the block-then-token variant (top blocks, then top tokens inside them).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hga_oracle.c")
_LIB = os.path.join(_HERE, "libhga_oracle.so")


def build(force: bool = False) -> str:
    """Compile hga_oracle.c into libhga_oracle.so (gcc -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", "-std=c11", "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        i32, i64, dbl, vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_double.restype = dbl
        L.oracle_bf16_rne.argtypes = [dbl]
        L.oracle_bf16_rne.restype = ctypes.c_uint16
        L.oracle_summaries.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp]
        L.oracle_summaries.restype = None
        L.oracle_chunk_scores.argtypes = [vp, i32, i64, i32, i32, vp, i32, vp]
        L.oracle_chunk_scores.restype = None
        L.oracle_group_scores.argtypes = [vp, i32, i64, i32, i32, vp, i32, vp]
        L.oracle_group_scores.restype = None
        L.oracle_route_block.argtypes = [vp, i32, i64, i32, i32, vp, vp, i32, i32, i32, i32, i32,
                                         vp, i32, vp, vp]
        L.oracle_route_block.restype = i32
        L.oracle_route.argtypes = [vp, i32, i32, vp, vp, i32, i32, i32, i32, i32, vp, i32]
        L.oracle_route.restype = i32
        L.oracle_attend.argtypes = [vp, i32, i32, vp, vp, vp, i32, dbl, vp, vp]
        L.oracle_attend.restype = None
        L.oracle_prefill_block.argtypes = [vp, i32, i64, i32, i32, vp, vp, vp, i32, i32, dbl, vp]
        L.oracle_prefill_block.restype = None
        L.oracle_hisa_route.argtypes = [vp, i32, i32, vp, vp, i32, i32, i32, i32, vp, i32, vp]
        L.oracle_hisa_route.restype = i32
        _lib = L
    return _lib


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def bf16_to_f64(a) -> np.ndarray:
    """bfloat16 bit patterns -> float64 (exact), vectorised."""
    a = np.asarray(a, dtype=np.uint16)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_rne(x: float) -> int:
    return int(lib().oracle_bf16_rne(float(x)))


def summaries(K, C: int, g: int, with_f64: bool = False):
    """Chunk and group summaries of one (sequence, KV head); K is [L][d] bf16 bits.

    Returns chunk_sum [nf][d] and group_sum [nf][C/g][d] (bf16 bits), plus the
    unrounded float64 means when ``with_f64``.
    """
    K = _u16(K)
    L, d = K.shape
    nf, gpc = L // C, C // g
    cs = np.zeros((nf, d), dtype=np.uint16)
    gs = np.zeros((nf, gpc, d), dtype=np.uint16)
    cf = np.zeros((nf, d), dtype=np.float64) if with_f64 else None
    gf = np.zeros((nf, gpc, d), dtype=np.float64) if with_f64 else None
    lib().oracle_summaries(_p(K), L, d, C, g, _p(cs), _p(gs), _p(cf), _p(gf))
    return (cs, gs, cf, gf) if with_f64 else (cs, gs)


def chunk_scores(q, chunk_sum) -> np.ndarray:
    """Routing scores of every chunk summary. q is [R][d] (decode) or [n_q][R][d] (block)."""
    q = _u16(q)
    if q.ndim == 2:
        q = q[None]
    n_q, R, d = q.shape
    cs = _u16(chunk_sum)
    out = np.zeros(cs.shape[0], dtype=np.float64)
    lib().oracle_chunk_scores(_p(q), n_q, R * d, R, d, _p(cs), cs.shape[0], _p(out))
    return out


def group_scores(q, group_sum_chunk) -> np.ndarray:
    q = _u16(q)
    if q.ndim == 2:
        q = q[None]
    n_q, R, d = q.shape
    gs = _u16(group_sum_chunk)
    out = np.zeros(gs.shape[0], dtype=np.float64)
    lib().oracle_group_scores(_p(q), n_q, R * d, R, d, _p(gs), gs.shape[0], _p(out))
    return out


def max_routed(L: int, C: int, g: int, k: int, G: int) -> int:
    nf = L // C
    if nf <= 2:
        return L
    return C + min(k, nf - 2) * min(G, C // g) * g + (L - (nf - 1) * C)


def route(q, chunk_sum, group_sum, L: int, C: int, g: int, k: int, G: int, return_chunks: bool = False):
    """Routed token positions (ascending) for one (sequence, KV head).

    q is [R][d] for a decode query or [n_q][R][d] for a prefill block (max over
    the block's queries).
    """
    q = _u16(q)
    if q.ndim == 2:
        q = q[None]
    n_q, R, d = q.shape
    cap = max_routed(L, C, g, k, G)
    tok = np.zeros(max(cap, 1), dtype=np.int32)
    kept = np.zeros(max(L // C, 1), dtype=np.int32)
    nk = ctypes.c_int32(0)
    n = lib().oracle_route_block(_p(q), n_q, R * d, R, d, _p(_u16(chunk_sum)), _p(_u16(group_sum)), L,
                                 C, g, k, G, _p(tok), cap, _p(kept), ctypes.byref(nk))
    if n < 0:
        raise RuntimeError("oracle_route_block: capacity")
    return (tok[:n].copy(), kept[:nk.value].copy()) if return_chunks else tok[:n].copy()


def hisa_candidates(L: int, C: int, m: int) -> int:
    """Tokens the block-then-token route scores for one query: first block + top-m blocks + last block
    and tail (every token when nf <= 2)."""
    nf = L // C
    if nf <= 2:
        return L
    return C + min(m, nf - 2) * C + (L - (nf - 1) * C)


def hisa_route(q, chunk_sum, K, L: int, C: int, m: int, k_tok: int, return_scored: bool = False):
    """Block-then-token routed positions (ascending) of one decode query q [R][d] over K [L][d]: the
    top-m chunks (plus the first and last) by their summaries, then the top k_tok tokens inside them."""
    q = _u16(q)
    R, d = q.shape
    K = _u16(K)
    if K.shape[0] < L:
        raise IndexError("K shorter than L")
    cap = max(min(k_tok, hisa_candidates(L, C, m)), 1)
    tok = np.zeros(cap, dtype=np.int32)
    scored = ctypes.c_int64(0)
    n = lib().oracle_hisa_route(_p(q), R, d, _p(_u16(chunk_sum)), _p(K), L, C, m, k_tok, _p(tok), cap,
                                ctypes.byref(scored))
    if n < 0:
        raise RuntimeError("oracle_hisa_route: capacity")
    return (tok[:n].copy(), int(scored.value)) if return_scored else tok[:n].copy()


def token_scores(q, K) -> np.ndarray:
    """Head-summed indexer score of every key row of K [n][d] for q [R][d] (the token step's score)."""
    return chunk_scores(q, K)


def attend(q, K, V, tokens, scale: float | None = None, with_lse: bool = False):
    """Exact softmax attention of q [R][d] over K/V rows ``tokens``; float64 [R][d]."""
    q = _u16(q)
    K = _u16(K)
    V = _u16(V)
    R, d = q.shape
    tokens = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
    if tokens.size and (tokens.min() < 0 or tokens.max() >= K.shape[0]):
        raise IndexError("token outside K")
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = np.zeros((R, d), dtype=np.float64)
    lse = np.zeros(R, dtype=np.float64)
    lib().oracle_attend(_p(q), R, d, _p(K), _p(V), _p(tokens), tokens.size, sc, _p(out), _p(lse))
    return (out, lse) if with_lse else out


def prefill_block(q_block, K, V, cache_tokens, P: int, scale: float | None = None):
    """Block of queries at P.. sharing cache_tokens, plus causal own tokens; [n_q][R][d]."""
    q = _u16(q_block)
    n_q, R, d = q.shape
    K = _u16(K)
    V = _u16(V)
    ct = np.ascontiguousarray(np.asarray(cache_tokens, dtype=np.int32))
    if P + n_q > K.shape[0]:
        raise IndexError("block outside K")
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = np.zeros((n_q, R, d), dtype=np.float64)
    lib().oracle_prefill_block(_p(q), n_q, R * d, R, d, _p(K), _p(V), _p(ct), ct.size, P, sc, _p(out))
    return out


def decode_one(q, K, V, L: int, C: int, g: int, k: int, G: int, scale: float | None = None):
    """Whole decode step for one (sequence, KV head) from raw keys: summaries, routing, attention."""
    cs, gs = summaries(K[:L], C, g)
    tok = route(q, cs, gs, L, C, g, k, G)
    return attend(q, K, V, tok, scale), tok
