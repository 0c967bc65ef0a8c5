"""Seeded synthetic inputs for routed-attention decode and prefill.

The arithmetic lives in ``hga_synth.c`` (SplitMix64 counter streams, Box-Muller
normals, rotate-half rotary embedding in double precision, planted chunks,
bfloat16 round-to-nearest-even). This module builds that file into
``libhga_synth.so``, binds it with ctypes, and lays the results out as the
library expects: K/V head-major ``[B][Hkv][L][d]`` (or a shuffled page pool),
q ``[B][Hq][d]``, all bfloat16 bit patterns in ``numpy.uint16`` arrays.

The workloads mirror the shapes of the Hierarchical Global Attention abstract
(Qwen3-30B-A3B attention: 32 query heads, 4 KV heads, head dim 128, contexts of
4K to 64K tokens, about 3% of tokens routed). Nothing here routes or attends.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hga_synth.c")
_LIB = os.path.join(_HERE, "libhga_synth.so")

ROPE_THETA = 1.0e6
SEED_BASE = 20260701


def build(force: bool = False) -> str:
    """Compile hga_synth.c into libhga_synth.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", _LIB, _SRC, "-lm"]
        )
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        i32, i64, u64, dbl = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_double
        vp = ctypes.c_void_p
        L.synth_u64.argtypes = [u64, u64, u64]
        L.synth_u64.restype = u64
        L.synth_normal.argtypes = [u64, u64, u64]
        L.synth_normal.restype = dbl
        L.synth_bf16_rne.argtypes = [dbl]
        L.synth_bf16_rne.restype = ctypes.c_uint16
        L.synth_plant_chunks.argtypes = [u64, i32, i32, i32, vp]
        L.synth_plant_chunks.restype = i32
        L.synth_sequence.argtypes = [u64, i32, i32, i32, vp, i32, i32, i32, dbl, i32, i32, i32,
                                     vp, vp, vp, i64, vp]
        L.synth_sequence.restype = i32
        L.synth_permutation.argtypes = [u64, u64, i32, vp]
        L.synth_permutation.restype = None
        L.synth_uniform_ints.argtypes = [u64, u64, i32, i32, i32, vp]
        L.synth_uniform_ints.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------


@dataclass(frozen=True)
class Workload:
    """One synthetic routed-attention workload (sizes and routing parameters)."""

    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ctx_len: int  # decode: tokens in cache (query sits at ctx_len-1); prefill: cache length
    chunk: int
    group: int
    top_chunks: int
    top_groups: int
    n_plant: int  # planted chunks per sequence (-1: one per 8 full chunks)
    seed: int
    paged: bool = False
    page_size: int = 128
    min_len: int = 0  # ragged batches: lengths uniform over [min_len, ctx_len]
    n_new: int = 0  # prefill: new query tokens
    block: int = 0  # prefill: queries sharing one routing decision


TINY_DECODE_4K = Workload("tiny_decode_4k", 1, 4, 1, 64, 4096, 64, 16, 8, 2, 4, SEED_BASE + 0)
DECODE_16K = Workload("decode_16k", 1, 32, 4, 128, 16384, 128, 16, 16, 4, 16, SEED_BASE + 1)
DECODE_64K = Workload("decode_64k", 1, 32, 4, 128, 65536, 128, 16, 32, 4, 64, SEED_BASE + 2)
BATCHED_PAGED = Workload("batched_paged_16x4k_64k", 16, 32, 4, 128, 65536, 128, 16, 32, 4, -1,
                         SEED_BASE + 3, paged=True, page_size=128, min_len=4096)
PREFILL_64K = Workload("prefill_2048_on_63488", 1, 32, 4, 128, 63488, 128, 16, 32, 4, -1,
                       SEED_BASE + 4, n_new=2048, block=64)

WORKLOADS = {w.name: w for w in (TINY_DECODE_4K, DECODE_16K, DECODE_64K, BATCHED_PAGED, PREFILL_64K)}
SWEEP_LENGTHS = (4096, 8192, 16384, 32768, 65536)


def n_plant_for(w: Workload, n_chunks: int) -> int:
    return n_chunks // 8 if w.n_plant < 0 else w.n_plant


# ---------------------------------------------------------------------------
# generation
# ---------------------------------------------------------------------------


@dataclass
class Sequence:
    q: np.ndarray  # [n_q][Hq][d] uint16
    k: np.ndarray  # [Hkv][L][d] uint16
    v: np.ndarray
    planted: np.ndarray  # int32 chunk ids
    q_pos: np.ndarray  # int32 positions of the queries


def sequence(w: Workload, seq: int, length: int, q_pos, plant_chunks: int | None = None,
             out_k: np.ndarray | None = None, out_v: np.ndarray | None = None) -> Sequence:
    """Generate one sequence: K/V for positions [0, length) and q at q_pos.

    ``out_k``/``out_v`` may be [Hkv][Lmax][d] views to write into (Lmax >= length).
    """
    q_pos = np.ascontiguousarray(np.asarray(q_pos, dtype=np.int32).reshape(-1))
    n_q = q_pos.shape[0]
    H, Hkv, d = w.n_q_heads, w.n_kv_heads, w.head_dim
    q = np.empty((n_q, H, d), dtype=np.uint16)
    if out_k is None:
        out_k = np.empty((Hkv, length, d), dtype=np.uint16)
        out_v = np.empty((Hkv, length, d), dtype=np.uint16)
    assert out_k.flags.c_contiguous and out_v.flags.c_contiguous
    assert out_k.shape[0] == Hkv and out_k.shape[1] >= length and out_k.shape[2] == d
    stride = out_k.shape[1] * d
    pc = (length // w.chunk) if plant_chunks is None else plant_chunks
    n_plant = n_plant_for(w, pc)
    planted = np.zeros(max(n_plant, 1), dtype=np.int32)
    n = lib().synth_sequence(w.seed, seq, length, n_q, _ptr(q_pos), H, Hkv, d, ROPE_THETA, w.chunk,
                             pc, n_plant, _ptr(q), _ptr(out_k), _ptr(out_v), stride, _ptr(planted))
    if n < 0:
        raise RuntimeError("synth_sequence failed")
    return Sequence(q=q, k=out_k[:, :length], v=out_v[:, :length], planted=planted[:n].copy(),
                    q_pos=q_pos)


@dataclass
class DecodeInputs:
    w: Workload
    q: np.ndarray  # [B][Hq][d]
    k: np.ndarray  # [B][Hkv][Lmax][d]
    v: np.ndarray
    seq_lens: np.ndarray  # [B] int32
    planted: list = field(default_factory=list)


def decode_inputs(w: Workload, lengths=None, max_len: int | None = None, replicas_of: int | None = None) -> DecodeInputs:
    """Contiguous decode inputs: one query per sequence at position len-1.

    ``lengths`` defaults to ``ctx_len`` for every sequence. With ``replicas_of=n``
    only the first n sequences are drawn and the rest repeat them (distinct
    memory, same values), which keeps large batches quick to build.
    """
    B = w.batch
    if lengths is None:
        lengths = [w.ctx_len] * B
    lengths = [int(x) for x in lengths]
    B = len(lengths)
    Lmax = max(lengths) if max_len is None else max_len
    H, Hkv, d = w.n_q_heads, w.n_kv_heads, w.head_dim
    q = np.empty((B, H, d), dtype=np.uint16)
    k = np.zeros((B, Hkv, Lmax, d), dtype=np.uint16)
    v = np.zeros((B, Hkv, Lmax, d), dtype=np.uint16)
    planted = []
    for b in range(B):
        src = b if replicas_of is None else b % replicas_of
        if src != b and lengths[src] == lengths[b]:
            q[b] = q[src]
            k[b] = k[src]
            v[b] = v[src]
            planted.append(planted[src])
            continue
        s = sequence(w, src, lengths[b], [lengths[b] - 1], out_k=k[b], out_v=v[b])
        q[b] = s.q[0]
        planted.append(s.planted)
    return DecodeInputs(w=w, q=q, k=k, v=v, seq_lens=np.asarray(lengths, dtype=np.int32), planted=planted)


@dataclass
class PagedInputs:
    w: Workload
    q: np.ndarray  # [B][Hq][d]
    k_pool: np.ndarray  # [P][Hkv][page][d]
    v_pool: np.ndarray
    page_table: np.ndarray  # [B][max_pages] int32 (unused slots -1)
    seq_lens: np.ndarray  # [B] int32
    planted: list = field(default_factory=list)

    def contiguous(self, b: int):
        """K, V of sequence b gathered back to [Hkv][L][d] through the page table."""
        L = int(self.seq_lens[b])
        ps = self.w.page_size
        n = (L + ps - 1) // ps
        pages = self.page_table[b, :n]
        k = self.k_pool[pages].transpose(1, 0, 2, 3).reshape(self.w.n_kv_heads, n * ps, -1)[:, :L]
        v = self.v_pool[pages].transpose(1, 0, 2, 3).reshape(self.w.n_kv_heads, n * ps, -1)[:, :L]
        return np.ascontiguousarray(k), np.ascontiguousarray(v)


def seq_lengths(w: Workload) -> np.ndarray:
    """Ragged lengths, seeded, uniform over [min_len, ctx_len] inclusive."""
    out = np.zeros(w.batch, dtype=np.int32)
    lib().synth_uniform_ints(w.seed, 1_000_003, w.batch, w.min_len, w.ctx_len, _ptr(out))
    return out


def paged_inputs(w: Workload, lengths=None) -> PagedInputs:
    """Ragged batched decode with a paged K/V pool and a shuffled page table."""
    ps = w.page_size
    lens = seq_lengths(w) if lengths is None else np.asarray(lengths, dtype=np.int32)
    B = len(lens)
    H, Hkv, d = w.n_q_heads, w.n_kv_heads, w.head_dim
    n_pages = [(int(L) + ps - 1) // ps for L in lens]
    total = int(sum(n_pages))
    max_pages = max(n_pages)
    perm = np.zeros(total, dtype=np.int32)
    lib().synth_permutation(w.seed, 1_000_004, total, _ptr(perm))
    k_pool = np.zeros((total, Hkv, ps, d), dtype=np.uint16)
    v_pool = np.zeros((total, Hkv, ps, d), dtype=np.uint16)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    q = np.empty((B, H, d), dtype=np.uint16)
    planted = []
    off = 0
    for b in range(B):
        L = int(lens[b])
        s = sequence(w, b, L, [L - 1])
        q[b] = s.q[0]
        planted.append(s.planted)
        pages = perm[off:off + n_pages[b]]
        off += n_pages[b]
        table[b, :n_pages[b]] = pages
        pad = n_pages[b] * ps - L
        kk = np.pad(s.k, ((0, 0), (0, pad), (0, 0))).reshape(Hkv, n_pages[b], ps, d)
        vv = np.pad(s.v, ((0, 0), (0, pad), (0, 0))).reshape(Hkv, n_pages[b], ps, d)
        k_pool[pages] = kk.transpose(1, 0, 2, 3)
        v_pool[pages] = vv.transpose(1, 0, 2, 3)
    return PagedInputs(w=w, q=q, k_pool=k_pool, v_pool=v_pool, page_table=table, seq_lens=lens,
                       planted=planted)


@dataclass
class PrefillInputs:
    w: Workload
    q: np.ndarray  # [T][Hq][d], positions cache_len .. cache_len+T-1
    k: np.ndarray  # [1][Hkv][cache_len+T][d]
    v: np.ndarray
    cache_len: int
    planted: np.ndarray


def prefill_inputs(w: Workload, cache_len: int | None = None, n_new: int | None = None) -> PrefillInputs:
    """Chunked prefill: n_new queries right after a cache of cache_len tokens.

    Planted chunks are drawn among the cache's full chunks, shifted along the
    normalised sum of all new queries (per KV head).
    """
    L0 = w.ctx_len if cache_len is None else cache_len
    T = w.n_new if n_new is None else n_new
    Hkv, d = w.n_kv_heads, w.head_dim
    k = np.zeros((1, Hkv, L0 + T, d), dtype=np.uint16)
    v = np.zeros((1, Hkv, L0 + T, d), dtype=np.uint16)
    s = sequence(w, 0, L0 + T, np.arange(L0, L0 + T, dtype=np.int32), plant_chunks=L0 // w.chunk,
                 out_k=k[0], out_v=v[0])
    return PrefillInputs(w=w, q=s.q, k=k, v=v, cache_len=L0, planted=s.planted)


def with_len(w: Workload, L: int) -> Workload:
    """The same routing parameters at another context length (planted count scales 1/8)."""
    return replace(w, name=f"{w.name}@{L}", ctx_len=L, n_plant=(L // w.chunk) // 8)
