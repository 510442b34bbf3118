"""CPU oracle for MiniMax-M3 block-sparse attention over a paged KV cache.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline / reference arm are the only code allowed to import this package.  The GPU product
path never imports, loads or calls it, and it imports nothing from that path.

The arithmetic lives in ``msa_oracle.c`` (plain loops, fp64).  This module only compiles it
with gcc, loads it with ctypes and marshals numpy arrays.  See ``msa_oracle.c`` for the
definition each function follows and the readings taken where the pages are silent.

Parity pins (tests/test_oracle_pins.py) check it against numpy brute force, torch's own
bf16 / float8_e4m3fn decoders, closed forms of attention and hand-worked selection cases.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_LIB = os.path.join(_HERE, "libmsa_oracle.so")

BLOCK = 128
HEAD_DIM = 128


def build(force: bool = False) -> str:
    """Compile msa_oracle.c into libmsa_oracle.so with gcc (OpenMP, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
             "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.orc_bf16_value.restype = ctypes.c_double
        lib.orc_bf16_value.argtypes = [ctypes.c_uint16]
        lib.orc_e4m3_value.restype = ctypes.c_double
        lib.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.orc_e2m1_value.restype = ctypes.c_double
        lib.orc_e2m1_value.argtypes = [ctypes.c_uint8]
        lib.orc_ue8m0_value.restype = ctypes.c_double
        lib.orc_ue8m0_value.argtypes = [ctypes.c_uint8]
        lib.orc_index_scores.restype = None
        lib.orc_index_scores.argtypes = [I, P, P, P, I, P, I, P, P, I, I, I, P]
        lib.orc_select_blocks.restype = None
        lib.orc_select_blocks.argtypes = [I, P, P, I, I, P, I, I, I, I, P, P]
        lib.orc_select_blocks_shared.restype = None
        lib.orc_select_blocks_shared.argtypes = [I, P, P, I, I, P, I, I, I, I, P, P]
        lib.orc_latent_attention.restype = None
        lib.orc_latent_attention.argtypes = [I, P, P, I, I, P, I, I, P, P, I, P, I, I, P, I, P,
                                             I, P, ctypes.c_double, P]
        lib.orc_attention.restype = None
        lib.orc_attention.argtypes = [I, P, P, P, I, P, P, P, I, I, I, P, P, I,
                                      ctypes.c_double, P]
        _lib = lib
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def bf16_value(bits: int) -> float:
    return _load().orc_bf16_value(int(bits))


def e4m3_value(code: int) -> float:
    return _load().orc_e4m3_value(int(code))


def e2m1_value(code: int) -> float:
    return _load().orc_e2m1_value(int(code))


def ue8m0_value(code: int) -> float:
    return _load().orc_ue8m0_value(int(code))


IDX_FORMATS = {"bf16": 0, "fp8": 1, "fp4": 2}


def _bits16(x):
    """Raw 16-bit patterns of a bf16 array given as a torch tensor or a uint16/int16 ndarray."""
    if hasattr(x, "view") and hasattr(x, "dtype") and "torch" in str(type(x)):
        import torch
        return x.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    return np.asarray(x).view(np.uint16)


def _bytes8(x):
    if hasattr(x, "dtype") and "torch" in str(type(x)):
        import torch
        return x.detach().contiguous().cpu().view(torch.uint8).numpy()
    return np.asarray(x).view(np.uint8)


def _ints(x):
    if hasattr(x, "dtype") and "torch" in str(type(x)):
        return x.detach().cpu().numpy().astype(np.int32)
    return np.asarray(x, dtype=np.int32)


def index_scores(row_off, cache_len, table, q_idx, k_idx, max_blocks, k_idx_scale=None,
                 idx_dtype="bf16"):
    """Block scores [total_q, H_kv, max_blocks] in fp64 (-inf where the block is not visible).

    q_idx bf16 [total_q, H_kv, 128]; k_idx by ``idx_dtype``: "bf16" bf16 [num_pages, H_idxk,
    128, 128]; "fp8" e4m3 bytes [num_pages, H_idxk, 128, 128] with k_idx_scale float32
    [num_pages, H_idxk, 128]; "fp4" e2m1 pairs uint8 [num_pages, H_idxk, 128, 64] with
    k_idx_scale ue8m0 uint8 [num_pages, H_idxk, 128, 4].
    """
    lib = _load()
    fmt = IDX_FORMATS[idx_dtype]
    row_off, p_off = _c(_ints(row_off), np.int32)
    cache_len, p_cl = _c(_ints(cache_len), np.int32)
    table, p_tab = _c(_ints(table), np.int32)
    qb, p_q = _c(_bits16(q_idx), np.uint16)
    if fmt == 0:
        kb, p_k = _c(_bits16(k_idx), np.uint16)
        p_s = None
    else:
        kb, p_k = _c(_bytes8(k_idx), np.uint8)
        assert kb.shape[3] == (128 if fmt == 1 else 64), kb.shape
        if fmt == 1:
            sc = np.asarray(k_idx_scale.detach().cpu().numpy() if hasattr(k_idx_scale, "detach")
                            else k_idx_scale, dtype=np.float32)
            sc, p_s = _c(sc, np.float32)
            assert sc.shape == kb.shape[:3]
        else:
            sc, p_s = _c(_bytes8(k_idx_scale), np.uint8)
            assert sc.shape == kb.shape[:3] + (4,)
    total_q, H_kv, _ = qb.shape
    H_idxk = kb.shape[1]
    batch = row_off.shape[0] - 1
    out = np.empty((total_q, H_kv, max_blocks), dtype=np.float64)
    lib.orc_index_scores(batch, p_off, p_cl, p_tab, table.shape[1], p_q, fmt, p_k, p_s, H_kv,
                         H_idxk, max_blocks, out.ctypes.data_as(ctypes.c_void_p))
    return out


def select_blocks(row_off, cache_len, scores, top_k, init_blocks, local_blocks):
    """Selected block ids [total_q, H_kv, S] (ascending, -1 padded) and counts [total_q, H_kv].

    ``scores`` may be fp64 or fp32; comparisons are made on its values as given.
    """
    lib = _load()
    row_off, p_off = _c(_ints(row_off), np.int32)
    cache_len, p_cl = _c(_ints(cache_len), np.int32)
    sc, p_sc = _c(np.asarray(scores, dtype=np.float64), np.float64)
    total_q, H_kv, max_blocks = sc.shape
    S = init_blocks + local_blocks + top_k
    ids = np.empty((total_q, H_kv, S), dtype=np.int32)
    counts = np.empty((total_q, H_kv), dtype=np.int32)
    lib.orc_select_blocks(row_off.shape[0] - 1, p_off, p_cl, H_kv, max_blocks, p_sc, top_k,
                          init_blocks, local_blocks, S, ids.ctypes.data_as(ctypes.c_void_p),
                          counts.ctypes.data_as(ctypes.c_void_p))
    return ids, counts


def select_blocks_shared(row_off, cache_len, scores, top_k, init_blocks, local_blocks):
    """The selection with the indexer top-k shared across a sequence's new tokens: the top-k
    of the first new token's candidates, plus each token's own forced blocks, ascending.  Only
    the first new token's row of ``scores`` is read."""
    lib = _load()
    row_off, p_off = _c(_ints(row_off), np.int32)
    cache_len, p_cl = _c(_ints(cache_len), np.int32)
    sc, p_sc = _c(np.asarray(scores, dtype=np.float64), np.float64)
    total_q, H_kv, max_blocks = sc.shape
    S = init_blocks + local_blocks + top_k
    ids = np.empty((total_q, H_kv, S), dtype=np.int32)
    counts = np.empty((total_q, H_kv), dtype=np.int32)
    lib.orc_select_blocks_shared(row_off.shape[0] - 1, p_off, p_cl, H_kv, max_blocks, p_sc,
                                 top_k, init_blocks, local_blocks, S,
                                 ids.ctypes.data_as(ctypes.c_void_p),
                                 counts.ctypes.data_as(ctypes.c_void_p))
    return ids, counts


def attention(row_off, cache_len, table, q, k_cache, v_cache, kv_fp8, ids, counts, scale):
    """Attention output [total_q, H_q, 128] in fp64 over the selected, causally clipped
    positions.  q bf16 [total_q, H_q, 128]; caches bf16 or e4m3 [num_pages, H_kv, 128, 128]."""
    lib = _load()
    row_off, p_off = _c(_ints(row_off), np.int32)
    cache_len, p_cl = _c(_ints(cache_len), np.int32)
    table, p_tab = _c(_ints(table), np.int32)
    qb, p_q = _c(_bits16(q), np.uint16)
    if kv_fp8:
        kb, p_k = _c(_bytes8(k_cache), np.uint8)
        vb, p_v = _c(_bytes8(v_cache), np.uint8)
    else:
        kb, p_k = _c(_bits16(k_cache), np.uint16)
        vb, p_v = _c(_bits16(v_cache), np.uint16)
    ids, p_ids = _c(_ints(ids), np.int32)
    counts, p_cnt = _c(_ints(counts), np.int32)
    total_q, H_q, _ = qb.shape
    H_kv = kb.shape[1]
    S = ids.shape[2]
    out = np.empty((total_q, H_q, HEAD_DIM), dtype=np.float64)
    lib.orc_attention(row_off.shape[0] - 1, p_off, p_cl, p_tab, table.shape[1], p_q, p_k, p_v,
                      int(bool(kv_fp8)), H_q, H_kv, p_ids, p_cnt, S, float(scale),
                      out.ctypes.data_as(ctypes.c_void_p))
    return out


def forward(inp, top_k, init_blocks, local_blocks, scale, max_blocks, share=False):
    """The whole path: scores -> selection -> attention.  ``inp`` is a mapping with the
    tensors named as in the C-ABI (row_off, cache_len, table, q, q_idx, k_idx, k, v, kv_fp8).
    ``share``: the indexer top-k shared across each sequence's new tokens."""
    sc = index_scores(inp["row_off"], inp["cache_len"], inp["table"], inp["q_idx"],
                      inp["k_idx"], max_blocks, inp.get("k_idx_scale"),
                      inp.get("idx_dtype", "bf16"))
    sel = select_blocks_shared if share else select_blocks
    ids, counts = sel(inp["row_off"], inp["cache_len"], sc, top_k, init_blocks, local_blocks)
    out = attention(inp["row_off"], inp["cache_len"], inp["table"], inp["q"], inp["k"],
                    inp["v"], inp["kv_fp8"], ids, counts, scale)
    return sc, ids, counts, out


def latent_attention(row_off, q, window, swa_kv, swa_layer, swa_len, swa_table, comp_kv,
                     comp_layer, comp_table, comp_idx, sink, scale):
    """Latent sparse attention [total_q, H, 128] in fp64: K = V latent rows from the
    sliding-window leaf (the ``window`` positions ending at each query's position
    swa_len[b] + i) and from the compressed leaf (comp_idx [total_q, n_entries], -1 padding),
    with the per-head sink in the denominator.  Leaves bf16 [pages, layers, 128, 128]."""
    lib = _load()
    row_off, p_off = _c(_ints(row_off), np.int32)
    qb, p_q = _c(_bits16(q), np.uint16)
    sw, p_sw = _c(_bits16(swa_kv), np.uint16)
    cp, p_cp = _c(_bits16(comp_kv), np.uint16)
    sl, p_sl = _c(_ints(swa_len), np.int32)
    st, p_st = _c(_ints(swa_table), np.int32)
    ct, p_ct = _c(_ints(comp_table), np.int32)
    ci, p_ci = _c(_ints(comp_idx), np.int32)
    sk = np.asarray(sink.detach().cpu().numpy() if hasattr(sink, "detach") else sink,
                    dtype=np.float32)
    sk, p_sk = _c(sk, np.float32)
    total_q, H, _ = qb.shape
    out = np.empty((total_q, H, HEAD_DIM), dtype=np.float64)
    lib.orc_latent_attention(row_off.shape[0] - 1, p_off, p_q, H, int(window), p_sw,
                             sw.shape[1], int(swa_layer), p_sl, p_st, st.shape[1], p_cp,
                             cp.shape[1], int(comp_layer), p_ct, ct.shape[1], p_ci,
                             ci.shape[1], p_sk, float(scale),
                             out.ctypes.data_as(ctypes.c_void_p))
    return out
