"""ctypes binding of libmsa.so (include/msa.h), one Python function per C entry point.

Argument marshalling only: every step of the path runs in the library's CUDA kernels.  Torch
tensors supply device memory and the current CUDA stream.  The library is loaded on first use
and a missing or unloadable library raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa.so")

MSA_OK, MSA_ERR_INVALID_ARG, MSA_ERR_UNSUPPORTED, MSA_ERR_CUDA = 0, 1, 2, 3
MSA_KV_BF16, MSA_KV_FP8_E4M3 = 0, 1
MSA_IDX_BF16, MSA_IDX_FP8_E4M3, MSA_IDX_FP4_E2M1 = 0, 1, 2
IDX_DTYPES = {"bf16": MSA_IDX_BF16, "fp8": MSA_IDX_FP8_E4M3, "fp4": MSA_IDX_FP4_E2M1}
MSA_DEVERR_PAGE_ID, MSA_DEVERR_LENGTHS, MSA_DEVERR_BLOCK_ID = 1, 2, 4
MSA_DEVERR_NUM_SELECTED, MSA_DEVERR_TIMEOUT = 8, 16
MSA_SHARE_ACROSS_DRAFTS = 1
BLOCK = 128
HEAD_DIM = 128


class MSAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {msa_status_string(status)} ({status})")
        self.status = status


class RaggedPaged(ctypes.Structure):
    """msa_ragged_paged_t."""
    _fields_ = [("input_row_offsets", ctypes.c_void_p), ("cache_lengths", ctypes.c_void_p),
                ("kv_lookup_table", ctypes.c_void_p), ("batch", ctypes.c_int32),
                ("total_q", ctypes.c_int32), ("max_q_len", ctypes.c_int32),
                ("max_pages_per_seq", ctypes.c_int32), ("num_pages", ctypes.c_int32)]


class IndexK(ctypes.Structure):
    """msa_index_k_t: the index-K cache in one of the msa_idx_dtype_t formats."""
    _fields_ = [("dtype", ctypes.c_int32), ("codes", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("num_heads", ctypes.c_int32)]


def index_k(codes, scales, num_heads: int, idx_dtype: str = "bf16") -> IndexK:
    """The msa_index_k_t view of an index-K cache (no copies)."""
    return IndexK(IDX_DTYPES[idx_dtype], _ptr(codes), _ptr(scales), int(num_heads))


class LatentLeaf(ctypes.Structure):
    """msa_latent_leaf_t: one paged leaf of the latent sparse attention."""
    _fields_ = [("kv", ctypes.c_void_p), ("cache_lengths", ctypes.c_void_p),
                ("lookup_table", ctypes.c_void_p), ("max_pages_per_seq", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("num_layers", ctypes.c_int32),
                ("layer", ctypes.c_int32)]


def latent_leaf(kv, cache_lengths, lookup_table, layer: int) -> LatentLeaf:
    """The msa_latent_leaf_t view of a leaf (kv bf16 [pages, layers, 128, 128]; no copies)."""
    return LatentLeaf(_ptr(kv), _ptr(cache_lengths), _ptr(lookup_table),
                      int(lookup_table.shape[-1]), int(kv.shape[0]), int(kv.shape[1]),
                      int(layer))


_lib: Optional[ctypes.CDLL] = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmsa.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m block_sparse_paged_scores_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    RP = ctypes.POINTER(RaggedPaged)
    lib.msa_index_scores.restype = I
    lib.msa_index_scores.argtypes = [RP, P, P, I, I, I, P, P, P]
    lib.msa_select_blocks.restype = I
    lib.msa_select_blocks.argtypes = [RP, P, I, I, I, I, I, P, P, P, P]
    lib.msa_index_select.restype = I
    lib.msa_index_select.argtypes = [RP, P, P, I, I, I, I, I, I, P, P, P, P, P, P]
    IK = ctypes.POINTER(IndexK)
    U = ctypes.c_uint32
    lib.msa_index_scores_k.restype = I
    lib.msa_index_scores_k.argtypes = [RP, P, IK, I, I, U, P, P, P]
    lib.msa_index_select_k.restype = I
    lib.msa_index_select_k.argtypes = [RP, P, IK, I, I, I, I, I, U, P, P, P, P, P, P]
    lib.msa_index_select_counters.restype = ctypes.c_size_t
    lib.msa_index_select_counters.argtypes = [RP, I]
    lib.msa_sparse_attn_paged.restype = I
    lib.msa_sparse_attn_paged.argtypes = [RP, P, P, P, I, P, P, I, I, I, I, F, I, P,
                                          ctypes.c_size_t, P, P, P]
    lib.msa_select_sparse_attn_paged.restype = I
    lib.msa_select_sparse_attn_paged.argtypes = [RP, P, I, I, I, P, P, P, I, I, I, I, F, I, P,
                                                 ctypes.c_size_t, P, P, P, P, P]
    lib.msa_decode_step_workspace_bytes.restype = ctypes.c_size_t
    lib.msa_decode_step_workspace_bytes.argtypes = [RP, I, I, I, I, I, I]
    lib.msa_decode_step.restype = I
    lib.msa_decode_step.argtypes = [RP, P, IK, I, I, I, P, P, P, I, I, I, I, F, I, P,
                                    ctypes.c_size_t, P, P, P, P, P, P]
    lib.msa_splitk_combine.restype = I
    lib.msa_splitk_combine.argtypes = [P, P, I, I, I, P, P]
    lib.msa_attn_workspace_bytes.restype = ctypes.c_size_t
    lib.msa_attn_workspace_bytes.argtypes = [RP, I, I, I, I, I]
    lib.msa_default_num_splits.restype = I
    lib.msa_default_num_splits.argtypes = [I, I, I, I, I]
    lib.msa_sparse_attn_paged_noalloc.restype = I
    lib.msa_sparse_attn_paged_noalloc.argtypes = [RP, P, P, P, I, P, P, I, I, I, I, F, I, P, P,
                                                  P]
    lib.msa_attn_partials.restype = I
    lib.msa_attn_partials.argtypes = [RP, I, I, I, I, I, ctypes.POINTER(ctypes.c_size_t),
                                      ctypes.POINTER(ctypes.c_size_t)]
    LL = ctypes.POINTER(LatentLeaf)
    lib.msa_latent_sparse_attn_paged.restype = I
    lib.msa_latent_sparse_attn_paged.argtypes = [P, I, I, I, P, I, LL, I, LL, P, I, P, F, I, P,
                                                 ctypes.c_size_t, P, P, P]
    lib.msa_latent_workspace_bytes.restype = ctypes.c_size_t
    lib.msa_latent_workspace_bytes.argtypes = [I, I, I]
    lib.msa_latent_default_splits.restype = I
    lib.msa_latent_default_splits.argtypes = [I, I, I, I, I]
    lib.msa_selftest_bounded_wait.restype = I
    lib.msa_selftest_bounded_wait.argtypes = [ctypes.c_uint32, P, P, P]
    lib.msa_status_string.restype = ctypes.c_char_p
    lib.msa_status_string.argtypes = [I]
    _lib = lib
    return lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, status: int):
    if status != MSA_OK:
        raise MSAError(fn, status)


def ragged_paged(input_row_offsets, cache_lengths, kv_lookup_table, total_q: int, max_q_len: int,
                 num_pages: int) -> RaggedPaged:
    """Build the msa_ragged_paged_t view of int32 device tensors (no copies)."""
    return RaggedPaged(_ptr(input_row_offsets), _ptr(cache_lengths), _ptr(kv_lookup_table),
                       int(input_row_offsets.numel()) - 1, int(total_q), int(max_q_len),
                       int(kv_lookup_table.shape[-1]), int(num_pages))


def msa_status_string(status: int) -> str:
    return load().msa_status_string(int(status)).decode()


def msa_default_num_splits(batch: int, max_q_len: int, num_kv_heads: int, S: int,
                           num_sms: int) -> int:
    return int(load().msa_default_num_splits(batch, max_q_len, num_kv_heads, S, num_sms))


def msa_attn_workspace_bytes(rp: RaggedPaged, S: int, num_q_heads: int, num_kv_heads: int,
                             max_blocks: int, num_splits: int) -> int:
    return int(load().msa_attn_workspace_bytes(ctypes.byref(rp), S, num_q_heads, num_kv_heads,
                                               max_blocks, num_splits))


def msa_attn_partials(rp: RaggedPaged, S: int, num_q_heads: int, num_kv_heads: int,
                      max_blocks: int, num_splits: int):
    """(number of partial split indices, partial_o byte offset, partial_lse byte offset)."""
    o, l_ = ctypes.c_size_t(0), ctypes.c_size_t(0)
    n = load().msa_attn_partials(ctypes.byref(rp), S, num_q_heads, num_kv_heads, max_blocks,
                                 num_splits, ctypes.byref(o), ctypes.byref(l_))
    return int(n), int(o.value), int(l_.value)


def msa_index_scores(rp: RaggedPaged, q_idx, k_idx_cache, num_kv_heads: int,
                     num_idx_k_heads: int, max_blocks: int, scores, dev_err=None, stream=None):
    _check("msa_index_scores", load().msa_index_scores(
        ctypes.byref(rp), _ptr(q_idx), _ptr(k_idx_cache), num_kv_heads, num_idx_k_heads,
        max_blocks, _ptr(scores), _ptr(dev_err), _stream(stream)))


def msa_select_blocks(rp: RaggedPaged, scores, num_kv_heads: int, max_blocks: int, top_k: int,
                      init_blocks: int, local_blocks: int, block_ids, num_selected, dev_err=None,
                      stream=None):
    _check("msa_select_blocks", load().msa_select_blocks(
        ctypes.byref(rp), _ptr(scores), num_kv_heads, max_blocks, top_k, init_blocks,
        local_blocks, _ptr(block_ids), _ptr(num_selected), _ptr(dev_err), _stream(stream)))


def msa_index_scores_k(rp: RaggedPaged, q_idx, k_idx: IndexK, num_kv_heads: int,
                       max_blocks: int, flags: int, scores, dev_err=None, stream=None):
    _check("msa_index_scores_k", load().msa_index_scores_k(
        ctypes.byref(rp), _ptr(q_idx), ctypes.byref(k_idx), num_kv_heads, max_blocks,
        int(flags), _ptr(scores), _ptr(dev_err), _stream(stream)))


def msa_index_select_k(rp: RaggedPaged, q_idx, k_idx: IndexK, num_kv_heads: int,
                       max_blocks: int, top_k: int, init_blocks: int, local_blocks: int,
                       flags: int, scores, block_ids, num_selected, counters, dev_err=None,
                       stream=None):
    _check("msa_index_select_k", load().msa_index_select_k(
        ctypes.byref(rp), _ptr(q_idx), ctypes.byref(k_idx), num_kv_heads, max_blocks, top_k,
        init_blocks, local_blocks, int(flags), _ptr(scores), _ptr(block_ids),
        _ptr(num_selected), _ptr(counters), _ptr(dev_err), _stream(stream)))


def msa_index_select_counters(rp: RaggedPaged, num_idx_k_heads: int) -> int:
    return int(load().msa_index_select_counters(ctypes.byref(rp), num_idx_k_heads))


def msa_index_select(rp: RaggedPaged, q_idx, k_idx_cache, num_kv_heads: int,
                     num_idx_k_heads: int, max_blocks: int, top_k: int, init_blocks: int,
                     local_blocks: int, scores, block_ids, num_selected, counters, dev_err=None,
                     stream=None):
    _check("msa_index_select", load().msa_index_select(
        ctypes.byref(rp), _ptr(q_idx), _ptr(k_idx_cache), num_kv_heads, num_idx_k_heads,
        max_blocks, top_k, init_blocks, local_blocks, _ptr(scores), _ptr(block_ids),
        _ptr(num_selected), _ptr(counters), _ptr(dev_err), _stream(stream)))


def msa_sparse_attn_paged(rp: RaggedPaged, q, k_cache, v_cache, kv_dtype: int, block_ids,
                          num_selected, S: int, num_q_heads: int, num_kv_heads: int,
                          max_blocks: int, scale: float, num_splits: int, workspace, out,
                          dev_err=None, stream=None, workspace_bytes: Optional[int] = None):
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("msa_sparse_attn_paged", load().msa_sparse_attn_paged(
        ctypes.byref(rp), _ptr(q), _ptr(k_cache), _ptr(v_cache), int(kv_dtype), _ptr(block_ids),
        _ptr(num_selected), S, num_q_heads, num_kv_heads, max_blocks, float(scale), num_splits,
        _ptr(workspace), int(workspace_bytes), _ptr(out), _ptr(dev_err), _stream(stream)))


def msa_select_sparse_attn_paged(rp: RaggedPaged, scores, top_k: int, init_blocks: int,
                                 local_blocks: int, q, k_cache, v_cache, kv_dtype: int,
                                 num_q_heads: int, num_kv_heads: int, max_blocks: int,
                                 scale: float, num_splits: int, workspace, block_ids,
                                 num_selected, out, dev_err=None, stream=None,
                                 workspace_bytes: Optional[int] = None):
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("msa_select_sparse_attn_paged", load().msa_select_sparse_attn_paged(
        ctypes.byref(rp), _ptr(scores), top_k, init_blocks, local_blocks, _ptr(q), _ptr(k_cache),
        _ptr(v_cache), int(kv_dtype), num_q_heads, num_kv_heads, max_blocks, float(scale),
        num_splits, _ptr(workspace), int(workspace_bytes), _ptr(block_ids), _ptr(num_selected),
        _ptr(out), _ptr(dev_err), _stream(stream)))


def msa_decode_step_workspace_bytes(rp: RaggedPaged, S: int, num_q_heads: int,
                                    num_kv_heads: int, num_idx_k_heads: int, max_blocks: int,
                                    num_splits: int) -> int:
    return int(load().msa_decode_step_workspace_bytes(ctypes.byref(rp), S, num_q_heads,
                                                      num_kv_heads, num_idx_k_heads, max_blocks,
                                                      num_splits))


def msa_decode_step(rp: RaggedPaged, q_idx, k_idx: IndexK, top_k: int, init_blocks: int,
                    local_blocks: int, q, k_cache, v_cache, kv_dtype: int, num_q_heads: int,
                    num_kv_heads: int, max_blocks: int, scale: float, num_splits: int,
                    workspace, scores, block_ids, num_selected, out, dev_err=None, stream=None,
                    workspace_bytes: Optional[int] = None):
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("msa_decode_step", load().msa_decode_step(
        ctypes.byref(rp), _ptr(q_idx), ctypes.byref(k_idx), top_k, init_blocks, local_blocks,
        _ptr(q), _ptr(k_cache), _ptr(v_cache), int(kv_dtype), num_q_heads, num_kv_heads,
        max_blocks, float(scale), num_splits, _ptr(workspace), int(workspace_bytes),
        _ptr(scores), _ptr(block_ids), _ptr(num_selected), _ptr(out), _ptr(dev_err),
        _stream(stream)))


def msa_sparse_attn_paged_noalloc(rp: RaggedPaged, q, k_cache, v_cache, kv_dtype: int,
                                  block_ids, num_selected, S: int, num_q_heads: int,
                                  num_kv_heads: int, max_blocks: int, scale: float,
                                  num_splits: int, out, dev_err=None, stream=None):
    """msa_sparse_attn_paged with its scratch in the library's own device array (for callers
    that cannot allocate a workspace); see include/msa.h for the size limit."""
    _check("msa_sparse_attn_paged_noalloc", load().msa_sparse_attn_paged_noalloc(
        ctypes.byref(rp), _ptr(q), _ptr(k_cache), _ptr(v_cache), int(kv_dtype), _ptr(block_ids),
        _ptr(num_selected), S, num_q_heads, num_kv_heads, max_blocks, float(scale), num_splits,
        _ptr(out), _ptr(dev_err), _stream(stream)))


def msa_latent_workspace_bytes(total_q: int, num_heads: int, num_splits: int) -> int:
    return int(load().msa_latent_workspace_bytes(total_q, num_heads, num_splits))


def msa_latent_default_splits(total_q: int, num_heads: int, window: int, n_entries: int,
                              num_sms: int) -> int:
    return int(load().msa_latent_default_splits(total_q, num_heads, window, n_entries, num_sms))


def msa_latent_sparse_attn_paged(input_row_offsets, batch: int, total_q: int, max_q_len: int,
                                 q, num_heads: int, swa: LatentLeaf, window: int,
                                 comp: LatentLeaf, comp_indices, n_entries: int, attn_sink,
                                 scale: float, num_splits: int, workspace, out, dev_err=None,
                                 stream=None, workspace_bytes: Optional[int] = None):
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("msa_latent_sparse_attn_paged", load().msa_latent_sparse_attn_paged(
        _ptr(input_row_offsets), batch, total_q, max_q_len, _ptr(q), num_heads,
        ctypes.byref(swa), window, ctypes.byref(comp), _ptr(comp_indices), n_entries,
        _ptr(attn_sink), float(scale), num_splits, _ptr(workspace), int(workspace_bytes),
        _ptr(out), _ptr(dev_err), _stream(stream)))


class LatentPath:
    """One latent sparse attention problem (a dict laid out as workload.generate_latent
    returns) with its output, workspace and error word allocated once; ``run()`` enqueues
    msa_latent_sparse_attn_paged on the current stream."""

    def __init__(self, prob: dict, num_splits: int = 0):
        self.p = prob
        dev = prob["q"].device
        self.swa = latent_leaf(prob["swa_kv"], prob["swa_len"], prob["swa_table"],
                               prob["swa_layer"])
        self.comp = latent_leaf(prob["comp_kv"], prob["comp_len"], prob["comp_table"],
                                prob["comp_layer"])
        self.num_splits = num_splits or msa_latent_default_splits(
            prob["total_q"], prob["H"], prob["window"], prob["n_entries"],
            torch.cuda.get_device_properties(dev).multi_processor_count)
        ws = msa_latent_workspace_bytes(prob["total_q"], prob["H"], self.num_splits)
        self.workspace = torch.empty((max(ws, 1),), dtype=torch.uint8, device=dev)
        self.workspace_bytes = ws
        self.out = torch.empty((prob["total_q"], prob["H"], HEAD_DIM), dtype=torch.bfloat16,
                               device=dev)
        self.dev_err = torch.zeros((1,), dtype=torch.int32, device=dev)

    def run(self, stream=None):
        p = self.p
        msa_latent_sparse_attn_paged(p["row_off"], p["batch"], p["total_q"], p["max_q_len"],
                                     p["q"], p["H"], self.swa, p["window"], self.comp,
                                     p["comp_idx"], p["n_entries"], p["sink"], p["scale"],
                                     self.num_splits, self.workspace, self.out, self.dev_err,
                                     stream, workspace_bytes=self.workspace_bytes)
        return self.out


def msa_selftest_bounded_wait(limit_us: int, dev_err, result, stream=None):
    """Diagnostic: the library's bounded pipeline wait made to run out (see include/msa.h)."""
    _check("msa_selftest_bounded_wait", load().msa_selftest_bounded_wait(
        int(limit_us), _ptr(dev_err), _ptr(result), _stream(stream)))


def msa_splitk_combine(partial_o, partial_lse, num_splits: int, total_q: int, num_q_heads: int,
                       out, stream=None):
    _check("msa_splitk_combine", load().msa_splitk_combine(
        _ptr(partial_o), _ptr(partial_lse), num_splits, total_q, num_q_heads, _ptr(out),
        _stream(stream)))


# ------------------------------------------------------------------ whole-path convenience
class Path:
    """The three stages over one problem (a dict laid out as ``workload.generate`` returns),
    with every output and the workspace allocated once on the problem's device.  ``run()``
    enqueues index scores -> selection -> attention on the current stream: by default the
    last two as one msa_select_sparse_attn_paged call (``select_in_attention``); with
    ``fused_select`` the first two as one msa_index_select call; with neither, three separate
    calls.  ``share_selection``: the indexer top-k shared across each sequence's draft tokens
    (MSA_SHARE_ACROSS_DRAFTS, through msa_index_select_k), then the attention.  ``one_call``
    (with ``select_in_attention``): the whole step as one msa_decode_step call, whose own
    workspace (flags and counters first, zeroed once here) is ``step_workspace``."""

    def __init__(self, prob: dict, num_splits: int = 0, max_blocks: Optional[int] = None,
                 fused_select: bool = False, select_in_attention: bool = True,
                 share_selection: bool = False, one_call: bool = True):
        self.p = prob
        self.share_selection = share_selection
        self.fused_select = fused_select or share_selection
        self.select_in_attention = select_in_attention
        dev = prob["q"].device
        self.max_blocks = int(max_blocks or prob["max_blocks"])
        self.rp = ragged_paged(prob["row_off"], prob["cache_len"], prob["table"], prob["total_q"],
                               prob["max_q_len"], prob["num_pages"])
        tq, hkv, S = prob["total_q"], prob["H_kv"], prob["S"]
        self.scores = torch.empty((tq, hkv, self.max_blocks), dtype=torch.float32, device=dev)
        self.block_ids = torch.empty((tq, hkv, S), dtype=torch.int32, device=dev)
        self.num_selected = torch.empty((tq, hkv), dtype=torch.int32, device=dev)
        self.out = torch.empty((tq, prob["H_q"], HEAD_DIM), dtype=torch.bfloat16, device=dev)
        self.dev_err = torch.zeros((1,), dtype=torch.int32, device=dev)
        self.num_splits = num_splits
        ws = msa_attn_workspace_bytes(self.rp, S, prob["H_q"], hkv, self.max_blocks, num_splits)
        self.workspace = torch.empty((max(ws, 1),), dtype=torch.uint8, device=dev)
        self.workspace_bytes = ws
        self.kv_dtype = MSA_KV_FP8_E4M3 if prob["kv_fp8"] else MSA_KV_BF16
        nc = msa_index_select_counters(self.rp, prob["H_idxk"])
        self.counters = torch.zeros((max(nc, 1),), dtype=torch.int32, device=dev)
        self.idx_dtype = prob.get("idx_dtype", "bf16")
        self.kidx = index_k(prob["k_idx"], prob.get("k_idx_scale"), prob["H_idxk"],
                            self.idx_dtype)
        self.index_flags = MSA_SHARE_ACROSS_DRAFTS if share_selection else 0
        self.one_call = one_call and select_in_attention and not self.fused_select
        if self.one_call:
            sb = msa_decode_step_workspace_bytes(self.rp, S, prob["H_q"], hkv, prob["H_idxk"],
                                                 self.max_blocks, num_splits)
            self.step_workspace = torch.zeros((max(sb, 256),), dtype=torch.uint8, device=dev)

    def index_scores(self, stream=None):
        p = self.p
        if self.idx_dtype == "bf16" and not self.index_flags:
            msa_index_scores(self.rp, p["q_idx"], p["k_idx"], p["H_kv"], p["H_idxk"],
                             self.max_blocks, self.scores, self.dev_err, stream)
        else:
            msa_index_scores_k(self.rp, p["q_idx"], self.kidx, p["H_kv"], self.max_blocks,
                               self.index_flags, self.scores, self.dev_err, stream)

    def index_select(self, stream=None):
        """Stages 1 and 2 in one call (one launch on the decode route and on most speculative
        shapes; two where the scores run on the tensor cores)."""
        p = self.p
        msa_index_select_k(self.rp, p["q_idx"], self.kidx, p["H_kv"], self.max_blocks,
                           p["top_k"], p["init_blocks"], p["local_blocks"], self.index_flags,
                           self.scores, self.block_ids, self.num_selected, self.counters,
                           self.dev_err, stream)

    def select(self, scores=None, stream=None):
        p = self.p
        msa_select_blocks(self.rp, self.scores if scores is None else scores, p["H_kv"],
                          self.max_blocks, p["top_k"], p["init_blocks"], p["local_blocks"],
                          self.block_ids, self.num_selected, self.dev_err, stream)

    def attend(self, block_ids=None, num_selected=None, stream=None, combine=True):
        """Stage 3.  With combine=False on the decode / speculative routes only the split-K
        partials are written (into the workspace); ``combine()`` then merges them."""
        p = self.p
        msa_sparse_attn_paged(self.rp, p["q"], p["k"], p["v"], self.kv_dtype,
                              self.block_ids if block_ids is None else block_ids,
                              self.num_selected if num_selected is None else num_selected,
                              p["S"], p["H_q"], p["H_kv"], self.max_blocks, p["scale"],
                              self.num_splits, self.workspace, self.out if combine else 0,
                              self.dev_err, stream, workspace_bytes=self.workspace_bytes)

    def select_attend(self, stream=None, combine=True):
        """Stages 2 and 3 in one call (msa_select_sparse_attn_paged: one launch on decode).
        With combine=False on the decode / speculative routes only the split-K partials are
        written; ``combine()`` then merges them."""
        p = self.p
        msa_select_sparse_attn_paged(self.rp, self.scores, p["top_k"], p["init_blocks"],
                                     p["local_blocks"], p["q"], p["k"], p["v"], self.kv_dtype,
                                     p["H_q"], p["H_kv"], self.max_blocks, p["scale"],
                                     self.num_splits, self.workspace, self.block_ids,
                                     self.num_selected, self.out if combine else 0,
                                     self.dev_err, stream, workspace_bytes=self.workspace_bytes)

    def partials(self):
        n, o_off, l_off = msa_attn_partials(self.rp, self.p["S"], self.p["H_q"], self.p["H_kv"],
                                            self.max_blocks, self.num_splits)
        return n, self.workspace.data_ptr() + o_off, self.workspace.data_ptr() + l_off

    def combine(self, stream=None):
        n, o_ptr, l_ptr = self.partials()
        msa_splitk_combine(o_ptr, l_ptr, n, self.p["total_q"], self.p["H_q"], self.out, stream)

    def step(self, stream=None):
        """The whole step as one msa_decode_step call."""
        p = self.p
        msa_decode_step(self.rp, p["q_idx"], self.kidx, p["top_k"], p["init_blocks"],
                        p["local_blocks"], p["q"], p["k"], p["v"], self.kv_dtype, p["H_q"],
                        p["H_kv"], self.max_blocks, p["scale"], self.num_splits,
                        self.step_workspace, self.scores, self.block_ids, self.num_selected,
                        self.out, self.dev_err, stream)

    def run(self, stream=None):
        if self.one_call:
            self.step(stream)
            return self.out
        if self.fused_select:
            self.index_select(stream)
        elif self.select_in_attention:
            self.index_scores(stream)
            self.select_attend(stream)
            return self.out
        else:
            self.index_scores(stream)
            self.select(stream=stream)
        self.attend(stream=stream)
        return self.out


class HostPipeline:
    """Steps whose per-step inputs arrive in pinned host memory and whose output goes back to
    pinned host memory, pipelined two deep: step i's host->device copy runs on one copy stream
    while step i-1 computes, and its device->host copy on another while step i+1 computes.

    The KV caches (``k``, ``v``, ``k_idx``) stay resident and are shared.  The per-step inputs
    (``PER_STEP``) of one step travel as one packed buffer (``pack``: each tensor at a 256-byte
    aligned offset), so a step costs one host->device copy; on the device they live twice, in
    two staging buffers that the two Paths read in place, and alternate between steps with every
    output.  Stream order keeps each buffer's writer after its last reader: copy-in(i) waits for
    compute(i-2), compute(i) waits for copy-in(i) and for copy-out(i-2), copy-out(i) waits for
    compute(i).
    """

    PER_STEP = ("q", "q_idx", "row_off", "cache_len", "table")

    def __init__(self, prob: dict, **path_kw):
        self.layout, off = [], 0
        for k in self.PER_STEP:
            t = prob[k]
            n = t.numel() * t.element_size()
            self.layout.append((k, off, t.dtype, tuple(t.shape), n))
            off = (off + n + 255) // 256 * 256
        self.step_bytes = off
        dev = prob["q"].device
        self.stage = [torch.empty((off,), dtype=torch.uint8, device=dev) for _ in range(2)]
        self.paths = []
        for b in range(2):
            p = dict(prob)
            for k, o, dt, shape, n in self.layout:
                p[k] = self.stage[b][o:o + n].view(dt).view(shape)
                p[k].copy_(prob[k])
            self.paths.append(Path(p, **path_kw))
        self.compute = torch.cuda.Stream(dev)
        self.h2d = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)
        self.copied_in = [torch.cuda.Event() for _ in range(2)]
        self.computed = [torch.cuda.Event() for _ in range(2)]
        self.copied_out = [torch.cuda.Event() for _ in range(2)]
        self.i = 0

    def pack(self, host_in: dict) -> torch.Tensor:
        """One step's PER_STEP tensors (host) packed into a new pinned buffer for submit()."""
        buf = torch.empty((self.step_bytes,), dtype=torch.uint8).pin_memory()
        for k, o, dt, shape, n in self.layout:
            t = host_in[k]
            assert t.dtype == dt and tuple(t.shape) == shape, k
            buf[o:o + n].view(dt).view(shape).copy_(t)
        return buf

    def start(self, after: Optional[torch.cuda.Event] = None):
        """Order the three streams after ``after`` (e.g. a timing event) and restart at step 0."""
        for s in (self.compute, self.h2d, self.d2h):
            if after is not None:
                s.wait_event(after)
        self.i = 0

    def submit(self, host_packed: torch.Tensor, host_out: torch.Tensor) -> torch.cuda.Event:
        """Enqueue one step: ``host_packed`` is a pinned buffer from pack(), ``host_out``
        (pinned) receives the step's output.  Returns the event after which ``host_out``
        holds it."""
        b = self.i % 2
        path = self.paths[b]
        with torch.cuda.stream(self.h2d):
            if self.i >= 2:
                self.h2d.wait_event(self.computed[b])
            self.stage[b].copy_(host_packed, non_blocking=True)
            self.copied_in[b].record(self.h2d)
        self.compute.wait_event(self.copied_in[b])
        if self.i >= 2:
            self.compute.wait_event(self.copied_out[b])
        path.run(self.compute)
        self.computed[b].record(self.compute)
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(self.computed[b])
            host_out.copy_(path.out, non_blocking=True)
            self.copied_out[b].record(self.d2h)
        self.i += 1
        return self.copied_out[b]

    def finish(self, stream: torch.cuda.Stream):
        """Order ``stream`` after every step submitted so far."""
        for s in (self.compute, self.h2d, self.d2h):
            stream.wait_stream(s)
