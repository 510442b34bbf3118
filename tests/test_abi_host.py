"""Host-side checks of the C ABI that need no GPU: the library builds and loads, exports every
entry point include/msa.h declares, and its host-only helpers and argument validation behave
as documented (no call here launches device work)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from block_sparse_paged_scores_b200 import build as msa_build
from block_sparse_paged_scores_b200 import msa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")


@pytest.fixture(scope="module")
def lib():
    msa_build.build()
    return msa.load()


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"MSA_API\s+[\w\s\*]+?\b(msa_\w+)\s*\(", src)))


def test_header_declares_the_four_stages_and_helpers():
    names = _declared()
    for n in ("msa_index_scores", "msa_select_blocks", "msa_sparse_attn_paged",
              "msa_splitk_combine", "msa_attn_workspace_bytes", "msa_default_num_splits",
              "msa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", msa.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for n in _declared():
        assert n in exported, n
        assert hasattr(lib, n)
    # nothing else leaks out of the library
    assert {e for e in exported if e.startswith("msa")} == set(_declared())


def test_header_compiles_as_plain_c(tmp_path):
    src = tmp_path / "use.c"
    src.write_text('#include "msa.h"\nint main(void){return (int)msa_status_string(MSA_OK)[0] == 0;}\n')
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-c", f"-I{ROOT}/include",
                           str(src), "-o", str(tmp_path / "use.o")])


def test_status_strings(lib):
    assert msa.msa_status_string(0) == "MSA_OK"
    assert msa.msa_status_string(1) == "MSA_ERR_INVALID_ARG"
    assert msa.msa_status_string(2) == "MSA_ERR_UNSUPPORTED"
    assert msa.msa_status_string(3) == "MSA_ERR_CUDA"
    assert msa.msa_status_string(99) == "MSA_ERR_UNKNOWN"


def test_default_splits_fill_the_sms(lib):
    # decode / speculative: one persistent partition per SM, fewer for tiny work lists
    assert msa.msa_default_num_splits(32, 1, 8, 19, 148) == 148
    assert msa.msa_default_num_splits(1, 1, 1, 6, 148) == 1       # 6 entries, >= 8 per CTA
    assert msa.msa_default_num_splits(1, 1, 4, 6, 148) == 3       # 24 entries
    assert msa.msa_default_num_splits(128, 1, 8, 69, 148) == 148
    assert msa.msa_default_num_splits(64, 4, 8, 35, 148) == 148
    assert msa.msa_default_num_splits(8, 4096, 8, 67, 148) == 1   # prefill: one partition
    assert msa.msa_default_num_splits(0, 1, 8, 19, 148) == 1


def _rp(batch=2, total_q=2, max_q_len=1, max_pages=16, num_pages=64):
    fake = 0x10000  # never dereferenced by host-only paths
    return msa.RaggedPaged(fake, fake, fake, batch, total_q, max_q_len, max_pages, num_pages)


def test_workspace_bytes(lib):
    rows = 4 * 64
    rp = _rp(batch=4, total_q=4, max_q_len=1)
    # one partition covering all 4 x 8 items of 19 slots: one piece per row
    ws1 = msa.msa_attn_workspace_bytes(rp, 19, 64, 8, 16, 1)
    assert ws1 >= rows * 128 * 4 + rows * 4
    assert msa.msa_attn_partials(rp, 19, 64, 8, 16, 1)[0] == 1
    # three partitions: some item straddles two of them -> two pieces
    ws3 = msa.msa_attn_workspace_bytes(rp, 19, 64, 8, 16, 3)
    assert ws3 >= 2 * rows * 128 * 4 + 2 * rows * 4
    n, o_off, l_off = msa.msa_attn_partials(rp, 19, 64, 8, 16, 3)
    assert n == 2 and o_off == 0 and l_off >= 2 * rows * 128 * 4
    rp = _rp(batch=2, total_q=8, max_q_len=4)
    ws = msa.msa_attn_workspace_bytes(rp, 35, 64, 8, 16, 1)              # speculative: + plan
    assert ws >= 8 * 64 * 128 * 4 + 2 * 8 * 16 * 8
    rp = _rp(batch=2, total_q=600, max_q_len=300)
    ws = msa.msa_attn_workspace_bytes(rp, 35, 64, 8, 16, 0)              # prefill: plan only
    assert 0 < ws < 600 * 64 * 128 * 4
    assert msa.msa_attn_partials(rp, 35, 64, 8, 16, 0)[0] == 0           # writes out directly
    assert msa.msa_attn_workspace_bytes(rp, 0, 64, 8, 16, 1) == 0        # invalid -> 0
    assert msa.msa_attn_workspace_bytes(rp, 35, 63, 8, 16, 1) == 0


def test_invalid_arguments_are_rejected_before_any_launch(lib):
    rp = _rp()
    P = 0x10000
    stat = lib.msa_index_scores(ctypes.byref(rp), None, P, 8, 1, 16, P, None, None)
    assert stat == msa.MSA_ERR_INVALID_ARG
    stat = lib.msa_index_scores(ctypes.byref(rp), P, P, 8, 3, 16, P, None, None)   # H_idxk
    assert stat == msa.MSA_ERR_INVALID_ARG
    stat = lib.msa_index_scores(ctypes.byref(rp), P, P, 8, 1, 17, P, None, None)   # > max_pages
    assert stat == msa.MSA_ERR_INVALID_ARG
    stat = lib.msa_index_scores(ctypes.byref(rp), P, P + 2, 8, 1, 16, P, None, None)  # align
    assert stat == msa.MSA_ERR_INVALID_ARG
    stat = lib.msa_index_scores(ctypes.byref(rp), P + 8, P, 8, 1, 16, P, None, None)  # q_idx
    assert stat == msa.MSA_ERR_INVALID_ARG
    stat = lib.msa_index_scores(ctypes.byref(rp), P, P, 64, 1, 16, P, None, None)  # group > 32
    assert stat == msa.MSA_ERR_UNSUPPORTED
    stat = lib.msa_select_blocks(ctypes.byref(rp), P, 8, 16, 0, 0, 0, P, P, None, None)  # S = 0
    assert stat == msa.MSA_ERR_INVALID_ARG
    # fused index + select: the decode route needs counters; S = 0 and null outputs rejected
    fused = lambda **kw: lib.msa_index_select(
        ctypes.byref(kw.get("rp", rp)), P, P, 8, 1, 16, kw.get("top_k", 4), 1, 1,
        kw.get("scores", P), kw.get("ids", P), P, kw.get("counters", P), None, None)
    assert fused(counters=None) == msa.MSA_ERR_INVALID_ARG
    assert fused(top_k=-1) == msa.MSA_ERR_INVALID_ARG
    assert fused(scores=None) == msa.MSA_ERR_INVALID_ARG
    assert fused(ids=None) == msa.MSA_ERR_INVALID_ARG
    assert fused(counters=P + 2) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_index_select(ctypes.byref(rp), P, P, 8, 1, 16, 0, 0, 0, P, P, P, P, None,
                                None) == msa.MSA_ERR_INVALID_ARG                   # S = 0
    assert msa.msa_index_select_counters(_rp(batch=5, max_q_len=3, total_q=9), 8) == 5 * 3 * 8
    # select + attention in one call: the selection's and the attention's validation, up front
    sa = lambda **kw: lib.msa_select_sparse_attn_paged(
        ctypes.byref(rp), kw.get("scores", P), kw.get("top_k", 4), 1, 1, P, P, P, 0, 64, 8, 16,
        ctypes.c_float(kw.get("scale", 0.088)), 0, None, 0, kw.get("ids", P), P,
        kw.get("out", P), None, None)
    assert sa(scores=None) == msa.MSA_ERR_INVALID_ARG
    assert sa(top_k=-1) == msa.MSA_ERR_INVALID_ARG
    assert sa(ids=None) == msa.MSA_ERR_INVALID_ARG
    assert sa(scale=0.0) == msa.MSA_ERR_INVALID_ARG
    assert sa(out=P + 8) == msa.MSA_ERR_INVALID_ARG
    assert sa() == msa.MSA_ERR_INVALID_ARG          # the decode route needs a workspace
    stat = lib.msa_select_blocks(ctypes.byref(rp), P, 8, 16, -1, 1, 1, P, P, None, None)
    assert stat == msa.MSA_ERR_INVALID_ARG
    bad = msa.RaggedPaged(P, P, P, 0, 2, 1, 16, 64)                                 # batch 0
    stat = lib.msa_select_blocks(ctypes.byref(bad), P, 8, 16, 4, 1, 1, P, P, None, None)
    assert stat == msa.MSA_ERR_INVALID_ARG
    f = ctypes.c_float
    args = lambda **kw: dict(dict(q=P, k=P, v=P, dt=0, ids=P, cnt=P, S=19, hq=64, hkv=8, mb=16,
                                  scale=0.088, ns=0, ws=None, wsb=0, out=P), **kw)

    def attn(**kw):
        a = args(**kw)
        return lib.msa_sparse_attn_paged(ctypes.byref(rp), a["q"], a["k"], a["v"], a["dt"],
                                         a["ids"], a["cnt"], a["S"], a["hq"], a["hkv"], a["mb"],
                                         f(a["scale"]), a["ns"], a["ws"], a["wsb"], a["out"],
                                         None, None)
    assert attn(q=None) == msa.MSA_ERR_INVALID_ARG
    assert attn(dt=7) == msa.MSA_ERR_INVALID_ARG
    assert attn(S=0) == msa.MSA_ERR_INVALID_ARG
    assert attn(hq=60) == msa.MSA_ERR_INVALID_ARG          # not a multiple of H_kv
    assert attn(scale=0.0) == msa.MSA_ERR_INVALID_ARG
    assert attn(scale=float("nan")) == msa.MSA_ERR_INVALID_ARG
    assert attn(ns=-1) == msa.MSA_ERR_INVALID_ARG
    assert attn(k=P + 8) == msa.MSA_ERR_INVALID_ARG        # cache not 16-byte aligned
    assert attn(out=P + 8) == msa.MSA_ERR_INVALID_ARG      # output not 16-byte aligned
    assert attn(hq=8 * 128) == msa.MSA_ERR_UNSUPPORTED     # GQA group 128 > 64
    assert attn(ns=4) == msa.MSA_ERR_INVALID_ARG           # partials need a workspace
    assert attn(ns=5000) == msa.MSA_ERR_INVALID_ARG        # more partitions than allowed
    stat = lib.msa_splitk_combine(None, P, 2, 4, 8, P, None)
    assert stat == msa.MSA_ERR_INVALID_ARG
    stat = lib.msa_splitk_combine(P, P, 0, 4, 8, P, None)
    assert stat == msa.MSA_ERR_INVALID_ARG


def test_binding_raises_on_error_status(lib):
    rp = _rp()
    with pytest.raises(msa.MSAError) as ei:
        msa.msa_select_blocks(rp, 0x10000, 8, 16, 0, 0, 0, 0x10000, 0x10000, stream=0)
    assert ei.value.status == msa.MSA_ERR_INVALID_ARG


def test_decode_step_workspace_and_refusals(lib):
    """msa_decode_step: its workspace is the step's flag and counter words (rounded to 256 bytes)
    in front of the attention's; invalid arguments are refused before anything is enqueued."""
    rp = _rp(batch=4, total_q=4, max_q_len=1)
    attn = msa.msa_attn_workspace_bytes(rp, 19, 64, 8, 16, 2)
    words = 2 + 2 * 4 * 1 * 1                      # epoch, done, counters, flags (1 index head)
    assert msa.msa_decode_step_workspace_bytes(rp, 19, 64, 8, 1, 16, 2) == \
        (words * 4 + 255) // 256 * 256 + attn
    many = msa.msa_decode_step_workspace_bytes(_rp(batch=100, total_q=100), 19, 64, 8, 8, 16, 2)
    assert many - msa.msa_attn_workspace_bytes(_rp(batch=100, total_q=100), 19, 64, 8, 16, 2) \
        == ((2 + 2 * 100 * 8) * 4 + 255) // 256 * 256
    assert msa.msa_decode_step_workspace_bytes(rp, 19, 64, 8, 0, 16, 2) == 0  # no index heads
    P = 0x10000
    k = msa.IndexK(msa.MSA_IDX_BF16, P, 0, 1)

    def step(**kw):
        return lib.msa_decode_step(
            ctypes.byref(kw.get("rp", rp)), P, ctypes.byref(kw.get("k", k)), kw.get("top_k", 16),
            1, 2, P, P, P, 0, 64, 8, 16, 0.1, 0, kw.get("ws", P), kw.get("ws_bytes", 1 << 20),
            kw.get("scores", P), P, P, P, None, None)
    assert step(top_k=-1) == msa.MSA_ERR_INVALID_ARG
    assert step(scores=None) == msa.MSA_ERR_INVALID_ARG
    assert step(ws=None) == msa.MSA_ERR_INVALID_ARG
    assert step(ws=P + 64) == msa.MSA_ERR_INVALID_ARG               # 256-byte alignment
    assert step(ws_bytes=8) == msa.MSA_ERR_INVALID_ARG              # no room for the flags
    assert step(k=msa.IndexK(msa.MSA_IDX_BF16, P, 0, 0)) == msa.MSA_ERR_INVALID_ARG
    empty = _rp(batch=4, total_q=0, max_q_len=1)
    assert step(rp=empty, scores=None) == msa.MSA_OK                # nothing to do
