"""C-ABI checks that need no GPU: the library loads, exports every entry point
include/sf.h declares, and rejects bad arguments with a status code before any
CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sf():
    from chunked_linear_recurrence_chunkwise_b200 import build
    build.build()
    from chunked_linear_recurrence_chunkwise_b200 import sf as sfm
    return sfm


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(sf_\w+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_symbols()
    for must in ("sf_fwd", "sf_bwd", "sf_fwd_seq", "sf_bwd_seq", "sf_workspace_bytes",
                 "sf_seq_workspace_bytes", "sf_check", "sf_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol(sf):
    out = subprocess.check_output(["nm", "-D", "--defined-only", sf.LIB_PATH], text=True)
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    missing = [n for n in declared_symbols() if n not in exported]
    assert not missing, missing
    for n in declared_symbols():
        assert hasattr(sf._lib, n)


def test_status_strings(sf):
    for code in range(6):
        assert sf.sf_status_string(code)
    assert "unknown" in sf.sf_status_string(99)


def _call_fwd(sf, sh, q=16, k=16, v=16, o=16, ws=256, ws_bytes=1 << 30):
    P = ctypes.c_void_p
    return sf.raw_call("sf_fwd", ctypes.byref(sh), P(q), P(k), P(v), None, None, None, P(o), None,
                       P(ws), ctypes.c_size_t(ws_bytes), None)


def test_argument_errors_return_codes_without_launching(sf):
    ok = sf.shape(1, 128, 2, 64, 64, sf.SF_BF16)
    assert sf.sf_workspace_bytes(ok, sf.SF_OP_FWD) > 0
    assert sf.sf_workspace_bytes(ok, sf.SF_OP_BWD) > sf.sf_workspace_bytes(ok, sf.SF_OP_FWD)
    bad_chunk = sf.shape(1, 128, 2, 64, 64, sf.SF_BF16, chunk=32)
    assert sf.sf_workspace_bytes(bad_chunk, 0) == 0
    assert _call_fwd(sf, bad_chunk) == sf.SF_ERR_UNSUPPORTED
    assert _call_fwd(sf, sf.shape(1, 128, 2, 0, 64, sf.SF_F32)) == sf.SF_ERR_UNSUPPORTED
    assert _call_fwd(sf, sf.shape(1, 128, 2, 256, 64, sf.SF_F32)) == sf.SF_ERR_UNSUPPORTED
    assert _call_fwd(sf, sf.shape(1, 128, 2, 64, 64, 7)) == sf.SF_ERR_UNSUPPORTED
    assert _call_fwd(sf, sf.shape(1, 128, 2, 64, 64, sf.SF_F32, ld_t=100)) == sf.SF_ERR_INVALID
    assert _call_fwd(sf, sf.shape(-1, 128, 2, 64, 64, sf.SF_F32)) == sf.SF_ERR_INVALID
    assert _call_fwd(sf, ok, q=0) == sf.SF_ERR_INVALID            # NULL input
    assert _call_fwd(sf, ok, o=17) == sf.SF_ERR_INVALID           # misaligned output
    assert _call_fwd(sf, ok, ws=0) == sf.SF_ERR_WORKSPACE         # no workspace
    assert _call_fwd(sf, ok, ws_bytes=1024) == sf.SF_ERR_WORKSPACE
    assert _call_fwd(sf, ok, ws=272) == sf.SF_ERR_WORKSPACE       # not 256-byte aligned
    assert sf.raw_call("sf_fwd", None, *([None] * 8), None, ctypes.c_size_t(0), None) == sf.SF_ERR_INVALID


def test_backward_gradient_pointer_rules(sf):
    P = ctypes.c_void_p
    sh = sf.shape(1, 128, 2, 64, 64, sf.SF_F32)
    args = [P(16)] * 3 + [P(16), None, None, P(16), None] + [P(16)] * 3 + [None, None, None]
    # g given but dg NULL -> invalid
    rc = sf.raw_call("sf_bwd", ctypes.byref(sh), *args, P(256), ctypes.c_size_t(1 << 30), None)
    assert rc == sf.SF_ERR_INVALID


def test_sequence_lengths_must_sum_to_T(sf):
    sh = sf.shape(1, 300, 2, 64, 64, sf.SF_F32)
    assert sf.sf_seq_workspace_bytes(sh, [100, 100], 0) == 0
    assert sf.sf_seq_workspace_bytes(sh, [100, 0, 200], 0) == 0
    assert sf.sf_seq_workspace_bytes(sh, [100, 200], 0) > 0
    lens = (ctypes.c_int * 2)(100, 100)
    P = ctypes.c_void_p
    rc = sf.raw_call("sf_fwd_seq", ctypes.byref(sh), 2, lens, P(16), P(16), P(16), None, None, None,
                     P(16), None, None, P(256), ctypes.c_size_t(1 << 30), None, None)
    assert rc == sf.SF_ERR_INVALID


def test_keep_drivers_check_the_kept_buffer(sf):
    """The no-recompute drivers reject a missing, short or misaligned keep buffer
    (and a bad cut) before any CUDA call."""
    sh = sf.shape(1, 300, 2, 64, 64, sf.SF_F32)
    assert sf.sf_keep_bytes(sh, [100, 100]) == 0
    need = sf.sf_keep_bytes(sh, [100, 200])
    assert need > 0
    # more pieces keep more (each piece's chunks are padded to 64 tokens)
    assert sf.sf_keep_bytes(sh, [100] * 3) > sf.sf_keep_bytes(sh, [300])
    tc = sf.shape(1, 256, 2, 128, 128, sf.SF_BF16)
    assert sf.sf_keep_bytes(tc, [256]) > 0
    lens = (ctypes.c_int * 2)(100, 200)
    P, S = ctypes.c_void_p, ctypes.c_size_t

    def fwd(keep, keep_bytes, lens_=lens):
        return sf.raw_call("sf_fwd_seq_keep", ctypes.byref(sh), 2, lens_, P(16), P(16), P(16), None,
                           None, None, P(16), None, P(keep) if keep else None, S(keep_bytes),
                           P(256), S(1 << 30), None, None)

    def bwd(keep, keep_bytes):
        return sf.raw_call("sf_bwd_seq_keep", ctypes.byref(sh), 2, lens, P(16), P(16), P(16), None,
                           None, P(keep) if keep else None, S(keep_bytes), P(16), None, P(16), P(16),
                           P(16), None, None, None, P(256), S(1 << 30), None, None)

    assert fwd(0, need) == sf.SF_ERR_WORKSPACE
    assert fwd(256, need - 1) == sf.SF_ERR_WORKSPACE
    assert fwd(272, need) == sf.SF_ERR_WORKSPACE       # not 256-byte aligned
    assert fwd(256, need, (ctypes.c_int * 2)(100, 100)) == sf.SF_ERR_INVALID
    assert bwd(0, need) == sf.SF_ERR_WORKSPACE
    assert bwd(256, need - 1) == sf.SF_ERR_WORKSPACE


def test_product_path_does_not_reference_the_oracle():
    pkg = os.path.join(ROOT, "chunked_linear_recurrence_chunkwise_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".h", ".cuh", ".cpp")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in text and "from oracle" not in text, fn
                assert "sf_oracle" not in text and "sfo_" not in text, fn


def test_sequence_accumulation_memory_is_flat_in_T(sf):
    """The memory property of Sequence Accumulation (atlas.scime.ai page, Key
    results: device memory stays constant as the context grows) at the layer: with
    pieces of a fixed length, the recompute drivers' workspace does not grow with
    T, while the buffer of the drivers that keep the intermediates grows in
    proportion to T."""
    for dtype, d in ((sf.SF_BF16, 128), (sf.SF_F32, 64)):
        ws, keep = {}, {}
        for n in (4, 16, 64):
            sh = sf.shape(1, 4096 * n, 32, d, d, dtype)
            lens = [4096] * n
            ws[n] = (sf.sf_seq_workspace_bytes(sh, lens, sf.SF_OP_FWD),
                     sf.sf_seq_workspace_bytes(sh, lens, sf.SF_OP_BWD))
            keep[n] = sf.sf_keep_bytes(sh, lens)
        assert ws[4] == ws[16] == ws[64]
        assert keep[16] == 4 * keep[4] and keep[64] == 16 * keep[4]
        assert ws[64][1] < keep[64] / 8
