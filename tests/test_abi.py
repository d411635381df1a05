"""C-ABI boundary checks that need no GPU: the library loads, exports every
symbol include/resa.h declares, implements the Eq. 5 budget, sizes its
workspace, and rejects invalid arguments before touching the device."""
import ctypes
import os
import re

import pytest

import oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "resa.h")


@pytest.fixture(scope="module")
def resa():
    import __graft_entry__
    __graft_entry__.build()
    import block_sparse_attention_quest_b200 as m
    return m


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"RESA_API\s+[\w\s\*]+?\b(resa_\w+)\s*\(", txt)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("resa_build_desc", "resa_decode_sparse", "resa_rectify", "resa_num_selected",
              "resa_select_blocks", "resa_attend_blocks",
              "resa_workspace_bytes", "resa_decode_dense", "resa_status_string",
              "resa_workspace_status"):
        assert n in names


def test_library_exports_every_declared_symbol(resa):
    lib = ctypes.CDLL(resa.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(resa.EXPORTED) <= set(_declared())


def test_num_selected_matches_oracle(resa):
    for length in (1, 15, 16, 17, 2048, 2112, 32768, 131072, 131073, 262144, 65536):
        for r in (0.05, 0.1, 0.2, 0.3, 1.0):
            for n_min in (1, 4, 16):
                M = orc.num_blocks(length)
                assert resa.num_selected(length, r, n_min) == orc.num_selected(M, r, n_min)


def test_num_selected_rejects(resa):
    lib = resa._lib
    assert lib.resa_num_selected(0, 16, 0.1, 4) == resa.RESA_ERR_INVALID_ARG
    assert lib.resa_num_selected(100, 32, 0.1, 4) == resa.RESA_ERR_INVALID_ARG
    assert lib.resa_num_selected(100, 16, 0.0, 4) == resa.RESA_ERR_INVALID_ARG
    assert lib.resa_num_selected(100, 16, 1.5, 4) == resa.RESA_ERR_INVALID_ARG
    assert lib.resa_num_selected(100, 16, 0.1, 0) == resa.RESA_ERR_INVALID_ARG


def _dims(resa, **kw):
    d = dict(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, block_size=16,
             dtype=resa.RESA_BF16, max_len=4096)
    d.update(kw)
    return resa.Dims(**d)


def test_workspace_bytes(resa):
    d = _dims(resa)
    small = resa.workspace_bytes(d, 1000, 32)
    big = resa.workspace_bytes(d, 4000, 32)
    assert 0 < small <= big and big % 256 == 0
    assert resa._lib.resa_workspace_bytes(ctypes.byref(_dims(resa, head_dim=96)), 100, 32) == 0


FAKE = 0x10000   # aligned, never dereferenced: validation fails first


def _decode(resa, d, **kw):
    a = dict(q=FAKE, k_new=None, v_new=None, k=FAKE, v=FAKE, desc=FAKE, length=100, r=0.1,
             n_min=4, scale=1.0, out=FAKE, lse=None, sel=None, ws=FAKE, ws_bytes=1 << 30)
    a.update(kw)
    return resa._lib.resa_decode_sparse(ctypes.byref(d), a["q"], a["k_new"], a["v_new"], a["k"],
                                        a["v"], a["desc"], a["length"], a["r"], a["n_min"],
                                        a["scale"], a["out"], a["lse"], a["sel"], a["ws"],
                                        a["ws_bytes"], None)


def test_decode_rejects_invalid_arguments(resa):
    E = resa
    d = _dims(resa)
    assert _decode(resa, d, q=None) == E.RESA_ERR_INVALID_ARG
    assert _decode(resa, d, desc=None) == E.RESA_ERR_INVALID_ARG
    assert _decode(resa, d, q=FAKE + 4) == E.RESA_ERR_INVALID_ARG          # misaligned
    assert _decode(resa, d, ws=FAKE + 16) == E.RESA_ERR_INVALID_ARG        # ws not 256-aligned
    assert _decode(resa, d, k_new=FAKE) == E.RESA_ERR_INVALID_ARG          # v_new missing
    assert _decode(resa, d, length=0) == E.RESA_ERR_INVALID_ARG
    assert _decode(resa, d, length=4097) == E.RESA_ERR_CAPACITY
    assert _decode(resa, d, r=0.0) == E.RESA_ERR_INVALID_ARG
    assert _decode(resa, d, r=1.01) == E.RESA_ERR_INVALID_ARG
    assert _decode(resa, d, n_min=0) == E.RESA_ERR_INVALID_ARG
    assert _decode(resa, d, scale=float("nan")) == E.RESA_ERR_INVALID_ARG
    assert _decode(resa, d, scale=-1.0) == E.RESA_ERR_INVALID_ARG
    assert _decode(resa, d, scale=0.0) == E.RESA_ERR_INVALID_ARG
    assert _decode(resa, d, ws_bytes=1024) == E.RESA_ERR_WORKSPACE
    assert _decode(resa, _dims(resa, head_dim=96)) == E.RESA_ERR_UNSUPPORTED
    assert _decode(resa, _dims(resa, block_size=32)) == E.RESA_ERR_UNSUPPORTED
    assert _decode(resa, _dims(resa, n_q_heads=72, n_kv_heads=8)) == E.RESA_ERR_UNSUPPORTED
    assert _decode(resa, _dims(resa, n_q_heads=30)) == E.RESA_ERR_INVALID_ARG
    assert _decode(resa, _dims(resa, max_len=4008)) == E.RESA_ERR_INVALID_ARG
    assert _decode(resa, _dims(resa, dtype=7)) == E.RESA_ERR_INVALID_ARG


def test_rectify_and_build_desc_reject_invalid_arguments(resa):
    E = resa
    d = _dims(resa)
    lib = resa._lib

    def rect(length=100, f=32, ws_bytes=1 << 30, k_f=FAKE):
        return lib.resa_rectify(ctypes.byref(d), FAKE, k_f, FAKE, FAKE, FAKE, FAKE, length, f, 1.0,
                                FAKE, FAKE, ws_bytes, None)
    assert rect(f=0) == E.RESA_ERR_INVALID_ARG
    assert rect(f=101) == E.RESA_ERR_INVALID_ARG
    assert rect(k_f=None) == E.RESA_ERR_INVALID_ARG
    assert rect(length=5000) == E.RESA_ERR_CAPACITY
    assert rect(ws_bytes=256) == E.RESA_ERR_WORKSPACE
    assert lib.resa_build_desc(ctypes.byref(d), FAKE, 0, FAKE, None) == E.RESA_ERR_INVALID_ARG
    assert lib.resa_build_desc(ctypes.byref(d), FAKE, 4097, FAKE, None) == E.RESA_ERR_CAPACITY
    assert lib.resa_build_desc(ctypes.byref(d), None, 10, FAKE, None) == E.RESA_ERR_INVALID_ARG


def test_status_strings(resa):
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert resa.status_string(code) != "unknown status"
    assert resa.status_string(-99) == "unknown status"


def test_varlen_calls_reject_invalid_arguments(resa):
    """The *_varlen calls need a 4-byte aligned lens array and apply the
    fixed-length checks to len_bound; nothing is launched when they fail."""
    E = resa
    d = _dims(resa)
    lib = resa._lib
    dr = ctypes.byref(d)

    def dec(lens=FAKE, bound=100, ws_bytes=1 << 30, r=0.1):
        return lib.resa_decode_sparse_varlen(dr, FAKE, None, None, FAKE, FAKE, FAKE, lens, bound,
                                             r, 4, 1.0, FAKE, None, None, FAKE, ws_bytes, None)
    assert dec(lens=None) == E.RESA_ERR_INVALID_ARG
    assert dec(lens=FAKE + 2) == E.RESA_ERR_INVALID_ARG
    assert dec(bound=0) == E.RESA_ERR_INVALID_ARG
    assert dec(bound=4097) == E.RESA_ERR_CAPACITY
    assert dec(ws_bytes=512) == E.RESA_ERR_WORKSPACE
    assert dec(r=0.0) == E.RESA_ERR_INVALID_ARG

    def dense(lens=FAKE, bound=100):
        return lib.resa_decode_dense_varlen(dr, FAKE, None, None, FAKE, FAKE, None, lens, bound,
                                            1.0, FAKE, None, FAKE, 1 << 30, None)
    assert dense(lens=None) == E.RESA_ERR_INVALID_ARG
    assert dense(bound=4097) == E.RESA_ERR_CAPACITY

    def rect(lens=FAKE, bound=100, f=32):
        return lib.resa_rectify_varlen(dr, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, lens, win, bound,
                                       f, 1.0, FAKE, FAKE, 1 << 30, None)
    win = None
    assert rect(lens=None) == E.RESA_ERR_INVALID_ARG
    win = FAKE + 1                                  # misaligned windows
    assert rect() == E.RESA_ERR_INVALID_ARG
    win = None
    assert rect(f=101) == E.RESA_ERR_INVALID_ARG
    assert rect(f=0) == E.RESA_ERR_INVALID_ARG
    assert rect(bound=4097) == E.RESA_ERR_CAPACITY

    assert lib.resa_build_desc_varlen(dr, FAKE, None, 100, FAKE, None) == E.RESA_ERR_INVALID_ARG
    assert lib.resa_build_desc_varlen(dr, FAKE, FAKE, 4097, FAKE, None) == E.RESA_ERR_CAPACITY
    assert lib.resa_build_desc_varlen(dr, FAKE, FAKE, 0, FAKE, None) == E.RESA_ERR_INVALID_ARG


def test_workspace_covers_every_smaller_window(resa):
    """A workspace sized for window f serves every window f' <= f (a smaller
    window may take more splits per row)."""
    for kw in (dict(batch=5), dict(batch=1), dict(batch=3, n_q_heads=12, n_kv_heads=4)):
        d = _dims(resa, **kw)
        big = resa.workspace_bytes(d, 4000, 64)
        for f in range(1, 65):
            assert resa.workspace_bytes(d, 4000, f) <= big, (kw, f)


def test_decode_only_workspace_does_not_serve_a_rectification(resa):
    """A workspace sized for decoding only (f = 0) holds no room for the
    rectification's split partials: it is smaller than one sized for f = 1,
    and a rectification given one is rejected before anything is launched."""
    d = _dims(resa)
    dec = resa.workspace_bytes(d, 4000, 0)
    assert 0 < dec < resa.workspace_bytes(d, 4000, 1) <= resa.workspace_bytes(d, 4000, 32)
    rc = resa._lib.resa_rectify(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4000, 32, 1.0,
                                FAKE, FAKE, dec, None)
    assert rc == resa.RESA_ERR_WORKSPACE
    # two 128-row tiles per KV head (f = 64, 4 query heads per KV head) need
    # room for the partials of both
    assert resa.workspace_bytes(d, 4000, 64) >= resa.workspace_bytes(d, 4000, 32)


def test_prefill_rejects_invalid_arguments(resa):
    E = resa
    lib = resa._lib

    def pre(d, q=FAKE, desc=FAKE, length=100, scale=1.0, ws_bytes=1 << 30):
        return lib.resa_prefill(ctypes.byref(d), q, FAKE, FAKE, desc, length, scale, FAKE, FAKE,
                                ws_bytes, None)
    d = _dims(resa)
    assert pre(d, q=None) == E.RESA_ERR_INVALID_ARG
    assert pre(d, desc=None) == E.RESA_ERR_INVALID_ARG
    assert pre(d, length=0) == E.RESA_ERR_INVALID_ARG
    assert pre(d, length=4097) == E.RESA_ERR_CAPACITY
    assert pre(d, scale=0.0) == E.RESA_ERR_INVALID_ARG
    assert pre(d, ws_bytes=64) == E.RESA_ERR_WORKSPACE
    assert pre(_dims(resa, dtype=resa.RESA_F32)) == E.RESA_ERR_UNSUPPORTED
    assert pre(_dims(resa, n_q_heads=24)) == E.RESA_ERR_UNSUPPORTED      # group of 3


def test_wait_check_rejects_invalid_arguments(resa):
    lib = resa._lib
    E = resa
    assert lib.resa_wait_check(None, 1, 1000, FAKE, None) == E.RESA_ERR_INVALID_ARG
    assert lib.resa_wait_check(FAKE + 2, 1, 1000, FAKE, None) == E.RESA_ERR_INVALID_ARG
    assert lib.resa_wait_check(FAKE, 1, 1000, FAKE + 16, None) == E.RESA_ERR_INVALID_ARG
    assert lib.resa_wait_check(FAKE, 1, 0, FAKE, None) == E.RESA_ERR_INVALID_ARG
    assert lib.resa_wait_check(FAKE, 1, 2000001, FAKE, None) == E.RESA_ERR_INVALID_ARG


def test_decode_rejects_more_blocks_than_the_selection_takes(resa):
    """262145 blocks (4M + 16 tokens) is one block past the selection's limit:
    rejected on the host before anything is launched."""
    d = _dims(resa, n_q_heads=4, n_kv_heads=1, max_len=16 * 262145)
    assert _decode(resa, d, length=16 * 262144 + 1, ws_bytes=1 << 40) == resa.RESA_ERR_UNSUPPORTED
