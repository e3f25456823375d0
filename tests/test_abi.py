"""C ABI checks that need no GPU: the library loads, exports every entry point that
include/tk_route.h declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tk_route.h")


@pytest.fixture(scope="module")
def tk():
    from token_routing_gate_b200 import build

    build.build()
    from token_routing_gate_b200 import tk as mod

    return mod


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^TK_API\s+[\w\s\*]+?\b(tk_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_four_steps():
    names = _declared()
    for n in ("tk_gate_topk", "tk_route_map", "tk_expand", "tk_reduce"):
        assert n in names


def test_library_exports_every_declared_symbol(tk):
    L = ctypes.CDLL(tk.LIB_PATH)
    for name in _declared():
        assert hasattr(L, name), name
    assert sorted(tk.ABI_SYMBOLS) == _declared()


def test_sizes_and_strings(tk):
    assert tk.max_rows(8192, 256, 8, 1) == 65536
    assert tk.max_rows(16384, 256, 8, 128) == 16384 * 8 + 256 * 127
    # E rows of per-tile counts, tiles of 128 tokens, each row padded to a multiple of 4 tiles
    assert tk.route_map_workspace_bytes(8192, 256, 8) == 64 * 256 * 4
    assert tk.route_map_workspace_bytes(8193, 256, 8) == 68 * 256 * 4
    assert tk.route_map_workspace_bytes(0, 16, 2) == 4 * 16 * 4
    assert tk.lib.tk_status_str(0) == b"TK_OK"
    assert tk.lib.tk_status_str(1) == b"TK_ERR_INVALID_ARG"
    assert tk.lib.tk_abi_version() >> 16 == 1
    assert tk.lib.tk_abi_version() & 0xFFFF >= 3  # the self-tests and the window route map are there


FAKE = ctypes.c_void_p(0x10000)      # never dereferenced: the calls fail validation first
MISALIGNED = ctypes.c_void_p(0x10008)


@pytest.mark.parametrize("args,what", [
    ((FAKE, None, -1, 16, 2, 0, 1, FAKE, FAKE, None), "T"),
    ((FAKE, None, 4, 0, 1, 0, 1, FAKE, FAKE, None), "E"),
    ((FAKE, None, 4, 2000, 2, 0, 1, FAKE, FAKE, None), "E"),
    ((FAKE, None, 4, 16, 0, 0, 1, FAKE, FAKE, None), "k"),
    ((FAKE, None, 4, 16, 17, 0, 1, FAKE, FAKE, None), "k"),
    ((FAKE, None, 4, 64, 33, 0, 1, FAKE, FAKE, None), "k"),
    ((FAKE, None, 4, 16, 2, 7, 1, FAKE, FAKE, None), "score_fn"),
    ((FAKE, FAKE, 4, 16, 2, 0, 1, FAKE, FAKE, None), "bias"),
    ((None, None, 4, 16, 2, 1, 1, FAKE, FAKE, None), "NULL"),
])
def test_gate_rejects(tk, args, what):
    assert tk.lib.tk_gate_topk(*args) == 1
    assert what in tk.lib.tk_last_error_detail().decode()


def test_gate_empty_is_a_no_op(tk):
    assert tk.lib.tk_gate_topk(None, None, 0, 16, 2, 0, 1, None, None, None) == 0


def test_route_map_rejects(tk):
    L = tk.lib
    ws = tk.route_map_workspace_bytes(300, 16, 2)
    ok = (FAKE, 300, 16, 2, 1, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None, None)
    bad = [
        (dict(i=4, v=0), "align"),
        (dict(i=4, v=5000), "align"),
        (dict(i=10, v=ws - 4), "workspace"),
        (dict(i=9, v=MISALIGNED), "aligned"),
        (dict(i=5, v=None), "NULL"),
        (dict(i=8, v=None), "token_of"),
        (dict(i=3, v=33), "k"),
    ]
    for change, what in bad:
        a = list(ok)
        a[change["i"]] = change["v"]
        assert L.tk_route_map(*a) == 1, what
        assert what in L.tk_last_error_detail().decode()
    # the worst-case row count must fit int32
    assert L.tk_route_map(FAKE, 2**27, 1024, 32, 1, FAKE, FAKE, FAKE, FAKE, FAKE, 2**40, None, None) == 1


def test_expand_rejects(tk):
    L = tk.lib
    ok = [FAKE, FAKE, FAKE, FAKE, 64, 16, 2, 256, 1, 0, FAKE, None, None, None]
    cases = [
        (7, 12, "H"), (7, 0, "H"), (9, 5, "out_dtype"), (8, 0, "align"), (0, MISALIGNED, "aligned"),
        (10, MISALIGNED, "aligned"), (0, None, "NULL"), (6, 0, "k"),
    ]
    for i, v, what in cases:
        a = list(ok)
        a[i] = v
        assert L.tk_expand(*a) == 1, what
        assert what in L.tk_last_error_detail().decode()
    a = list(ok)
    a[9] = 1          # E4M3 output
    a[7] = 264        # not a multiple of 128
    a[11] = FAKE
    assert L.tk_expand(*a) == 1 and "128" in L.tk_last_error_detail().decode()
    a[7] = 256
    a[11] = None      # scales missing
    assert L.tk_expand(*a) == 1 and "out_scale" in L.tk_last_error_detail().decode()
    a = list(ok)
    a[8] = 128        # align > 1 needs token_of
    a[3] = None
    assert L.tk_expand(*a) == 1 and "token_of" in L.tk_last_error_detail().decode()


def test_reduce_rejects(tk):
    L = tk.lib
    ok = [FAKE, 128, FAKE, None, 64, 2, 256, FAKE, None, None]
    for i, v, what in [(5, 0, "k"), (5, 33, "k"), (6, 7, "H"), (1, -1, "y_rows"),
                       (0, MISALIGNED, "aligned"), (7, MISALIGNED, "aligned"), (2, None, "NULL")]:
        a = list(ok)
        a[i] = v
        assert L.tk_reduce(*a) == 1, what
        assert what in L.tk_last_error_detail().decode()
    assert L.tk_reduce(None, 0, None, None, 0, 2, 256, None, None, None) == 0


def test_reduce_masked_validates_like_reduce(tk):
    L = tk.lib
    ok = [FAKE, 10, FAKE, None, 4, 2, 256, FAKE, None, None]
    for i, v, what in [(5, 0, "k"), (5, 33, "k"), (6, 12, "H"), (1, -1, "y_rows"), (2, None, "NULL"),
                       (7, MISALIGNED, "aligned")]:
        a = list(ok)
        a[i] = v
        assert L.tk_reduce_masked(*a) == 1, what
        detail = L.tk_last_error_detail().decode()
        assert what in detail and "tk_reduce_masked" in detail
    a = list(ok)
    a[4] = 0
    assert L.tk_reduce_masked(*a) == 0      # T = 0: nothing to do


def test_binding_raises_with_detail(tk):
    with pytest.raises(tk.TkError) as ei:
        tk._check("tk_reduce", tk.lib.tk_reduce(FAKE, 1, FAKE, None, 4, 0, 256, FAKE, None, None))
    assert "k=0" in str(ei.value)


def test_next_rows_reject_bad_arguments(tk):
    L = tk.lib
    ws = L.tk_balance_stats_workspace_bytes(128, 16)
    assert ws == 2 * 16 * 8
    ok = [FAKE, FAKE, 128, 16, 2, 1, FAKE, FAKE, FAKE, FAKE, ws, None]
    for i, v, what in [(4, 17, "k"), (5, 3, "score_fn"), (10, ws - 8, "workspace"), (9, MISALIGNED, "aligned"),
                       (1, None, "NULL")]:
        a = list(ok)
        a[i] = v
        assert L.tk_balance_stats(*a) == 1, what
        assert what in L.tk_last_error_detail().decode()
    for args, what in [((FAKE, 10, 2, 16, 3, 0, FAKE, None), "divide"),
                       ((FAKE, 10, 2, 16, 4, 4, FAKE, None), "tp_rank"),
                       ((FAKE, 10, 0, 16, 4, 0, FAKE, None), "k")]:
        assert L.tk_tp_mask(*args) == 1 and what in L.tk_last_error_detail().decode()
    wsb = L.tk_reduce_backward_workspace_bytes(64, 4)
    assert wsb == 64 * 4 * 4 * 8
    ok = [FAKE, FAKE, 256, FAKE, FAKE, FAKE, None, 64, 16, 4, 256, FAKE, FAKE, FAKE, wsb, None, None]
    for i, v, what in [(10, 12, "H"), (9, 0, "k"), (14, wsb - 8, "workspace"), (0, MISALIGNED, "aligned"),
                       (4, None, "together"), (13, None, "NULL")]:
        a = list(ok)
        a[i] = v
        assert L.tk_reduce_backward(*a) == 1, what
        assert what in L.tk_last_error_detail().decode()
    assert L.tk_expand_backward(FAKE, 10, FAKE, 4, 0, 256, FAKE, None, None) == 1


def test_selftest_rejects_bad_limits(tk):
    assert tk.lib.tk_selftest_bounded_wait(0, FAKE, None) == 1
    assert tk.lib.tk_selftest_bounded_wait(3_000_000_000, FAKE, None) == 1
    assert tk.lib.tk_selftest_bounded_wait(1000, None, None) == 1


def test_ep_entries_reject_bad_arguments(tk):
    L = tk.lib
    T, G = 64, 4
    ws = L.tk_ep_layout_workspace_bytes(T, G)
    assert ws >= T * G * 4 and L.tk_ep_layout_workspace_bytes(T, 33) == 0
    ok = [FAKE, T, 16, 2, G, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None, None]
    for i, v, what in [(4, 0, "G="), (4, 33, "G="), (2, 18, "multiple of G"), (3, 33, "k="),
                       (10, ws - 16, "workspace"), (9, MISALIGNED, "aligned"), (7, None, "NULL")]:
        a = list(ok)
        a[i] = v
        assert L.tk_ep_layout(*a) == 1, what
        assert what in L.tk_last_error_detail().decode(), what
    peers = (tk.EpPeer * G)(*[tk.EpPeer(FAKE, None, FAKE, FAKE, 0, 100) for _ in range(G)])
    ok = [FAKE, FAKE, FAKE, FAKE, FAKE, T, 16, 2, 256, G, 0, peers, None, None]
    for i, v, what in [(9, 33, "G="), (6, 18, "multiple of G"), (8, 12, "H="), (10, 5, "out_dtype"),
                       (11, None, "peers"), (0, MISALIGNED, "aligned")]:
        a = list(ok)
        a[i] = v
        assert L.tk_ep_dispatch(*a) == 1, what
        assert what in L.tk_last_error_detail().decode(), what
    a = list(ok)
    a[8], a[10] = 200, 1                   # E4M3 needs H % 128 == 0
    assert L.tk_ep_dispatch(*a) == 1 and "128" in L.tk_last_error_detail().decode()
    bad = (tk.EpPeer * G)(*[tk.EpPeer(None, None, FAKE, FAKE, 0, 100) for _ in range(G)])
    a = list(ok)
    a[11] = bad
    assert L.tk_ep_dispatch(*a) == 1 and "receive buffers" in L.tk_last_error_detail().decode()
    parts = (ctypes.c_void_p * G)(*[FAKE] * G)
    base = (ctypes.c_int64 * G)(*[0] * G)
    rows = (ctypes.c_int64 * G)(*[10] * G)
    assert L.tk_ep_combine(parts, base, rows, FAKE, FAKE, T, 33, 256, FAKE, None, None) == 1
    assert L.tk_ep_combine(parts, base, rows, FAKE, FAKE, T, G, 12, FAKE, None, None) == 1
    assert L.tk_ep_combine(parts, base, rows, FAKE, FAKE, T, G, 256, MISALIGNED, None, None) == 1
    neg = (ctypes.c_int64 * G)(*[-1] * G)
    assert L.tk_ep_combine(parts, base, neg, FAKE, FAKE, T, G, 256, FAKE, None, None) == 1
    assert L.tk_ep_combine(parts, base, rows, FAKE, FAKE, 0, G, 256, FAKE, None, None) == 0


def test_binding_without_library_raises(tmp_path):
    """A copy of the package without libtk_route.so: importing the binding fails loudly; there is
    no CPU path to fall back on."""
    import shutil
    import subprocess
    import sys

    pkg = os.path.join(ROOT, "token_routing_gate_b200")
    dst = tmp_path / "token_routing_gate_b200"
    dst.mkdir()
    for name in os.listdir(pkg):
        if name.endswith(".py"):
            shutil.copy(os.path.join(pkg, name), dst / name)
    code = "import token_routing_gate_b200.tk"
    r = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode != 0
    assert "is not built" in r.stderr and "no CPU path" in r.stderr, r.stderr[-2000:]


def test_product_modules_do_not_reach_the_oracle():
    """The package never imports, loads or runs anything under oracle/."""
    pkg = os.path.join(ROOT, "token_routing_gate_b200")
    for name in sorted(os.listdir(pkg)):
        if name.endswith(".py"):
            text = open(os.path.join(pkg, name)).read()
            assert not re.search(r"^\s*(from|import)\s+oracle\b", text, flags=re.M), name
            assert "tk_oracle" not in text and "liboracle" not in text, name
    csrc = os.path.join(pkg, "csrc")
    for name in sorted(os.listdir(csrc)):
        text = open(os.path.join(csrc, name)).read()
        assert "oracle" not in text.lower(), name


def test_route_map_window_rejects_bad_windows(tk):
    L = tk.lib
    ws = L.tk_route_map_workspace_bytes(128, 32, 8)
    ok = [FAKE, 128, 256, 8, 64, 32, 1, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None, None]
    for i, v, what in [(4, -1, "window"), (4, 225, "window"), (5, 0, "E=0"), (5, 257, "window"), (5, 1025, "E=1025"),
                       (3, 33, "k"), (6, 0, "align"), (12, ws - 16, "workspace"), (7, None, "NULL")]:
        a = list(ok)
        a[i] = v
        assert L.tk_route_map_window(*a) == 1, what
        detail = L.tk_last_error_detail().decode()
        assert what in detail and "tk_route_map_window" in detail, detail
    a = list(ok)
    a[11] = MISALIGNED
    assert L.tk_route_map_window(*a) == 1 and "aligned" in L.tk_last_error_detail().decode()
