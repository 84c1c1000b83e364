"""C-ABI checks that need no GPU: the library loads, exports every declared
symbol, and rejects bad arguments on the host before anything reaches CUDA."""
import ctypes
import os
import re

import pytest

import gated_token_recurrence_b200 as gtr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*[\w\s\*]+?\b(gtr_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    assert "gtr_gla_fwd" in names and "gtr_gla_fwd_ex" in names
    assert set(gtr.EXPORTED) <= set(names)


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(gtr.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_status_strings_and_version():
    assert gtr.status_string(0) == "GTR_OK"
    assert gtr.status_string(4) == "GTR_ERR_TIMEOUT"
    assert gtr.status_string(99) == "GTR_ERR_UNKNOWN"
    assert gtr.version() >= 100


def _fwd_ex(**kw):
    a = dict(q=16, k=16, v=16, g=16, out=16, B=1, heads=2, H=4, W=4, dk=64, dv=64, direction=0,
             din=gtr.F16, dout=gtr.F16, path=0, ws=None, ws_bytes=0)
    a.update(kw)
    return gtr.lib.gtr_gla_fwd_ex(a["q"], a["k"], a["v"], a["g"], a["out"], a["B"], a["heads"],
                                  a["H"], a["W"], a["dk"], a["dv"], a["direction"], a["din"],
                                  a["dout"], a["path"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(out=None), 1), (dict(g=8), 1),          # null / misaligned
    (dict(B=0), 1), (dict(heads=-1), 1), (dict(H=0), 1), (dict(W=-3), 1),
    (dict(direction=4), 1), (dict(direction=-1), 1), (dict(din=7), 1), (dict(path=9), 1),
    (dict(dk=48), 2), (dict(dk=128), 2), (dict(dv=128), 2),           # valid but unsupported
    (dict(din=gtr.F32, dout=gtr.F16), 2), (dict(din=gtr.BF16, dout=gtr.F16), 2),
    (dict(ws=None, ws_bytes=0), 5),                                   # workspace missing
])
def test_bad_arguments_rejected_on_host(kw, code):
    assert _fwd_ex(**kw) == code


def test_workspace_query():
    n = gtr.workspace_bytes(1, 6, 40, 40, 64, 64, gtr.F16, "split")
    units = 6 * 25
    assert n == 256 + 2048 + units * (2 * 64 * 64 + 64) * 4
    assert gtr.workspace_bytes(1, 6, 40, 40, 64, 64, gtr.F16, "auto") >= n
    assert gtr.workspace_bytes(0, 6, 40, 40) == 0
    assert gtr.workspace_bytes(1, 6, 40, 40, 48, 64) == 0
    assert gtr.workspace_bytes(1, 6, 40, 40, 32, 64) > 0   # d_k = 32 is supported


def test_typed_entries_validate_too():
    f = gtr.lib.gtr_gla_fwd_f16
    assert f(None, 16, 16, 16, 16, 1, 1, 8, 8, 64, 64, 0, None) == 1
    assert gtr.lib.gtr_gla_fwd_f32(16, 16, 16, 16, 16, 1, 1, 8, 8, 64, 64, 9, None) == 1
    assert gtr.lib.gtr_gla_fwd_bf16(16, 16, 16, 16, 16, 1, 1, 8, 8, 48, 64, 0, None) == 2


def test_dispatcher_plan():
    assert gtr.plan(1, 6, 40, 40, in_dtype=gtr.F16) == ("fused", 1)
    assert gtr.plan(8, 6, 48, 80, in_dtype=gtr.BF16) == ("fused", 1)
    assert gtr.plan(1, 2, 16, 16, in_dtype=gtr.F32) == ("split", 3)
    assert gtr.status_string(6) == "GTR_ERR_RANGE"


def test_short_sequences_take_the_split_path_whatever_is_requested():
    """Shorter than one chunk: a requested fused path runs the split path, so the
    workspace query for that request is the split path's size."""
    split = gtr.workspace_bytes(1, 2, 7, 9, 64, 64, gtr.F16, "split")
    assert gtr.workspace_bytes(1, 2, 7, 9, 64, 64, gtr.F16, "fused") == split
    assert gtr.workspace_bytes(1, 2, 7, 9, 64, 64, gtr.F16, "fused_sequential") == split
    assert gtr.plan(1, 2, 7, 9, in_dtype=gtr.F16) == ("split", 3)


# ---------------------------------------------------------------- gtr_gla_fwd_noalloc (host side)
def _noalloc(B, heads, H, W, q=256, out=256, din=gtr.F16, dout=gtr.F16, dk=64):
    # the pointers are never dereferenced: every case below is decided on the host
    return gtr.lib.gtr_gla_fwd_noalloc(q, 256, 256, 256, out, B, heads, H, W, dk, 64, 0, din, dout, None)


def test_noalloc_unit_limit_matches_its_array():
    """634 chunk units of split-path scratch fit the fixed 20 MiB array, 635 do not."""
    array = 20 << 20
    fits = gtr.workspace_bytes(1, 2, 64, 317, 64, 64, gtr.F16, "split")   # 2 x 317 = 634 units
    over = gtr.workspace_bytes(1, 1, 64, 635, 64, 64, gtr.F16, "split")   # 635 units
    assert fits <= array < over
    assert _noalloc(1, 1, 64, 635) == 5          # GTR_ERR_WORKSPACE, nothing enqueued
    assert _noalloc(5, 127, 1, 64) == 5          # 635 units spread over (batch, head)


def test_noalloc_validates_arguments_before_the_size_limit():
    """Argument errors keep their own codes on a problem that is also too large."""
    assert _noalloc(1, 1, 64, 635, q=None) == 1                       # null pointer
    assert _noalloc(1, 1, 64, 635, out=8) == 1                        # misaligned
    assert _noalloc(1, 1, 64, 635, din=gtr.BF16, dout=gtr.F16) == 2   # unsupported pairing
    assert _noalloc(1, 1, 64, 635, dk=48) == 2                        # unsupported d_k


# ---------------------------------------------------------------- gtr_gla_block_fwd (host side)
def _block(**kw):
    a = dict(q=256, k=256, v=256, lg=256, z=None, w2=None, b=None, rank=0, tau=16.0, og=None, nw=None,
             eps=1e-6, out=256, B=1, heads=2, H=8, W=8, dk=64, dv=64, direction=0, din=gtr.F16, dout=gtr.F16,
             path=0, ws=None, wsb=0)
    a.update(kw)
    return gtr.lib.gtr_gla_block_fwd(a["q"], a["k"], a["v"], a["lg"], a["z"], a["w2"], a["b"], a["rank"],
                                     a["tau"], a["og"], a["nw"], a["eps"], a["out"], a["B"], a["heads"], a["H"],
                                     a["W"], a["dk"], a["dv"], a["direction"], a["din"], a["dout"], a["path"],
                                     a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(lg=None), 1),                                               # no gates at all
    (dict(z=256, w2=256, b=256, rank=16), 1),                         # both gate sources
    (dict(lg=None, z=256, w2=None, b=256, rank=16), 1),               # factor missing
    (dict(lg=None, z=256, w2=256, b=256, rank=4), 1),                 # ranks 8 and 16 only
    (dict(lg=None, z=256, w2=256, b=256, rank=12), 1),
    (dict(lg=None, z=256, w2=256, b=256, rank=20), 1),
    (dict(lg=None, z=256, w2=256, b=256, rank=16, tau=0.0), 1),       # tau must be positive
    (dict(lg=None, z=256, w2=256, b=256, rank=16, tau=float("inf")), 1),
    (dict(og=256, nw=None), 1),                                       # norm weight missing
    (dict(og=264, nw=256), 1),                                        # misaligned output gate
    (dict(og=256, nw=256, eps=-1.0), 1),                              # negative eps
    (dict(path=7), 1), (dict(dk=48), 2), (dict(din=gtr.BF16, dout=gtr.F16), 2),
    (dict(ws=256, wsb=16), 5),                                        # caller workspace too small
])
def test_block_arguments_rejected_on_host(kw, code):
    assert _block(**kw) == code


@pytest.mark.parametrize("args,code", [
    ((None, 256, 256, None, 256, 1, 8, 8, 64, 1), 1),      # null xg
    ((256, 256, 256, None, 264, 1, 8, 8, 64, 1), 1),       # misaligned out
    ((256, 256, 256, None, 256, 0, 8, 8, 64, 1), 1),       # B = 0
    ((256, 256, 256, None, 256, 1, 8, 8, 64, 5), 1),       # bad dtype
    ((256, 256, 256, None, 256, 1, 8, 8, 96, 1), 2),       # C not whole 64-channel blocks (16-bit)
    ((256, 256, 256, None, 256, 1, 8, 8, 48, 0), 2),       # C not whole 32-channel blocks (fp32)
])
def test_stencil_arguments_rejected_on_host(args, code):
    assert gtr.lib.gtr_sswiglu_dwconv(*args, None) == code
