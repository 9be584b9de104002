"""The C-ABI library on the host: it loads, exports every declared symbol, and
rejects bad arguments before touching the GPU (no compute calls here)."""

import ctypes
import os
import re

import pytest

import attention_tiled_attn_b200 as attn
from attention_tiled_attn_b200 import build as attn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn_b200.h")


@pytest.fixture(scope="module")
def lib():
    attn_build.build()
    return attn.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(attn_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("attn_fwd", "attn_status_string", "attn_release_workspace", "attn_device_status", "attn_version"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def declared_parameters():
    """{name: [kind of each parameter]} for every function the header declares,
    kind one of "ptr", "float", "int" ((void) gives an empty list)."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"^\s*(?:const\s+)?\w+\**\s+\**(attn_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.M | re.S):
        params = m.group(2).strip()
        kinds = []
        if params not in ("", "void"):
            for prm in params.split(","):
                kinds.append("ptr" if "*" in prm else "float" if re.search(r"\bfloat\b", prm) else "int")
        out[m.group(1)] = kinds
    return out


def test_binding_argtypes_match_the_header(lib):
    """Every function the binding gives argtypes takes the header's parameters, in
    number and kind, so a changed C signature cannot be called with a stale one."""
    decl = declared_parameters()
    assert set(decl) == set(declared_functions())
    kind_of = {ctypes.c_void_p: "ptr", ctypes.c_char_p: "ptr", ctypes.c_float: "float", ctypes.c_int: "int",
               ctypes.c_uint: "int", ctypes.c_size_t: "int"}
    checked = 0
    for name, kinds in decl.items():
        argtypes = getattr(getattr(lib, name), "argtypes", None)
        if argtypes is not None:
            assert [kind_of[a] for a in argtypes] == kinds, name
            checked += 1
    assert checked >= 8


def test_status_strings(lib):
    assert attn.status_string(0) == "ok"
    for st in range(-18, 0):
        s = attn.status_string(st)
        assert s and s != "unknown status"
    assert attn.status_string(-99) == "unknown status"
    assert attn.version() == 10000


P = 0x10000  # a 16-byte aligned fake device address; never dereferenced on the error paths


def call(**kw):
    a = dict(q=P, k=P, v=P, out=P, lse=P, N=1, Hq=2, H=1, L=8, S=8, E=64, Ev=64, scale=0.125, mode=0,
             sink=None, mask_kind=0, window=0, bias=None, dtype=0, stream=None)
    a.update(kw)
    return attn.attn_fwd_raw(a["q"], a["k"], a["v"], a["out"], a["lse"], a["N"], a["Hq"], a["H"], a["L"], a["S"],
                             a["E"], a["Ev"], a["scale"], a["mode"], a["sink"], a["mask_kind"], a["window"],
                             a["bias"], a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), -1), (dict(v=None), -1), (dict(out=None), -1),
    (dict(N=0), -2), (dict(L=0), -2), (dict(S=-3), -2), (dict(Hq=0), -2),
    (dict(Hq=3, H=2), -3),
    (dict(E=96), -4), (dict(Ev=32), -4), (dict(E=256), -4),
    (dict(scale=0.0), -5), (dict(scale=-1.0), -5), (dict(scale=float("inf")), -5), (dict(scale=float("nan")), -5),
    (dict(mode=3), -6), (dict(mode=-1), -6),
    (dict(mask_kind=3), -7), (dict(mask_kind=2, window=0), -8),
    (dict(mode=2, sink=None), -9),
    (dict(dtype=2), -10),
    (dict(q=P + 8), -11), (dict(out=P + 4), -11), (dict(bias=P + 8), -11), (dict(lse=P + 2), -11),
    (dict(N=1 << 20, Hq=1 << 12, H=1 << 12), -2),
    (dict(dtype=1, N=1, Hq=70000, H=70000), -2),
])
def test_argument_validation(lib, kw, status):
    assert call(**kw) == status


def call_streaming(**kw):
    a = dict(q=P, k=P, v=P, out=P, lse=P, N=1, Hq=2, H=1, L=8, S=8, E=64, Ev=64, scale=0.125, mode=0,
             sink=None, window=4, keep=2, bias=None, dtype=0, stream=None)
    a.update(kw)
    return attn.attn_fwd_streaming_raw(a["q"], a["k"], a["v"], a["out"], a["lse"], a["N"], a["Hq"], a["H"], a["L"],
                                       a["S"], a["E"], a["Ev"], a["scale"], a["mode"], a["sink"], a["window"],
                                       a["keep"], a["bias"], a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(window=0), -8), (dict(window=-5), -8), (dict(keep=-1), -18),
    (dict(q=None), -1), (dict(Hq=3, H=2), -3), (dict(E=96), -4), (dict(scale=0.0), -5),
    (dict(mode=2, sink=None), -9), (dict(dtype=2), -10), (dict(k=P + 8), -11),
])
def test_streaming_argument_validation(lib, kw, status):
    assert call_streaming(**kw) == status


def call_indexed(**kw):
    a = dict(q=P, k=P, v=P, out=P, lse=P, idx=P, n_sel=8, N=1, Hq=2, H=1, L=1, S=64, E=64, Ev=64, scale=0.125,
             sink=None, mask_kind=0, window=0, bias=None, stream=None)
    a.update(kw)
    return attn.attn_decode_indexed_raw(a["q"], a["k"], a["v"], a["out"], a["lse"], a["idx"], a["n_sel"], a["N"],
                                        a["Hq"], a["H"], a["L"], a["S"], a["E"], a["Ev"], a["scale"], a["sink"],
                                        a["mask_kind"], a["window"], a["bias"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(idx=None), -1), (dict(q=None), -1), (dict(n_sel=0), -2), (dict(n_sel=-4), -2),
    (dict(N=0), -2), (dict(Hq=3, H=2), -3), (dict(E=96), -4), (dict(scale=0.0), -5),
    (dict(mask_kind=3), -7), (dict(mask_kind=2, window=0), -8),
    (dict(idx=P + 2), -11), (dict(v=P + 8), -11),
    (dict(Hq=32, H=1), -17), (dict(Hq=4, H=1, L=5), -17),
])
def test_indexed_argument_validation(lib, kw, status):
    assert call_indexed(**kw) == status


def call_padded(**kw):
    a = dict(q=P, k=P, v=P, out=P, lse=P, N=1, Hq=2, H=1, L=8, S=8, E=64, Ev=64, scale=0.125, mode=0,
             sink=None, mask_kind=1, window=0, bits=P, start=P, end=P, dtype=0, stream=None)
    a.update(kw)
    return attn.attn_fwd_padded_raw(a["q"], a["k"], a["v"], a["out"], a["lse"], a["N"], a["Hq"], a["H"], a["L"],
                                    a["S"], a["E"], a["Ev"], a["scale"], a["mode"], a["sink"], a["mask_kind"],
                                    a["window"], a["bits"], a["start"], a["end"], a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(mask_kind=3), -7), (dict(mask_kind=2, window=0), -8),
    (dict(bits=P + 2), -11), (dict(start=P + 1), -11), (dict(end=P + 3), -11),
    (dict(q=None), -1), (dict(Hq=3, H=2), -3), (dict(E=96), -4), (dict(scale=-1.0), -5), (dict(mode=2), -9),
    (dict(dtype=5), -10),
])
def test_padded_argument_validation(lib, kw, status):
    assert call_padded(**kw) == status


def call_bwd(**kw):
    a = dict(q=P, k=P, v=P, out=P, dout=P, lse=P, dq=P, dk=P, dv=P, dsink=None, N=1, Hq=2, H=1, L=8, S=8, E=64,
             Ev=64, scale=0.125, mode=0, sink=None, mask_kind=1, window=0, stream=None, keep=0, bits=None,
             start=None, end=None)
    a.update(kw)
    return attn.attn_bwd_raw(a["q"], a["k"], a["v"], a["out"], a["dout"], a["lse"], a["dq"], a["dk"], a["dv"],
                             a["dsink"], a["N"], a["Hq"], a["H"], a["L"], a["S"], a["E"], a["Ev"], a["scale"],
                             a["mode"], a["sink"], a["mask_kind"], a["window"], a["stream"], a["keep"], a["bits"],
                             a["start"], a["end"])


@pytest.mark.parametrize("kw,status", [
    (dict(out=None), -1), (dict(dout=None), -1), (dict(lse=None), -1), (dict(dq=None), -1), (dict(dk=None), -1),
    (dict(dv=None), -1), (dict(q=None), -1),
    (dict(N=0), -2), (dict(Hq=3, H=2), -3), (dict(E=96), -4), (dict(scale=0.0), -5), (dict(mode=7), -6),
    (dict(mask_kind=3), -7), (dict(mask_kind=2, window=0), -8), (dict(mode=2), -9),
    (dict(dq=P + 4), -11), (dict(dk=P + 8), -11), (dict(out=P + 2), -11), (dict(lse=P + 2), -11),
    (dict(keep=-1), -18), (dict(keep=3, mask_kind=1), -18), (dict(keep=3, mask_kind=0), -18),
    (dict(bits=P + 2), -11), (dict(start=P + 1), -11), (dict(end=P + 3), -11),
])
def test_bwd_argument_validation(lib, kw, status):
    assert call_bwd(**kw) == status


def test_python_binding_rejects_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        attn.attn_fwd(q, q, q, scale=0.1)


@pytest.mark.parametrize("call", [
    lambda q: attn.attn_fwd(q, q, q, scale=0.1, mode="cosine"),
    lambda q: attn.attn_fwd(q, q, q, scale=0.1, mask_kind="diagonal"),
    lambda q: attn.attn_fwd(q, q, q, scale=0.1, mask_kind="causal", keep_first=4),
    lambda q: attn.attn_fwd(q, q, q, scale=0.1, mask_kind="window", window=8, keep_first=4),
    lambda q: attn.attn_bwd(q, q, q, q, q, q, scale=0.1, mode="cosine"),
    lambda q: attn.attn_bwd(q, q, q, q, q, q, scale=0.1, mask_kind="window", window=8, keep_first=4),
    lambda q: attn.attn_decode_indexed(q, q, q, q, scale=0.1, mask_kind="streaming"),
], ids=["fwd_mode", "fwd_mask", "fwd_keep_causal", "fwd_keep_window", "bwd_mode", "bwd_keep_window",
        "indexed_streaming"])
def test_python_binding_rejects_unknown_kinds_and_stray_kept_keys(lib, call):
    """Unknown mode or mask strings, and kept keys without the streaming mask, are
    rejected before any tensor is looked at (so this holds on a host without a GPU)."""
    import torch
    q = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="unknown mode|unknown mask kind|keep_first needs"):
        call(q)
