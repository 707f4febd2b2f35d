"""The C-ABI library builds, loads without a GPU, and exports every entry
point that include/moe.h declares; the binding's ctypes prototypes take the
declared number and kinds of arguments; host-side argument checks answer
without launching anything."""
import ctypes
import os
import re

import pytest

import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.findall(r"^\s*(?:MOE_API\s+)?(?:const\s+char\s*\*|moe_status)\s+(moe_\w+)\s*\(", src, flags=re.M)


@pytest.fixture(scope="module")
def L():
    build.build()
    return moe.lib()


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("moe_route", "moe_dispatch_layout", "moe_permute", "moe_grouped_swiglu",
              "moe_combine", "moe_forward"):
        assert n in names
    assert sorted(names) == sorted(moe.SYMBOLS)


def test_library_exports_every_declared_symbol(L):
    for n in _declared():
        assert hasattr(L, n), n


def test_status_strings(L):
    for code, name in moe.STATUS_NAMES.items():
        assert L.moe_status_string(code).decode() == name


def _size(fn, **kw):
    s = moe.moe_shape(**{**dict(T=2048, d=256, E=16, k=4, f=256, ep=1, dtype=moe.MOE_F32), **kw})
    n = ctypes.c_size_t(0)
    return fn(ctypes.byref(s), ctypes.byref(n)), n.value


@pytest.mark.parametrize("kw,expect", [
    (dict(), moe.MOE_OK),
    (dict(E=0), moe.MOE_ERR_INVALID_ARG),
    (dict(E=257), moe.MOE_ERR_INVALID_ARG),
    (dict(k=0), moe.MOE_ERR_INVALID_ARG),
    (dict(k=17, E=64), moe.MOE_ERR_INVALID_ARG),
    (dict(k=5, E=4), moe.MOE_ERR_INVALID_ARG),
    (dict(ep=3), moe.MOE_ERR_INVALID_ARG),     # 16 % 3 != 0
    (dict(ep=32), moe.MOE_ERR_INVALID_ARG),    # more ranks than experts
    (dict(T=-1), moe.MOE_ERR_INVALID_ARG),
    (dict(T=1 << 29, k=4), moe.MOE_ERR_INVALID_ARG),  # T*k >= 2^31
    (dict(d=100), moe.MOE_ERR_UNSUPPORTED),
    (dict(f=96), moe.MOE_ERR_UNSUPPORTED),
    (dict(d=8192, dtype=moe.MOE_F32), moe.MOE_ERR_UNSUPPORTED),
    (dict(d=8192, dtype=moe.MOE_BF16), moe.MOE_OK),
    (dict(dtype=7), moe.MOE_ERR_INVALID_ARG),
    (dict(T=0), moe.MOE_OK),
])
def test_shape_checks(L, kw, expect):
    for fn in (L.moe_scratch_size, L.moe_forward_workspace_size, L.moe_packed_weights_size):
        st, n = _size(fn, **kw)
        assert st == expect
        if st == moe.MOE_OK:
            assert n > 0


def test_workspace_sizes_grow_with_tokens(L):
    _, a = _size(L.moe_forward_workspace_size, T=1024)
    _, b = _size(L.moe_forward_workspace_size, T=4096)
    assert b > a
    _, p = _size(L.moe_packed_weights_size, d=256, E=16, f=256)
    assert p >= 4 * (16 * 256 + 3 * 16 * 256 * 256)


def test_bad_placement_rejected_before_any_launch(L):
    s = moe.moe_shape(T=8, d=256, E=16, k=2, f=256, ep=4, dtype=moe.MOE_F32)
    lay = moe.moe_layout(*([ctypes.c_void_p(256)] * 9))
    ws = ctypes.c_void_p(1 << 20)
    # rank 0 owns 5 experts, rank 3 owns 3: not a partition
    bad = (ctypes.c_int32 * 16)(*([0] * 5 + [1] * 4 + [2] * 4 + [3] * 3))
    assert L.moe_dispatch_layout(ctypes.byref(s), ctypes.c_void_p(256), bad, ctypes.byref(lay),
                                 ws, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    out_of_range = (ctypes.c_int32 * 16)(*([0] * 4 + [1] * 4 + [2] * 4 + [4] * 4))
    assert L.moe_dispatch_layout(ctypes.byref(s), ctypes.c_void_p(256), out_of_range,
                                 ctypes.byref(lay), ws, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    # too small a workspace
    assert L.moe_dispatch_layout(ctypes.byref(s), ctypes.c_void_p(256), None, ctypes.byref(lay),
                                 ws, 16, None) == moe.MOE_ERR_WORKSPACE
    # misaligned index pointer
    assert L.moe_dispatch_layout(ctypes.byref(s), ctypes.c_void_p(258), None, ctypes.byref(lay),
                                 ws, 1 << 30, None) == moe.MOE_ERR_ALIGNMENT
    # missing send-layout outputs with ep > 1
    lay2 = moe.moe_layout(*([ctypes.c_void_p(256)] * 4 + [None] * 5))
    assert L.moe_dispatch_layout(ctypes.byref(s), ctypes.c_void_p(256), None, ctypes.byref(lay2),
                                 ws, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [
    dict(E=0), dict(E=257), dict(k=0), dict(k=17, E=64), dict(ep=3), dict(T=-1),
    dict(T=1 << 29, k=4), dict(d=100), dict(f=96), dict(d=8192, dtype=moe.MOE_F32), dict(dtype=7),
])
def test_static_layout_validates_like_the_workspace_layout(L, kw):
    """moe_dispatch_layout_static takes the same inputs as
    moe_dispatch_layout and rejects the same shapes with the same status,
    before any launch (so no GPU is needed)."""
    s = moe.moe_shape(**{**dict(T=2048, d=256, E=16, k=4, f=256, ep=1, dtype=moe.MOE_F32), **kw})
    lay = moe.moe_layout(*([ctypes.c_void_p(256)] * 9))
    a = L.moe_dispatch_layout(ctypes.byref(s), ctypes.c_void_p(256), None, ctypes.byref(lay),
                              ctypes.c_void_p(1 << 20), 1 << 30, None)
    b = L.moe_dispatch_layout_static(ctypes.byref(s), ctypes.c_void_p(256), None,
                                     ctypes.byref(lay), None, None)
    assert a == b != moe.MOE_OK


def test_static_layout_rejects_bad_placements_and_pointers(L):
    s = moe.moe_shape(T=8, d=256, E=16, k=2, f=256, ep=4, dtype=moe.MOE_F32)
    lay = moe.moe_layout(*([ctypes.c_void_p(256)] * 9))
    bad = (ctypes.c_int32 * 16)(*([0] * 5 + [1] * 4 + [2] * 4 + [3] * 3))
    assert L.moe_dispatch_layout_static(ctypes.byref(s), ctypes.c_void_p(256), bad,
                                        ctypes.byref(lay), None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_dispatch_layout_static(ctypes.byref(s), ctypes.c_void_p(258), None,
                                        ctypes.byref(lay), None, None) == moe.MOE_ERR_ALIGNMENT
    lay2 = moe.moe_layout(*([ctypes.c_void_p(256)] * 4 + [None] * 5))
    assert L.moe_dispatch_layout_static(ctypes.byref(s), ctypes.c_void_p(256), None,
                                        ctypes.byref(lay2), None, None) == moe.MOE_ERR_INVALID_ARG


def test_misaligned_tensors_rejected(L):
    s = moe.moe_shape(T=8, d=256, E=16, k=2, f=256, ep=1, dtype=moe.MOE_BF16)
    P = ctypes.c_void_p
    assert L.moe_permute(ctypes.byref(s), P(8), P(256), P(4096), None) == moe.MOE_ERR_ALIGNMENT
    assert L.moe_combine(ctypes.byref(s), P(4096), P(256), None, P(4100), None) == moe.MOE_ERR_ALIGNMENT
    assert L.moe_permute(ctypes.byref(s), None, P(256), P(4096), None) == moe.MOE_ERR_INVALID_ARG


def _declared_params():
    """Entry point -> its parameter count, from include/moe.h."""
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"(?:MOE_API\s+)?(?:const\s+char\s*\*|moe_status)\s+(moe_\w+)\s*\(([^)]*)\)\s*;",
                         src):
        params = [p.strip() for p in m.group(2).split(",") if p.strip()]
        out[m.group(1)] = 0 if params == ["void"] else len(params)
    return out


def test_binding_argument_counts_match_the_header(L):
    """Each ctypes prototype takes as many arguments as the C declaration,
    so no call can shift or drop an argument."""
    decl = _declared_params()
    assert sorted(decl) == sorted(moe.SYMBOLS)
    for name, n in decl.items():
        fn = getattr(L, name)
        assert fn.argtypes is not None, name
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)


def _c_kind(param: str) -> str:
    p = " ".join(param.split())
    if "*" in p or p.startswith(("moe_stream_t", "moe_event_t")):
        return "ptr"
    if p.startswith(("size_t", "const size_t", "uint64_t")):
        return "size"  # unsigned 64-bit: ctypes' c_size_t is c_uint64
    if p.startswith(("double", "const double")):
        return "f64"
    if "int64_t" in p:
        return "i64"
    if p.startswith(("int32_t", "int ", "const int32_t", "moe_status", "moe_dtype")):
        return "i32"
    raise AssertionError(f"unclassified parameter {param!r}")


def _py_kind(t) -> str:
    if t is ctypes.c_void_p or t is ctypes.c_char_p or isinstance(t, type(ctypes.POINTER(ctypes.c_int))):
        return "ptr"
    if t is ctypes.c_size_t:
        return "size"
    if t is ctypes.c_double:
        return "f64"
    if ctypes.sizeof(t) == 8:
        return "i64"
    if ctypes.sizeof(t) == 4:
        return "i32"
    raise AssertionError(f"unclassified ctypes type {t!r}")


def test_binding_argument_kinds_match_the_header(L):
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    for m in re.finditer(r"(?:MOE_API\s+)?(?:const\s+char\s*\*|moe_status)\s+(moe_\w+)\s*\(([^)]*)\)\s*;",
                         src):
        params = [p.strip() for p in m.group(2).split(",") if p.strip()]
        fn = getattr(L, m.group(1))
        kinds_c = [_c_kind(p) for p in params]
        kinds_py = [_py_kind(t) for t in fn.argtypes]
        assert kinds_py == kinds_c, (m.group(1), kinds_py, kinds_c)


def test_struct_layouts_match_the_header(tmp_path):
    """sizeof / offsetof of the ABI structs as a C compiler lays them out
    from include/moe.h, against the binding's ctypes structures (and the
    device-resident moe_stats words that stats_dict decodes)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    structs = {
        "moe_shape": [f for f, _ in moe.moe_shape._fields_],
        "moe_layout": [f for f, _ in moe.moe_layout._fields_],
        "moe_forward_buffers": [f for f, _ in moe.moe_forward_buffers._fields_],
        "moe_router_counts": [f for f, _ in moe.moe_router_counts._fields_],
        "moe_ep_peer_dest": [f for f, _ in moe.moe_ep_peer_dest._fields_],
        "moe_ep_peer_return": [f for f, _ in moe.moe_ep_peer_return._fields_],
        "moe_stats": ["rows_sent", "dup_removed", "tokens_single_rank", "home_rank_rows",
                      "max_expert_rows", "min_expert_rows"],
    }
    lines = ['#include <stdio.h>', '#include "moe.h"', "int main(void) {"]
    for s, fields in structs.items():
        lines.append(f'  printf("{s} size %zu\\n", sizeof({s}));')
        for f in fields:
            lines.append(f'  printf("{s} {f} %zu\\n", offsetof({s}, {f}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.check_call([cc, "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    got = {}
    for line in subprocess.check_output([str(exe)], text=True).splitlines():
        s, f, v = line.split()
        got[(s, f)] = int(v)
    for s, cls in (("moe_shape", moe.moe_shape), ("moe_layout", moe.moe_layout),
                   ("moe_forward_buffers", moe.moe_forward_buffers),
                   ("moe_router_counts", moe.moe_router_counts),
                   ("moe_ep_peer_dest", moe.moe_ep_peer_dest),
                   ("moe_ep_peer_return", moe.moe_ep_peer_return)):
        assert got[(s, "size")] == ctypes.sizeof(cls), s
        for f in structs[s]:
            assert got[(s, f)] == getattr(cls, f).offset, (s, f)
    # stats_dict reads six int64 words: the four counters, then max (low half)
    # and min (high half) of word 4
    assert [got[("moe_stats", f)] for f in structs["moe_stats"]] == [0, 8, 16, 24, 32, 36]
    assert got[("moe_stats", "size")] <= 6 * 8


def test_peer_entry_points_reject_bad_arguments(L):
    """Argument checks of the peer-memory exchange, all before any launch."""
    s = moe.Shape(T=64, d=128, E=8, k=2, f=128, ep=2).c
    lay = moe.moe_layout()
    dests = (moe.moe_ep_peer_dest * 2)()
    dests[0] = moe.moe_ep_peer_dest(None, None, None, 0, -1)
    assert L.moe_ep_dispatch_peer(ctypes.byref(s), None, None, None, None, ctypes.byref(lay),
                                  dests, None) == moe.MOE_ERR_INVALID_ARG
    dests[0] = moe.moe_ep_peer_dest(None, None, None, 0, 3)  # rows but no buffers
    assert L.moe_ep_dispatch_peer(ctypes.byref(s), None, None, None, None, ctypes.byref(lay),
                                  dests, None) == moe.MOE_ERR_INVALID_ARG
    dests[0] = moe.moe_ep_peer_dest(8, 16, 16, 0, 3)  # recv_x not 16-byte aligned
    assert L.moe_ep_dispatch_peer(ctypes.byref(s), None, None, None, None, ctypes.byref(lay),
                                  dests, None) == moe.MOE_ERR_ALIGNMENT
    assert L.moe_ep_dispatch_peer(ctypes.byref(s), None, None, None, None, ctypes.byref(lay),
                                  None, None) == moe.MOE_ERR_INVALID_ARG
    one = moe.Shape(T=64, d=128, E=8, k=2, f=128, ep=1).c
    dests[0] = moe.moe_ep_peer_dest(None, None, None, 0, 0)
    assert L.moe_ep_dispatch_peer(ctypes.byref(one), None, None, None, None, ctypes.byref(lay),
                                  dests, None) == moe.MOE_ERR_INVALID_ARG
    # returns: blocks must tile the received rows
    rets = (moe.moe_ep_peer_return * 2)()
    rets[0] = moe.moe_ep_peer_return(256, 0, 30)
    rets[1] = moe.moe_ep_peer_return(256, 0, 30)
    assert L.moe_ep_expert_forward_peer(ctypes.byref(s), 256, 256, 256, 256, rets, 256, 1 << 30,
                                        None) == moe.MOE_ERR_INVALID_ARG
    rets[1] = moe.moe_ep_peer_return(8, 0, 34)
    assert L.moe_ep_expert_forward_peer(ctypes.byref(s), 256, 256, 256, 256, rets, 256, 1 << 30,
                                        None) == moe.MOE_ERR_ALIGNMENT
    rets[1] = moe.moe_ep_peer_return(256, -1, 34)
    assert L.moe_ep_expert_forward_peer(ctypes.byref(s), 256, 256, 256, 256, rets, 256, 1 << 30,
                                        None) == moe.MOE_ERR_INVALID_ARG
    # rendezvous
    flags = (ctypes.c_void_p * 2)(256, 256)
    assert L.moe_ep_signal_wait(flags, 0, 2, 0, 256, None) == moe.MOE_ERR_INVALID_ARG  # epoch 0
    assert L.moe_ep_signal_wait(flags, 2, 2, 1, 256, None) == moe.MOE_ERR_INVALID_ARG  # rank
    assert L.moe_ep_signal_wait(flags, 0, 0, 1, 256, None) == moe.MOE_ERR_INVALID_ARG  # P
    assert L.moe_ep_signal_wait(flags, 0, 2, 1, None, None) == moe.MOE_ERR_INVALID_ARG  # ws
    assert L.moe_ep_signal_wait(flags, 0, 2, 1, 260, None) == moe.MOE_ERR_ALIGNMENT
    bad = (ctypes.c_void_p * 2)(256, 260)
    assert L.moe_ep_signal_wait(bad, 0, 2, 1, 256, None) == moe.MOE_ERR_ALIGNMENT
    nul = (ctypes.c_void_p * 2)(256, None)
    assert L.moe_ep_signal_wait(nul, 0, 2, 1, 256, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_debug_ep_signal_wait(flags, 0, 2, 1, 256, 0, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_debug_ep_signal_wait(flags, 0, 2, 1, 256, 2_000_000_000,
                                      None) == moe.MOE_ERR_INVALID_ARG


def test_forward_options_reject_unknown_bits(L):
    """moe_debug_forward_options: only MOE_FWD_COMBINE_IN_DOWN is defined;
    any other bit is an invalid argument, before any check of the rest."""
    s = moe.Shape(T=64, d=128, E=8, k=2, f=128).c
    for bad in (2, 4, 1 << 30, -1):
        assert L.moe_debug_forward_options(ctypes.byref(s), None, None, None, None, None, None,
                                           None, 0, bad, None) == moe.MOE_ERR_INVALID_ARG
