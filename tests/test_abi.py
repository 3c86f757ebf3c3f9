"""The C ABI without a GPU: the library loads, exports every symbol that
include/ckv.h declares, sizes workspaces on the host, and rejects bad
arguments with the documented status before touching the device.

Every call below fails a host-side check, so none of them reaches a CUDA
call; a test asserts that explicitly (status is never CKV_OK or
CKV_ERR_CUDA)."""
import ctypes
import os
import re

import pytest

import graph_community_sparse_b200 as ckv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ckv.h")

OK, INVALID, MISALIGNED, UNSUPPORTED, CAPACITY, WORKSPACE, CUDA = range(7)


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"CKV_API\s+[\w\s\*]+?\b(ckv_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(ckv.lib, n), n
    assert sorted(ckv.EXPORTED) == names


def test_abi_version_and_status_strings():
    ver = int(re.search(r"#define CKV_ABI_VERSION (\d+)", open(HEADER).read()).group(1))
    assert ckv.ckv_abi_version() == ver
    for i, name in enumerate(["CKV_OK", "CKV_ERR_INVALID_ARG", "CKV_ERR_MISALIGNED", "CKV_ERR_UNSUPPORTED",
                              "CKV_ERR_CAPACITY", "CKV_ERR_WORKSPACE", "CKV_ERR_CUDA"]):
        assert ckv.ckv_status_string(i) == name
        assert re.search(rf"\b{name} = {i}\b", open(HEADER).read())


def test_struct_layouts_match_header_order():
    src = open(HEADER).read()
    for cls, tag in [(ckv.CacheDesc, "ckv_cache_desc"), (ckv.GraphDesc, "ckv_graph_desc"),
                     (ckv.SelectionDesc, "ckv_selection_desc")]:
        body = re.search(r"typedef struct \{([^{}]*)\}\s*" + tag + ";", src).group(1)
        body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
        fields = re.findall(r"\**\s*(\w+)\s*(?=[,;])", body)
        assert [f[0] for f in cls._fields_] == fields, tag


# ---------------------------------------------------------------------------
# fake descriptors: plausible device addresses that are never dereferenced
# ---------------------------------------------------------------------------
FAKE = 0x7F0000000000


def _cache(**kw):
    c = dict(dtype=1, B=2, Hkv=8, Hq=32, d=128, T_cap=4096, k=FAKE, v=FAKE + (1 << 30),
             stride_b=8 * 4096 * 128, stride_h=4096 * 128, stride_t=128)
    c.update(kw)
    return ckv.CacheDesc(**c)


def _graph(**kw):
    g = dict(mode=0, S=4, Cmax=128, max_tail=16, T_cap=4096)
    for i, f in enumerate(["comm_of", "offs", "tok", "cnt", "cent", "cent_q", "cent_qs", "num_comm", "tail_tok",
                           "tail_comm", "tail_len", "dev_err"]):
        g[f] = FAKE + (i + 2) * (1 << 28)
    g.update(kw)
    return ckv.GraphDesc(**g)


def _sel(**kw):
    s = dict(tok_cap=4096)
    for i, f in enumerate(["sel_comm", "n_sel", "sel_tok", "n_tok", "tok_prefix", "tail_sel", "unit_prefix"]):
        s[f] = FAKE + (i + 20) * (1 << 28)
    s.update(kw)
    return ckv.SelectionDesc(**s)


def _ws_size(cache, graph=None, sel=None):
    out = ctypes.c_size_t(0)
    st = ckv.lib.ckv_workspace_size(ctypes.byref(cache), ctypes.byref(graph) if graph else None,
                                    ctypes.byref(sel) if sel else None, ctypes.byref(out))
    return st, out.value


def test_workspace_size_is_host_only_and_monotone():
    st, a = _ws_size(_cache())
    assert st == OK and a > 0
    st, b = _ws_size(_cache(), _graph())
    assert st == OK and b >= a
    st, c = _ws_size(_cache(), _graph(Cmax=1024))
    assert st == OK and c >= b
    st, _ = _ws_size(_cache(d=96))
    assert st == UNSUPPORTED


def _call_build(cache, graph, labels=FAKE, stride=4096, T=4096, ws=FAKE, ws_bytes=1 << 40):
    return ckv.lib.ckv_build_centroids(ctypes.byref(cache), labels, stride, T, ctypes.byref(graph), ws,
                                       ws_bytes, None)


def _call_select(cache, graph, sel, q=FAKE, budget=128, ws=FAKE, ws_bytes=1 << 40):
    return ckv.lib.ckv_score_select(ctypes.byref(cache), ctypes.byref(graph), q, budget, ctypes.byref(sel),
                                    ws, ws_bytes, None)


def _call_decode(cache, graph, sel, q=FAKE, out=FAKE, nbr=FAKE, ws=FAKE, ws_bytes=1 << 40):
    return ckv.lib.ckv_sparse_decode(ctypes.byref(cache), q, ctypes.byref(graph), ctypes.byref(sel), out, nbr,
                                     ws, ws_bytes, None)


def _call_edges(cache, mode=0, S=4, T=4096, q=FAKE, nbr=FAKE, pair_cap=1024, ws=FAKE, ws_bytes=1 << 40):
    return ckv.lib.ckv_build_edges(ctypes.byref(cache), mode, S, q, T, nbr, None, FAKE, FAKE, FAKE, FAKE,
                                   pair_cap, FAKE, ws, ws_bytes, None)


def test_edges_workspace_size_is_host_only():
    out = ctypes.c_size_t(0)
    assert ckv.lib.ckv_edges_workspace_size(ctypes.byref(_cache()), 0, 4, 1000, ctypes.byref(out)) == OK
    small = out.value
    assert ckv.lib.ckv_edges_workspace_size(ctypes.byref(_cache()), 1, 4, 4000, ctypes.byref(out)) == OK
    assert out.value > small > 0
    assert ckv.lib.ckv_edges_workspace_size(ctypes.byref(_cache()), 0, 4, 5000, ctypes.byref(out)) == INVALID


CASES = [
    ("dtype", lambda: _call_build(_cache(dtype=7), _graph()), UNSUPPORTED),
    ("head dim", lambda: _call_build(_cache(d=80), _graph()), UNSUPPORTED),
    ("gqa ratio", lambda: _call_build(_cache(Hq=48), _graph()), UNSUPPORTED),
    ("Hq % Hkv", lambda: _call_build(_cache(Hq=30), _graph()), INVALID),
    ("null K", lambda: _call_build(_cache(k=None), _graph()), INVALID),
    ("misaligned K", lambda: _call_build(_cache(k=FAKE + 8), _graph()), MISALIGNED),
    ("misaligned stride", lambda: _call_build(_cache(stride_t=132), _graph()), MISALIGNED),
    ("graph T_cap", lambda: _call_build(_cache(), _graph(T_cap=2048)), INVALID),
    ("Cmax 0", lambda: _call_build(_cache(), _graph(Cmax=0)), UNSUPPORTED),
    ("Cmax too big", lambda: _call_build(_cache(), _graph(Cmax=100000)), UNSUPPORTED),
    ("graph mode", lambda: _call_build(_cache(), _graph(mode=5)), INVALID),
    ("assign rule", lambda: _call_build(_cache(), _graph(assign_rule=2)), INVALID),
    ("negative assign rule", lambda: ckv.lib.ckv_assign_update(ctypes.byref(_cache()),
                                                              ctypes.byref(_graph(assign_rule=-1)), 5, FAKE, FAKE,
                                                              None), INVALID),
    ("null graph array", lambda: _call_build(_cache(), _graph(cent=None)), INVALID),
    ("null cent_q", lambda: _call_build(_cache(), _graph(cent_q=None)), INVALID),
    ("null cent_qs", lambda: _call_build(_cache(), _graph(cent_qs=None)), INVALID),
    ("misaligned cent_q", lambda: _call_build(_cache(), _graph(cent_q=FAKE + 8)), MISALIGNED),
    ("misaligned cent_qs", lambda: _call_build(_cache(), _graph(cent_qs=FAKE + 4)), MISALIGNED),
    ("too many units", lambda: _call_build(_cache(B=400), _graph(mode=1)), UNSUPPORTED),
    ("null labels", lambda: _call_build(_cache(), _graph(), labels=None), INVALID),
    ("T > T_cap", lambda: _call_build(_cache(), _graph(), T=5000, stride=5000), CAPACITY),
    ("T < S", lambda: _call_build(_cache(), _graph(), T=2), INVALID),
    ("labels stride", lambda: _call_build(_cache(), _graph(), stride=100), INVALID),
    ("build ws small", lambda: _call_build(_cache(), _graph(), ws_bytes=16), WORKSPACE),
    ("build ws null", lambda: _call_build(_cache(), _graph(), ws=None), WORKSPACE),
    ("build ws misaligned", lambda: _call_build(_cache(), _graph(), ws=FAKE + 64), WORKSPACE),
    ("negative budget", lambda: _call_select(_cache(), _graph(), _sel(), budget=-1), INVALID),
    ("null q", lambda: _call_select(_cache(), _graph(), _sel(), q=None), INVALID),
    ("misaligned q", lambda: _call_select(_cache(), _graph(), _sel(), q=FAKE + 4), MISALIGNED),
    ("tok_cap < S", lambda: _call_select(_cache(), _graph(), _sel(tok_cap=2)), INVALID),
    ("null selection array", lambda: _call_select(_cache(), _graph(), _sel(unit_prefix=None)), INVALID),
    ("null run offsets", lambda: _call_select(_cache(), _graph(), _sel(tok_prefix=None)), INVALID),
    ("null tail communities", lambda: _call_decode(_cache(), _graph(), _sel(tail_sel=None)), INVALID),
    ("select ws small", lambda: _call_select(_cache(), _graph(), _sel(), ws_bytes=100), WORKSPACE),
    ("null out", lambda: _call_decode(_cache(), _graph(), _sel(), out=None), INVALID),
    ("misaligned out", lambda: _call_decode(_cache(), _graph(), _sel(), out=FAKE + 4), MISALIGNED),
    ("decode ws small", lambda: _call_decode(_cache(), _graph(), _sel(), ws_bytes=1000), WORKSPACE),
    ("assign pos", lambda: ckv.lib.ckv_assign_update(ctypes.byref(_cache()), ctypes.byref(_graph()), 4096,
                                                     FAKE, FAKE, None), CAPACITY),
    ("assign null nbr", lambda: ckv.lib.ckv_assign_update(ctypes.byref(_cache()), ctypes.byref(_graph()), 5,
                                                          None, FAKE, None), INVALID),
    ("append pos", lambda: ckv.lib.ckv_append_assign(ctypes.byref(_cache()), ctypes.byref(_graph()), -1,
                                                     FAKE, FAKE, FAKE, FAKE, None), CAPACITY),
    ("append null k_new", lambda: ckv.lib.ckv_append_assign(ctypes.byref(_cache()), ctypes.byref(_graph()), 5,
                                                            None, FAKE, FAKE, FAKE, None), INVALID),
    ("append misaligned v_new", lambda: ckv.lib.ckv_append_assign(ctypes.byref(_cache()), ctypes.byref(_graph()),
                                                                  5, FAKE, FAKE + 8, FAKE, FAKE, None), INVALID),
    ("append null nbr", lambda: ckv.lib.ckv_append_assign(ctypes.byref(_cache()), ctypes.byref(_graph()), 5,
                                                          FAKE, FAKE, None, FAKE, None), INVALID),
    ("fused pos", lambda: ckv.lib.ckv_sparse_decode_append(ctypes.byref(_cache()), FAKE, ctypes.byref(_graph()),
                                                           ctypes.byref(_sel()), FAKE, None, 4096, FAKE, FAKE,
                                                           None, FAKE, 1 << 40, None), CAPACITY),
    ("fused null v_new", lambda: ckv.lib.ckv_sparse_decode_append(ctypes.byref(_cache()), FAKE, ctypes.byref(_graph()),
                                                                  ctypes.byref(_sel()), FAKE, None, 5, FAKE, None,
                                                                  None, FAKE, 1 << 40, None), INVALID),
    ("fused ws small", lambda: ckv.lib.ckv_sparse_decode_append(ctypes.byref(_cache()), FAKE, ctypes.byref(_graph()),
                                                                ctypes.byref(_sel()), FAKE, None, 5, FAKE, FAKE,
                                                                None, FAKE, 1000, None), WORKSPACE),
    ("dense T", lambda: ckv.lib.ckv_dense_decode(ctypes.byref(_cache()), FAKE, 0, FAKE, FAKE, 1 << 40, None),
     CAPACITY),
    ("dense ws", lambda: ckv.lib.ckv_dense_decode(ctypes.byref(_cache()), FAKE, 100, FAKE, FAKE, 8, None),
     WORKSPACE),
    ("null cache", lambda: ckv.lib.ckv_dense_decode(None, FAKE, 100, FAKE, FAKE, 1 << 40, None), INVALID),
    ("kernel times null", lambda: ckv.lib.ckv_kernel_times(None, None, 6), INVALID),
    ("kernel times short", lambda: ckv.lib.ckv_kernel_times((ctypes.c_float * 6)(), (ctypes.c_int32 * 6)(), 5),
     INVALID),
    ("device error null graph", lambda: ckv.lib.ckv_get_device_error(None, None, ctypes.byref(ctypes.c_int32()), 0),
     INVALID),
    ("device error null code", lambda: ckv.lib.ckv_get_device_error(ctypes.byref(_graph()), None, None, 0), INVALID),
    ("device error null word", lambda: ckv.lib.ckv_get_device_error(ctypes.byref(_graph(dev_err=None)), None,
                                                                     ctypes.byref(ctypes.c_int32()), 0), INVALID),
    ("edges: fp32 cache", lambda: _call_edges(_cache(dtype=0)), UNSUPPORTED),
    ("edges: T above T_cap", lambda: _call_edges(_cache(), T=5000), CAPACITY),
    ("edges: T below S", lambda: _call_edges(_cache(), S=8, T=4), INVALID),
    ("edges: graph mode", lambda: _call_edges(_cache(), mode=3), INVALID),
    ("edges: null nbr", lambda: _call_edges(_cache(), nbr=None), INVALID),
    ("edges: misaligned q", lambda: _call_edges(_cache(), q=FAKE + 4), MISALIGNED),
    ("edges: pair_cap 0", lambda: _call_edges(_cache(), pair_cap=0), INVALID),
    ("edges: small workspace", lambda: _call_edges(_cache(), ws_bytes=1024), WORKSPACE),
]


@pytest.mark.parametrize("name,call,want", CASES, ids=[c[0] for c in CASES])
def test_host_validation(name, call, want):
    st = call()
    assert st not in (OK, CUDA)
    assert st == want, (name, ckv.ckv_status_string(st), ckv.ckv_last_error())
    assert ckv.ckv_last_error() != ""


def test_python_binding_raises():
    with pytest.raises(ckv.CKVError) as e:
        ckv._check(UNSUPPORTED, "x")
    assert e.value.status == UNSUPPORTED


def test_kernel_timing_is_host_side_until_used():
    """Turning timing on and off and reading an empty record touch no device."""
    assert ckv.lib.ckv_kernel_timing(1) == 0 and ckv.lib.ckv_kernel_timing(0) == 0
    times = ckv.ckv_kernel_times()
    assert list(times) == list(ckv.KERNEL_KINDS) and all(v == (0.0, 0) for v in times.values())
    hdr = open(HEADER).read()
    assert int(re.search(r"#define CKV_KERNEL_KINDS (\d+)", hdr).group(1)) == len(ckv.KERNEL_KINDS)
