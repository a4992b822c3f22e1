"""The C-ABI library loads and exports every symbol include/am_b200.h
declares; host-side argument errors come back synchronously (no GPU needed:
each of these returns before the first CUDA call)."""
import ctypes
import os
import re

import pytest

import attention_matching_b200 as am

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "am_b200.h")


def declared_functions():
    src = open(HDR).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(am_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert "am_compact_heads" in names and len(names) >= 6
    L = am.lib()
    for n in names:
        assert hasattr(L, n), n


@pytest.mark.parametrize("cname,mirror", [("am_opts_t", "AmOpts"), ("am_workspace_view_t", "AmWorkspaceView")])
def test_struct_layout_matches_header(tmp_path, cname, mirror):
    """Each ctypes mirror has the size and field offsets a C compiler gives
    the header's struct."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    cls = getattr(am, mirror)
    fields = [f[0] for f in cls._fields_]
    src = tmp_path / "layout.c"
    src.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"am_b200.h\"\n"
                   f"int main(void) {{\n  printf(\"%zu\\n\", sizeof({cname}));\n"
                   + "".join(f"  printf(\"%zu\\n\", offsetof({cname}, {f}));\n" for f in fields)
                   + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    include = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run([cc, "-std=c99", "-I", include, str(src), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], check=True, capture_output=True,
                                          text=True).stdout.split()]
    assert got[0] == ctypes.sizeof(cls)
    assert got[1:] == [getattr(cls, f).offset for f in fields]


def test_defaults_and_status_strings():
    o = am.make_opts()
    assert (o.in_dtype, o.topk, o.refit_every) == (am.BF16, 1, 1)
    assert abs(o.ridge - 1e-6) < 1e-12 and abs(o.w_floor_rel - 1e-12) < 1e-18
    L = am.lib()
    for code in range(11):
        assert L.am_status_string(code)
    assert L.am_version() >= 100


def test_workspace_size_scales_with_features():
    o = am.make_opts(am.BF16, 4, 2)
    a = am.workspace_size(8192, 8192, 128, [164] * 8, o)
    assert a >= 8 * 8192 * 8192 * 4
    assert am.workspace_size(1000, 1100, 128, [13, 22, 8], o) < a


@pytest.mark.parametrize("bad", [
    dict(budgets=[0]), dict(budgets=[301]), dict(topk=0), dict(refit_every=0),
    dict(topk=16, refit_every=8), dict(d=300), dict(ridge=-1.0), dict(w_floor_rel=0.0),
    dict(T=4096, budgets=[2049]),
])
def test_workspace_size_rejects(bad):
    args = dict(n=512, T=300, d=64, budgets=[16], topk=1, refit_every=1, ridge=1e-6, w_floor_rel=1e-12)
    args.update(bad)
    o = am.make_opts(am.FP32, args["topk"], args["refit_every"], ridge=args["ridge"],
                     w_floor_rel=args["w_floor_rel"])
    with pytest.raises(am.AmError):
        am.workspace_size(args["n"], args["T"], args["d"], args["budgets"], o)


def _call(**over):
    L = am.lib()
    o = am.make_opts(am.FP32)
    H, n, T, d = 1, 64, 32, 16
    budgets = (ctypes.c_int32 * H)(4)
    offs = (ctypes.c_int64 * (H + 1))(0, 4)
    args = dict(Q=1 << 20, K=1 << 21, V=1 << 22, n=n, T=T, d=d, H=H, budgets=budgets, opts=ctypes.byref(o),
                ws=None, ws_bytes=0, offs=offs, Ck=1 << 23, beta=1 << 24, Cv=1 << 25, idx=1 << 26)
    args.update(over)
    return L.am_compact_heads(args["Q"], args["K"], args["V"], args["n"], args["T"], args["d"], args["H"],
                              args["budgets"], args["opts"], args["ws"], args["ws_bytes"], args["offs"],
                              args["Ck"], args["beta"], args["Cv"], args["idx"], None)


def test_compact_heads_argument_errors_are_synchronous():
    assert _call(Q=None) == 1                       # null input
    assert _call(n=0) == 1                          # bad size
    bad_budget = (ctypes.c_int32 * 1)(33)
    assert _call(budgets=bad_budget) == 2           # budget > T
    bad_offs = (ctypes.c_int64 * 2)(0, 5)
    assert _call(offs=bad_offs) == 1                # offsets disagree with budgets
    assert _call(ws=None) == 3                      # no workspace
    assert _call(ws=4096 + 8, ws_bytes=1 << 30) == 3  # misaligned workspace
    assert _call(ws=4096, ws_bytes=16) == 3          # too small


def test_attend_packed_argument_errors():
    """am_attend_packed rejects missing buffers and unsupported sizes before
    any GPU work."""
    L = am.lib()
    v = ctypes.c_void_p(16)
    args = dict(Q=v, nq=4, d=64, H=2, dt=am.BF16, Ck=v, beta=v, Cv=v, cu=v, Kn=None, Vn=None, Tn=0,
                scale=ctypes.c_float(0.0), out=v, stream=None)

    def call(**kw):
        a = dict(args, **kw)
        return L.am_attend_packed(a["Q"], a["nq"], a["d"], a["H"], a["dt"], a["Ck"], a["beta"], a["Cv"],
                                  a["cu"], a["Kn"], a["Vn"], a["Tn"], a["scale"], a["out"], a["stream"])

    code = {v: k for k, v in am.STATUS.items()}
    assert call(Q=None) == code["AM_ERR_INVALID_ARG"]
    assert call(Tn=5) == code["AM_ERR_INVALID_ARG"]          # fresh keys without buffers
    assert call(d=300) == code["AM_ERR_UNSUPPORTED"]
    assert call(dt=7) == code["AM_ERR_INVALID_ARG"]
    assert call(nq=0) == code["AM_ERR_INVALID_ARG"]


@pytest.mark.parametrize("n,T,d,budgets,select", [
    (512, 256, 64, [16], 0), (1000, 1100, 128, [13, 22, 8], 0), (8192, 8192, 128, [164] * 8, 0),
    (700, 900, 128, [70, 45], 1), (33, 1, 16, [1], 0),
])
def test_workspace_view_regions_fit_align_and_do_not_overlap(n, T, d, budgets, select):
    """The feature regions and call statistics am_workspace_view reports lie
    inside the size am_workspace_size asks for, start 16-byte aligned and are
    disjoint."""
    dt = am.BF16 if d in (64, 128) else am.FP32
    o = am.make_opts(dt, 4, 2, select_mode=select)
    size = am.workspace_size(n, T, d, budgets, o)
    v = am.AmWorkspaceView()
    H, S = len(budgets), sum(budgets)
    arr = (ctypes.c_int32 * H)(*budgets)
    assert am.lib().am_workspace_view(n, T, d, H, arr, ctypes.byref(o), ctypes.byref(v)) == 0
    ldn = v.ldn
    assert ldn % 32 == 0 and ldn >= n
    regions = [(v.phiT, H * T * ldn * 4), (v.mass, H * ldn * 8), (v.target, H * n * d * 4), (v.shift, H * 4),
               (v.weights, S * 8), (v.resid, H * ldn * 4), (v.rows_evaluated, H * 8),
               (v.column_norms, H * T * 8), (v.nnls_refits, H * 4), (v.nnls_solves, H * 4)]
    for off, sz in regions:
        assert off % 16 == 0 and off + sz <= size, (off, sz, size)
    spans = sorted(regions)
    for (a, sa), (b, _) in zip(spans, spans[1:]):
        assert a + sa <= b, (a, sa, b)


def test_highest_attention_mode_argument_rules():
    """Highest-attention selection ignores topk and refit_every (a k·R the
    OMP path rejects is accepted) and needs T <= 16384 for its per-head sort."""
    code = {v: k for k, v in am.STATUS.items()}
    ok = am.make_opts(am.BF16, 64, 64, select_mode=am.SELECT_HIGHEST)
    assert am.workspace_size(512, 4096, 128, [100, 200], ok) > 0
    with pytest.raises(am.AmError) as e:
        am.workspace_size(512, 4096, 128, [100], am.make_opts(am.BF16, 64, 64))
    assert e.value.code == code["AM_ERR_UNSUPPORTED"]
    with pytest.raises(am.AmError) as e:
        am.workspace_size(512, 20000, 128, [100], ok)
    assert e.value.code == code["AM_ERR_UNSUPPORTED"]
    with pytest.raises(am.AmError) as e:
        am.workspace_size(512, 4096, 128, [100], am.make_opts(am.BF16, 4, 2, select_mode=5))
    assert e.value.code == code["AM_ERR_INVALID_ARG"]


def _opts_with_offsets(offsets, dtype=None):
    o = am.make_opts(am.BF16 if dtype is None else dtype, 8, 2)
    arr = (ctypes.c_int64 * len(offsets))(*offsets)
    o.key_offsets = ctypes.cast(arr, ctypes.c_void_p)
    return o, arr


def test_key_offsets_argument_rules():
    """Per-head key counts: offsets start at 0 and grow by at least one key,
    the largest count equals T, and each budget fits its own head."""
    code = {v: k for k, v in am.STATUS.items()}
    o, keep = _opts_with_offsets([0, 1024, 2048, 2500])
    assert am.workspace_size(768, 1024, 128, [103, 103, 46], o) > 0
    for offs, T, budgets, want in [
        ([1, 1024, 2048, 2500], 1024, [10, 10, 10], "AM_ERR_INVALID_ARG"),    # does not start at 0
        ([0, 1024, 1024, 2500], 1476, [10, 10, 10], "AM_ERR_INVALID_ARG"),    # an empty head
        ([0, 1024, 2048, 2500], 2048, [10, 10, 10], "AM_ERR_INVALID_ARG"),    # T is not the largest count
        ([0, 1024, 2048, 2500], 1024, [10, 10, 453], "AM_ERR_BUDGET"),        # t above the head's 452 keys
    ]:
        o, keep = _opts_with_offsets(offs)
        with pytest.raises(am.AmError) as e:
            am.workspace_size(768, T, 128, budgets, o)
        assert e.value.code == code[want], (offs, T, budgets)


def test_wave_workspace_sizes():
    """Waves of consecutive heads: one wave of every head is the ordinary
    workspace; smaller waves need less, never less than the largest single
    head, and the size grows with the wave."""
    o = am.make_opts(am.BF16, 8, 2)
    budgets = [819] * 7 + [266]
    offs = [0]
    for h in range(8):
        offs.append(offs[-1] + (8192 if h < 7 else 2656))
    o, keep = _opts_with_offsets(offs)
    full = am.workspace_size(8192, 8192, 128, budgets, o)
    assert am.workspace_size(8192, 8192, 128, budgets, o, wave_heads=8) == full
    assert am.workspace_size(8192, 8192, 128, budgets, o, wave_heads=100) == full
    sizes = [am.workspace_size(8192, 8192, 128, budgets, o, wave_heads=w) for w in (1, 2, 4, 8)]
    assert sizes == sorted(sizes) and sizes[0] < sizes[1] < sizes[3]
    assert sizes[0] >= 8192 * 8192 * 4        # one head's stored features
    assert sizes[1] < 3 * 8192 * 8192 * 4     # two heads' worth, not eight


def test_workspace_below_one_head_is_rejected_before_any_work():
    """A workspace that cannot hold one head's wave is refused synchronously."""
    o = am.make_opts(am.FP32)
    one = am.workspace_size(64, 32, 16, [4], o)
    assert _call(ws=4096, ws_bytes=one - 4096) == 3
