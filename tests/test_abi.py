"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, its host-only arithmetic matches the oracle's definitions,
and argument validation rejects bad calls before anything is enqueued."""
from __future__ import annotations

import ctypes as C
import os
import re

import numpy as np
import pytest

import oracle
import mixed_length_paged_b200 as hpa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hpa.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*HPA_API\s+(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(hpa_[a-z0-9_]+)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    from mixed_length_paged_b200 import build
    build.build()
    return hpa.lib()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ["hpa_decode_plan", "hpa_decode_run", "hpa_kv_prologue",
              "hpa_decode_workspace_size", "hpa_default_num_ctas", "hpa_status_string",
              "hpa_plan_grid", "hpa_workspace_layout", "hpa_read_status"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    missing = [n for n in _declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_only_declared_symbols_are_exported(L):
    out = os.popen(f"nm -D --defined-only {hpa.library_path}").read()
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    ours = {s for s in exported if s.startswith("hpa_")}
    assert ours == set(_declared_functions())


def test_status_strings(L):
    for code, name in [(0, b"HPA_OK"), (1, b"HPA_ERR_INVALID_ARG"), (2, b"HPA_ERR_UNSUPPORTED"),
                       (3, b"HPA_ERR_WORKSPACE"), (4, b"HPA_ERR_CUDA")]:
        assert L.hpa_status_string(code) == name
    assert L.hpa_version() == 100


@pytest.mark.parametrize("kind", [0, 1, 2, 3])
@pytest.mark.parametrize("B,Hkv,P,param,maxlen", [
    (32, 8, 148, 0, 131072), (64, 8, 148, 0, 512), (2, 2, 148, 0, 200), (2, 2, 148, 3, 200),
    (5, 4, 7, 5, 65), (1, 1, 1, 0, 1), (256, 8, 148, 0, 16384), (3, 2, 5, 0, 0),
])
def test_plan_grid_matches_oracle(L, kind, B, Hkv, P, param, maxlen):
    assert hpa.plan_grid(kind, B, Hkv, P, param, maxlen) == \
        oracle.plan_grid(kind, B, Hkv, P, param, maxlen)


def test_workspace_layout_is_aligned_and_ordered(L):
    for kind, args in [(0, (32, 8, 64, 128, 148)), (1, (2, 2, 8, 64, 148)),
                       (2, (256, 8, 64, 128, 4864)), (3, (32, 8, 64, 128, 148))]:
        lay = hpa.workspace_layout(kind, *args)
        offs = [lay[k] for k in ["header", "lens", "tile_start", "cta_desc", "seg_desc",
                                 "part_ml", "part_acc", "total"]]
        assert all(o % 256 == 0 for o in offs)
        assert offs == sorted(offs)
        B, Hkv, Hq, D, grid = args
        G = Hq // Hkv
        V = 5 * grid if kind == 0 else grid  # dynamic: primary ranges + tail chunks
        assert lay["part_acc"] - lay["part_ml"] >= 2 * V * G * 8
        assert lay["total"] - lay["part_acc"] >= 2 * V * G * D * 4
        assert lay["cta_desc"] - lay["tile_start"] >= (B + 1) * 4
        assert lay["seg_desc"] - lay["cta_desc"] >= 32 * V
        assert lay["part_ml"] - lay["seg_desc"] >= 8 * B * Hkv
        assert hpa.decode_workspace_size(kind, *args) == lay["total"]
    assert L.hpa_decode_workspace_size(0, 0, 8, 64, 128, 148) == 0
    assert L.hpa_decode_workspace_size(0, 2, 3, 8, 64, 148) == 0  # Hq % Hkv != 0
    assert L.hpa_decode_workspace_size(7, 2, 2, 8, 64, 148) == 0  # unknown plan kind


def _plan(L, **kw):
    a = dict(seq_lens=1, batch=2, num_kv_heads=2, num_q_heads=8, head_dim=64, pt_stride=4,
             kind=0, num_ctas=148, param=0, max_seq_len=0, workspace=256, ws_bytes=1 << 20)
    a.update(kw)
    g = C.c_int(-7)
    rc = L.hpa_decode_plan(a["seq_lens"], a["batch"], a["num_kv_heads"], a["num_q_heads"],
                           a["head_dim"], a["pt_stride"], a["kind"], a["num_ctas"], a["param"],
                           a["max_seq_len"], a["workspace"], a["ws_bytes"], C.byref(g), None)
    return rc, g.value


@pytest.mark.parametrize("bad,expect", [
    (dict(seq_lens=None), 1), (dict(workspace=None), 1), (dict(batch=0), 1),
    (dict(num_kv_heads=0), 1), (dict(num_q_heads=7), 1), (dict(pt_stride=0), 1),
    (dict(num_ctas=0), 1), (dict(kind=4), 1), (dict(param=-1), 1), (dict(ws_bytes=16), 3),
    (dict(workspace=256 + 8), 3),
    (dict(batch=32769), 2),  # more sequences than one plan holds
    (dict(num_ctas=65537), 2),  # dynamic plans over at most 65536 CTAs
    (dict(kind=3, num_ctas=65537), 2),
    (dict(kind=3, param=(1 << 20) + 1), 2),  # smallest end piece at most 2^20 tiles
])
def test_plan_rejects_bad_arguments_without_launching(L, bad, expect):
    rc, grid = _plan(L, **bad)
    assert rc == expect
    assert grid == -7  # nothing reported, nothing enqueued


def _plan_shape(L, **kw):
    a = dict(seq_lens=1, batch=2, num_kv_heads=2, num_q_heads=8, head_dim=64, pt_stride=4,
             kind=0, num_ctas=148, param=0, tail_den=8, tail_chunks=4, tail_min=32,
             unit_cost=1, end_cost=0, workspace=256, ws_bytes=1 << 20)
    a.update(kw)
    g = C.c_int(-7)
    rc = L.hpa_decode_plan_shape(a["seq_lens"], a["batch"], a["num_kv_heads"], a["num_q_heads"],
                                 a["head_dim"], a["pt_stride"], a["kind"], a["num_ctas"],
                                 a["param"], a["tail_den"], a["tail_chunks"], a["tail_min"],
                                 a["unit_cost"], a["end_cost"], a["workspace"], a["ws_bytes"],
                                 C.byref(g), None)
    return rc, g.value


@pytest.mark.parametrize("bad,expect", [
    (dict(kind=1), 1), (dict(kind=2), 1),           # the static kinds have no tail
    (dict(tail_den=-1), 1), (dict(tail_den=(1 << 20) + 1), 1),
    (dict(tail_chunks=0), 1), (dict(tail_chunks=hpa.TAIL_CHUNKS_MAX + 1), 1),
    (dict(tail_den=0, tail_chunks=0), 1), (dict(tail_min=-1), 1), (dict(tail_min=(1 << 20) + 1), 1),
    (dict(seq_lens=None), 1), (dict(ws_bytes=16), 3), (dict(num_ctas=65537), 2),
    (dict(unit_cost=0), 1), (dict(unit_cost=hpa.COST_MAX + 1), 1), (dict(end_cost=-1), 1),
    (dict(end_cost=hpa.COST_MAX + 1), 1), (dict(unit_cost=-2, end_cost=3), 1),
])
def test_plan_shape_rejects_bad_arguments_without_launching(L, bad, expect):
    rc, grid = _plan_shape(L, **bad)
    assert rc == expect
    assert grid == -7


def test_plan_shape_defaults_match_the_header():
    src = open(HEADER).read()
    for name, val in [("HPA_TAIL_DEN_DEFAULT", hpa.TAIL_DEN_DEFAULT),
                      ("HPA_TAIL_CHUNKS_DEFAULT", hpa.TAIL_CHUNKS_DEFAULT),
                      ("HPA_TAIL_MIN_DEFAULT", hpa.TAIL_MIN_DEFAULT),
                      ("HPA_TAIL_CHUNKS_MAX", hpa.TAIL_CHUNKS_MAX),
                      ("HPA_COST_UNIT_DEFAULT", hpa.COST_UNIT_DEFAULT),
                      ("HPA_COST_END_DEFAULT", hpa.COST_END_DEFAULT),
                      ("HPA_COST_END_DEFAULT_FP8", hpa.COST_END_DEFAULT_FP8),
                      ("HPA_COST_MAX", hpa.COST_MAX)]:
        assert re.search(rf"#define {name} {val}\b", src), name


def _run(L, **kw):
    a = dict(q=256, k=256, v=256, ks=None, vs=None, kvd=0, pt=256, pts=4, pages=8, out=256,
             outd=0, B=2, Hq=8, Hkv=2, D=64, scale=0.125, kind=0, grid=148, ws=256, wsb=1 << 24)
    a.update(kw)
    return L.hpa_decode_run(a["q"], a["k"], a["v"], a["ks"], a["vs"], a["kvd"], a["pt"], a["pts"],
                            a["pages"], a["out"], a["outd"], a["B"], a["Hq"], a["Hkv"], a["D"],
                            C.c_float(a["scale"]), a["kind"], a["grid"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("bad,expect", [
    (dict(q=None), 1), (dict(k=None), 1), (dict(out=None), 1), (dict(ws=None), 1),
    (dict(B=0), 1), (dict(Hq=6, Hkv=4), 1), (dict(kvd=5), 1), (dict(outd=2), 1),
    (dict(scale=0.0), 1), (dict(scale=float("nan")), 1), (dict(kvd=1), 1),  # fp8 w/o scales
    (dict(Hq=66, Hkv=2), 2),   # G = 33: more rows than four MMA n-tiles
    (dict(Hq=128, Hkv=2), 2),  # G = 64
    (dict(D=96), 2), (dict(D=256), 2), (dict(kvd=1, ks=256, vs=256), 2),  # fp8 needs D = 128
    (dict(pages=1 << 26, Hkv=8, Hq=8), 2),  # rows overflow int32 TMA coordinates
    (dict(k=256 + 8), 1), (dict(q=256 + 2), 1), (dict(q=256 + 8), 1), (dict(out=256 + 2), 1),
    (dict(wsb=64), 3), (dict(ws=256 + 16), 3), (dict(kind=9), 1),
])
def test_run_rejects_bad_arguments_without_launching(L, bad, expect):
    assert _run(L, **bad) == expect


def _run_multi(L, **kw):
    a = dict(q=256, k=256, v=256, ks=None, vs=None, kvd=0, pt=256, pts=4, pages=8, out=256,
             outd=0, B=2, T=2, Hq=8, Hkv=2, D=64, scale=0.125, kind=0, grid=148, ws=256,
             wsb=1 << 24)
    a.update(kw)
    return L.hpa_decode_run_multi(a["q"], a["k"], a["v"], a["ks"], a["vs"], a["kvd"], a["pt"],
                                  a["pts"], a["pages"], a["out"], a["outd"], a["B"], a["T"],
                                  a["Hq"], a["Hkv"], a["D"], C.c_float(a["scale"]), a["kind"],
                                  a["grid"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("bad,expect", [
    (dict(T=0), 1), (dict(T=-3), 1), (dict(T=17, Hq=2, Hkv=2), 2),
    (dict(T=5, Hq=64, Hkv=8), 2),    # G * T = 40 rows > 32
    (dict(T=3, Hq=16, Hkv=1), 2),    # G = 16: room for two tokens, not three
    (dict(T=2, Hq=32, Hkv=1), 2),    # G = 32: no room for a second token
    (dict(q=None), 1), (dict(q=256 + 8), 1), (dict(wsb=64), 3), (dict(kind=9), 1),
])
def test_run_multi_rejects_bad_arguments_without_launching(L, bad, expect):
    assert _run_multi(L, **bad) == expect


def test_multi_token_workspace_counts_rows_of_all_tokens(L):
    # a 4-token step of G = 2 needs the workspace of G * T = 8 rows per kv head
    assert hpa.decode_workspace_size(0, 32, 8, 16 * 4, 128, 296) == \
        hpa.decode_workspace_size(0, 32, 8, 64, 128, 296)
    assert _run_multi(L, T=4, Hq=4, Hkv=2,
                      wsb=hpa.decode_workspace_size(0, 2, 2, 4, 64, 148)) == 3  # sized for T=1


def _run_pro(L, **kw):
    a = dict(qr=256, kr=256, vr=256, gq=256, gk=256, eps=1e-6, theta=1e4, kc=256, vc=256, qo=None,
             pt=256, pts=4, pages=8, out=256, outd=0, B=2, Hq=8, Hkv=2, D=64, scale=0.125,
             kind=0, grid=148, ws=256, wsb=1 << 24)
    a.update(kw)
    return L.hpa_decode_run_prologue(
        a["qr"], a["kr"], a["vr"], a["gq"], a["gk"], C.c_float(a["eps"]), C.c_float(a["theta"]),
        a["kc"], a["vc"], a["qo"], a["pt"], a["pts"], a["pages"], a["out"], a["outd"], a["B"],
        a["Hq"], a["Hkv"], a["D"], C.c_float(a["scale"]), a["kind"], a["grid"], a["ws"], a["wsb"],
        None)


@pytest.mark.parametrize("bad,expect", [
    (dict(qr=None), 1), (dict(kr=None), 1), (dict(vr=None), 1), (dict(gq=None), 1),
    (dict(gk=None), 1), (dict(kc=None), 1), (dict(out=None), 1), (dict(ws=None), 1),
    (dict(kr=256 + 8), 1), (dict(vr=256 + 4), 1), (dict(qr=256 + 8), 1), (dict(qo=256 + 1), 1),
    (dict(eps=-1.0), 1), (dict(eps=float("inf")), 1), (dict(theta=0.0), 1),
    (dict(theta=float("nan")), 1), (dict(scale=0.0), 1), (dict(D=96), 2),
    (dict(Hq=34, Hkv=2), 2),  # G = 17: the fused prologue takes at most 16 rows per kv head
    (dict(wsb=64), 3), (dict(kind=9), 1),
])
def test_run_prologue_rejects_bad_arguments_without_launching(L, bad, expect):
    assert _run_pro(L, **bad) == expect


def _prologue(L, **kw):
    a = dict(qr=256, kr=256, vr=256, gq=256, gk=256, eps=1e-6, theta=1e4, pos=256, pt=256, pts=4,
             kc=256, vc=256, qo=256, B=2, Hq=8, Hkv=2, D=64, pages=8, status=None)
    a.update(kw)
    return L.hpa_kv_prologue(a["qr"], a["kr"], a["vr"], a["gq"], a["gk"], C.c_float(a["eps"]),
                             C.c_float(a["theta"]), a["pos"], a["pt"], a["pts"], a["kc"], a["vc"],
                             a["qo"], a["B"], a["Hq"], a["Hkv"], a["D"], a["pages"], a["status"],
                             None)


@pytest.mark.parametrize("bad,expect", [
    (dict(qr=None), 1), (dict(gk=None), 1), (dict(pos=None), 1), (dict(B=0), 1),
    (dict(Hq=7), 1), (dict(eps=-1.0), 1), (dict(theta=0.0), 1), (dict(theta=float("inf")), 1),
    (dict(D=80), 2),
])
def test_prologue_rejects_bad_arguments_without_launching(L, bad, expect):
    assert _prologue(L, **bad) == expect


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(hpa, "_lib", None)
    monkeypatch.setattr(hpa, "library_path", "/nonexistent/libhpa.so")
    with pytest.raises(hpa.HpaLibraryMissing):
        hpa.lib()
    with pytest.raises(hpa.HpaLibraryMissing):
        hpa.decode_workspace_size(0, 2, 2, 8, 64, 148)


def test_product_path_does_not_reference_the_oracle():
    pkg = os.path.join(ROOT, "mixed_length_paged_b200")
    for dirpath, _, files in os.walk(pkg):
        if "_build" in dirpath:
            continue
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "liboracle" not in text, f


def test_decode_num_ctas_rejects_bad_geometry(L):
    assert L.hpa_decode_num_ctas(0, 0, 8, 1) == -1
    assert L.hpa_decode_num_ctas(0, 64, 0, 1) == -1
    assert L.hpa_decode_num_ctas(0, 64, 8, 0) == -1
    assert L.hpa_decode_num_ctas(0, 60, 8, 1) == -1  # Hq not a multiple of Hkv
    assert L.hpa_decode_num_ctas(0, 64, 8, 5) == -1  # 40 rows per kv head
    assert L.hpa_decode_num_ctas(0, 33, 1, 1) == -1


def test_num_ctas_environment_override():
    # runs in a child process: the override is read from the environment at
    # each call, and this needs no GPU
    import subprocess
    import sys
    code = ("import mixed_length_paged_b200 as h; L = h.lib(); "
            "print(L.hpa_default_num_ctas(0), L.hpa_decode_num_ctas(0, 64, 8, 2))")
    for val, want in (("77", "77 77"), ("1", "1 1")):
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                           env={**os.environ, "HPA_NUM_CTAS": val},
                           cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        assert r.stdout.split() == want.split(), r.stderr


def _step_call(L, **kw):
    a = dict(sl=256, q=256, k=256, v=256, ks=None, vs=None, kvd=0, pt=256, pts=4, pages=8,
             out=256, outd=0, B=2, T=1, Hq=8, Hkv=2, D=64, scale=0.125, n=148, ws=256,
             wsb=1 << 24)
    a.update(kw)
    return L.hpa_decode_step(a["sl"], a["q"], a["k"], a["v"], a["ks"], a["vs"], a["kvd"], a["pt"],
                             a["pts"], a["pages"], a["out"], a["outd"], a["B"], a["T"], a["Hq"],
                             a["Hkv"], a["D"], C.c_float(a["scale"]), a["n"], a["ws"], a["wsb"],
                             None)


@pytest.mark.parametrize("bad,expect", [
    (dict(sl=None), 1), (dict(q=None), 1), (dict(B=0), 1), (dict(n=0), 1),
    (dict(B=513), 2),                  # tile offsets of at most 512 sequences in shared memory
    (dict(n=65537), 2), (dict(T=5, Hq=64, Hkv=8), 2), (dict(wsb=64), 3), (dict(D=96), 2),
])
def test_step_rejects_bad_arguments_without_launching(L, bad, expect):
    assert _step_call(L, **bad) == expect


def test_step_prologue_rejects_bad_arguments_without_launching(L):
    def call(**kw):
        a = dict(sl=256, qr=256, kr=256, vr=256, gq=256, gk=256, eps=1e-6, theta=1e4, kc=256,
                 vc=256, qo=None, pt=256, pts=4, pages=8, out=256, outd=0, B=2, Hq=8, Hkv=2, D=64,
                 scale=0.125, n=148, ws=256, wsb=1 << 24)
        a.update(kw)
        return L.hpa_decode_step_prologue(
            a["sl"], a["qr"], a["kr"], a["vr"], a["gq"], a["gk"], C.c_float(a["eps"]),
            C.c_float(a["theta"]), a["kc"], a["vc"], a["qo"], a["pt"], a["pts"], a["pages"],
            a["out"], a["outd"], a["B"], a["Hq"], a["Hkv"], a["D"], C.c_float(a["scale"]), a["n"],
            a["ws"], a["wsb"], None)
    assert call(sl=None) == 1
    assert call(kr=None) == 1
    assert call(eps=-1.0) == 1
    assert call(B=513) == 2
    assert call(n=65537) == 2
    assert call(wsb=64) == 3


def test_step_lse_rejects_bad_arguments_without_launching(L):
    def call(lse=256, **kw):
        a = dict(sl=256, q=256, k=256, v=256, ks=None, vs=None, kvd=0, pt=256, pts=4, pages=8,
                 out=256, outd=1, B=2, T=1, Hq=8, Hkv=2, D=64, scale=0.125, n=148, ws=256,
                 wsb=1 << 24)
        a.update(kw)
        return L.hpa_decode_step_lse(a["sl"], a["q"], a["k"], a["v"], a["ks"], a["vs"], a["kvd"],
                                     a["pt"], a["pts"], a["pages"], a["out"], a["outd"], lse,
                                     a["B"], a["T"], a["Hq"], a["Hkv"], a["D"],
                                     C.c_float(a["scale"]), a["n"], a["ws"], a["wsb"], None)
    assert call(lse=None) == 1          # the log-sum-exps are the point of the call
    assert call(lse=258) == 1           # fp32, 4-byte aligned
    assert call(sl=None) == 1
    assert call(B=513) == 2
    assert call(D=96) == 2
    assert call(wsb=64) == 3


def test_merge_states_rejects_bad_arguments_without_launching(L):
    def call(n=2, parts=None, lparts=None, rows=10, D=128, out=256, outd=1, lse_out=None):
        o = (C.c_void_p * max(n, 1))(*([256] * max(n, 1))) if parts is None else parts
        l = (C.c_void_p * max(n, 1))(*([512] * max(n, 1))) if lparts is None else lparts
        return L.hpa_merge_states(o, l, n, rows, D, out, outd, lse_out, None)
    assert call(n=0) == 1
    assert call(n=17) == 2                          # at most 16 states per call
    assert call(D=96) == 2
    assert call(rows=-1) == 1
    assert call(outd=7) == 1
    assert call(out=None) == 1
    assert call(parts=(C.c_void_p * 2)(256, None)) == 1
    assert call(parts=(C.c_void_p * 2)(256, 264)) == 1      # o parts 16-byte aligned
    assert call(lparts=(C.c_void_p * 2)(512, 514)) == 1     # lse parts 4-byte aligned
    assert call(out=264, outd=1) == 1               # fp32 out: 16-byte aligned
    assert call(out=260, outd=0) == 1               # bf16 out: 8-byte aligned
    assert call(lse_out=258) == 1
    assert L.hpa_merge_states(None, None, 1, 1, 128, 256, 1, None, None) == 1
    # no rows: nothing to enqueue, so this succeeds without a GPU
    assert call(rows=0) == 0


def test_length_aware_workspace_equals_dynamic(L):
    # the length-aware plan has the dynamic plan's ranges, grid and tail, so
    # its workspace is laid out the same way
    for args in [(32, 8, 64, 128, 296), (1, 1, 8, 64, 7), (512, 8, 64, 128, 296)]:
        assert hpa.decode_workspace_size(3, *args) == hpa.decode_workspace_size(0, *args)
        assert hpa.workspace_layout(3, *args) == hpa.workspace_layout(0, *args)


def test_read_cta_times_rejects_bad_arguments(L):
    buf = (C.c_uint64 * 8)()
    assert L.hpa_read_cta_times(None, 0, 2, 2, 8, 64, 2, buf, None) == 1
    assert L.hpa_read_cta_times(256, 0, 2, 2, 8, 64, 2, None, None) == 1
    assert L.hpa_read_cta_times(256, 0, 0, 2, 8, 64, 2, buf, None) == 1   # batch 0
    assert L.hpa_read_cta_times(256, 9, 2, 2, 8, 64, 2, buf, None) == 1   # unknown kind


def test_workspace_has_room_for_the_cta_trace(L):
    # the trace region (grid x 4 uint64) sits after the partials
    for grid in (1, 148, 296, 4864):
        lay = hpa.workspace_layout(0, 32, 8, 64, 128, grid)
        assert lay["total"] - lay["part_acc"] >= 2 * 5 * grid * 8 * 128 * 4 + grid * 32
