"""fp64 CPU oracle for paged mixed-length decode attention (ctypes binding).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg import this package; the CUDA library and its Python binding
never do.  The arithmetic lives in ``oracle.c`` (plain fp64 loops, each
function citing the passage it follows); this module only marshals numpy
arrays.  Arrays of dtype uint16 are bf16 bit patterns; uint8 are e4m3 codes.

Every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` against closed forms, library routines and
brute force, not against itself.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = C.CDLL(path)
        _declare(_lib)
    return _lib


_P = C.c_void_p
_I = C.c_int
_L = C.c_long
_D = C.c_double


def _declare(L):
    L.oracle_bf16_to_f64.restype = _D
    L.oracle_bf16_to_f64.argtypes = [C.c_uint16]
    L.oracle_bf16_from_f64.restype = C.c_uint16
    L.oracle_bf16_from_f64.argtypes = [_D]
    L.oracle_e4m3_decode.restype = _D
    L.oracle_e4m3_decode.argtypes = [C.c_uint8]
    L.oracle_e4m3_encode.restype = C.c_uint8
    L.oracle_e4m3_encode.argtypes = [_D]
    L.oracle_quantize_kv_e4m3.restype = None
    L.oracle_quantize_kv_e4m3.argtypes = [_P, _P, _I, _I, _I, _I, C.c_uint8, _P, _P]
    L.oracle_rmsnorm.restype = None
    L.oracle_rmsnorm.argtypes = [_P, _P, _I, _D, _P]
    L.oracle_rope.restype = None
    L.oracle_rope.argtypes = [_P, _I, _D, _D, _P]
    L.oracle_prologue.restype = _I
    L.oracle_prologue.argtypes = [_P, _P, _P, _P, _P, _D, _D, _P, _P, _I, _P, _P, _P,
                                  _I, _I, _I, _I, _I, _I]
    L.oracle_paged_decode_multi.restype = _I
    L.oracle_paged_decode_multi.argtypes = [_P, _P, _P, _P, _I, _P, _P, _P, _I, _P, _I, _I, _I,
                                            _I, _I, _I, _I, _D, _P, _I, _P, _I]
    L.oracle_paged_decode.restype = _I
    L.oracle_paged_decode.argtypes = [_P, _P, _P, _P, _I, _P, _P, _P, _I, _P, _I, _I, _I, _I,
                                      _I, _I, _D, _P, _I, _P, _I]
    L.oracle_partial.restype = _I
    L.oracle_partial.argtypes = [_P, _P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _I, _D,
                                 _I, _I, _L, _L, _P, _P, _P]
    L.oracle_lse_merge.restype = None
    L.oracle_lse_merge.argtypes = [_P, _P, _P, _I, _I, _P]
    L.oracle_plan_grid.restype = _L
    L.oracle_plan_grid.argtypes = [_I, _I, _I, _I, _I, _I, _I]
    L.oracle_plan.restype = _I
    L.oracle_plan.argtypes = [_P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P,
                              _P, _P, _P]
    L.oracle_num_threads.restype = _I
    L.oracle_num_threads.argtypes = []


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    pass


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what}: oracle status {rc} (1 bad argument, 2 page id out of range)")


# ---------------------------------------------------------------- codecs

def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns -> fp64 (exact)."""
    b = _c(bits, np.uint16)
    u = b.astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):
        return u.view(np.float32).astype(np.float64)


def bf16_from_f64(x) -> np.ndarray:
    """fp64 -> bf16 bit patterns, round to nearest even (per element, in C)."""
    L = lib()
    x = np.asarray(x, dtype=np.float64)
    return np.array([L.oracle_bf16_from_f64(float(v)) for v in x.ravel()],
                    dtype=np.uint16).reshape(x.shape)


def e4m3_decode(codes) -> np.ndarray:
    L = lib()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([L.oracle_e4m3_decode(int(v)) for v in c.ravel()],
                    dtype=np.float64).reshape(c.shape)


def e4m3_encode(x) -> np.ndarray:
    L = lib()
    x = np.asarray(x, dtype=np.float64)
    return np.array([L.oracle_e4m3_encode(float(v)) for v in x.ravel()],
                    dtype=np.uint8).reshape(x.shape)


def quantize_kv_e4m3(values, live, dead_code: int = 0x7F):
    """fp32 cache values [P][Hkv][S][D] -> (e4m3 codes, fp32 scales [P][Hkv])."""
    v = _c(values, np.float32)
    P, Hkv, S, D = v.shape
    lv = _c(live, np.int32)
    codes = np.empty(v.shape, dtype=np.uint8)
    scales = np.empty((P, Hkv), dtype=np.float32)
    lib().oracle_quantize_kv_e4m3(_ptr(v), _ptr(lv), P, Hkv, S, D, dead_code, _ptr(codes),
                                  _ptr(scales))
    return codes, scales


# ---------------------------------------------------------------- prologue

def rmsnorm(x, gamma, eps: float) -> np.ndarray:
    x = _c(x, np.float64)
    g = _c(gamma, np.float64)
    y = np.empty_like(x)
    lib().oracle_rmsnorm(_ptr(x), _ptr(g), x.shape[0], eps, _ptr(y))
    return y


def rope(x, pos: float, theta: float) -> np.ndarray:
    x = _c(x, np.float64)
    y = np.empty_like(x)
    lib().oracle_rope(_ptr(x), x.shape[0], float(pos), float(theta), _ptr(y))
    return y


def prologue(q_raw, k_raw, v_raw, q_gamma, k_gamma, eps, theta, positions, page_table,
             k_cache, v_cache, page_size: int = 64):
    """Fused prologue on host copies.  k_cache/v_cache (uint16 bf16 bits,
    [P][Hkv][S][D]) are updated in place; returns q_out fp64 [B][Hq][D]."""
    q_raw = _c(q_raw, np.uint16)
    k_raw = _c(k_raw, np.uint16)
    v_raw = _c(v_raw, np.uint16)
    B, Hq, D = q_raw.shape
    Hkv = k_raw.shape[1]
    assert k_cache.dtype == np.uint16 and k_cache.flags.c_contiguous
    assert v_cache.dtype == np.uint16 and v_cache.flags.c_contiguous
    pt = _c(page_table, np.int32)
    pos = _c(positions, np.int32)
    q_out = np.empty((B, Hq, D), dtype=np.float64)
    rc = lib().oracle_prologue(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw),
                               _ptr(_c(q_gamma, np.float32)), _ptr(_c(k_gamma, np.float32)),
                               float(eps), float(theta), _ptr(pos), _ptr(pt), pt.shape[1],
                               _ptr(k_cache), _ptr(v_cache), _ptr(q_out), B, Hq, Hkv, D,
                               page_size, k_cache.shape[0])
    _check(rc, "prologue")
    return q_out


# ---------------------------------------------------------------- attention

def paged_decode(q, k_cache, v_cache, page_table, seq_lens, num_kv_heads: int, scale: float,
                 *, kv_fp8: bool = False, k_scale=None, v_scale=None, rows=None,
                 page_size: int = 64, num_threads: int = 0) -> np.ndarray:
    """Decode attention, fp64 [B][Hq][D].  q: uint16 bf16 bits or float64.
    Only the sequences in ``rows`` are computed (others left zero)."""
    q = np.asarray(q)
    q16 = _c(q, np.uint16) if q.dtype == np.uint16 else None
    q64 = None if q16 is not None else _c(q, np.float64)
    B, Hq, D = q.shape
    kc = _c(k_cache, np.uint8 if kv_fp8 else np.uint16)
    vc = _c(v_cache, np.uint8 if kv_fp8 else np.uint16)
    ks = _c(k_scale, np.float32) if kv_fp8 else None
    vs = _c(v_scale, np.float32) if kv_fp8 else None
    pt = _c(page_table, np.int32)
    sl = _c(seq_lens, np.int32)
    r = None if rows is None else _c(rows, np.int32)
    out = np.zeros((B, Hq, D), dtype=np.float64)
    rc = lib().oracle_paged_decode(_ptr(q16), _ptr(q64), _ptr(kc), _ptr(vc), int(kv_fp8),
                                   _ptr(ks), _ptr(vs), _ptr(pt), pt.shape[1], _ptr(sl), B, Hq,
                                   num_kv_heads, D, page_size, kc.shape[0], float(scale),
                                   _ptr(r), 0 if r is None else r.shape[0], _ptr(out),
                                   num_threads)
    _check(rc, "paged_decode")
    return out


def paged_decode_multi(q, k_cache, v_cache, page_table, seq_lens, num_kv_heads: int,
                       scale: float, *, kv_fp8: bool = False, k_scale=None, v_scale=None,
                       rows=None, page_size: int = 64, num_threads: int = 0) -> np.ndarray:
    """Multi-token decode attention, fp64 [B][T][Hq][D]: q is [B][T][Hq][D]
    (uint16 bf16 bits or float64); query token i of sequence b sees the
    first seq_lens[b] - T + i + 1 tokens (the T new tokens are the last T of
    the sequence, causal among themselves)."""
    q = np.asarray(q)
    q16 = _c(q, np.uint16) if q.dtype == np.uint16 else None
    q64 = None if q16 is not None else _c(q, np.float64)
    B, T, Hq, D = q.shape
    kc = _c(k_cache, np.uint8 if kv_fp8 else np.uint16)
    vc = _c(v_cache, np.uint8 if kv_fp8 else np.uint16)
    ks = _c(k_scale, np.float32) if kv_fp8 else None
    vs = _c(v_scale, np.float32) if kv_fp8 else None
    pt = _c(page_table, np.int32)
    sl = _c(seq_lens, np.int32)
    r = None if rows is None else _c(rows, np.int32)
    out = np.zeros((B, T, Hq, D), dtype=np.float64)
    rc = lib().oracle_paged_decode_multi(_ptr(q16), _ptr(q64), _ptr(kc), _ptr(vc), int(kv_fp8),
                                         _ptr(ks), _ptr(vs), _ptr(pt), pt.shape[1], _ptr(sl), B,
                                         T, Hq, num_kv_heads, D, page_size, kc.shape[0],
                                         float(scale), _ptr(r), 0 if r is None else r.shape[0],
                                         _ptr(out), num_threads)
    _check(rc, "paged_decode_multi")
    return out


def partial(q, k_cache, v_cache, page_table, num_kv_heads: int, scale: float, b: int, h: int,
            t0: int, t1: int, *, kv_fp8=False, k_scale=None, v_scale=None,
            page_size: int = 64):
    """(acc[D], m, l) of one (b, h) over tokens [t0, t1)."""
    q = np.asarray(q)
    q16 = _c(q, np.uint16) if q.dtype == np.uint16 else None
    q64 = None if q16 is not None else _c(q, np.float64)
    B, Hq, D = q.shape
    kc = _c(k_cache, np.uint8 if kv_fp8 else np.uint16)
    vc = _c(v_cache, np.uint8 if kv_fp8 else np.uint16)
    ks = _c(k_scale, np.float32) if kv_fp8 else None
    vs = _c(v_scale, np.float32) if kv_fp8 else None
    pt = _c(page_table, np.int32)
    acc = np.zeros(D, dtype=np.float64)
    m = C.c_double()
    l = C.c_double()
    rc = lib().oracle_partial(_ptr(q16), _ptr(q64), _ptr(kc), _ptr(vc), int(kv_fp8), _ptr(ks),
                              _ptr(vs), _ptr(pt), pt.shape[1], Hq, num_kv_heads, D, page_size,
                              kc.shape[0], float(scale), b, h, t0, t1, _ptr(acc), C.byref(m),
                              C.byref(l))
    _check(rc, "partial")
    return acc, m.value, l.value


def lse_merge(acc, m, l) -> np.ndarray:
    acc = _c(acc, np.float64)
    n, D = acc.shape
    out = np.empty(D, dtype=np.float64)
    lib().oracle_lse_merge(_ptr(acc), _ptr(_c(m, np.float64)), _ptr(_c(l, np.float64)), n, D,
                           _ptr(out))
    return out


def attention_state(q, k_cache, v_cache, page_table, num_kv_heads: int, scale: float, b: int,
                    h: int, t0: int, t1: int, **kw):
    """(o[D], lse) of row (b, h) over tokens [t0, t1): the normalised output
    o = sum_j softmax_j v_j and its log-sum-exp lse = log sum_j exp(scale
    q.k_j), the state a split-KV piece hands to the merge (xiaodao.ai
    "HPC-Ops TPOT -48.8%", Attention section).  An empty range has the state
    (0, -inf), which every merge ignores."""
    D = np.asarray(q).shape[-1]
    if t1 <= t0:
        return np.zeros(D), -np.inf
    acc, m, l = partial(q, k_cache, v_cache, page_table, num_kv_heads, scale, b, h, t0, t1, **kw)
    return acc / l, m + np.log(l)


def merge_states(o, lse):
    """Log-sum-exp merge of n states (o_i[D], lse_i) of one row, computed over
    disjoint key sets: with M = max_i lse_i and w_i = exp(lse_i - M), the
    merged state is (sum_i w_i o_i / sum_i w_i, M + log sum_i w_i), folded in
    index order; states with lse = -inf contribute nothing, and a row whose
    states are all -inf merges to (0, -inf)."""
    o = np.asarray(o, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    n, D = o.shape
    M = -np.inf
    for i in range(n):
        M = max(M, lse[i])
    if M == -np.inf:
        return np.zeros(D), -np.inf
    num = np.zeros(D)
    den = 0.0
    for i in range(n):
        if lse[i] == -np.inf:
            continue
        w = np.exp(lse[i] - M)
        num += w * o[i]
        den += w
    return num / den, M + np.log(den)


# ---------------------------------------------------------------- planner

PLAN_DYNAMIC, PLAN_STATIC_NSPLIT, PLAN_STATIC_CHUNK, PLAN_LENGTH_AWARE = 0, 1, 2, 3


def plan_grid(kind, batch, num_kv_heads, num_ctas, param=0, max_seq_len=0, page_size=64) -> int:
    return int(lib().oracle_plan_grid(kind, batch, num_kv_heads, num_ctas, param, max_seq_len,
                                      page_size))


def plan(seq_lens, num_kv_heads: int, *, kind: int = 0, num_ctas: int, param: int = 0,
         max_seq_len: int = 0, capacity_tokens: int, tail: tuple[int, int, int],
         cost: tuple[int, int] = (1, 0), page_size: int = 64) -> dict:
    """The plan of ``kind`` (oracle.c, oracle_plan).  ``tail = (den, k, mn)``
    and ``cost = (q, e)`` pick the member of the dynamic family (kinds 0 and
    3): if U >= mn P, the last min(U // den, U - P) units in min(k P, that)
    run-time chunks; the primary ranges split the cost of the other units
    evenly, q per unit and e more per segment end.  tail = (0, 1, 0) with
    cost = (1, 0) is the plain even partition.  The tail is required, so that
    every caller states which member it checks; cost (1, 0) -- the units
    themselves split evenly -- is the default."""
    sl = _c(seq_lens, np.int32)
    B = sl.shape[0]
    grid = plan_grid(kind, B, num_kv_heads, num_ctas, param, max_seq_len, page_size)
    S = B * num_kv_heads
    lens = np.zeros(B, dtype=np.int32)
    tile_start = np.zeros(B + 1, dtype=np.int32)
    cta = np.zeros((5 * grid, 2), dtype=np.int32)
    split_count = np.zeros(S, dtype=np.int32)
    first_slot = np.zeros(S, dtype=np.int32)
    n_units = C.c_int32()
    n_ranges = C.c_int32()
    rc = lib().oracle_plan(_ptr(sl), B, num_kv_heads, page_size, capacity_tokens, kind,
                           num_ctas, param, max_seq_len, int(tail[0]), int(tail[1]),
                           int(tail[2]), int(cost[0]), int(cost[1]),
                           _ptr(lens), _ptr(tile_start),
                           _ptr(cta), _ptr(split_count), _ptr(first_slot), C.byref(n_units),
                           C.byref(n_ranges))
    _check(rc, "plan")
    V = int(n_ranges.value)
    return {"grid": grid, "ranges": V, "lens": lens, "tile_start": tile_start, "cta": cta[:V],
            "split_count": split_count, "first_slot": first_slot,
            "n_units": int(n_units.value)}


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def available_cores() -> int:
    return len(os.sched_getaffinity(0))
