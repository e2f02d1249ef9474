"""Python binding of libhpa.so: paged mixed-length decode attention on B200.

Argument marshalling only -- every step of the decode path (prologue, plan,
run, split merge) executes in the library's CUDA kernels.  PyTorch supplies
device memory and streams.  The library must have been built
(``python -m mixed_length_paged_b200.build``); importing the binding without
it raises ``HpaLibraryMissing`` -- there is no fallback implementation.

The functions mirror the C ABI in ``include/hpa.h``:

    decode_workspace_size, plan_grid, default_num_ctas, decode_num_ctas,
    workspace_layout, decode_plan (with ``tail=`` / ``cost=`` for hpa_decode_plan_shape),
    decode_run, decode_step (+ ``lse=``: hpa_decode_step_lse), decode_step_prologue,
    decode_run_multi, decode_run_prologue, kv_prologue, merge_states,
    read_status, read_cta_times, decode_noalloc, noalloc_read_status

plus ``tail_idle`` (a summary of read_cta_times), and ``PagedDecoder``
bundles a workspace with plan + run for callers who do not want to manage
it.  ``mixed_length_paged_b200.sharding`` spreads a batch over the ranks of a
process group (by kv head, or by page with a log-sum-exp merge of the ranks'
states).
"""
from __future__ import annotations

import ctypes as C
import os

import torch

__all__ = [
    "HpaError", "HpaLibraryMissing", "lib", "library_path", "PLAN_DYNAMIC", "PLAN_STATIC_NSPLIT",
    "PLAN_STATIC_CHUNK", "PLAN_LENGTH_AWARE", "TAIL_DEN_DEFAULT", "TAIL_CHUNKS_DEFAULT",
    "TAIL_MIN_DEFAULT", "TAIL_CHUNKS_MAX", "COST_UNIT_DEFAULT", "COST_END_DEFAULT", "COST_END_DEFAULT_FP8",
    "COST_MAX",
    "DEVICE_LEN_CLAMPED", "DEVICE_BAD_PAGE", "DEVICE_BAD_PLAN",
    "DEVICE_BAD_POSITION", "DEVICE_TIMEOUT", "decode_workspace_size", "plan_grid",
    "default_num_ctas", "decode_num_ctas", "workspace_layout", "decode_plan", "decode_run",
    "decode_step", "decode_step_prologue", "MAX_STEP_BATCH", "decode_run_multi",
    "decode_run_prologue",
    "kv_prologue", "read_status", "PagedDecoder", "version", "decode_noalloc", "noalloc_read_status", "NOALLOC_SCRATCH_BYTES",
    "merge_states", "MAX_MERGE_STATES", "read_cta_times", "tail_idle",
]

PLAN_DYNAMIC, PLAN_STATIC_NSPLIT, PLAN_STATIC_CHUNK, PLAN_LENGTH_AWARE = 0, 1, 2, 3
KV_BF16, KV_FP8_E4M3 = 0, 1
OUT_BF16, OUT_F32 = 0, 1
DEVICE_LEN_CLAMPED, DEVICE_BAD_PAGE, DEVICE_BAD_PLAN = 0x1, 0x2, 0x4
DEVICE_BAD_POSITION, DEVICE_TIMEOUT = 0x8, 0x10
PAGE_SIZE = 64
# run-time tail of the dynamic plans (hpa.h: HPA_TAIL_DEN_DEFAULT, ...)
TAIL_DEN_DEFAULT, TAIL_CHUNKS_DEFAULT, TAIL_MIN_DEFAULT, TAIL_CHUNKS_MAX = 8, 4, 32, 4
# cost weights of their primary ranges (hpa.h: HPA_COST_UNIT_DEFAULT, ...); the
# in-kernel plans use COST_END_DEFAULT_FP8 for e4m3 caches
COST_UNIT_DEFAULT, COST_END_DEFAULT, COST_END_DEFAULT_FP8, COST_MAX = 1, 0, 2, 4
NOALLOC_SCRATCH_BYTES = 16 << 20

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libhpa.so")


class HpaError(RuntimeError):
    pass


class HpaLibraryMissing(ImportError):
    pass


_STATUS = {0: "HPA_OK", 1: "HPA_ERR_INVALID_ARG", 2: "HPA_ERR_UNSUPPORTED",
           3: "HPA_ERR_WORKSPACE", 4: "HPA_ERR_CUDA"}
_lib = None

_V, _I, _F, _Z = C.c_void_p, C.c_int, C.c_float, C.c_size_t


def lib():
    """The loaded libhpa.so (loaded on first use; raises if it was never built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise HpaLibraryMissing(
                f"{library_path} not found; build it with `python -m mixed_length_paged_b200.build`")
        L = C.CDLL(library_path)
        L.hpa_status_string.restype = C.c_char_p
        L.hpa_status_string.argtypes = [_I]
        L.hpa_last_cuda_error.restype = C.c_char_p
        L.hpa_last_cuda_error.argtypes = []
        L.hpa_version.restype = _I
        L.hpa_version.argtypes = []
        L.hpa_default_num_ctas.restype = _I
        L.hpa_default_num_ctas.argtypes = [_I]
        L.hpa_decode_num_ctas.restype = _I
        L.hpa_decode_num_ctas.argtypes = [_I, _I, _I, _I]
        L.hpa_plan_grid.restype = _I
        L.hpa_plan_grid.argtypes = [_I, _I, _I, _I, _I, _I]
        L.hpa_decode_workspace_size.restype = _Z
        L.hpa_decode_workspace_size.argtypes = [_I, _I, _I, _I, _I, _I]
        L.hpa_workspace_layout.restype = _I
        L.hpa_workspace_layout.argtypes = [_I, _I, _I, _I, _I, _I, C.POINTER(_Z)]
        L.hpa_decode_plan.restype = _I
        L.hpa_decode_plan.argtypes = [_V, _I, _I, _I, _I, _I, _I, _I, _I, _I, _V, _Z,
                                      C.POINTER(_I), _V]
        L.hpa_decode_plan_shape.restype = _I
        L.hpa_decode_plan_shape.argtypes = [_V, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                                            _I, _V, _Z, C.POINTER(_I), _V]
        L.hpa_decode_run.restype = _I
        L.hpa_decode_run.argtypes = [_V, _V, _V, _V, _V, _I, _V, _I, _I, _V, _I, _I, _I, _I, _I,
                                     _F, _I, _I, _V, _Z, _V]
        L.hpa_decode_step_prologue.restype = _I
        L.hpa_decode_step_prologue.argtypes = [_V, _V, _V, _V, _V, _V, _F, _F, _V, _V, _V, _V, _I,
                                               _I, _V, _I, _I, _I, _I, _I, _F, _I, _V, _Z, _V]
        L.hpa_decode_step.restype = _I
        L.hpa_decode_step.argtypes = [_V, _V, _V, _V, _V, _V, _I, _V, _I, _I, _V, _I, _I, _I, _I,
                                      _I, _I, _F, _I, _V, _Z, _V]
        L.hpa_decode_step_lse.restype = _I
        L.hpa_decode_step_lse.argtypes = [_V, _V, _V, _V, _V, _V, _I, _V, _I, _I, _V, _I, _V, _I,
                                          _I, _I, _I, _I, _F, _I, _V, _Z, _V]
        L.hpa_merge_states.restype = _I
        L.hpa_merge_states.argtypes = [_V, _V, _I, C.c_longlong, _I, _V, _I, _V, _V]
        L.hpa_decode_run_multi.restype = _I
        L.hpa_decode_run_multi.argtypes = [_V, _V, _V, _V, _V, _I, _V, _I, _I, _V, _I, _I, _I,
                                           _I, _I, _I, _F, _I, _I, _V, _Z, _V]
        L.hpa_decode_run_prologue.restype = _I
        L.hpa_decode_run_prologue.argtypes = [_V, _V, _V, _V, _V, _F, _F, _V, _V, _V, _V, _I, _I,
                                              _V, _I, _I, _I, _I, _I, _F, _I, _I, _V, _Z, _V]
        L.hpa_kv_prologue.restype = _I
        L.hpa_kv_prologue.argtypes = [_V, _V, _V, _V, _V, _F, _F, _V, _V, _I, _V, _V, _V, _I, _I,
                                      _I, _I, _I, _V, _V]
        L.hpa_decode_noalloc.restype = _I
        L.hpa_decode_noalloc.argtypes = [_V, _V, _V, _V, _V, _I, _V, _I, _I, _V, _V, _I, _I, _I,
                                         _I, _I, _F, _I, _V]
        L.hpa_noalloc_read_status.restype = _I
        L.hpa_noalloc_read_status.argtypes = [C.POINTER(C.c_int32), _I, _V]
        L.hpa_read_cta_times.restype = _I
        L.hpa_read_cta_times.argtypes = [_V, _I, _I, _I, _I, _I, _I, _V, _V]
        L.hpa_read_status.restype = _I
        L.hpa_read_status.argtypes = [_V, C.POINTER(C.c_int32), _V]
        _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc != 0:
        msg = f"{what} failed: {_STATUS.get(rc, rc)}"
        if rc == 4:
            msg += " (" + lib().hpa_last_cuda_error().decode() + ")"
        raise HpaError(msg)


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _dev(t: torch.Tensor, name: str, dtypes, ndim=None):
    if not t.is_cuda:
        raise HpaError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise HpaError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise HpaError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise HpaError(f"{name} must have {ndim} dims, got {t.dim()}")


def version() -> int:
    return int(lib().hpa_version())


def default_num_ctas(device: int | None = None) -> int:
    d = torch.cuda.current_device() if device is None else device
    n = lib().hpa_default_num_ctas(d)
    if n < 1:
        raise HpaError("hpa_default_num_ctas: " + lib().hpa_last_cuda_error().decode())
    return n


def decode_num_ctas(num_q_heads: int, num_kv_heads: int, q_tokens: int = 1,
                    device: int | None = None) -> int:
    """Persistent CTA count matching the run kernel's residency for this head
    geometry (hpa_decode_num_ctas)."""
    d = torch.cuda.current_device() if device is None else device
    n = lib().hpa_decode_num_ctas(d, num_q_heads, num_kv_heads, q_tokens)
    if n < 1:
        raise HpaError("hpa_decode_num_ctas: invalid arguments or no device")
    return n


def plan_grid(kind: int, batch: int, num_kv_heads: int, num_ctas: int, param: int = 0,
              max_seq_len: int = 0) -> int:
    g = lib().hpa_plan_grid(kind, batch, num_kv_heads, num_ctas, param, max_seq_len)
    if g < 1:
        raise HpaError("hpa_plan_grid: invalid arguments")
    return g


def decode_workspace_size(kind: int, batch: int, num_kv_heads: int, num_q_heads: int,
                          head_dim: int, grid: int) -> int:
    n = lib().hpa_decode_workspace_size(kind, batch, num_kv_heads, num_q_heads, head_dim, grid)
    if n == 0:
        raise HpaError("hpa_decode_workspace_size: invalid arguments")
    return int(n)


def workspace_layout(kind, batch, num_kv_heads, num_q_heads, head_dim, grid) -> dict:
    off = (_Z * 8)()
    _check(lib().hpa_workspace_layout(kind, batch, num_kv_heads, num_q_heads, head_dim, grid, off),
           "hpa_workspace_layout")
    names = ["header", "lens", "tile_start", "cta_desc", "seg_desc", "part_ml", "part_acc",
             "total"]
    return {n: int(v) for n, v in zip(names, off)}


def decode_plan(seq_lens: torch.Tensor, *, num_kv_heads: int, num_q_heads: int, head_dim: int,
                pt_stride: int, workspace: torch.Tensor, kind: int = PLAN_DYNAMIC,
                num_ctas: int | None = None, param: int = 0, max_seq_len: int = 0,
                tail: tuple[int, int, int] | None = None, cost: tuple[int, int] | None = None,
                stream=None) -> int:
    """Enqueue the tile plan; returns the grid to pass to decode_run.

    ``tail = (tail_den, tail_chunks, tail_min)`` sets the run-time tail of a
    DYNAMIC or LENGTH_AWARE plan ((0, 1, 0): no tail) and ``cost =
    (unit_cost, end_cost)`` the cost weights of its primary ranges ((1, 0):
    the units split evenly), both through hpa_decode_plan_shape; None keeps
    the library's default (TAIL_*_DEFAULT, COST_*_DEFAULT)."""
    _dev(seq_lens, "seq_lens", (torch.int32,), 1)
    _dev(workspace, "workspace", (torch.uint8,))
    if num_ctas is None:
        num_ctas = default_num_ctas(seq_lens.device.index)
    grid = C.c_int(0)
    if tail is not None or cost is not None:
        t = (TAIL_DEN_DEFAULT, TAIL_CHUNKS_DEFAULT, TAIL_MIN_DEFAULT) if tail is None else tail
        c = (COST_UNIT_DEFAULT, COST_END_DEFAULT) if cost is None else cost
        rc = lib().hpa_decode_plan_shape(_ptr(seq_lens), seq_lens.shape[0], num_kv_heads,
                                         num_q_heads, head_dim, pt_stride, kind, num_ctas, param,
                                         int(t[0]), int(t[1]), int(t[2]), int(c[0]), int(c[1]),
                                         _ptr(workspace), workspace.numel(), C.byref(grid),
                                         _stream(stream))
        _check(rc, "hpa_decode_plan_shape")
        return grid.value
    rc = lib().hpa_decode_plan(_ptr(seq_lens), seq_lens.shape[0], num_kv_heads, num_q_heads,
                               head_dim, pt_stride, kind, num_ctas, param, max_seq_len,
                               _ptr(workspace), workspace.numel(), C.byref(grid), _stream(stream))
    _check(rc, "hpa_decode_plan")
    return grid.value


def decode_run(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
               page_table: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor, grid: int,
               softmax_scale: float, *, kind: int = PLAN_DYNAMIC,
               k_scale: torch.Tensor | None = None, v_scale: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """Enqueue the persistent decode kernel (and the split merge); writes and
    returns ``out``.  ``kind``/``grid``: those of the plan in ``workspace``.

    k_cache/v_cache: bf16, or uint8 / float8_e4m3fn codes with k_scale/v_scale."""
    _dev(q, "q", (torch.bfloat16,), 3)
    fp8 = k_cache.dtype in (torch.uint8, torch.float8_e4m3fn)
    cache_types = (torch.uint8, torch.float8_e4m3fn) if fp8 else (torch.bfloat16,)
    _dev(k_cache, "k_cache", cache_types, 4)
    _dev(v_cache, "v_cache", cache_types, 4)
    _dev(page_table, "page_table", (torch.int32,), 2)
    _dev(out, "out", (torch.bfloat16, torch.float32), 3)
    _dev(workspace, "workspace", (torch.uint8,))
    if fp8:
        if k_scale is None or v_scale is None:
            raise HpaError("FP8 caches need k_scale and v_scale")
        _dev(k_scale, "k_scale", (torch.float32,), 2)
        _dev(v_scale, "v_scale", (torch.float32,), 2)
    B, Hq, D = q.shape
    num_pages, Hkv, S, Dk = k_cache.shape
    if S != PAGE_SIZE or Dk != D or tuple(v_cache.shape) != tuple(k_cache.shape) \
            or tuple(out.shape) != tuple(q.shape) or page_table.shape[0] != B:
        raise HpaError("decode_run: inconsistent shapes")
    rc = lib().hpa_decode_run(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale),
                              _ptr(v_scale), KV_FP8_E4M3 if fp8 else KV_BF16, _ptr(page_table),
                              page_table.shape[1], num_pages, _ptr(out),
                              OUT_F32 if out.dtype == torch.float32 else OUT_BF16, B, Hq, Hkv, D,
                              float(softmax_scale), kind, grid, _ptr(workspace),
                              workspace.numel(), _stream(stream))
    _check(rc, "hpa_decode_run")
    return out


MAX_STEP_BATCH = 512  # sequences hpa_decode_step plans in the kernel


def decode_step(seq_lens: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                v_cache: torch.Tensor, page_table: torch.Tensor, out: torch.Tensor,
                workspace: torch.Tensor, num_ctas: int, softmax_scale: float, *,
                k_scale: torch.Tensor | None = None, v_scale: torch.Tensor | None = None,
                lse: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One decode step with the dynamic plan made inside the decode kernel
    (hpa_decode_step).  q/out are [B][Hq][D], or [B][T][Hq][D] for T query
    tokens per sequence.  The workspace must be zero-filled before its first
    use (or last written by decode_plan).  With ``lse`` (fp32, q's shape
    without D) each row's log-sum-exp is written too (hpa_decode_step_lse),
    for merge_states."""
    _dev(seq_lens, "seq_lens", (torch.int32,), 1)
    if q.dim() not in (3, 4):
        raise HpaError("q must be [B][Hq][D] or [B][T][Hq][D]")
    _dev(q, "q", (torch.bfloat16,), q.dim())
    fp8 = k_cache.dtype in (torch.uint8, torch.float8_e4m3fn)
    cache_types = (torch.uint8, torch.float8_e4m3fn) if fp8 else (torch.bfloat16,)
    _dev(k_cache, "k_cache", cache_types, 4)
    _dev(v_cache, "v_cache", cache_types, 4)
    _dev(page_table, "page_table", (torch.int32,), 2)
    _dev(out, "out", (torch.bfloat16, torch.float32), q.dim())
    _dev(workspace, "workspace", (torch.uint8,))
    if fp8:
        if k_scale is None or v_scale is None:
            raise HpaError("FP8 caches need k_scale and v_scale")
        _dev(k_scale, "k_scale", (torch.float32,), 2)
        _dev(v_scale, "v_scale", (torch.float32,), 2)
    if q.dim() == 3:
        B, Hq, D = q.shape
        T = 1
    else:
        B, T, Hq, D = q.shape
    num_pages, Hkv, S, Dk = k_cache.shape
    if S != PAGE_SIZE or Dk != D or tuple(v_cache.shape) != tuple(k_cache.shape) \
            or tuple(out.shape) != tuple(q.shape) or page_table.shape[0] != B \
            or seq_lens.shape[0] != B:
        raise HpaError("decode_step: inconsistent shapes")
    out_kind = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    kv_kind = KV_FP8_E4M3 if fp8 else KV_BF16
    if lse is not None:
        _dev(lse, "lse", (torch.float32,), q.dim() - 1)
        if tuple(lse.shape) != tuple(q.shape[:-1]):
            raise HpaError("decode_step: lse must have q's shape without the head dim")
        rc = lib().hpa_decode_step_lse(_ptr(seq_lens), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                       _ptr(k_scale), _ptr(v_scale), kv_kind, _ptr(page_table),
                                       page_table.shape[1], num_pages, _ptr(out), out_kind,
                                       _ptr(lse), B, T, Hq, Hkv, D, float(softmax_scale),
                                       num_ctas, _ptr(workspace), workspace.numel(),
                                       _stream(stream))
        _check(rc, "hpa_decode_step_lse")
        return out
    rc = lib().hpa_decode_step(_ptr(seq_lens), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                               _ptr(k_scale), _ptr(v_scale), kv_kind, _ptr(page_table),
                               page_table.shape[1], num_pages, _ptr(out), out_kind, B, T, Hq, Hkv,
                               D, float(softmax_scale), num_ctas, _ptr(workspace),
                               workspace.numel(), _stream(stream))
    _check(rc, "hpa_decode_step")
    return out


MAX_MERGE_STATES = 16  # states hpa_merge_states combines in one call


def merge_states(o_parts, lse_parts, out: torch.Tensor, lse_out: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """Log-sum-exp merge of attention states over disjoint key sets of the
    same rows (hpa_merge_states): o_parts are fp32 tensors of out's shape
    [..., D], lse_parts fp32 tensors of out's shape without D.  A part may
    live on a peer GPU whose memory this context can address."""
    o_parts, lse_parts = list(o_parts), list(lse_parts)
    n = len(o_parts)
    if n != len(lse_parts) or not 1 <= n <= MAX_MERGE_STATES:
        raise HpaError(f"merge_states: 1..{MAX_MERGE_STATES} (o, lse) pairs, got {n} and "
                       f"{len(lse_parts)}")
    _dev(out, "out", (torch.bfloat16, torch.float32))
    D = out.shape[-1]
    rows = out.numel() // D if D else 0
    for i, (o, l) in enumerate(zip(o_parts, lse_parts)):
        _dev(o, f"o_parts[{i}]", (torch.float32,), out.dim())
        _dev(l, f"lse_parts[{i}]", (torch.float32,), out.dim() - 1)
        if tuple(o.shape) != tuple(out.shape) or tuple(l.shape) != tuple(out.shape[:-1]):
            raise HpaError("merge_states: part shapes must match out")
    if lse_out is not None:
        _dev(lse_out, "lse_out", (torch.float32,), out.dim() - 1)
        if tuple(lse_out.shape) != tuple(out.shape[:-1]):
            raise HpaError("merge_states: lse_out must have out's shape without D")
    o_ptrs = (C.c_void_p * n)(*[o.data_ptr() for o in o_parts])
    l_ptrs = (C.c_void_p * n)(*[l.data_ptr() for l in lse_parts])
    rc = lib().hpa_merge_states(o_ptrs, l_ptrs, n, rows, D, _ptr(out),
                                OUT_F32 if out.dtype == torch.float32 else OUT_BF16,
                                _ptr(lse_out), _stream(stream))
    _check(rc, "hpa_merge_states")
    return out


def decode_step_prologue(seq_lens: torch.Tensor, q_raw: torch.Tensor, k_raw: torch.Tensor,
                         v_raw: torch.Tensor, q_gamma: torch.Tensor, k_gamma: torch.Tensor,
                         k_cache: torch.Tensor, v_cache: torch.Tensor, page_table: torch.Tensor,
                         out: torch.Tensor, workspace: torch.Tensor, num_ctas: int,
                         softmax_scale: float, *, q_out: torch.Tensor | None = None,
                         eps: float = 1e-6, rope_theta: float = 10000.0,
                         stream=None) -> torch.Tensor:
    """A whole decode step -- prologue, dynamic plan, attention, merge -- in two
    launches (hpa_decode_step_prologue); seq_lens are post-append lengths."""
    _dev(seq_lens, "seq_lens", (torch.int32,), 1)
    for t, n, nd in ((q_raw, "q_raw", 3), (k_raw, "k_raw", 3), (v_raw, "v_raw", 3),
                     (k_cache, "k_cache", 4), (v_cache, "v_cache", 4)):
        _dev(t, n, (torch.bfloat16,), nd)
    if q_out is not None:
        _dev(q_out, "q_out", (torch.bfloat16,), 3)
    _dev(q_gamma, "q_gamma", (torch.float32,), 1)
    _dev(k_gamma, "k_gamma", (torch.float32,), 1)
    _dev(page_table, "page_table", (torch.int32,), 2)
    _dev(out, "out", (torch.bfloat16, torch.float32), 3)
    _dev(workspace, "workspace", (torch.uint8,))
    B, Hq, D = q_raw.shape
    num_pages, Hkv, S, Dk = k_cache.shape
    if S != PAGE_SIZE or Dk != D or tuple(v_cache.shape) != tuple(k_cache.shape) \
            or tuple(out.shape) != tuple(q_raw.shape) or page_table.shape[0] != B \
            or tuple(k_raw.shape) != (B, Hkv, D) or tuple(v_raw.shape) != (B, Hkv, D) \
            or seq_lens.shape[0] != B or q_gamma.numel() != D or k_gamma.numel() != D \
            or (q_out is not None and tuple(q_out.shape) != tuple(q_raw.shape)):
        raise HpaError("decode_step_prologue: inconsistent shapes")
    rc = lib().hpa_decode_step_prologue(
        _ptr(seq_lens), _ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(q_gamma), _ptr(k_gamma),
        float(eps), float(rope_theta), _ptr(k_cache), _ptr(v_cache), _ptr(q_out),
        _ptr(page_table), page_table.shape[1], num_pages, _ptr(out),
        OUT_F32 if out.dtype == torch.float32 else OUT_BF16, B, Hq, Hkv, D,
        float(softmax_scale), num_ctas, _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "hpa_decode_step_prologue")
    return out


def decode_run_multi(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                     page_table: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                     grid: int, softmax_scale: float, *, kind: int = PLAN_DYNAMIC,
                     k_scale: torch.Tensor | None = None, v_scale: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Multi-token decode: q and out are [B][T][Hq][D]; query token i of a
    sequence of L tokens sees its first L - T + i + 1 tokens.  The plan in
    ``workspace`` must have been made with num_q_heads = Hq * T."""
    _dev(q, "q", (torch.bfloat16,), 4)
    fp8 = k_cache.dtype in (torch.uint8, torch.float8_e4m3fn)
    cache_types = (torch.uint8, torch.float8_e4m3fn) if fp8 else (torch.bfloat16,)
    _dev(k_cache, "k_cache", cache_types, 4)
    _dev(v_cache, "v_cache", cache_types, 4)
    _dev(page_table, "page_table", (torch.int32,), 2)
    _dev(out, "out", (torch.bfloat16, torch.float32), 4)
    _dev(workspace, "workspace", (torch.uint8,))
    if fp8:
        if k_scale is None or v_scale is None:
            raise HpaError("FP8 caches need k_scale and v_scale")
        _dev(k_scale, "k_scale", (torch.float32,), 2)
        _dev(v_scale, "v_scale", (torch.float32,), 2)
    B, T, Hq, D = q.shape
    num_pages, Hkv, S, Dk = k_cache.shape
    if S != PAGE_SIZE or Dk != D or tuple(v_cache.shape) != tuple(k_cache.shape) \
            or tuple(out.shape) != tuple(q.shape) or page_table.shape[0] != B:
        raise HpaError("decode_run_multi: inconsistent shapes")
    rc = lib().hpa_decode_run_multi(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale),
                                    _ptr(v_scale), KV_FP8_E4M3 if fp8 else KV_BF16,
                                    _ptr(page_table), page_table.shape[1], num_pages, _ptr(out),
                                    OUT_F32 if out.dtype == torch.float32 else OUT_BF16, B, T, Hq,
                                    Hkv, D, float(softmax_scale), kind, grid, _ptr(workspace),
                                    workspace.numel(), _stream(stream))
    _check(rc, "hpa_decode_run_multi")
    return out


def decode_run_prologue(q_raw: torch.Tensor, k_raw: torch.Tensor, v_raw: torch.Tensor,
                        q_gamma: torch.Tensor, k_gamma: torch.Tensor, k_cache: torch.Tensor,
                        v_cache: torch.Tensor, page_table: torch.Tensor, out: torch.Tensor,
                        workspace: torch.Tensor, grid: int, softmax_scale: float, *,
                        q_out: torch.Tensor | None = None, eps: float = 1e-6,
                        rope_theta: float = 10000.0, kind: int = PLAN_DYNAMIC,
                        stream=None) -> torch.Tensor:
    """decode_run with the prologue (RMSNorm + RoPE of q and of the new K row,
    the K/V slot write) fused into the decode kernel; writes and returns
    ``out``.  The plan in ``workspace`` must hold the post-append lengths; the
    new token goes to position seq_len - 1.  bf16 caches only."""
    for t, n, nd in ((q_raw, "q_raw", 3), (k_raw, "k_raw", 3), (v_raw, "v_raw", 3),
                     (k_cache, "k_cache", 4), (v_cache, "v_cache", 4)):
        _dev(t, n, (torch.bfloat16,), nd)
    if q_out is not None:
        _dev(q_out, "q_out", (torch.bfloat16,), 3)
    _dev(q_gamma, "q_gamma", (torch.float32,), 1)
    _dev(k_gamma, "k_gamma", (torch.float32,), 1)
    _dev(page_table, "page_table", (torch.int32,), 2)
    _dev(out, "out", (torch.bfloat16, torch.float32), 3)
    _dev(workspace, "workspace", (torch.uint8,))
    B, Hq, D = q_raw.shape
    num_pages, Hkv, S, Dk = k_cache.shape
    if S != PAGE_SIZE or Dk != D or tuple(v_cache.shape) != tuple(k_cache.shape) \
            or tuple(out.shape) != tuple(q_raw.shape) or page_table.shape[0] != B \
            or tuple(k_raw.shape) != (B, Hkv, D) or tuple(v_raw.shape) != (B, Hkv, D) \
            or q_gamma.numel() != D or k_gamma.numel() != D \
            or (q_out is not None and tuple(q_out.shape) != tuple(q_raw.shape)):
        raise HpaError("decode_run_prologue: inconsistent shapes")
    rc = lib().hpa_decode_run_prologue(
        _ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(q_gamma), _ptr(k_gamma), float(eps),
        float(rope_theta), _ptr(k_cache), _ptr(v_cache), _ptr(q_out), _ptr(page_table),
        page_table.shape[1], num_pages, _ptr(out),
        OUT_F32 if out.dtype == torch.float32 else OUT_BF16, B, Hq, Hkv, D,
        float(softmax_scale), kind, grid, _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "hpa_decode_run_prologue")
    return out


def kv_prologue(q_raw, k_raw, v_raw, q_gamma, k_gamma, positions, page_table, k_cache, v_cache,
                q_out, *, eps: float = 1e-6, rope_theta: float = 10000.0, status=None,
                stream=None) -> torch.Tensor:
    """Enqueue the fused RMSNorm + RoPE + KV-write prologue; returns q_out."""
    for t, n, nd in ((q_raw, "q_raw", 3), (k_raw, "k_raw", 3), (v_raw, "v_raw", 3),
                     (q_out, "q_out", 3), (k_cache, "k_cache", 4), (v_cache, "v_cache", 4)):
        _dev(t, n, (torch.bfloat16,), nd)
    _dev(q_gamma, "q_gamma", (torch.float32,), 1)
    _dev(k_gamma, "k_gamma", (torch.float32,), 1)
    _dev(positions, "positions", (torch.int32,), 1)
    _dev(page_table, "page_table", (torch.int32,), 2)
    if status is not None:
        _dev(status, "status", (torch.int32,))
    B, Hq, D = q_raw.shape
    Hkv = k_raw.shape[1]
    rc = lib().hpa_kv_prologue(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(q_gamma),
                               _ptr(k_gamma), float(eps), float(rope_theta), _ptr(positions),
                               _ptr(page_table), page_table.shape[1], _ptr(k_cache),
                               _ptr(v_cache), _ptr(q_out), B, Hq, Hkv, D, k_cache.shape[0],
                               _ptr(status), _stream(stream))
    _check(rc, "hpa_kv_prologue")
    return q_out


def decode_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                   page_table: torch.Tensor, seq_lens: torch.Tensor, out: torch.Tensor,
                   softmax_scale: float, *, k_scale: torch.Tensor | None = None,
                   v_scale: torch.Tensor | None = None, num_ctas: int = 0,
                   stream=None) -> torch.Tensor:
    """One decode step (dynamic plan + run) without a caller workspace.

    For callers that cannot allocate device memory where the step is issued:
    the scratch is the library's static 16 MiB device array, shared by every
    call on the device (calls that overlap on the GPU race on it).  The first
    call on a device looks the array up; make it before any stream capture."""
    _dev(q, "q", (torch.bfloat16,), 3)
    fp8 = k_cache.dtype in (torch.uint8, torch.float8_e4m3fn)
    cache_types = (torch.uint8, torch.float8_e4m3fn) if fp8 else (torch.bfloat16,)
    _dev(k_cache, "k_cache", cache_types, 4)
    _dev(v_cache, "v_cache", cache_types, 4)
    _dev(page_table, "page_table", (torch.int32,), 2)
    _dev(seq_lens, "seq_lens", (torch.int32,), 1)
    _dev(out, "out", (torch.bfloat16, torch.float32), 3)
    if fp8:
        if k_scale is None or v_scale is None:
            raise HpaError("FP8 caches need k_scale and v_scale")
        _dev(k_scale, "k_scale", (torch.float32,), 2)
        _dev(v_scale, "v_scale", (torch.float32,), 2)
    # the call uses the current device's scratch array and stream: every
    # tensor must live on that device
    cur = torch.cuda.current_device()
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                    ("page_table", page_table), ("seq_lens", seq_lens), ("out", out),
                    ("k_scale", k_scale), ("v_scale", v_scale)):
        if t is not None and t.device.index != cur:
            raise HpaError(f"decode_noalloc: {name} is on {t.device}, the current device is "
                           f"cuda:{cur}")
    B, Hq, D = q.shape
    num_pages, Hkv = k_cache.shape[0], k_cache.shape[1]
    rc = lib().hpa_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale),
                                  _ptr(v_scale), KV_FP8_E4M3 if fp8 else KV_BF16,
                                  _ptr(page_table), page_table.shape[1], num_pages,
                                  _ptr(seq_lens), _ptr(out),
                                  OUT_F32 if out.dtype == torch.float32 else OUT_BF16, B, Hq,
                                  Hkv, D, float(softmax_scale), num_ctas, _stream(stream))
    _check(rc, "hpa_decode_noalloc")
    return out


def noalloc_read_status(clear: bool = False, stream=None) -> int:
    """Status word (DEVICE_* bits) of decode_noalloc's static array on the
    current device (hpa_noalloc_read_status); ``clear`` resets it to 0
    afterwards.  Synchronises the stream."""
    v = C.c_int32(0)
    _check(lib().hpa_noalloc_read_status(C.byref(v), int(bool(clear)), _stream(stream)),
           "hpa_noalloc_read_status")
    return int(v.value)


def read_status(workspace: torch.Tensor, stream=None) -> int:
    """Device status word of a plan's workspace (synchronises the stream)."""
    v = C.c_int32(0)
    _check(lib().hpa_read_status(_ptr(workspace), C.byref(v), _stream(stream)), "hpa_read_status")
    return int(v.value)


def read_cta_times(workspace: torch.Tensor, kind: int, batch: int, num_kv_heads: int,
                   num_q_heads: int, head_dim: int, grid: int, stream=None):
    """Per-CTA timeline of the last run on ``workspace`` (hpa_read_cta_times):
    an int64 tensor [grid][4] of (start ns, producer done ns, epilogue done ns,
    units streamed).  The shape arguments are those the workspace was sized
    with; synchronises the stream."""
    t = torch.zeros((grid, 4), dtype=torch.int64)
    _check(lib().hpa_read_cta_times(_ptr(workspace), kind, batch, num_kv_heads, num_q_heads,
                                    head_dim, grid, t.data_ptr(), _stream(stream)),
           "hpa_read_cta_times")
    return t


def tail_idle(times: torch.Tensor) -> dict:
    """Load balance of one run from its CTA timeline: the span from the first
    CTA start to the last epilogue, the spread of the CTAs' finishing times and
    the idle fraction sum_c (last end - end_c) / (CTAs x span) -- the share of
    the CTAs' time spent waiting for the slowest one."""
    t = times.to(torch.float64)
    t0, end = t[:, 0].min(), t[:, 2]
    span = float(end.max() - t0)
    ends = (end - t0).sort().values
    n = ends.numel()
    return {"span_us": span / 1e3,
            "end_min_us": float(ends[0]) / 1e3,
            "end_median_us": float(ends[n // 2]) / 1e3,
            "end_max_us": float(ends[-1]) / 1e3,
            "idle_fraction": float((ends[-1] - ends).sum()) / (n * span) if span > 0 else 0.0,
            "units_min": int(times[:, 3].min()), "units_max": int(times[:, 3].max())}


class PagedDecoder:
    """A workspace sized for one batch shape, plus plan + run in one call.
    ``q_tokens`` > 1: multi-token decode (q and out [B][T][Hq][D])."""

    def __init__(self, batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                 pt_stride: int, *, kind: int = PLAN_DYNAMIC, num_ctas: int | None = None,
                 param: int = 0, max_seq_len: int = 0, q_tokens: int = 1, device=None):
        self.device = torch.device("cuda" if device is None else device)
        self.num_ctas = num_ctas or decode_num_ctas(num_q_heads, num_kv_heads, q_tokens,
                                                    self.device.index or 0)
        self.kind, self.param, self.max_seq_len = kind, param, max_seq_len
        self.q_tokens = q_tokens
        self.shape = (batch, num_q_heads, num_kv_heads, head_dim, pt_stride)
        grid = plan_grid(kind, batch, num_kv_heads, self.num_ctas, param, max_seq_len)
        # a multi-token plan counts G * T rows per kv head; zero-filled so that
        # step() can use it from the first call
        self.workspace = torch.zeros(decode_workspace_size(kind, batch, num_kv_heads,
                                                           num_q_heads * q_tokens, head_dim, grid),
                                     dtype=torch.uint8, device=self.device)
        self.grid = grid

    def plan(self, seq_lens: torch.Tensor, stream=None) -> int:
        B, Hq, Hkv, D, pts = self.shape
        self.grid = decode_plan(seq_lens, num_kv_heads=Hkv, num_q_heads=Hq * self.q_tokens,
                                head_dim=D,
                                pt_stride=pts, workspace=self.workspace, kind=self.kind,
                                num_ctas=self.num_ctas, param=self.param,
                                max_seq_len=self.max_seq_len, stream=stream)
        return self.grid

    def run(self, q, k_cache, v_cache, page_table, out, softmax_scale, *, k_scale=None,
            v_scale=None, stream=None):
        if q.dim() == 4:  # [B][T][Hq][D]: the multi-token entry (any T)
            return decode_run_multi(q, k_cache, v_cache, page_table, out, self.workspace,
                                    self.grid, softmax_scale, kind=self.kind, k_scale=k_scale,
                                    v_scale=v_scale, stream=stream)
        return decode_run(q, k_cache, v_cache, page_table, out, self.workspace, self.grid,
                          softmax_scale, kind=self.kind, k_scale=k_scale, v_scale=v_scale,
                          stream=stream)

    def step(self, q, k_cache, v_cache, page_table, seq_lens, out, softmax_scale, *,
             k_scale=None, v_scale=None, lse=None, stream=None):
        """plan + run as one decode_step (the dynamic plan made inside the
        decode kernel) when the plan is dynamic and the batch fits, else the
        two calls.  ``lse`` (the rows' log-sum-exp) needs the first form."""
        if self.kind == PLAN_DYNAMIC and self.shape[0] <= MAX_STEP_BATCH:
            return decode_step(seq_lens, q, k_cache, v_cache, page_table, out, self.workspace,
                               self.num_ctas, softmax_scale, k_scale=k_scale, v_scale=v_scale,
                               lse=lse, stream=stream)
        if lse is not None:
            raise HpaError(f"step: lse needs the dynamic plan and batch <= {MAX_STEP_BATCH}")
        self.plan(seq_lens, stream=stream)
        return self.run(q, k_cache, v_cache, page_table, out, softmax_scale, k_scale=k_scale,
                        v_scale=v_scale, stream=stream)

    def step_prologue(self, q_raw, k_raw, v_raw, q_gamma, k_gamma, k_cache, v_cache, page_table,
                      seq_lens, out, softmax_scale, stream=None, **kw):
        """A whole step with the prologue: decode_step_prologue when the plan is
        dynamic and the batch fits, else plan + run_prologue."""
        if self.kind == PLAN_DYNAMIC and self.shape[0] <= MAX_STEP_BATCH:
            return decode_step_prologue(seq_lens, q_raw, k_raw, v_raw, q_gamma, k_gamma, k_cache,
                                        v_cache, page_table, out, self.workspace, self.num_ctas,
                                        softmax_scale, stream=stream, **kw)
        self.plan(seq_lens, stream=stream)
        return self.run_prologue(q_raw, k_raw, v_raw, q_gamma, k_gamma, k_cache, v_cache,
                                 page_table, out, softmax_scale, stream=stream, **kw)

    def run_prologue(self, q_raw, k_raw, v_raw, q_gamma, k_gamma, k_cache, v_cache, page_table,
                     out, softmax_scale, **kw):
        """The planned step with the prologue fused in (decode_run_prologue)."""
        return decode_run_prologue(q_raw, k_raw, v_raw, q_gamma, k_gamma, k_cache, v_cache,
                                   page_table, out, self.workspace, self.grid, softmax_scale,
                                   kind=self.kind, **kw)

    def __call__(self, q, k_cache, v_cache, page_table, seq_lens, out, softmax_scale, **kw):
        self.plan(seq_lens, stream=kw.get("stream"))
        return self.run(q, k_cache, v_cache, page_table, out, softmax_scale, **kw)

    def status(self, stream=None) -> int:
        return read_status(self.workspace, stream)

    def cta_times(self, stream=None) -> torch.Tensor:
        """Per-CTA timeline of the last run (read_cta_times)."""
        B, Hq, Hkv, D, _ = self.shape
        return read_cta_times(self.workspace, self.kind, B, Hkv, Hq * self.q_tokens, D,
                              self.grid, stream)
