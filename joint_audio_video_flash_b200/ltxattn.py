"""ctypes binding of libltxattn.so (the C ABI in include/ltxattn.h).

Argument marshalling only: torch tensors are checked for dtype, device, shape and
contiguity, and their device pointers are passed to the library together with
the current CUDA stream.  There is no fallback: if the library is missing or a
call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import math
import os
import re
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
# LTXATTN_DEBUG=1 selects the guard-word build (libltxattn_debug.so, see build.build(debug=True))
LIB_PATH = os.path.join(_PKG, "libltxattn_debug.so" if os.environ.get("LTXATTN_DEBUG") == "1"
                        else "libltxattn.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "ltxattn.h")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_MISALIGNED, ERR_CUDA, ERR_DEVICE_TIMEOUT, \
    ERR_NOT_INITIALIZED, ERR_WORKSPACE_GUARD = range(8)

_lock = threading.Lock()
_lib = None


class LtxAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def load() -> ctypes.CDLL:
    """Load libltxattn.so (built by ``joint_audio_video_flash_b200.build``); raise if absent."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: run joint_audio_video_flash_b200.build"
                                  + (" with debug=True" if LIB_PATH.endswith("_debug.so") else ""))
            lib = ctypes.CDLL(LIB_PATH)
            vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
            lib.ltxattn_create.argtypes = []
            lib.ltxattn_forward.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, vp]
            lib.ltxattn_forward_ex.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci,
                                               ctypes.POINTER(ci), vp]
            lib.ltxattn_check.argtypes = [vp]
            lib.ltxattn_destroy.argtypes = []
            lib.ltxattn_status_string.argtypes = [ci]
            lib.ltxattn_status_string.restype = ctypes.c_char_p
            lib.ltxattn_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, vp]
            lib.ltxattn_num_entry_points.argtypes = []
            lib.ltxattn_qk_norm_rope.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci,
                                                 cf, vp]
            lib.ltxattn_na3d_forward.argtypes = [vp, vp, vp, vp] + [ci] * 9 + [cf, vp]
            lib.ltxattn_na3d_plan.argtypes = [ci] * 6 + [vp, vp]
            lib.ltxattn_forward_plan.argtypes = [ci] * 8 + [vp, vp]
            lib.ltxattn_forward_partial.argtypes = [vp, vp, vp, vp, vp] + [ci] * 6 + [cf, vp]
            lib.ltxattn_combine.argtypes = [vp, vp, vp] + [ci] * 5 + [vp]
            lib.ltxattn_forward_grouped.argtypes = [vp, ci, vp]
            lib.ltxattn_entry_point_name.argtypes = [ci]
            lib.ltxattn_entry_point_name.restype = ctypes.c_char_p
            _lib = lib
    return _lib


def header_entry_points() -> list[str]:
    """Function names declared in include/ltxattn.h."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"^\s*(?:LTXATTN_API\s+)?(?:int|const char\*)\s+(ltxattn_\w+)\s*\(", text, flags=re.M)


def status_string(status: int) -> str:
    return load().ltxattn_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise LtxAttnError(status, where)


def create() -> None:
    _check(load().ltxattn_create(), "ltxattn_create")


def destroy() -> None:
    _check(load().ltxattn_destroy(), "ltxattn_destroy")


def _stream_handle(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def check(stream=None) -> None:
    """Synchronise the stream and raise if a kernel recorded a stalled wait."""
    _check(load().ltxattn_check(ctypes.c_void_p(_stream_handle(stream))), "ltxattn_check")


def selftest_wait_timeout(timeout_ns: int = 1_000_000, stream=None) -> int:
    """Run the bounded-wait self-test; returns the raw status (DEVICE_TIMEOUT expected)."""
    return int(load().ltxattn_selftest_wait_timeout(ctypes.c_ulonglong(int(timeout_ns)),
                                                      ctypes.c_void_p(_stream_handle(stream))))


def _check_attention_tensors(q, k, v, out) -> None:
    """Checks the library cannot make from raw pointers: bf16, contiguous 4-D BSHD, k and v
    shaped [batch, kv_len, heads, head_dim] like q, out shaped like q, every tensor on the
    current CUDA device (the C ABI works on the current device's context).  `out` may be
    None (checked later, once allocated)."""
    import torch
    named = [("q", q), ("k", k), ("v", v)] + ([("out", out)] if out is not None else [])
    for name, t in named:
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a bfloat16 CUDA tensor")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous [batch, len, heads, head_dim] tensor")
        if t.device.index != torch.cuda.current_device():
            raise ValueError(f"{name} is on {t.device}, not on the current device "
                             f"cuda:{torch.cuda.current_device()}")
    batch, _, heads, head_dim = q.shape
    kv_len = k.shape[1]
    if tuple(k.shape) != (batch, kv_len, heads, head_dim) or v.shape != k.shape:
        raise ValueError("k and v must be [batch, kv_len, heads, head_dim] matching q")
    if out is not None and out.shape != q.shape:
        raise ValueError("out must be shaped like q")


def forward(q, k, v, out=None, *, kv_valid_len: int | None = None, scale: float | None = None,
            num_splits: int = 0, stream=None, return_splits: bool = False):
    """O = softmax(scale q k^T, keys < kv_valid_len) v for bf16 BSHD CUDA tensors.

    q: [B, Lq, H, D]; k, v: [B, Lkv, H, D]; out (optional): [B, Lq, H, D].
    """
    import torch
    if out is None:
        _check_attention_tensors(q, k, v, None)
        out = torch.empty_like(q)
    _check_attention_tensors(q, k, v, out)
    batch, q_len, heads, head_dim = q.shape
    kv_len = k.shape[1]
    if kv_valid_len is None:
        kv_valid_len = kv_len
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    used = ctypes.c_int(0)
    st = load().ltxattn_forward_ex(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()), int(q_len), int(kv_len),
        int(kv_valid_len), int(batch), int(heads), int(head_dim), ctypes.c_float(scale),
        int(num_splits), ctypes.byref(used), ctypes.c_void_p(_stream_handle(stream)))
    _check(st, "ltxattn_forward")
    return (out, used.value) if return_splits else out


class _Call(ctypes.Structure):
    """``ltxattn_call`` of include/ltxattn.h."""
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("out", ctypes.c_void_p), ("q_len", ctypes.c_int), ("kv_len", ctypes.c_int),
                ("kv_valid_len", ctypes.c_int), ("batch", ctypes.c_int),
                ("heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("scale", ctypes.c_float)]


def forward_grouped(calls, *, stream=None):
    """Several independent attention calls through ``ltxattn_forward_grouped``.

    ``calls``: a sequence of dicts with keys q, k, v, out (tensors as for ``forward``; out
    required) and optional kv_valid_len and scale.  Calls at head_dim 64 whose valid keys
    fit in one 128-key tile (a2v, audio self-attention) share one launch.  Returns the
    list of outputs.
    """
    arr = (_Call * len(calls))()
    outs = []
    for i, c in enumerate(calls):
        q, k, v, out = c["q"], c["k"], c["v"], c["out"]
        _check_attention_tensors(q, k, v, out)
        batch, q_len, heads, head_dim = q.shape
        kv_len = k.shape[1]
        kv_valid = c.get("kv_valid_len")
        scale = c.get("scale")
        arr[i] = _Call(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), int(q_len),
                       int(kv_len), int(kv_len if kv_valid is None else kv_valid), int(batch),
                       int(heads), int(head_dim),
                       float(1.0 / math.sqrt(head_dim) if scale is None else scale))
        outs.append(out)
    st = load().ltxattn_forward_grouped(ctypes.cast(arr, ctypes.c_void_p), len(calls),
                                        ctypes.c_void_p(_stream_handle(stream)))
    _check(st, "ltxattn_forward_grouped")
    return outs


def forward_split_noalloc(q, k, v, out, *, kv_valid_len: int | None = None,
                          scale: float | None = None, num_splits: int = 0, stream=None) -> int:
    """Key-split forward that allocates no device memory (``ltxattn_forward_split_noalloc``).

    For callers that must not let the library allocate (a plugin host that owns all
    device memory, a serving loop with a fixed memory plan, a hard memory quota):
    key-split fp32 partials go to the library's built-in 16 MiB scratch array (one key
    part needs none).  ``out`` is required (this call allocates nothing, not even the
    output).  Tensors are checked as for ``forward``.  Returns the raw status; calls whose
    GPU work overlaps race on the shared scratch; ``check()`` reports a kernel wait that
    ran out in the last such call.
    """
    _check_attention_tensors(q, k, v, out)
    lib = load()
    fn = lib.ltxattn_forward_split_noalloc
    vp, ci = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ctypes.c_float, ci, vp]
    batch, q_len, heads, head_dim = q.shape
    kv_len = k.shape[1]
    if kv_valid_len is None:
        kv_valid_len = kv_len
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    return int(fn(vp(q.data_ptr()), vp(k.data_ptr()), vp(v.data_ptr()), vp(out.data_ptr()),
                  int(q_len), int(kv_len), int(kv_valid_len), int(batch), int(heads),
                  int(head_dim), ctypes.c_float(scale), int(num_splits),
                  vp(_stream_handle(stream))))


def qk_norm_rope(q, k, q_weight, k_weight, cos, sin, q_out=None, k_out=None, *,
                 eps: float = 1e-6, stream=None):
    """Norm and rotary step of queries and keys (``ltxattn_qk_norm_rope``); returns (q', k').

    q, k: bf16 CUDA [B, L, H, D]; weights: bf16 [H * D]; cos, sin: fp32 [L, D / 2].  The
    outputs may be the inputs (in place).
    """
    import torch
    for name, t in (("q", q), ("k", k)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda \
                or t.dim() != 4 or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous bf16 CUDA [batch, len, heads, dim] tensor")
    if k.shape != q.shape:
        raise ValueError("q and k must have the same shape")
    batch, seq_len, heads, head_dim = q.shape
    for name, t, dt, shape in (("q_weight", q_weight, torch.bfloat16, (heads * head_dim,)),
                               ("k_weight", k_weight, torch.bfloat16, (heads * head_dim,)),
                               ("cos", cos, torch.float32, (seq_len, head_dim // 2)),
                               ("sin", sin, torch.float32, (seq_len, head_dim // 2))):
        if (not isinstance(t, torch.Tensor) or t.dtype != dt or not t.is_cuda
                or tuple(t.shape) != shape or not t.is_contiguous()):
            raise TypeError(f"{name} must be a contiguous {dt} CUDA tensor of shape {shape}")
    q_out = torch.empty_like(q) if q_out is None else q_out
    k_out = torch.empty_like(k) if k_out is None else k_out
    for name, t in (("q_out", q_out), ("k_out", k_out)):
        if t.dtype != torch.bfloat16 or t.shape != q.shape or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 tensor shaped like q")
    st = load().ltxattn_qk_norm_rope(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(q_out.data_ptr()), ctypes.c_void_p(k_out.data_ptr()),
        ctypes.c_void_p(q_weight.data_ptr()), ctypes.c_void_p(k_weight.data_ptr()),
        ctypes.c_void_p(cos.data_ptr()), ctypes.c_void_p(sin.data_ptr()), int(batch),
        int(seq_len), int(heads), int(head_dim), ctypes.c_float(eps),
        ctypes.c_void_p(_stream_handle(stream)))
    _check(st, "ltxattn_qk_norm_rope")
    return q_out, k_out


def na3d_forward(q, k, v, grid, window, out=None, *, scale: float | None = None, stream=None):
    """3-D neighbourhood attention (``ltxattn_na3d_forward``) of bf16 CUDA tensors.

    q, k, v: [B, T*Y*X, H, D] with tokens in raster order of the grid (T, Y, X); window
    (kT, kY, kX): odd sizes, each at most its grid axis.  Returns out [B, T*Y*X, H, D].
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a bfloat16 CUDA tensor")
        if t.dim() != 4 or not t.is_contiguous() or t.shape != q.shape:
            raise ValueError(f"{name} must be a contiguous [batch, tokens, heads, head_dim] "
                             "tensor shaped like q")
    grid_t, grid_y, grid_x = (int(x) for x in grid)
    win_t, win_y, win_x = (int(x) for x in window)
    batch, tokens, heads, head_dim = q.shape
    if tokens != grid_t * grid_y * grid_x:
        raise ValueError(f"{tokens} tokens but grid {tuple(grid)}")
    if out is None:
        out = torch.empty_like(q)
    elif (out.dtype != torch.bfloat16 or out.shape != q.shape or not out.is_contiguous()
          or out.device != q.device):
        raise ValueError("out must be a contiguous bf16 tensor shaped like q on q's device")
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    st = load().ltxattn_na3d_forward(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()), int(batch), grid_t,
        grid_y, grid_x, int(heads), int(head_dim), win_t, win_y, win_x, ctypes.c_float(scale),
        ctypes.c_void_p(_stream_handle(stream)))
    _check(st, "ltxattn_na3d_forward")
    return out


# ltxattn_kernel values
KERNEL_ONE_TILE, KERNEL_TWO_TILES, KERNEL_ONE_TILE_DUAL = 0, 1, 2
KERNEL_SHORT_KV, KERNEL_A2V, KERNEL_PAIR = 3, 4, 5


def forward_plan(q_len: int, kv_len: int, kv_valid_len: int, batch: int, heads: int,
                 head_dim: int, num_splits: int = 0, num_sms: int = 148):
    """The kernel ``ltxattn_forward`` runs for these sizes and its key-range parts
    (``ltxattn_forward_plan``, host only): (one of the KERNEL_* values, parts)."""
    kernel = ctypes.c_int()
    parts = ctypes.c_int()
    st = load().ltxattn_forward_plan(int(q_len), int(kv_len), int(kv_valid_len), int(batch),
                                     int(heads), int(head_dim), int(num_splits), int(num_sms),
                                     ctypes.cast(ctypes.pointer(kernel), ctypes.c_void_p),
                                     ctypes.cast(ctypes.pointer(parts), ctypes.c_void_p))
    _check(st, "ltxattn_forward_plan")
    return kernel.value, parts.value


def na3d_plan(grid, window):
    """The blocking ``ltxattn_na3d_forward`` uses (``ltxattn_na3d_plan``, host only): the
    query brick (t, y, x), the key tile (t, y, x) and the key tiles per (batch, head)."""
    shape = (ctypes.c_int * 6)()
    tiles = ctypes.c_longlong()
    st = load().ltxattn_na3d_plan(*(int(x) for x in grid), *(int(x) for x in window),
                                  ctypes.cast(shape, ctypes.c_void_p),
                                  ctypes.cast(ctypes.pointer(tiles), ctypes.c_void_p))
    _check(st, "ltxattn_na3d_plan")
    return tuple(shape[:3]), tuple(shape[3:]), int(tiles.value)


def rows_pad(q_len: int) -> int:
    """Query rows per (batch, head) in the partial-result layout: q_len rounded up to 128."""
    return -(-int(q_len) // 128) * 128


def forward_partial(q, k, v, o_part=None, lse=None, *, kv_valid_len: int | None = None,
                    scale: float | None = None, stream=None):
    """Attention over one key range (``ltxattn_forward_partial``): returns (o_part, lse).

    q: [B, Lq, H, D]; k, v: [B, Lkv, H, D] (bf16 CUDA).  o_part: fp32 [B, H, rows_pad, D],
    lse: fp32 [B, H, rows_pad] base-2 log-sum-exp; rows past Lq are left unwritten.
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a bfloat16 CUDA tensor")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous [batch, len, heads, head_dim] tensor")
    batch, q_len, heads, head_dim = q.shape
    kv_len = k.shape[1]
    if tuple(k.shape) != (batch, kv_len, heads, head_dim) or v.shape != k.shape:
        raise ValueError("k and v must be [batch, kv_len, heads, head_dim] matching q")
    rp = rows_pad(q_len)
    if o_part is None:
        o_part = torch.empty(batch, heads, rp, head_dim, dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty(batch, heads, rp, dtype=torch.float32, device=q.device)
    if (o_part.dtype != torch.float32 or tuple(o_part.shape) != (batch, heads, rp, head_dim)
            or not o_part.is_contiguous() or lse.dtype != torch.float32
            or tuple(lse.shape) != (batch, heads, rp) or not lse.is_contiguous()):
        raise ValueError("o_part / lse must be contiguous fp32 [B, H, rows_pad, D] / [B, H, rows_pad]")
    if kv_valid_len is None:
        kv_valid_len = kv_len
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    st = load().ltxattn_forward_partial(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o_part.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()), int(q_len), int(kv_len), int(kv_valid_len), int(batch),
        int(heads), int(head_dim), ctypes.c_float(scale), ctypes.c_void_p(_stream_handle(stream)))
    _check(st, "ltxattn_forward_partial")
    return o_part, lse


def combine(o_parts, lses, q_len: int, out=None, *, stream=None):
    """Merge of key-range partial results (``ltxattn_combine``) into bf16 [B, q_len, H, D].

    o_parts: fp32 [P, B, H, rows_pad, D]; lses: fp32 [P, B, H, rows_pad].
    """
    import torch
    if (not isinstance(o_parts, torch.Tensor) or o_parts.dtype != torch.float32
            or o_parts.dim() != 5 or not o_parts.is_contiguous() or not o_parts.is_cuda):
        raise TypeError("o_parts must be a contiguous fp32 CUDA [P, B, H, rows_pad, D] tensor")
    parts, batch, heads, rp, head_dim = o_parts.shape
    if rp != rows_pad(q_len):
        raise ValueError(f"rows_pad {rp} does not match q_len {q_len}")
    if (lses.dtype != torch.float32 or tuple(lses.shape) != (parts, batch, heads, rp)
            or not lses.is_contiguous()):
        raise ValueError("lses must be a contiguous fp32 [P, B, H, rows_pad] tensor")
    if out is None:
        out = torch.empty(batch, q_len, heads, head_dim, dtype=torch.bfloat16,
                          device=o_parts.device)
    st = load().ltxattn_combine(
        ctypes.c_void_p(o_parts.data_ptr()), ctypes.c_void_p(lses.data_ptr()),
        ctypes.c_void_p(out.data_ptr()), int(parts), int(q_len), int(batch), int(heads),
        int(head_dim), ctypes.c_void_p(_stream_handle(stream)))
    _check(st, "ltxattn_combine")
    return out
