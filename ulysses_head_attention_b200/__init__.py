"""Python binding of libulysses.so (the Ulysses SP hot path on one B200).

Argument marshalling only: every function below checks that the tensors it
is handed are CUDA tensors of the documented shape/dtype, then calls the C
entry point of the same name (declared in include/ulysses.h) with their
device pointers and the current CUDA stream.  All arithmetic runs in the
library's kernels; there is no Python or CPU fallback.  Importing this module
fails loudly when the library has not been built.

Shapes (full sizes b, n, H, d; P virtual ranks):
    seq-sharded   (P, b, n/P, H, d)
    head-sharded  (P, b, n, H/P, d)
    lse           (P, b, h_q/P, n) float32
    position_ids  (b, n) int64, on the device
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# ULYSSES_DEBUG=1 loads the bounds-checked build (every global index and TMA
# tile coordinate checked; see ulysses_debug_status) instead of the release one.
DEBUG_BUILD = os.environ.get("ULYSSES_DEBUG", "0") == "1"
LIB_PATH = os.path.join(HERE, "libulysses_debug.so" if DEBUG_BUILD else "libulysses.so")

ULY_BF16, ULY_F32 = 0, 1
STATUS_NAMES = {0: "ULY_OK", 1: "ULY_ERR_INVALID_ARG", 2: "ULY_ERR_UNSUPPORTED", 3: "ULY_ERR_CUDA",
                4: "ULY_ERR_WORKSPACE", 5: "ULY_ERR_TIMEOUT", 6: "ULY_ERR_BOUNDS"}
# Every symbol include/ulysses.h declares.
EXPORTS = ("ulysses_seq_to_head", "ulysses_head_to_seq", "ulysses_kv_seq_to_head", "ulysses_kv_head_to_seq",
           "ulysses_transpose_runs", "ulysses_attn_fwd_workspace", "ulysses_attn_fwd",
           "ulysses_attn_bwd_workspace", "ulysses_attn_bwd", "ulysses_attn_bwd_timed", "ulysses_attn_fwd_noalloc",
           "ulysses_attn_fwd_noalloc_status",
           "ulysses_attn_fwd_kv_range", "ulysses_attn_bwd_kv_range", "ulysses_attn_lse_merge",
           "ulysses_sp_loss_aggregate", "ulysses_workspace_status", "ulysses_selftest_wait_timeout",
           "ulysses_seq_to_head_push", "ulysses_head_to_seq_push", "ulysses_wait_flags", "ulysses_release_flags",
           "ulysses_ipc_handle",
           "ulysses_ipc_open", "ulysses_ipc_close", "ulysses_attn_fwd_block", "ulysses_attn_bwd_block",
           "ulysses_accumulate", "ulysses_debug_status", "ulysses_layer_step_host_bytes", "ulysses_layer_step_host",
           "ulysses_layer_status", "ulysses_status_string")


class UlyShape(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("n", ctypes.c_int64), ("h_q", ctypes.c_int64),
                ("h_kv", ctypes.c_int64), ("d", ctypes.c_int64), ("P", ctypes.c_int32)]


class UlyssesError(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({status_string(status)})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python ulysses_head_attention_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    shp = ctypes.POINTER(UlyShape)
    sig = {
        "ulysses_seq_to_head": ([vp, vp, i64, i64, i64, i64, i32, i32, vp], i32),
        "ulysses_head_to_seq": ([vp, vp, i64, i64, i64, i64, i32, i32, vp], i32),
        "ulysses_kv_seq_to_head": ([vp, vp, i64, i64, i64, i64, i32, i32, vp], i32),
        "ulysses_kv_head_to_seq": ([vp, vp, i64, i64, i64, i64, i32, i32, vp], i32),
        "ulysses_transpose_runs": ([vp, vp, i64, i64, i64, vp], i32),
        "ulysses_attn_fwd_workspace": ([shp], sz),
        "ulysses_attn_fwd": ([vp, vp, vp, vp, shp, i32, f32, vp, i32, vp, vp, sz, vp], i32),
        "ulysses_attn_bwd_workspace": ([shp, i32], sz),
        "ulysses_attn_bwd": ([vp, vp, vp, vp, i32, vp, vp, vp, shp, i32, f32, vp, vp, vp, i32, vp, sz, vp], i32),
        "ulysses_attn_bwd_timed": ([vp, vp, vp, vp, i32, vp, vp, vp, shp, i32, f32, vp, vp, vp, i32, vp, sz, vp,
                                    ctypes.POINTER(vp)], i32),
        "ulysses_attn_fwd_noalloc": ([vp, vp, vp, vp, shp, i32, f32, vp, i32, vp, vp], i32),
        "ulysses_attn_fwd_kv_range": ([vp, vp, vp, vp, shp, i32, f32, i64, i64, vp, i32, vp, vp, sz, vp], i32),
        "ulysses_attn_bwd_kv_range": ([vp, vp, vp, vp, i32, vp, vp, vp, shp, i32, f32, i64, i64, vp, vp, vp, i32,
                                       vp, sz, vp], i32),
        "ulysses_attn_lse_merge": ([vp, vp, i32, shp, vp, i32, vp, vp], i32),
        "ulysses_sp_loss_aggregate": ([vp, vp, i64, i64, i32, i64, vp, vp, vp, vp], i32),
        "ulysses_workspace_status": ([vp, vp, ctypes.POINTER(ctypes.c_int32)], i32),
        "ulysses_attn_fwd_noalloc_status": ([vp, ctypes.POINTER(ctypes.c_int32)], i32),
        "ulysses_selftest_wait_timeout": ([vp, sz, ctypes.c_uint64, vp], i32),
        "ulysses_seq_to_head_push": ([vp, ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i64, i64, i64, i64, i32, i32,
                                      ctypes.c_uint32, vp, sz, vp], i32),
        "ulysses_head_to_seq_push": ([vp, ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i64, i64, i64, i64, i32, i32,
                                      ctypes.c_uint32, vp, sz, vp], i32),
        "ulysses_wait_flags": ([vp, i32, ctypes.c_uint32, ctypes.c_uint64, vp, vp], i32),
        "ulysses_release_flags": ([ctypes.POINTER(vp), i32, ctypes.c_uint32, vp], i32),
        "ulysses_ipc_handle": ([vp, ctypes.c_char_p], i32),
        "ulysses_ipc_open": ([ctypes.c_char_p, ctypes.POINTER(vp)], i32),
        "ulysses_ipc_close": ([vp], i32),
        "ulysses_attn_fwd_block": ([vp, vp, vp, vp, shp, i64, i64, i64, i64, f32, vp, i32, vp, vp, sz, vp], i32),
        "ulysses_attn_bwd_block": ([vp, vp, vp, vp, i32, vp, vp, vp, shp, i64, i64, i64, i64, f32, vp, vp, vp, i32,
                                    vp, sz, vp], i32),
        "ulysses_accumulate": ([vp, vp, i64, vp], i32),
        "ulysses_debug_status": ([vp, ctypes.POINTER(ctypes.c_int32)], i32),
        "ulysses_layer_step_host_bytes": ([shp], sz),
        "ulysses_layer_step_host": ([vp, vp, vp, vp, vp, shp, f32, vp, vp, vp, vp, vp, sz, vp, vp, vp,
                                     ctypes.POINTER(vp)], i32),
        "ulysses_layer_status": ([vp, shp, vp, ctypes.POINTER(ctypes.c_int32)], i32),
        "ulysses_status_string": ([i32], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.ulysses_status_string(status).decode()


def _check(status: int, what: str) -> None:
    if status != 0:
        raise UlyssesError(what, status)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return ULY_BF16
    if t.dtype == torch.float32:
        return ULY_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


_BF16, _F32, _I64, _OUT = (torch.bfloat16,), (torch.float32,), (torch.int64,), (torch.bfloat16, torch.float32)


def _expect(t, shape, dtypes, name: str) -> None:
    """Shape and dtype of one argument: the kernels index every buffer by the
    call's shape, so a smaller tensor would be read or written out of bounds."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} is {t.dtype}, expected {' or '.join(str(x) for x in dtypes)}")


def _one_device(stream, **tensors) -> None:
    """Every tensor on the CUDA device the kernels launch on (the stream's)."""
    for name, t in tensors.items():
        _dev(t, name)
    dev = (stream.device if stream is not None else torch.device("cuda", torch.cuda.current_device()))
    for name, t in tensors.items():
        if t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the launch is on {dev}")


def _check_attn(q_head, k_head, v_head, position_ids, o_head, lse, stream, do_head=None, dq_head=None,
                dk_head=None, dv_head=None, ws=None) -> None:
    """Layouts of the attention calls (head layout, per virtual rank)."""
    if not isinstance(q_head, torch.Tensor) or q_head.dim() != 5:
        raise ValueError("q_head must be [P][b][n][h_q/P][d]")
    P, b, n, hq, d = q_head.shape
    if not isinstance(k_head, torch.Tensor) or k_head.dim() != 5:
        raise ValueError("k_head must be [P][b][n][h_kv/P][d]")
    hkv = k_head.shape[3]
    _expect(q_head, (P, b, n, hq, d), _BF16, "q_head")
    _expect(k_head, (P, b, n, hkv, d), _BF16, "k_head")
    _expect(v_head, (P, b, n, hkv, d), _BF16, "v_head")
    _expect(position_ids, (b, n), _I64, "position_ids")
    _expect(o_head, (P, b, n, hq, d), _OUT, "o_head")
    _expect(lse, (P, b, hq, n), _F32, "lse")
    grads = {}
    if do_head is not None:
        _expect(do_head, (P, b, n, hq, d), _BF16, "do_head")
        _expect(dq_head, (P, b, n, hq, d), _OUT, "dq_head")
        _expect(dk_head, (P, b, n, hkv, d), (dq_head.dtype,), "dk_head")
        _expect(dv_head, (P, b, n, hkv, d), (dq_head.dtype,), "dv_head")
        grads = dict(do_head=do_head, dq_head=dq_head, dk_head=dk_head, dv_head=dv_head)
    if ws is not None:
        grads["ws"] = ws
    _one_device(stream, q_head=q_head, k_head=k_head, v_head=v_head, position_ids=position_ids, o_head=o_head,
                lse=lse, **grads)


def make_shape(b: int, n: int, h_q: int, h_kv: int, d: int, P: int) -> UlyShape:
    return UlyShape(b, n, h_q, h_kv, d, P)


def ulysses_seq_to_head(x_seq: torch.Tensor, x_head: torch.Tensor, stream=None) -> None:
    """x_seq (P, b, n/P, H, d) -> x_head (P, b, n, H/P, d)."""
    P, b, m, H, d = x_seq.shape
    if tuple(x_head.shape) != (P, b, m * P, H // P, d) or x_head.dtype != x_seq.dtype:
        raise ValueError("x_head shape/dtype does not match x_seq")
    _one_device(stream, x_seq=x_seq, x_head=x_head)
    _check(lib.ulysses_seq_to_head(_dev(x_seq, "x_seq"), _dev(x_head, "x_head"), b, m * P, H, d, P,
                                   _dtype_code(x_seq), _stream(stream)), "ulysses_seq_to_head")


def ulysses_head_to_seq(x_head: torch.Tensor, x_seq: torch.Tensor, stream=None) -> None:
    """x_head (P, b, n, H/P, d) -> x_seq (P, b, n/P, H, d)."""
    P, b, n, h, d = x_head.shape
    if tuple(x_seq.shape) != (P, b, n // P, h * P, d) or x_seq.dtype != x_head.dtype:
        raise ValueError("x_seq shape/dtype does not match x_head")
    _one_device(stream, x_head=x_head, x_seq=x_seq)
    _check(lib.ulysses_head_to_seq(_dev(x_head, "x_head"), _dev(x_seq, "x_seq"), b, n, h * P, d, P,
                                   _dtype_code(x_head), _stream(stream)), "ulysses_head_to_seq")


def ulysses_kv_seq_to_head(x_seq: torch.Tensor, x_head: torch.Tensor, stream=None) -> None:
    """K/V x_seq (P, b, n/P, H_kv, d) -> x_head (P, b, n, max(H_kv/P, 1), d); one
    replicated kv head per rank when H_kv < P."""
    P, b, m, H, d = x_seq.shape
    h = H // P if H >= P else 1
    if tuple(x_head.shape) != (P, b, m * P, h, d) or x_head.dtype != x_seq.dtype:
        raise ValueError("x_head shape/dtype does not match x_seq")
    _one_device(stream, x_seq=x_seq, x_head=x_head)
    _check(lib.ulysses_kv_seq_to_head(_dev(x_seq, "x_seq"), _dev(x_head, "x_head"), b, m * P, H, d, P,
                                      _dtype_code(x_seq), _stream(stream)), "ulysses_kv_seq_to_head")


def ulysses_kv_head_to_seq(x_head: torch.Tensor, x_seq: torch.Tensor, stream=None) -> None:
    """dK/dV x_head (P, b, n, max(H_kv/P, 1), d) -> x_seq (P, b, n/P, H_kv, d);
    the replicas are summed when H_kv < P."""
    P, b, m, H, d = x_seq.shape
    h = H // P if H >= P else 1
    if tuple(x_head.shape) != (P, b, m * P, h, d) or x_head.dtype != x_seq.dtype:
        raise ValueError("x_seq shape/dtype does not match x_head")
    _one_device(stream, x_head=x_head, x_seq=x_seq)
    _check(lib.ulysses_kv_head_to_seq(_dev(x_head, "x_head"), _dev(x_seq, "x_seq"), b, m * P, H, d, P,
                                      _dtype_code(x_seq), _stream(stream)), "ulysses_kv_head_to_seq")


def ulysses_transpose_runs(src: torch.Tensor, dst: torch.Tensor, A: int, B: int, run_bytes: int,
                           stream=None) -> None:
    """dst[j][i][:] = src[i][j][:] over runs of run_bytes bytes (i < A, j < B)."""
    if src.numel() * src.element_size() != A * B * run_bytes or dst.numel() * dst.element_size() != A * B * run_bytes:
        raise ValueError("buffer sizes do not match A * B * run_bytes")
    _one_device(stream, src=src, dst=dst)
    _check(lib.ulysses_transpose_runs(_dev(src, "src"), _dev(dst, "dst"), A, B, run_bytes, _stream(stream)),
           "ulysses_transpose_runs")


def _attn_shape(q_head: torch.Tensor, k_head: torch.Tensor) -> UlyShape:
    P, b, n, hq, d = q_head.shape
    Pk, bk, nk, hkv, dk = k_head.shape
    if (Pk, bk, nk, dk) != (P, b, n, d):
        raise ValueError("k_head shape does not match q_head")
    return UlyShape(b, n, hq * P, hkv * P, d, P)


def ulysses_attn_fwd_workspace(shape: UlyShape) -> int:
    return int(lib.ulysses_attn_fwd_workspace(ctypes.byref(shape)))


def ulysses_attn_bwd_workspace(shape: UlyShape, g_dtype: int) -> int:
    return int(lib.ulysses_attn_bwd_workspace(ctypes.byref(shape), g_dtype))


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """A zeroed uint8 workspace tensor (torch's allocator aligns to >= 256 B)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def ulysses_attn_fwd(q_head, k_head, v_head, position_ids, o_head, lse, ws, rank: int = -1,
                     softmax_scale: float = 0.0, stream=None) -> None:
    """Local causal attention of every rank (or `rank`) on its head slice."""
    _check_attn(q_head, k_head, v_head, position_ids, o_head, lse, stream, ws=ws)
    shape = _attn_shape(q_head, k_head)
    _check(lib.ulysses_attn_fwd(_dev(q_head, "q_head"), _dev(k_head, "k_head"), _dev(v_head, "v_head"),
                                _dev(position_ids, "position_ids"), ctypes.byref(shape), rank, softmax_scale,
                                _dev(o_head, "o_head"), _dtype_code(o_head), _dev(lse, "lse"),
                                _dev(ws, "ws"), ws.numel() * ws.element_size(), _stream(stream)),
           "ulysses_attn_fwd")


def ulysses_attn_fwd_noalloc(q_head, k_head, v_head, position_ids, o_head, lse, rank: int = -1,
                             softmax_scale: float = 0.0, stream=None) -> None:
    """ulysses_attn_fwd without a workspace, for callers that cannot allocate
    device memory: the library's fixed per-GPU scratch (b*n <= 524288 tokens)
    is used instead.  Calls that overlap on the GPU race on that scratch."""
    _check_attn(q_head, k_head, v_head, position_ids, o_head, lse, stream)
    shape = _attn_shape(q_head, k_head)
    _check(lib.ulysses_attn_fwd_noalloc(_dev(q_head, "q_head"), _dev(k_head, "k_head"), _dev(v_head, "v_head"),
                                        _dev(position_ids, "position_ids"), ctypes.byref(shape), rank,
                                        softmax_scale, _dev(o_head, "o_head"), _dtype_code(o_head),
                                        _dev(lse, "lse"), _stream(stream)),
           "ulysses_attn_fwd_noalloc")


def ulysses_attn_fwd_noalloc_status(stream=None) -> int:
    """Synchronize, then read and clear the status word of the current
    device's no-alloc scratch (0 = ok)."""
    code = ctypes.c_int32(-1)
    _check(lib.ulysses_attn_fwd_noalloc_status(_stream(stream), ctypes.byref(code)),
           "ulysses_attn_fwd_noalloc_status")
    return int(code.value)


def ulysses_attn_bwd(q_head, k_head, v_head, o_head, lse, do_head, position_ids, dq_head, dk_head, dv_head, ws,
                     rank: int = -1, softmax_scale: float = 0.0, stream=None) -> None:
    """Gradients dQ, dK, dV of the local attention (head layout)."""
    _check_attn(q_head, k_head, v_head, position_ids, o_head, lse, stream, do_head, dq_head, dk_head, dv_head,
                ws)
    shape = _attn_shape(q_head, k_head)
    _check(lib.ulysses_attn_bwd(_dev(q_head, "q_head"), _dev(k_head, "k_head"), _dev(v_head, "v_head"),
                                _dev(o_head, "o_head"), _dtype_code(o_head), _dev(lse, "lse"),
                                _dev(do_head, "do_head"), _dev(position_ids, "position_ids"), ctypes.byref(shape),
                                rank, softmax_scale, _dev(dq_head, "dq_head"), _dev(dk_head, "dk_head"),
                                _dev(dv_head, "dv_head"), _dtype_code(dq_head), _dev(ws, "ws"),
                                ws.numel() * ws.element_size(), _stream(stream)),
           "ulysses_attn_bwd")


def ulysses_attn_bwd_timed(q_head, k_head, v_head, o_head, lse, do_head, position_ids, dq_head, dk_head, dv_head,
                           ws, events, rank: int = -1, softmax_scale: float = 0.0, stream=None) -> None:
    """ulysses_attn_bwd that also records five torch.cuda.Events around its
    kernels (before sample tables, statistics, dK/dV, dQ; after dQ)."""
    if len(events) != 5:
        raise ValueError("five events are needed")
    _check_attn(q_head, k_head, v_head, position_ids, o_head, lse, stream, do_head, dq_head, dk_head, dv_head,
                ws)
    shape = _attn_shape(q_head, k_head)
    handles = []
    for ev in events:
        if ev.cuda_event == 0:   # torch creates the handle lazily, at the first record
            ev.record(torch.cuda.current_stream() if stream is None else stream)
        handles.append(ev.cuda_event)
    arr = (ctypes.c_void_p * 5)(*handles)
    _check(lib.ulysses_attn_bwd_timed(_dev(q_head, "q_head"), _dev(k_head, "k_head"), _dev(v_head, "v_head"),
                                      _dev(o_head, "o_head"), _dtype_code(o_head), _dev(lse, "lse"),
                                      _dev(do_head, "do_head"), _dev(position_ids, "position_ids"),
                                      ctypes.byref(shape), rank, softmax_scale, _dev(dq_head, "dq_head"),
                                      _dev(dk_head, "dk_head"), _dev(dv_head, "dv_head"), _dtype_code(dq_head),
                                      _dev(ws, "ws"), ws.numel() * ws.element_size(), _stream(stream), arr),
           "ulysses_attn_bwd_timed")


def ulysses_sp_loss_aggregate(losses, shift_labels, loss, good, dlosses, ignore_index: int = -100,
                              stream=None) -> None:
    """Weighted aggregation of per-rank losses: losses float32[P], shift_labels
    int64[P][b][n/P] (seq-sharded); writes loss float32[1], good int64[P],
    dlosses float32[P]."""
    if losses.dtype != torch.float32 or loss.dtype != torch.float32 or dlosses.dtype != torch.float32:
        raise TypeError("losses, loss and dlosses must be float32")
    if shift_labels.dtype != torch.int64 or good.dtype != torch.int64:
        raise TypeError("shift_labels and good must be int64")
    if shift_labels.dim() != 3:
        raise ValueError("shift_labels must be [P][b][n/P]")
    P, b, m = shift_labels.shape
    if losses.numel() != P or good.numel() != P or dlosses.numel() != P or loss.numel() != 1:
        raise ValueError("losses, good and dlosses need P elements, loss one")
    _one_device(stream, losses=losses, shift_labels=shift_labels, loss=loss, good=good, dlosses=dlosses)
    _check(lib.ulysses_sp_loss_aggregate(_dev(losses, "losses"), _dev(shift_labels, "shift_labels"), b, m * P, P,
                                         ignore_index, _dev(loss, "loss"), _dev(good, "good"),
                                         _dev(dlosses, "dlosses"), _stream(stream)),
           "ulysses_sp_loss_aggregate")


def ulysses_attn_fwd_kv_range(q_head, k_head, v_head, position_ids, o_head, lse, ws, k_lo: int, k_hi: int,
                              rank: int = -1, softmax_scale: float = 0.0, stream=None) -> None:
    """Forward over the keys [k_lo, k_hi) only (one ring block)."""
    _check_attn(q_head, k_head, v_head, position_ids, o_head, lse, stream, ws=ws)
    shape = _attn_shape(q_head, k_head)
    _check(lib.ulysses_attn_fwd_kv_range(_dev(q_head, "q_head"), _dev(k_head, "k_head"), _dev(v_head, "v_head"),
                                         _dev(position_ids, "position_ids"), ctypes.byref(shape), rank,
                                         softmax_scale, k_lo, k_hi, _dev(o_head, "o_head"), _dtype_code(o_head),
                                         _dev(lse, "lse"), _dev(ws, "ws"), ws.numel() * ws.element_size(),
                                         _stream(stream)), "ulysses_attn_fwd_kv_range")


def ulysses_attn_bwd_kv_range(q_head, k_head, v_head, o_head, lse, do_head, position_ids, dq_head, dk_head, dv_head,
                              ws, k_lo: int, k_hi: int, rank: int = -1, softmax_scale: float = 0.0,
                              stream=None) -> None:
    """One key block's share of the backward, given the merged O and LSE."""
    _check_attn(q_head, k_head, v_head, position_ids, o_head, lse, stream, do_head, dq_head, dk_head, dv_head,
                ws)
    shape = _attn_shape(q_head, k_head)
    _check(lib.ulysses_attn_bwd_kv_range(_dev(q_head, "q_head"), _dev(k_head, "k_head"), _dev(v_head, "v_head"),
                                         _dev(o_head, "o_head"), _dtype_code(o_head), _dev(lse, "lse"),
                                         _dev(do_head, "do_head"), _dev(position_ids, "position_ids"),
                                         ctypes.byref(shape), rank, softmax_scale, k_lo, k_hi,
                                         _dev(dq_head, "dq_head"), _dev(dk_head, "dk_head"), _dev(dv_head, "dv_head"),
                                         _dtype_code(dq_head), _dev(ws, "ws"), ws.numel() * ws.element_size(),
                                         _stream(stream)), "ulysses_attn_bwd_kv_range")


def _check_block(q_blk, k_blk, v_blk, position_ids, o_blk, lse_blk, stream, do_blk=None, dq_blk=None, dk_blk=None,
                 dv_blk=None, ws=None):
    """Layouts of the block calls: Q-side rows q_rows, K-side rows k_rows."""
    if not isinstance(q_blk, torch.Tensor) or q_blk.dim() != 5 or not isinstance(k_blk, torch.Tensor) \
            or k_blk.dim() != 5:
        raise ValueError("q_blk / k_blk must be [P][b][rows][heads][d]")
    P, b, qr, hq, d = q_blk.shape
    kr, hkv = k_blk.shape[2], k_blk.shape[3]
    if not isinstance(position_ids, torch.Tensor) or position_ids.dim() != 2:
        raise ValueError("position_ids must be [b][n]")
    n = position_ids.shape[1]
    _expect(q_blk, (P, b, qr, hq, d), _BF16, "q_blk")
    _expect(k_blk, (P, b, kr, hkv, d), _BF16, "k_blk")
    _expect(v_blk, (P, b, kr, hkv, d), _BF16, "v_blk")
    _expect(position_ids, (b, n), _I64, "position_ids")
    _expect(o_blk, (P, b, qr, hq, d), _OUT, "o_blk")
    _expect(lse_blk, (P, b, hq, qr), _F32, "lse_blk")
    more = {}
    if do_blk is not None:
        _expect(do_blk, (P, b, qr, hq, d), _BF16, "do_blk")
        _expect(dq_blk, (P, b, qr, hq, d), _OUT, "dq_blk")
        _expect(dk_blk, (P, b, kr, hkv, d), (dq_blk.dtype,), "dk_blk")
        _expect(dv_blk, (P, b, kr, hkv, d), (dq_blk.dtype,), "dv_blk")
        more = dict(do_blk=do_blk, dq_blk=dq_blk, dk_blk=dk_blk, dv_blk=dv_blk)
    if ws is not None:
        more["ws"] = ws
    _one_device(stream, q_blk=q_blk, k_blk=k_blk, v_blk=v_blk, position_ids=position_ids, o_blk=o_blk,
                lse_blk=lse_blk, **more)
    return UlyShape(b, n, hq * P, hkv * P, d, P), qr, kr


def ulysses_attn_fwd_block(q_blk, k_blk, v_blk, position_ids, o_blk, lse_blk, ws, q_base: int, k_base: int,
                           softmax_scale: float = 0.0, stream=None) -> None:
    """Partial attention of the query rows [q_base, q_base + q_rows) over the
    keys [k_base, k_base + k_rows), both stored compactly."""
    shape, qr, kr = _check_block(q_blk, k_blk, v_blk, position_ids, o_blk, lse_blk, stream, ws=ws)
    _check(lib.ulysses_attn_fwd_block(_dev(q_blk, "q_blk"), _dev(k_blk, "k_blk"), _dev(v_blk, "v_blk"),
                                      _dev(position_ids, "position_ids"), ctypes.byref(shape), q_base, qr, k_base, kr,
                                      softmax_scale, _dev(o_blk, "o_blk"), _dtype_code(o_blk), _dev(lse_blk, "lse_blk"),
                                      _dev(ws, "ws"), ws.numel() * ws.element_size(), _stream(stream)),
           "ulysses_attn_fwd_block")


def ulysses_attn_bwd_block(q_blk, k_blk, v_blk, o_blk, lse_blk, do_blk, position_ids, dq_blk, dk_blk, dv_blk, ws,
                           q_base: int, k_base: int, softmax_scale: float = 0.0, stream=None) -> None:
    """The key block's share of dQ and the query block's dK / dV contributions,
    given the query block's merged O and LSE."""
    shape, qr, kr = _check_block(q_blk, k_blk, v_blk, position_ids, o_blk, lse_blk, stream, do_blk, dq_blk, dk_blk,
                                 dv_blk, ws)
    _check(lib.ulysses_attn_bwd_block(_dev(q_blk, "q_blk"), _dev(k_blk, "k_blk"), _dev(v_blk, "v_blk"),
                                      _dev(o_blk, "o_blk"), _dtype_code(o_blk), _dev(lse_blk, "lse_blk"),
                                      _dev(do_blk, "do_blk"), _dev(position_ids, "position_ids"), ctypes.byref(shape),
                                      q_base, qr, k_base, kr, softmax_scale, _dev(dq_blk, "dq_blk"),
                                      _dev(dk_blk, "dk_blk"), _dev(dv_blk, "dv_blk"), _dtype_code(dq_blk),
                                      _dev(ws, "ws"), ws.numel() * ws.element_size(), _stream(stream)),
           "ulysses_attn_bwd_block")


def ulysses_accumulate(dst: torch.Tensor, src: torch.Tensor, stream=None) -> None:
    """dst += src (float32 tensors of the same shape)."""
    _expect(src, tuple(dst.shape), _F32, "src")
    _expect(dst, tuple(dst.shape), _F32, "dst")
    _one_device(stream, dst=dst, src=src)
    _check(lib.ulysses_accumulate(_dev(dst, "dst"), _dev(src, "src"), dst.numel(), _stream(stream)),
           "ulysses_accumulate")


def ulysses_attn_lse_merge(o_parts, lse_parts, o_head, lse, h_kv: int, stream=None) -> None:
    """Merge B partial results: o_parts float32 (B, P, b, n, h, d), lse_parts
    float32 (B, P, b, h, n) -> o_head (P, b, n, h, d), lse (P, b, h, n)."""
    if o_parts.dtype != torch.float32 or lse_parts.dtype != torch.float32 or lse.dtype != torch.float32:
        raise TypeError("o_parts, lse_parts and lse must be float32")
    if o_parts.dim() != 6:
        raise ValueError("o_parts must be [B][P][b][n][h_q/P][d]")
    B, P, b, n, h, d = o_parts.shape
    _expect(lse_parts, (B, P, b, h, n), _F32, "lse_parts")
    _expect(o_head, (P, b, n, h, d), _OUT, "o_head")
    _expect(lse, (P, b, h, n), _F32, "lse")
    _one_device(stream, o_parts=o_parts, lse_parts=lse_parts, o_head=o_head, lse=lse)
    shape = UlyShape(b, n, h * P, h_kv, d, P)
    _check(lib.ulysses_attn_lse_merge(_dev(o_parts, "o_parts"), _dev(lse_parts, "lse_parts"), B,
                                      ctypes.byref(shape), _dev(o_head, "o_head"), _dtype_code(o_head),
                                      _dev(lse, "lse"), _stream(stream)), "ulysses_attn_lse_merge")


def ulysses_debug_status(stream=None) -> int:
    """Debug build: synchronize, then read and clear the re-layout kernels'
    bounds record (0 = no index outside its buffer, 6 = ULY_ERR_BOUNDS).
    The release build has no checks and raises UlyssesError(ULY_ERR_UNSUPPORTED)."""
    code = ctypes.c_int32(-1)
    _check(lib.ulysses_debug_status(_stream(stream), ctypes.byref(code)), "ulysses_debug_status")
    return int(code.value)


def ulysses_workspace_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronize, then read and clear the workspace status word (0 = ok)."""
    code = ctypes.c_int32(-1)
    _check(lib.ulysses_workspace_status(_dev(ws, "ws"), _stream(stream), ctypes.byref(code)),
           "ulysses_workspace_status")
    return int(code.value)


def ulysses_selftest_wait_timeout(ws: torch.Tensor, limit_ns: int, stream=None) -> None:
    """Run the attention kernels' bounded-wait failure path on purpose: one
    CTA waits on a barrier nothing arrives at, gives up after limit_ns and
    records ULY_ERR_TIMEOUT in ws's status word (read it with
    ulysses_workspace_status)."""
    if not isinstance(ws, torch.Tensor) or ws.dtype != torch.uint8:
        raise TypeError("ws must be a uint8 CUDA tensor")
    _one_device(stream, ws=ws)
    _check(lib.ulysses_selftest_wait_timeout(_dev(ws, "ws"), ws.numel(), int(limit_ns), _stream(stream)),
           "ulysses_selftest_wait_timeout")


# ----------------------------------------------------------------------------- between GPUs
def _ptr_array(ptrs):
    arr = (ctypes.c_void_p * len(ptrs))()
    for i, p in enumerate(ptrs):
        arr[i] = int(p)
    return arr


def ulysses_seq_to_head_push(x_seq: torch.Tensor, dst_heads, dst_flags, rank: int, P: int, epoch: int,
                             ws: torch.Tensor, stream=None) -> None:
    """Store this rank's seq shard x_seq (b, n/P, H, d) into every rank's head
    buffer (b, n, H/P, d), then release dst_flags[s][rank] = epoch.  dst_heads /
    dst_flags: P device addresses (ints; peer-mapped for other GPUs), or
    tensors on this process's device (one GPU standing in for all ranks)."""
    b, m, H, d = x_seq.shape
    _dev(x_seq, "x_seq")
    _dev(ws, "ws")
    heads = [t.data_ptr() if isinstance(t, torch.Tensor) else int(t) for t in dst_heads]
    flags = [t.data_ptr() if isinstance(t, torch.Tensor) else int(t) for t in dst_flags]
    for t in list(dst_heads) + list(dst_flags):
        if isinstance(t, torch.Tensor):
            _one_device(stream, dst=t)
    if len(heads) != P or len(flags) != P:
        raise ValueError("dst_heads and dst_flags need one entry per rank")
    for t in dst_heads:
        if isinstance(t, torch.Tensor):
            _expect(t, (b, m * P, H // P, d), (x_seq.dtype,), "dst_heads[s]")
    _check(lib.ulysses_seq_to_head_push(x_seq.data_ptr(), _ptr_array(heads), _ptr_array(flags), rank, b, m * P, H, d,
                                        P, _dtype_code(x_seq), epoch, ws.data_ptr(), ws.numel() * ws.element_size(),
                                        _stream(stream)), "ulysses_seq_to_head_push")


def ulysses_head_to_seq_push(x_head: torch.Tensor, dst_seqs, dst_flags, rank: int, P: int, epoch: int,
                             ws: torch.Tensor, stream=None) -> None:
    """Store this rank's head slice x_head (b, n, H/P, d) into every rank's seq
    shard (b, n/P, H, d), then release dst_flags[s][rank] = epoch."""
    b, n, h, d = x_head.shape
    _dev(x_head, "x_head")
    _dev(ws, "ws")
    seqs = [t.data_ptr() if isinstance(t, torch.Tensor) else int(t) for t in dst_seqs]
    flags = [t.data_ptr() if isinstance(t, torch.Tensor) else int(t) for t in dst_flags]
    for t in list(dst_seqs) + list(dst_flags):
        if isinstance(t, torch.Tensor):
            _one_device(stream, dst=t)
    if len(seqs) != P or len(flags) != P:
        raise ValueError("dst_seqs and dst_flags need one entry per rank")
    for t in dst_seqs:
        if isinstance(t, torch.Tensor):
            _expect(t, (b, n // P, h * P, d), (x_head.dtype,), "dst_seqs[s]")
    _check(lib.ulysses_head_to_seq_push(x_head.data_ptr(), _ptr_array(seqs), _ptr_array(flags), rank, b, n, h * P, d,
                                        P, _dtype_code(x_head), epoch, ws.data_ptr(), ws.numel() * ws.element_size(),
                                        _stream(stream)), "ulysses_head_to_seq_push")


def ulysses_wait_flags(flags: torch.Tensor, epoch: int, limit_ns: int, ws: torch.Tensor, stream=None) -> None:
    """Enqueue a bounded wait until every slot of flags (uint32 as int32) holds epoch."""
    if flags.dtype not in (torch.int32,) or flags.dim() != 1:
        raise TypeError("flags must be a 1-D int32 tensor (uint32 slots)")
    _one_device(stream, flags=flags, ws=ws)
    _check(lib.ulysses_wait_flags(flags.data_ptr(), flags.numel(), epoch, int(limit_ns), ws.data_ptr(),
                                  _stream(stream)), "ulysses_wait_flags")


def ulysses_release_flags(slot_addrs, epoch: int, stream=None) -> None:
    """Store epoch into each uint32 slot (device addresses), with release
    semantics at system scope, after everything enqueued before it."""
    _check(lib.ulysses_release_flags(_ptr_array(slot_addrs), len(slot_addrs), epoch, _stream(stream)),
           "ulysses_release_flags")


def ulysses_ipc_handle(t: torch.Tensor) -> bytes:
    """The CUDA IPC handle (64 bytes) of the allocation at t's address."""
    buf = ctypes.create_string_buffer(64)
    _check(lib.ulysses_ipc_handle(_dev(t, "t"), buf), "ulysses_ipc_handle")
    return buf.raw


def ulysses_ipc_open(handle: bytes) -> int:
    """Open another process's allocation; returns its device address here."""
    if len(handle) != 64:
        raise ValueError("a CUDA IPC handle is 64 bytes")
    p = ctypes.c_void_p()
    _check(lib.ulysses_ipc_open(handle, ctypes.byref(p)), "ulysses_ipc_open")
    return int(p.value)


def ulysses_ipc_close(addr: int) -> None:
    _check(lib.ulysses_ipc_close(ctypes.c_void_p(addr)), "ulysses_ipc_close")


# ----------------------------------------------------------------------------- host to host
def _host(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


class LayerStepHost:
    """ulysses_layer_step_host with its device buffer, streams and events:
    one layer step from (pinned) host tensors to host tensors."""

    def __init__(self, b: int, n: int, h_q: int, h_kv: int, d: int, P: int, device=None):
        self.shape = UlyShape(b, n, h_q, h_kv, d, P)
        self.device = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        nbytes = int(lib.ulysses_layer_step_host_bytes(ctypes.byref(self.shape)))
        if nbytes == 0:
            raise ValueError("shape not accepted by the library")
        # zeroed once: the attention workspaces' status words inside it start clear
        self.dev = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        self.h2d, self.d2h = torch.cuda.Stream(self.device), torch.cuda.Stream(self.device)
        self.events = [torch.cuda.Event() for _ in range(3)]

    def step(self, q_seq, k_seq, v_seq, do_seq, position_ids, o_seq, dq_seq, dk_seq, dv_seq,
             softmax_scale: float = 0.0, stream=None) -> None:
        P, b, n, hq, hkv, d = (self.shape.P, self.shape.b, self.shape.n, self.shape.h_q, self.shape.h_kv,
                               self.shape.d)
        m = n // P
        _expect(q_seq, (P, b, m, hq, d), _BF16, "q_seq")
        _expect(k_seq, (P, b, m, hkv, d), _BF16, "k_seq")
        _expect(v_seq, (P, b, m, hkv, d), _BF16, "v_seq")
        _expect(do_seq, (P, b, m, hq, d), _BF16, "do_seq")
        _expect(position_ids, (b, n), _I64, "position_ids")
        _expect(o_seq, (P, b, m, hq, d), _F32, "o_seq")
        _expect(dq_seq, (P, b, m, hq, d), _F32, "dq_seq")
        _expect(dk_seq, (P, b, m, hkv, d), _F32, "dk_seq")
        _expect(dv_seq, (P, b, m, hkv, d), _F32, "dv_seq")
        for e in self.events:   # record once so the handles exist (a never-recorded event is complete)
            if e.cuda_event == 0:
                e.record(self.d2h)
        evs = (ctypes.c_void_p * 3)(*[e.cuda_event for e in self.events])
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        _check(lib.ulysses_layer_step_host(_host(q_seq, "q_seq"), _host(k_seq, "k_seq"), _host(v_seq, "v_seq"),
                                           _host(do_seq, "do_seq"), _host(position_ids, "position_ids"),
                                           ctypes.byref(self.shape), softmax_scale, _host(o_seq, "o_seq"),
                                           _host(dq_seq, "dq_seq"), _host(dk_seq, "dk_seq"), _host(dv_seq, "dv_seq"),
                                           self.dev.data_ptr(), self.dev.numel(), ctypes.c_void_p(s.cuda_stream),
                                           ctypes.c_void_p(self.h2d.cuda_stream), ctypes.c_void_p(self.d2h.cuda_stream),
                                           evs), "ulysses_layer_step_host")

    def done_event(self) -> torch.cuda.Event:
        """Completes once every output of the last step is on the host."""
        return self.events[2]

    def status(self) -> int:
        code = ctypes.c_int32(-1)
        _check(lib.ulysses_layer_status(self.dev.data_ptr(), ctypes.byref(self.shape),
                                        ctypes.c_void_p(torch.cuda.current_stream(self.device).cuda_stream),
                                        ctypes.byref(code)), "ulysses_layer_status")
        return int(code.value)

