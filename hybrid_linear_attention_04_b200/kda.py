"""Python binding of libkda (include/kda.h): argument marshalling only.

Each function takes torch tensors that already live where the C ABI wants
them (device tensors for device pointers, Python sequences or CPU tensors for
the _h host arrays), reads their shapes into a ``kda_dims``, and calls the
library function of the same name on the current CUDA stream. Every step of
the computation runs in libkda's kernels; there is no fallback of any kind. A
missing library raises ``KDAError`` at import of this module's first call.

The C functions take plain pointers and cannot see buffer sizes, so each
function here first checks every tensor's dtype, trailing dimensions and row
count against the rows the call reads or writes (``KDAError`` status 1), so
that a wrongly shaped argument fails on the host instead of addressing memory
outside its buffer on the device.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import numpy as np
import torch

_LIB_PATH = Path(__file__).resolve().parent / "libkda.so"
_lib = None

KDA_OK = 0
KDA_IO_BF16, KDA_IO_FP32 = 0, 1
STATUS_NAMES = {0: "KDA_OK", 1: "KDA_ERR_INVALID", 2: "KDA_ERR_UNSUPPORTED", 3: "KDA_ERR_ALIGN",
                4: "KDA_ERR_WORKSPACE", 5: "KDA_ERR_CUDA", 6: "KDA_ERR_TIMEOUT", 7: "KDA_ERR_RANGE"}


class KDAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class kda_dims(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("dk", ctypes.c_int32), ("dv", ctypes.c_int32),
                ("chunk", ctypes.c_int32), ("io", ctypes.c_int32), ("scale", ctypes.c_float)]


class kda_conv(ctypes.Structure):
    _fields_ = [("taps", ctypes.c_int32), ("w_q", ctypes.c_void_p), ("w_k", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I32, _I64 = ctypes.c_int32, ctypes.c_int64

_SIGNATURES = {
    "kda_snapshot_plan": (_I32, [_I32, _P, _P, _I32, _P, _P]),
    "kda_prefill_workspace_size": (_I32, [_P, _I32, _P, _P]),
    "kda_prefill": (_I32, [_P, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P,
                           ctypes.c_size_t, _P]),
    "kda_prefill_noalloc": (_I32, [_P, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P]),
    "kda_prefill_noalloc_capacity": (ctypes.c_size_t, []),
    "kda_decode": (_I32, [_P, _I32, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _P]),
    "kda_verify": (_I32, [_P, _I32, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _P, _P]),
    "kda_verify_commit": (_I32, [_P, _I32, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _I64, _P, _P,
                                 _P, _P, _P, _P, _P, _P, _I32, _P, _P, _P]),
    "kda_snapshot": (_I32, [_I32, _P, _P, _P, _I64, _P, _I64, _I32, _I32, _I32, _P]),
    "kda_state_map_apply": (_I32, [_I64, _I32, _I32, _P, _P, _P, _P, _P]),
    "kda_qk_frontend": (_I32, [_P, _P, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P]),
    "kda_decode_conv": (_I32, [_P, _P, _I32, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _P, _P]),
    "kda_verify_conv": (_I32, [_P, _P, _I32, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _P, _P, _P,
                               _P]),
    "kda_verify_commit_conv": (_I32, [_P, _P, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P,
                                      _P, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _P,
                                      _P]),
    "kda_status_string": (ctypes.c_char_p, [_I32]),
    "kda_check_device_status": (_I32, [_P]),
    "kda_launch_count": (_I64, []),
    "kda_last_cuda_error": (ctypes.c_char_p, []),
    "kda_test_fail_next_launches": (None, [_I32]),
    "kda_test_wait_timeout": (_I32, [_I32, _P]),
    "kda_internal_force_prefill_path": (None, [_I32]),
}


def library_path() -> Path:
    return _LIB_PATH


def lib():
    """The loaded libkda (ctypes). Raises KDAError if the library is missing."""
    global _lib
    if _lib is None:
        if not _LIB_PATH.exists():
            raise KDAError(-1, f"libkda.so not built at {_LIB_PATH} "
                               "(python -m hybrid_linear_attention_04_b200.build)")
        L = ctypes.CDLL(str(_LIB_PATH))
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != KDA_OK:
        if status == 5:
            where = f"{where} ({lib().kda_last_cuda_error().decode()})"
        raise KDAError(status, where)


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _dptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise KDAError(1, "device tensor expected")
    if not t.is_contiguous():
        raise KDAError(1, "contiguous tensor expected")
    return ctypes.c_void_p(t.data_ptr())


def _host_array(x, dtype):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x), dtype=dtype)


def _hptr(a):
    # the caller keeps `a` alive for the duration of the library call
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _io(t):
    if t.dtype == torch.bfloat16:
        return KDA_IO_BF16
    if t.dtype == torch.float32:
        return KDA_IO_FP32
    raise KDAError(2, f"unsupported io dtype {t.dtype}")


def _dims(q, v, chunk=0, scale=0.0):
    H, dk = q.shape[-2], q.shape[-1]
    return kda_dims(H, dk, v.shape[-1], chunk, _io(q), float(scale))


_F32, _I32T, _I64T, _U8 = torch.float32, torch.int32, torch.int64, torch.uint8


def _expect(t, name, dtype, rows, tail, required=True):
    """``t`` must be a tensor of ``dtype`` shaped [n, *tail] with n >= rows (the rows the
    call reads or writes). None passes where the call touches no row of it (rows == 0)
    or the argument is optional (required=False)."""
    if t is None:
        if required and rows > 0:
            raise KDAError(1, f"{name} is required")
        return
    try:
        shape, dt = t.shape, t.dtype
    except AttributeError:
        raise KDAError(1, f"{name} must be a tensor") from None
    if dt is not dtype or len(shape) != len(tail) + 1 or shape[1:] != tail or shape[0] < rows:
        if dt is not dtype:
            raise KDAError(1, f"{name} must be {dtype}, not {dt}")
        if len(shape) != len(tail) + 1 or shape[1:] != tail:
            raise KDAError(1, f"{name} must be shaped [n, {', '.join(map(str, tail))}], not {list(shape)}")
        raise KDAError(1, f"{name} has {shape[0]} rows; the call uses {rows}")


def _expect_tokens(q, k, v, g, beta, o, T, tag=""):
    """Packed token arrays of T rows: q, k [T, H, dk] and v, o [T, H, dv] in q's I/O type,
    g [T, H, dk] and beta [T, H] fp32 (o may be None where the call writes none)."""
    _io(q)
    io = q.dtype
    H, dk = q.shape[-2], q.shape[-1]
    dv = v.shape[-1] if v is not None else dk
    hk, hv = (H, dk), (H, dv)
    _expect(q, tag + "q", io, T, hk)
    _expect(k, tag + "k", io, T, hk)
    _expect(v, tag + "v", io, T, hv)
    _expect(g, tag + "g", _F32, T, hk)
    _expect(beta, tag + "beta", _F32, T, (H,))
    if o is not None:
        _expect(o, tag + "o", io, T, hv)
    return H, dk, dv


def _expect_len(a, name, n):
    if a is not None and len(a) != n:
        raise KDAError(1, f"{name} has {len(a)} entries; the call has {n} sequences")


def _cu(x, name):
    cu = _host_array(x, np.int32)
    if cu is None or cu.ndim != 1 or len(cu) < 1:
        raise KDAError(1, f"{name} must hold n_seq + 1 >= 1 offsets")
    return cu


def _snap_rows(cu, sp, snap_interval):
    if snap_interval <= 0:
        return 0
    return int(kda_snapshot_plan(cu, sp, snap_interval)[0][-1])


def kda_snapshot_plan(cu_seqlens, start_pos=None, snap_interval=0):
    """Snapshot rows per sequence: returns (offsets int64 [n_seq+1], positions int64 [total])."""
    cu = _host_array(cu_seqlens, np.int32)
    n_seq = len(cu) - 1
    sp = _host_array(start_pos, np.int64)
    offs = np.zeros(n_seq + 1, dtype=np.int64)
    _check(lib().kda_snapshot_plan(n_seq, _hptr(cu), _hptr(sp), snap_interval, _hptr(offs), None),
           "kda_snapshot_plan")
    pos = np.zeros(int(offs[-1]), dtype=np.int64)
    _check(lib().kda_snapshot_plan(n_seq, _hptr(cu), _hptr(sp), snap_interval, _hptr(offs),
                                   _hptr(pos)), "kda_snapshot_plan")
    return offs, pos


def kda_prefill_workspace_size(q, v, cu_seqlens, chunk=64) -> int:
    """Workspace bytes kda_prefill can use for these shapes (see include/kda.h)."""
    cu = _host_array(cu_seqlens, np.int32)
    dims = _dims(q, v, chunk)
    n = ctypes.c_size_t(0)
    _check(lib().kda_prefill_workspace_size(ctypes.byref(dims), len(cu) - 1, _hptr(cu),
                                            ctypes.byref(n)), "kda_prefill_workspace_size")
    return int(n.value)


def _expect_prefill(q, k, v, g, beta, cu, o, state_out, state_in, sp, snap_interval, snapshots):
    n = len(cu) - 1
    H, dk, dv = _expect_tokens(q, k, v, g, beta, o, int(cu[-1]))
    _expect_len(sp, "start_pos", n)
    _expect(state_in, "state_in", _F32, n, (H, dk, dv), required=False)
    _expect(state_out, "state_out", _F32, n, (H, dk, dv), required=False)
    _expect(snapshots, "snapshots", _F32, _snap_rows(cu, sp, snap_interval), (H, dk, dv))


def kda_prefill(q, k, v, g, beta, cu_seqlens, o, state_out=None, state_in=None, start_pos=None,
                snap_interval=0, snapshots=None, chunk=64, scale=0.0, stream=None,
                workspace="auto"):
    """Packed variable-length chunked prefill (see include/kda.h).

    ``workspace``: a device uint8 tensor of at least kda_prefill_workspace_size
    bytes, ``None`` for the single-launch kernel without scratch memory, or
    ``"auto"`` to allocate one of the required size on q's device (through
    PyTorch's allocator) for this call.
    """
    cu = _cu(cu_seqlens, "cu_seqlens")
    sp = _host_array(start_pos, np.int64)
    _expect_prefill(q, k, v, g, beta, cu, o, state_out, state_in, sp, snap_interval, snapshots)
    dims = _dims(q, v, chunk, scale)
    if isinstance(workspace, str):
        if workspace != "auto":
            raise KDAError(1, f"workspace must be a tensor, None or 'auto', not {workspace!r}")
        nbytes = kda_prefill_workspace_size(q, v, cu, chunk)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().kda_prefill(ctypes.byref(dims), len(cu) - 1, _hptr(cu), _hptr(sp), _dptr(q),
                             _dptr(k), _dptr(v), _dptr(g), _dptr(beta), _dptr(state_in),
                             _dptr(state_out), _dptr(o), int(snap_interval), _dptr(snapshots),
                             _dptr(workspace), ws_bytes, _stream(stream)), "kda_prefill")


def kda_prefill_noalloc(q, k, v, g, beta, cu_seqlens, o, state_out=None, state_in=None,
                        start_pos=None, snap_interval=0, snapshots=None, chunk=64, scale=0.0,
                        stream=None):
    """kda_prefill on the library's fixed device scratch: no allocation (see include/kda.h)."""
    cu = _cu(cu_seqlens, "cu_seqlens")
    sp = _host_array(start_pos, np.int64)
    _expect_prefill(q, k, v, g, beta, cu, o, state_out, state_in, sp, snap_interval, snapshots)
    dims = _dims(q, v, chunk, scale)
    _check(lib().kda_prefill_noalloc(ctypes.byref(dims), len(cu) - 1, _hptr(cu), _hptr(sp),
                                     _dptr(q), _dptr(k), _dptr(v), _dptr(g), _dptr(beta),
                                     _dptr(state_in), _dptr(state_out), _dptr(o),
                                     int(snap_interval), _dptr(snapshots), _stream(stream)),
           "kda_prefill_noalloc")


def kda_prefill_noalloc_capacity() -> int:
    return int(lib().kda_prefill_noalloc_capacity())


def kda_decode(q, k, v, g, beta, slots, state_pool, o, scale=0.0, stream=None):
    """One decode token per sequence, states updated in place (see include/kda.h)."""
    H, dk, dv = _expect_tokens(q, k, v, g, beta, o, q.shape[0])
    _expect(slots, "slots", _I32T, q.shape[0], ())
    _expect(state_pool, "state_pool", _F32, 0, (H, dk, dv))
    dims = _dims(q, v, 0, scale)
    _check(lib().kda_decode(ctypes.byref(dims), q.shape[0], _dptr(q), _dptr(k), _dptr(v),
                            _dptr(g), _dptr(beta), _dptr(slots), state_pool.shape[0],
                            _dptr(state_pool), _dptr(o), _stream(stream)), "kda_decode")


def kda_verify(q, k, v, g, beta, cu_draft, slots, state_pool, token_states, o, scale=0.0,
               stream=None):
    """Speculative verify with per-token states (see include/kda.h)."""
    cu = _cu(cu_draft, "cu_draft")
    T = int(cu[-1])
    H, dk, dv = _expect_tokens(q, k, v, g, beta, o, T)
    _expect(slots, "slots", _I32T, len(cu) - 1, ())
    _expect(state_pool, "state_pool", _F32, 0, (H, dk, dv))
    _expect(token_states, "token_states", _F32, T, (H, dk, dv))
    dims = _dims(q, v, 0, scale)
    _check(lib().kda_verify(ctypes.byref(dims), len(cu) - 1, _hptr(cu), _dptr(q), _dptr(k),
                            _dptr(v), _dptr(g), _dptr(beta), _dptr(slots), state_pool.shape[0],
                            _dptr(state_pool), _dptr(token_states), _dptr(o), _stream(stream)),
           "kda_verify")


def _expect_commit(pv, n_accept, cp, q, k, v, g, beta, cd, slots, state_pool, o, pos, snap_row,
                   snapshots, commit_new, conv):
    n, Tp, T = len(cd) - 1, int(cp[-1]), int(cd[-1])
    H, dk, dv = _expect_tokens(q, k, v, g, beta, o, T)
    _expect(pv.get("k"), "prev k", q.dtype, Tp, (H, dk))
    _expect(pv.get("v"), "prev v", q.dtype, Tp, (H, dv))
    _expect(pv.get("g"), "prev g", _F32, Tp, (H, dk))
    _expect(pv.get("beta"), "prev beta", _F32, Tp, (H,))
    if conv:
        _expect(pv.get("q"), "prev q", q.dtype, Tp, (H, dk))
    _expect(n_accept, "n_accept", _I32T, n, ())
    _expect(pos, "pos", _I64T, n, (), required=False)
    _expect(snap_row, "snap_row", _I64T, n, (), required=False)
    _expect(snapshots, "snapshots", _F32, 0, (H, dk, dv), required=False)
    _expect(commit_new, "commit_new", _U8, n, (), required=False)
    _expect(slots, "slots", _I32T, n, ())
    _expect(state_pool, "state_pool", _F32, 0, (H, dk, dv))
    return H, dk, dv


def kda_verify_commit(prev, n_accept, cu_prev, q, k, v, g, beta, cu_draft, slots, state_pool, o,
                      pos=None, snap_interval=0, snap_row=None, snapshots=None, commit_new=None,
                      scale=0.0, stream=None):
    """Speculative step with the previous step's commit fused in (see include/kda.h).

    ``prev``: dict of the previous batch's device tensors k, v, g, beta (packed by
    ``cu_prev``), or None when it is empty; ``n_accept``: device int32 [n_seq];
    ``commit_new``: device uint8 [n_seq] (mixed step: commit this step's tokens too).
    """
    cp = _cu(cu_prev, "cu_prev")
    cd = _cu(cu_draft, "cu_draft")
    if len(cp) != len(cd):
        raise KDAError(1, "cu_prev and cu_draft must describe the same sequences")
    pv = prev or {}
    _expect_commit(pv, n_accept, cp, q, k, v, g, beta, cd, slots, state_pool, o, pos, snap_row,
                   snapshots, commit_new, conv=False)
    dims = _dims(q, v, 0, scale)
    n_rows = 0 if snapshots is None else snapshots.shape[0]
    _check(lib().kda_verify_commit(
        ctypes.byref(dims), len(cd) - 1, _hptr(cp), _dptr(pv.get("k")), _dptr(pv.get("v")),
        _dptr(pv.get("g")), _dptr(pv.get("beta")), _dptr(n_accept), _dptr(pos), int(snap_interval),
        _dptr(snap_row), _dptr(snapshots), n_rows, _hptr(cd), _dptr(q), _dptr(k), _dptr(v),
        _dptr(g), _dptr(beta), _dptr(commit_new), _dptr(slots), state_pool.shape[0],
        _dptr(state_pool), _dptr(o), _stream(stream)), "kda_verify_commit")


def _conv_check(w_q, w_k, H=None, dk=None):
    if (w_q.shape != w_k.shape or w_q.dtype != torch.float32 or w_k.dtype != torch.float32
            or w_q.dim() != 3 or (H is not None and tuple(w_q.shape[:2]) != (H, dk))):
        raise KDAError(1, "conv weights must be fp32 [H, dk, taps], the same for q and k")


def _conv(w_q, w_k, H=None, dk=None):
    """kda_conv for weight tensors [H, dk, taps] (fp32, device)."""
    _conv_check(w_q, w_k, H, dk)
    _dptr(w_q), _dptr(w_k)
    return kda_conv(int(w_q.shape[-1]), w_q.data_ptr(), w_k.data_ptr())


def _conv_tail(H, dk, w):
    return (2, H, dk, int(w.shape[-1]) - 1)


def kda_qk_frontend(q_raw, k_raw, w_q, w_k, cu_seqlens, q_out, k_out, conv_in=None,
                    conv_out=None, start_pos=None, snap_interval=0, conv_snapshots=None,
                    chunk=64, stream=None):
    """Short conv + Swish + L2 front-end of a packed prefill batch (see include/kda.h)."""
    cu = _cu(cu_seqlens, "cu_seqlens")
    sp = _host_array(start_pos, np.int64)
    n, T = len(cu) - 1, int(cu[-1])
    _io(q_raw)
    H, dk = q_raw.shape[-2], q_raw.shape[-1]
    for t, name in ((q_raw, "q_raw"), (k_raw, "k_raw"), (q_out, "q_out"), (k_out, "k_out")):
        _expect(t, name, q_raw.dtype, T, (H, dk))
    _expect_len(sp, "start_pos", n)
    _conv_check(w_q, w_k, H, dk)
    ct = _conv_tail(H, dk, w_q)
    _expect(conv_in, "conv_in", _F32, n, ct, required=False)
    _expect(conv_out, "conv_out", _F32, n, ct, required=False)
    _expect(conv_snapshots, "conv_snapshots", _F32, _snap_rows(cu, sp, snap_interval), ct,
            required=False)
    conv = _conv(w_q, w_k, H, dk)
    dims = _dims(q_raw, q_raw, chunk)
    _check(lib().kda_qk_frontend(ctypes.byref(dims), ctypes.byref(conv), len(cu) - 1, _hptr(cu),
                                 _hptr(sp), _dptr(q_raw), _dptr(k_raw), _dptr(conv_in),
                                 _dptr(conv_out), _dptr(q_out), _dptr(k_out), int(snap_interval),
                                 _dptr(conv_snapshots), _stream(stream)), "kda_qk_frontend")


def kda_decode_conv(q, k, v, g, beta, slots, state_pool, conv_pool, o, w_q, w_k, scale=0.0,
                    stream=None):
    """kda_decode with the q/k front-end fused in (raw q, k; see include/kda.h)."""
    H, dk, dv = _expect_tokens(q, k, v, g, beta, o, q.shape[0])
    _expect(slots, "slots", _I32T, q.shape[0], ())
    _expect(state_pool, "state_pool", _F32, 0, (H, dk, dv))
    _conv_check(w_q, w_k, H, dk)
    _expect(conv_pool, "conv_pool", _F32, state_pool.shape[0], _conv_tail(H, dk, w_q))
    conv = _conv(w_q, w_k, H, dk)
    dims = _dims(q, v, 0, scale)
    _check(lib().kda_decode_conv(ctypes.byref(dims), ctypes.byref(conv), q.shape[0], _dptr(q),
                                 _dptr(k), _dptr(v), _dptr(g), _dptr(beta), _dptr(slots),
                                 state_pool.shape[0], _dptr(state_pool), _dptr(conv_pool),
                                 _dptr(o), _stream(stream)), "kda_decode_conv")


def kda_verify_conv(q, k, v, g, beta, cu_draft, slots, state_pool, conv_pool, token_states, o,
                    w_q, w_k, conv_token_states=None, scale=0.0, stream=None):
    """kda_verify with the q/k front-end fused in (see include/kda.h)."""
    cu = _cu(cu_draft, "cu_draft")
    T = int(cu[-1])
    H, dk, dv = _expect_tokens(q, k, v, g, beta, o, T)
    _expect(slots, "slots", _I32T, len(cu) - 1, ())
    _expect(state_pool, "state_pool", _F32, 0, (H, dk, dv))
    _expect(token_states, "token_states", _F32, T, (H, dk, dv))
    _conv_check(w_q, w_k, H, dk)
    ct = _conv_tail(H, dk, w_q)
    _expect(conv_pool, "conv_pool", _F32, state_pool.shape[0], ct)
    _expect(conv_token_states, "conv_token_states", _F32, T, ct, required=False)
    conv = _conv(w_q, w_k, H, dk)
    dims = _dims(q, v, 0, scale)
    _check(lib().kda_verify_conv(ctypes.byref(dims), ctypes.byref(conv), len(cu) - 1, _hptr(cu),
                                 _dptr(q), _dptr(k), _dptr(v), _dptr(g), _dptr(beta),
                                 _dptr(slots), state_pool.shape[0], _dptr(state_pool),
                                 _dptr(conv_pool), _dptr(token_states),
                                 _dptr(conv_token_states), _dptr(o), _stream(stream)),
           "kda_verify_conv")


def kda_verify_commit_conv(prev, n_accept, cu_prev, q, k, v, g, beta, cu_draft, slots,
                           state_pool, conv_pool, o, w_q, w_k, pos=None, snap_interval=0,
                           snap_row=None, snapshots=None, conv_snapshots=None, commit_new=None,
                           scale=0.0, stream=None):
    """kda_verify_commit with the q/k front-end fused in; ``prev`` holds raw q too."""
    cp = _cu(cu_prev, "cu_prev")
    cd = _cu(cu_draft, "cu_draft")
    if len(cp) != len(cd):
        raise KDAError(1, "cu_prev and cu_draft must describe the same sequences")
    pv = prev or {}
    H, dk, dv = _expect_commit(pv, n_accept, cp, q, k, v, g, beta, cd, slots, state_pool, o, pos,
                               snap_row, snapshots, commit_new, conv=True)
    _conv_check(w_q, w_k, H, dk)
    ct = _conv_tail(H, dk, w_q)
    _expect(conv_pool, "conv_pool", _F32, state_pool.shape[0], ct)
    n_rows = 0 if snapshots is None else snapshots.shape[0]
    _expect(conv_snapshots, "conv_snapshots", _F32, n_rows if snapshots is not None else 0, ct,
            required=False)
    conv = _conv(w_q, w_k, H, dk)
    dims = _dims(q, v, 0, scale)
    _check(lib().kda_verify_commit_conv(
        ctypes.byref(dims), ctypes.byref(conv), len(cd) - 1, _hptr(cp), _dptr(pv.get("q")),
        _dptr(pv.get("k")), _dptr(pv.get("v")), _dptr(pv.get("g")), _dptr(pv.get("beta")),
        _dptr(n_accept), _dptr(pos), int(snap_interval), _dptr(snap_row), _dptr(snapshots),
        _dptr(conv_snapshots), n_rows, _hptr(cd), _dptr(q), _dptr(k), _dptr(v), _dptr(g),
        _dptr(beta), _dptr(commit_new), _dptr(slots), state_pool.shape[0], _dptr(state_pool),
        _dptr(conv_pool), _dptr(o), _stream(stream)), "kda_verify_commit_conv")


def kda_state_map_apply(M, X, out, N=None, stream=None):
    """out = M X + N per leading index (see include/kda.h): M [..., dk, dk], X, N, out
    [..., dk, dv] fp32 device tensors; the leading dimensions are flattened."""
    dk, dv = X.shape[-2], X.shape[-1]
    n = X.numel() // (dk * dv)
    if M.shape[-2:] != (dk, dk) or M.numel() // (dk * dk) != n or out.shape != X.shape:
        raise KDAError(1, "kda_state_map_apply: shapes do not match")
    if N is not None and N.shape != X.shape:
        raise KDAError(1, "kda_state_map_apply: N must be shaped like X")
    if any(t is not None and t.dtype != _F32 for t in (M, X, N, out)):
        raise KDAError(1, "kda_state_map_apply: M, X, N and out must be fp32")
    _check(lib().kda_state_map_apply(n, dk, dv, _dptr(M), _dptr(X), _dptr(N), _dptr(out),
                                     _stream(stream)), "kda_state_map_apply")


def kda_snapshot(src_idx, dst_idx, src, dst, stream=None):
    """dst[dst_idx[i]] = src[src_idx[i]] for whole [H, dk, dv] states (see include/kda.h)."""
    if src.dim() != 4:
        raise KDAError(1, f"src must be shaped [n, H, dk, dv], not {list(src.shape)}")
    n, H, dk, dv = src_idx.shape[0], src.shape[1], src.shape[2], src.shape[3]
    _expect(src_idx, "src_idx", _I64T, n, ())
    _expect(dst_idx, "dst_idx", _I64T, n, ())
    _expect(src, "src", _F32, 0, (H, dk, dv))
    _expect(dst, "dst", _F32, 0, (H, dk, dv))
    _check(lib().kda_snapshot(n, _dptr(src_idx), _dptr(dst_idx), _dptr(src), src.shape[0],
                              _dptr(dst), dst.shape[0], H, dk, dv, _stream(stream)), "kda_snapshot")


def kda_check_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status code."""
    return int(lib().kda_check_device_status(_stream(stream)))


def kda_last_cuda_error() -> str:
    return lib().kda_last_cuda_error().decode()


def kda_launch_count() -> int:
    return int(lib().kda_launch_count())


def kda_status_string(status: int) -> str:
    return lib().kda_status_string(status).decode()
