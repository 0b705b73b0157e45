"""ctypes binding of the SAS C ABI (``include/sas.h``).

Argument marshalling only: every function takes torch tensors (device memory
owned by the caller), checks that they are contiguous, and passes their
pointers and sizes to the function of the same name in ``libsas_b200.so``.
All arithmetic runs in the library's CUDA kernels; there is no fallback. If the
library is missing, the first call raises ``RuntimeError``.
"""

from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsas_b200.so")
_lib = None

SAS_OK = 0
SAS_DT_F32 = 0
SAS_DT_BF16 = 1
BLOCK = 64

_c_int, _c_f, _vp, _sz = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t

# name -> (restype, argtypes), mirroring include/sas.h
_SIGNATURES = {
    "sas_status_string": (ctypes.c_char_p, [_c_int]),
    "sas_version": (_c_int, []),
    "sas_launch_count": (ctypes.c_uint64, []),
    "sas_set_wait_limit_ns": (ctypes.c_uint64, [ctypes.c_uint64]),
    "sas_gate_normalize": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp]),
    "sas_select_threshold": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp]),
    "sas_gate_normalize_select": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                           _vp]),
    "sas_gate_normalize_select_compact": (_c_int, [_vp, _vp, _vp, _vp, _vp] + [_c_int] * 6 + [_vp]),
    "sas_gate_normalize_select_varlen": (_c_int, [_vp, _vp, _vp, _vp, _vp] + [_c_int] * 6 + [_vp, _c_int, _vp]),
    "sas_select_noisy": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp]),
    "sas_gate_grad": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp]),
    "sas_fwd_workspace_size": (_c_int, [_c_int] * 8 + [ctypes.POINTER(_sz)]),
    "sas_bwd_workspace_size": (_c_int, [_c_int] * 8 + [ctypes.POINTER(_sz)]),
    "sas_decode_workspace_size": (_c_int, [_c_int] * 7 + [ctypes.POINTER(_sz)]),
    "sas_fwd": (_c_int, [_vp, _vp, _vp, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp] + [_c_int] * 7
                + [_c_f, _vp, _sz, _vp]),
    "sas_bwd": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
                + [_c_int] * 7 + [_c_f, _vp, _sz, _vp]),
    "sas_decode_fwd": (_c_int, [_vp, _vp, _vp, _c_int, _vp, _vp, _c_int, _c_int, _vp, _vp] + [_c_int] * 7
                       + [_c_f, _vp, _sz, _vp]),
    "sas_decode_fwd_paged": (_c_int, [_vp, _vp, _vp, _c_int, _vp, _c_int, _c_int, _vp, _vp, _c_int, _c_int, _vp,
                                      _vp] + [_c_int] * 6 + [_c_f, _vp, _sz, _vp]),
    "sas_decode_fwd_static": (_c_int, [_vp, _vp, _vp, _c_int, _vp, _vp, _c_int, _c_int, _vp, _vp] + [_c_int] * 7
                              + [_c_f, _vp]),
    "sas_decode_static_status": (_c_int, [_vp, ctypes.POINTER(ctypes.c_int32)]),
    "sas_device_status": (_c_int, [_vp, _vp, ctypes.POINTER(ctypes.c_int32)]),
    "sas_device_status_clear": (_c_int, [_vp, _vp]),
}


class SasError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {lib().sas_status_string(status).decode()} (status {status})")


def lib():
    """Load ``libsas_b200.so`` (once) and declare its signatures."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"SAS CUDA library not found at {_LIB_PATH}; build it with "
                "`python -m gated_block_sparse_flashattention_b200.build`")
        handle = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(handle, name)
            f.restype = res
            f.argtypes = args
        _lib = handle
    return _lib


def library_path() -> str:
    return _LIB_PATH


def _check(fn: str, status: int):
    if status != SAS_OK:
        raise SasError(fn, status)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("SAS tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SAS_DT_F32
    if t.dtype == torch.bfloat16:
        return SAS_DT_BF16
    raise ValueError(f"unsupported dtype {t.dtype}")


def launch_count() -> int:
    return int(lib().sas_launch_count())


def set_wait_limit_ns(ns: int) -> int:
    """Limit of each bounded wait in the fwd/bwd tensor-core kernels (0: the 1 s default); returns the old one."""
    return int(lib().sas_set_wait_limit_ns(int(ns)))


def status_string(status: int) -> str:
    return lib().sas_status_string(status).decode()


def sas_gate_normalize(s, logG, block=BLOCK, stream=None):
    B, Hkv, T, NB = s.shape
    _check("sas_gate_normalize", lib().sas_gate_normalize(_ptr(s), _ptr(logG), B, Hkv, T, NB, block, _stream(stream)))


def sas_select_threshold(logG, tau, tau_idx, sel, K, block=BLOCK, stream=None):
    B, Hkv, T, NB = logG.shape
    _check("sas_select_threshold", lib().sas_select_threshold(
        _ptr(logG), _ptr(tau), _ptr(tau_idx), _ptr(sel), B, Hkv, T, NB, block, K, _stream(stream)))


def sas_gate_normalize_select(s, logG, tau, tau_idx, sel, K, block=BLOCK, stream=None):
    B, Hkv, T, NB = s.shape
    _check("sas_gate_normalize_select", lib().sas_gate_normalize_select(
        _ptr(s), _ptr(logG), _ptr(tau), _ptr(tau_idx), _ptr(sel), B, Hkv, T, NB, block, K, _stream(stream)))


def sas_gate_normalize_select_compact(s, gate_lse, tau, tau_idx, sel, K, block=BLOCK, stream=None):
    B, Hkv, T, NB = s.shape
    _check("sas_gate_normalize_select_compact", lib().sas_gate_normalize_select_compact(
        _ptr(s), _ptr(gate_lse), _ptr(tau), _ptr(tau_idx), _ptr(sel), B, Hkv, T, NB, block, K, _stream(stream)))


def sas_gate_normalize_select_varlen(s, logG, tau, tau_idx, sel, K, cu_seqlens, block=BLOCK, stream=None):
    """cu_seqlens: host sequence of n_docs + 1 token offsets (multiples of 64, from 0 to T)."""
    B, Hkv, T, NB = s.shape
    cu = (ctypes.c_int32 * len(cu_seqlens))(*[int(x) for x in cu_seqlens])
    _check("sas_gate_normalize_select_varlen", lib().sas_gate_normalize_select_varlen(
        _ptr(s), _ptr(logG), _ptr(tau), _ptr(tau_idx), _ptr(sel), B, Hkv, T, NB, block, K,
        ctypes.cast(cu, ctypes.c_void_p), len(cu_seqlens) - 1, _stream(stream)))


def sas_select_noisy(logG, noise, logG_sel, tau, tau_idx, sel, K, block=BLOCK, stream=None):
    B, Hkv, T, NB = logG.shape
    _check("sas_select_noisy", lib().sas_select_noisy(
        _ptr(logG), _ptr(noise), _ptr(logG_sel), _ptr(tau), _ptr(tau_idx), _ptr(sel), B, Hkv, T, NB, block, K,
        _stream(stream)))


def sas_gate_grad(logG, dLogG, ds, block=BLOCK, stream=None, gate_lse=None):
    """gate_lse: the row log-sum-exp of compact gates (then logG holds the raw scores s)."""
    B, Hkv, T, NB = logG.shape
    _check("sas_gate_grad", lib().sas_gate_grad(
        _ptr(logG), _ptr(gate_lse), _ptr(dLogG), _ptr(ds), B, Hkv, T, NB, block, _stream(stream)))


def _ws_size(name, *args) -> int:
    out = _sz(0)
    _check(name, getattr(lib(), name)(*args, ctypes.byref(out)))
    return out.value


def sas_fwd_workspace_size(B, Hq, Hkv, T, d, K, dtype_code, block=BLOCK) -> int:
    return _ws_size("sas_fwd_workspace_size", B, Hq, Hkv, T, d, block, K, dtype_code)


def sas_bwd_workspace_size(B, Hq, Hkv, T, d, K, dtype_code, block=BLOCK) -> int:
    return _ws_size("sas_bwd_workspace_size", B, Hq, Hkv, T, d, block, K, dtype_code)


def sas_decode_workspace_size(B, Hq, Hkv, Lmax, d, K, block=BLOCK) -> int:
    return _ws_size("sas_decode_workspace_size", B, Hq, Hkv, Lmax, d, block, K)


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zeroed byte buffer of at least ``nbytes`` (torch allocations are 256-byte aligned)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def sas_fwd(Q, K, V, logG, tau, tau_idx, O, LSE, Kbudget, sm_scale, ws, block=BLOCK, stream=None, gate_lse=None,
            sel=None):
    """gate_lse: the row log-sum-exp of compact gates (then logG holds the raw scores s); sel: the
    selection call's index list [B, Hkv, T, Kbudget-1] (the row lists are then built from it)."""
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    _check("sas_fwd", lib().sas_fwd(
        _ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q), _ptr(logG), _ptr(gate_lse), _ptr(tau), _ptr(tau_idx), _ptr(sel),
        _ptr(O), _ptr(LSE),
        B, Hq, Hkv, T, d, block, int(Kbudget), float(sm_scale), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def sas_bwd(Q, K, V, O, dO, logG, tau, tau_idx, LSE, dQ, dK, dV, dLogG, Kbudget, sm_scale, ws, block=BLOCK,
            stream=None, gate_lse=None, sel=None):
    """gate_lse and sel as for ``sas_fwd``."""
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    _check("sas_bwd", lib().sas_bwd(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _dtype_code(Q), _ptr(logG), _ptr(gate_lse), _ptr(tau),
        _ptr(tau_idx), _ptr(sel),
        _ptr(LSE), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dLogG), B, Hq, Hkv, T, d, block, int(Kbudget),
        float(sm_scale), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def sas_decode_fwd(q, Kc, Vc, seqlen, s, K, o, ws, sm_scale, sel_out=None, apply_log_gate=False, block=BLOCK,
                   stream=None):
    B, Hq, d = q.shape
    Hkv, Lmax = Kc.shape[1], Kc.shape[2]
    NBmax = s.shape[-1]
    _check("sas_decode_fwd", lib().sas_decode_fwd(
        _ptr(q), _ptr(Kc), _ptr(Vc), _dtype_code(q), _ptr(seqlen), _ptr(s), K, 1 if apply_log_gate else 0,
        _ptr(o), _ptr(sel_out), B, Hq, Hkv, Lmax, NBmax, d, block, float(sm_scale), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def sas_decode_fwd_paged(q, Kp, Vp, page_table, seqlen, s, K, o, ws, sm_scale, sel_out=None, apply_log_gate=False,
                         block=BLOCK, stream=None):
    """Kp/Vp [num_pages, Hkv, 64, d]; page_table [B, max_pages] int32 on the device."""
    B, Hq, d = q.shape
    num_pages, Hkv = Kp.shape[0], Kp.shape[1]
    max_pages = page_table.shape[1]
    NBmax = s.shape[-1]
    _check("sas_decode_fwd_paged", lib().sas_decode_fwd_paged(
        _ptr(q), _ptr(Kp), _ptr(Vp), _dtype_code(q), _ptr(page_table), max_pages, num_pages, _ptr(seqlen), _ptr(s),
        K, 1 if apply_log_gate else 0, _ptr(o), _ptr(sel_out), B, Hq, Hkv, NBmax, d, block, float(sm_scale),
        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def sas_decode_fwd_static(q, Kc, Vc, seqlen, s, K, o, sm_scale, sel_out=None, apply_log_gate=False, block=BLOCK,
                          stream=None):
    """sas_decode_fwd with the library's built-in static scratch (no workspace argument)."""
    B, Hq, d = q.shape
    Hkv, Lmax = Kc.shape[1], Kc.shape[2]
    NBmax = s.shape[-1]
    _check("sas_decode_fwd_static", lib().sas_decode_fwd_static(
        _ptr(q), _ptr(Kc), _ptr(Vc), _dtype_code(q), _ptr(seqlen), _ptr(s), K, 1 if apply_log_gate else 0,
        _ptr(o), _ptr(sel_out), B, Hq, Hkv, Lmax, NBmax, d, block, float(sm_scale), _stream(stream)))


def sas_decode_static_status(stream=None) -> int:
    """Status word of the last sas_decode_fwd_static call on the current device (0: no kernel-side error)."""
    out = ctypes.c_int32(0)
    lib().sas_decode_static_status(_stream(stream), ctypes.byref(out))
    return out.value


def sas_device_status(ws, stream=None) -> int:
    out = ctypes.c_int32(0)
    lib().sas_device_status(_ptr(ws), _stream(stream), ctypes.byref(out))
    return out.value


def sas_device_status_clear(ws, stream=None):
    _check("sas_device_status_clear", lib().sas_device_status_clear(_ptr(ws), _stream(stream)))


# ---------------------------------------------------------------------------------------------
# Convenience wrappers that allocate outputs (torch device memory) and chain the calls.
# ---------------------------------------------------------------------------------------------
def gate_and_select(s, K, block=BLOCK, want_sel=False, stream=None):
    """logG, tau, tau_idx (and sel) from selector scores s [B,Hkv,T,NB] on the device."""
    B, Hkv, T, NB = s.shape
    logG = torch.empty_like(s)
    tau = torch.empty(B, Hkv, T, dtype=torch.float32, device=s.device)
    tidx = torch.empty(B, Hkv, T, dtype=torch.int32, device=s.device)
    sel = torch.empty(B, Hkv, T, max(K - 1, 1), dtype=torch.int32, device=s.device) if want_sel else None
    sas_gate_normalize_select(s, logG, tau, tidx, sel, K, block, stream)
    return logG, tau, tidx, sel


def gate_and_select_compact(s, K, block=BLOCK, want_sel=False, stream=None):
    """gate_lse, tau, tau_idx (and sel) of compact gates from selector scores s [B,Hkv,T,NB] on the device:
    pass s as the gates and gate_lse to forward / backward / gate_grad."""
    B, Hkv, T, NB = s.shape
    gate_lse = torch.empty(B, Hkv, T, dtype=torch.float32, device=s.device)
    tau = torch.empty(B, Hkv, T, dtype=torch.float32, device=s.device)
    tidx = torch.empty(B, Hkv, T, dtype=torch.int32, device=s.device)
    sel = torch.empty(B, Hkv, T, max(K - 1, 1), dtype=torch.int32, device=s.device) if want_sel else None
    sas_gate_normalize_select_compact(s, gate_lse, tau, tidx, sel, K, block, stream)
    return gate_lse, tau, tidx, sel


def gate_grad(logG, dLogG, block=BLOCK, stream=None, gate_lse=None):
    """ds = dL/ds [B,Hkv,T,NB] from the log-gate gradient of ``backward`` and the gates of ``gate_and_select``
    (or the scores and ``gate_lse`` of ``gate_and_select_compact``)."""
    ds = torch.empty_like(dLogG)
    sas_gate_grad(logG, dLogG, ds, block, stream, gate_lse=gate_lse)
    return ds


def _check_device_status(fn, ws, stream):
    st = sas_device_status(ws, stream)
    if st != 0:
        raise SasError(fn, -4)


def forward(Q, K, V, logG, tau, tau_idx, Kbudget, sm_scale, block=BLOCK, stream=None, ws=None, check=True,
            gate_lse=None, sel=None):
    """O, LSE of ``sas_fwd``. With ``check`` the stream is synchronised and the
    kernel status word is read (raises ``SasError`` on a kernel-side error).
    With ``gate_lse`` (compact gates) ``logG`` holds the raw scores s; ``sel`` is
    the selection's index list, from which the row lists are built."""
    B, Hq, T, d = Q.shape
    O = torch.empty_like(Q)
    LSE = torch.empty(B, Hq, T, dtype=torch.float32, device=Q.device)
    if ws is None:
        ws = workspace(sas_fwd_workspace_size(B, Hq, K.shape[1], T, d, Kbudget, _dtype_code(Q), block), Q.device)
    sas_fwd(Q, K, V, logG, tau, tau_idx, O, LSE, Kbudget, sm_scale, ws, block, stream, gate_lse=gate_lse, sel=sel)
    if check:
        _check_device_status("sas_fwd", ws, stream)
    return O, LSE


def backward(Q, K, V, O, dO, logG, tau, tau_idx, LSE, Kbudget, sm_scale, block=BLOCK, stream=None, ws=None,
             check=True, gate_lse=None, sel=None):
    """dQ, dK, dV, dLogG of ``sas_bwd`` (``check``, ``gate_lse`` and ``sel`` as in ``forward``)."""
    B, Hq, T, d = Q.shape
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    dLogG = torch.empty_like(logG)
    if ws is None:
        ws = workspace(sas_bwd_workspace_size(B, Hq, K.shape[1], T, d, Kbudget, _dtype_code(Q), block), Q.device)
    sas_bwd(Q, K, V, O, dO, logG, tau, tau_idx, LSE, dQ, dK, dV, dLogG, Kbudget, sm_scale, ws, block, stream,
            gate_lse=gate_lse, sel=sel)
    if check:
        _check_device_status("sas_bwd", ws, stream)
    return dQ, dK, dV, dLogG
