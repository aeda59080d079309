"""ctypes binding of libkata.so (the C ABI in include/kata.h).

Argument marshalling only: PyTorch provides device memory (outputs and
workspaces are torch allocations) and the current CUDA stream; every step of
the computation runs in libkata's kernels. There is no fallback: if the
library is missing, every call raises.
"""
from __future__ import annotations

import ctypes as C
import os
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
# KATA_DEBUG=1 in the environment loads the debug library (device-side bounds
# checks, include/kata.h kata_debug_build) instead of libkata.so.
LIB_PATH = _PKG / ("libkata_debug.so" if os.environ.get("KATA_DEBUG") == "1" else "libkata.so")

KATA_F32, KATA_BF16 = 0, 1
_DTYPE = {torch.float32: KATA_F32, torch.bfloat16: KATA_BF16}

_vp, _i, _f, _sz = C.c_void_p, C.c_int, C.c_float, C.c_size_t

# name -> (restype, argtypes), mirroring include/kata.h
SIGNATURES = {
    "kata_version": (_i, []),
    "kata_status_string": (C.c_char_p, [_i]),
    "kata_last_error": (C.c_char_p, []),
    "kata_packed_dim": (C.c_long, [_i]),
    "kata_launch_count": (C.c_ulonglong, []),
    "kata_sync_status": (_i, [_vp]),
    "kata_prefill_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "kata_prefill": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp, _vp,
                          _vp, _sz, _vp]),
    "kata_prefill_path": (_i, [_i, _i, _i, _i, _i, _i]),
    "kata_test_forced_timeout": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, C.c_uint, _vp]),
    "kata_debug_build": (_i, []),
    "kata_test_bounds_check": (_i, [_vp]),
    "kata_prefill_ex": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp, _vp,
                             _vp, _sz, _vp, _i]),
    "kata_quadratic_max_tokens": (_i, [_i]),
    "kata_prefill_auto_form": (_i, [_i, _i, _i, _i, _i, _i, _i]),
    "kata_prefill_host_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "kata_prefill_host": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _sz, _vp]),
    "kata_decode_step": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp]),
    "kata_decode_step_host": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp, _sz,
                                   _vp]),
    "lola_sre_workspace_bytes": (_sz, [_i, _i, _i, _i]),
    "lola_sre_score_topk": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp,
                                 _vp, _vp, _vp, _vp, _sz, _vp]),
    "lola_sre_score_topk_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f,
                                         _i, _vp, _vp, _vp, _vp, _vp]),
    "lola_readout_workspace_bytes": (_sz, [_i, _i, _i, _i]),
    "lola_hybrid_readout": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _i,
                                 _i, _vp, _vp, _f, _f, _vp, _vp, _sz, _vp]),
    "lola_prefill_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "lola_prefill": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _f, _vp, _vp, _vp, _vp,
                          _vp, _sz, _vp]),
    "lola_prefill_ex": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _f, _vp, _vp, _vp,
                             _vp, _vp, _sz, _vp, _i]),
    "lola_prefill_fused_applies": (_i, [_i, _i, _i, _i]),
    "kata_feature_dim": (C.c_long, [_i, _i, _i]),
    "kata_prefill_feature": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _vp, _vp,
                                  _vp, _vp, _vp, _vp, _sz, _vp]),
    "kata_decode_step_feature": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _vp, _vp, _vp,
                                      _vp]),
    "kata_state_prefix": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp]),
}

# multi-factor features (kata_prefill_feature, kata_decode_step_feature)
FEATURES = {"rank1": 0, "mg": 1, "sigmag": 2}

# lola_prefill_ex executions; "fusedN": the fused run with N CTAs per head
LOLA_RUNS = {"auto": 0, "segments": 1, "fused": 2, **{f"fused{n}": 10 + n for n in (6, 7, 8)}}

_lib = None


class KataError(RuntimeError):
    pass


def lib() -> C.CDLL:
    """The loaded libkata.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise KataError(f"{LIB_PATH} is missing: run __graft_entry__.build() or "
                            "python kernelized_linear_attention_chunked_b200/build.py")
        handle = C.CDLL(str(LIB_PATH))
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(name: str, status: int) -> None:
    if status != 0:
        L = lib()
        raise KataError(f"{name}: {L.kata_status_string(status).decode()}: "
                        f"{L.kata_last_error().decode()}")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dt(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPE:
        raise KataError(f"dtype {t.dtype} is not float32 or bfloat16")
    return _DTYPE[t.dtype]


def _dev(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise KataError("tensors must be contiguous CUDA tensors")


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def packed_dim(d: int) -> int:
    return int(lib().kata_packed_dim(d))


def launch_count() -> int:
    """Kernels libkata has launched in this process so far."""
    return int(lib().kata_launch_count())


def sync_status(stream=None) -> None:
    """Synchronise and raise if a kernel's bounded wait ran out."""
    _check("kata_sync_status", lib().kata_sync_status(_stream(stream)))


# kata_prefill_ex forms
FORMS = {"auto": 0, "chunked": 1, "quadratic": 2}


def prefill(q, k, v, chunk: int, eps: float = 1e-6, H_in=None, s_in=None, state: bool = True,
            output: bool = True, o=None, H_out=None, s_out=None, workspace=None, stream=None,
            form: str = "auto"):
    """Causal prefill. q, k, v [B, H, T, d]. Returns (o, H, s); o is None when
    ``output`` is False (state only), H and s are None when ``state`` is False.
    ``form``: "chunked", "quadratic" (o from a zero initial state; the final
    state, if asked for, by the state pass at the same time) or "auto"
    (kata_prefill's choice)."""
    _dev(q, k, v, H_in, s_in)
    B, Hh, T, d = q.shape
    D = d * (d + 1) // 2
    dt = _dt(q)
    if output and o is None:
        o = torch.empty(B, Hh, T, d, dtype=torch.float32, device=q.device)
    if state and H_out is None:
        H_out = torch.empty(B, Hh, D, d, dtype=torch.float32, device=q.device)
        s_out = torch.empty(B, Hh, D, dtype=torch.float32, device=q.device)
    L = lib()
    if workspace is None:
        workspace = _workspace(L.kata_prefill_workspace_bytes(B, Hh, T, d, chunk, dt), q.device)
    _check("kata_prefill_ex", L.kata_prefill_ex(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), dt, B, Hh, T, d, chunk, eps, _ptr(H_in),
        _ptr(s_in), _ptr(o), _ptr(H_out), _ptr(s_out), workspace.data_ptr(), workspace.numel(),
        _stream(stream), FORMS[form]))
    return o, H_out, s_out


def test_forced_timeout(q, k, v, polls: int, eps: float = 1e-6, o=None, stream=None):
    """kata_test_forced_timeout: the quadratic form with a wait that nothing
    completes (a failure-detection test hook). Returns o (not valid)."""
    _dev(q, k, v)
    B, Hh, T, d = q.shape
    if o is None:
        o = torch.empty(B, Hh, T, d, dtype=torch.float32, device=q.device)
    _check("kata_test_forced_timeout", lib().kata_test_forced_timeout(
        _ptr(q), _ptr(k), _ptr(v), B, Hh, T, d, eps, _ptr(o), polls, _stream(stream)))
    return o


def debug_build() -> bool:
    """True when the loaded library is libkata_debug.so (device-side bounds checks)."""
    return bool(lib().kata_debug_build())


def test_bounds_check(stream=None) -> None:
    """kata_test_bounds_check: one checked store past the end of a small device
    array (debug library only); the next sync_status() raises KATA_ERR_BOUNDS."""
    _check("kata_test_bounds_check", lib().kata_test_bounds_check(_stream(stream)))


def prefill_auto_form(B, H, T, d, chunk, dtype, with_state: bool = False) -> str:
    """The form kata_prefill takes for these sizes: "chunked" or "quadratic"
    (the latter only for calls without an initial or final state)."""
    f = int(lib().kata_prefill_auto_form(B, H, T, d, chunk, _DTYPE[dtype], int(with_state)))
    if f < 0:
        raise KataError(f"kata_prefill_auto_form: invalid arguments ({B}, {H}, {T}, {d}, {chunk})")
    return "quadratic" if f == FORMS["quadratic"] else "chunked"


def quadratic_max_tokens(d: int) -> int:
    """Largest T for which kata_prefill takes the quadratic form (0: never)."""
    return int(lib().kata_quadratic_max_tokens(d))


def prefill_uses_tensor_cores(B, H, T, d, chunk, dtype) -> bool:
    """True when kata_prefill runs the tcgen05 kernel for these sizes."""
    return int(lib().kata_prefill_path(B, H, T, d, chunk, _DTYPE[dtype])) == 1


def prefill_workspace_bytes(B, H, T, d, chunk, dtype) -> int:
    return int(lib().kata_prefill_workspace_bytes(B, H, T, d, chunk, _DTYPE[dtype]))


def prefill_host(q, k, v, chunk: int, eps: float, o, workspace, stream=None) -> None:
    """kata_prefill_host: q, k, v, o are (pinned) CPU tensors; asynchronous."""
    B, Hh, T, d = q.shape
    _check("kata_prefill_host", lib().kata_prefill_host(
        _ptr(q), _ptr(k), _ptr(v), _dt(q), B, Hh, T, d, chunk, eps, _ptr(o), _ptr(workspace),
        workspace.numel(), _stream(stream)))


def prefill_host_workspace_bytes(B, H, T, d, chunk, dtype) -> int:
    return int(lib().kata_prefill_host_workspace_bytes(B, H, T, d, chunk, _DTYPE[dtype]))


def decode_step(q, k, v, Hst, s, eps: float = 1e-6, o=None, stream=None):
    """One decode step, state updated in place. q, k, v [B, H, d]. Returns o."""
    _dev(q, k, v, Hst, s)
    B, Hh, d = q.shape
    if o is None:
        o = torch.empty(B, Hh, d, dtype=torch.float32, device=q.device)
    _check("kata_decode_step", lib().kata_decode_step(
        _ptr(q), _ptr(k), _ptr(v), _dt(q), B, Hh, d, eps, _ptr(Hst), _ptr(s), _ptr(o),
        _stream(stream)))
    return o


def feature_dim(d: int, feature: str, g: int) -> int:
    """Rows of the state of a multi-factor feature (0: invalid)."""
    return int(lib().kata_feature_dim(d, FEATURES[feature], g))


def prefill_feature(q, k, v, feature: str, g: int, chunk: int = 64, eps: float = 1e-6,
                    H_in=None, s_in=None, output: bool = True, state: bool = True,
                    workspace=None, stream=None):
    """Causal prefill with a multi-factor feature ("rank1", "mg", "sigmag").
    Returns (o or None, H [B, H, Df, d] or None, s [B, H, Df] or None)."""
    _dev(q, k, v, H_in, s_in)
    B, Hh, T, d = q.shape
    Df = feature_dim(d, feature, g)
    if Df <= 0:
        raise KataError(f"feature {feature!r} with g={g} is not available for d={d}")
    o = torch.empty(B, Hh, T, d, dtype=torch.float32, device=q.device) if output else None
    H_out = torch.empty(B, Hh, Df, d, dtype=torch.float32, device=q.device) if state else None
    s_out = torch.empty(B, Hh, Df, dtype=torch.float32, device=q.device) if state else None
    L = lib()
    if workspace is None:
        workspace = _workspace(L.kata_prefill_workspace_bytes(B, Hh, T, d, chunk, _dt(q)),
                               q.device)
    _check("kata_prefill_feature", L.kata_prefill_feature(
        _ptr(q), _ptr(k), _ptr(v), _dt(q), B, Hh, T, d, chunk, eps, FEATURES[feature], g,
        _ptr(H_in), _ptr(s_in), _ptr(o), _ptr(H_out), _ptr(s_out), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return o, H_out, s_out


def decode_step_feature(q, k, v, Hst, s, feature: str, g: int, eps: float = 1e-6, o=None,
                        stream=None):
    """One decode step with a multi-factor feature, state updated in place. Returns o."""
    _dev(q, k, v, Hst, s)
    B, Hh, d = q.shape
    if o is None:
        o = torch.empty(B, Hh, d, dtype=torch.float32, device=q.device)
    _check("kata_decode_step_feature", lib().kata_decode_step_feature(
        _ptr(q), _ptr(k), _ptr(v), _dt(q), B, Hh, d, eps, FEATURES[feature], g, _ptr(Hst),
        _ptr(s), _ptr(o), _stream(stream)))
    return o


def state_prefix(H_parts, s_parts, feature: str = "rank1", g: int = 1, stream=None):
    """Exclusive prefix sums over the parts' states: H_parts [n, B, H, Df, d],
    s_parts [n, B, H, Df] -> (H_prefix, s_prefix) of the same shapes, part z's
    prefix the sum of parts 0 .. z-1."""
    _dev(H_parts, s_parts)
    n, B, Hh, Df, d = H_parts.shape
    Hp, sp = torch.empty_like(H_parts), torch.empty_like(s_parts)
    _check("kata_state_prefix", lib().kata_state_prefix(
        _ptr(H_parts), _ptr(s_parts), n, B, Hh, d, FEATURES[feature], g, _ptr(Hp), _ptr(sp),
        _stream(stream)))
    return Hp, sp


def decode_step_host(q, k, v, Hst, s, eps, o, workspace, stream=None) -> None:
    B, Hh, d = q.shape
    _check("kata_decode_step_host", lib().kata_decode_step_host(
        _ptr(q), _ptr(k), _ptr(v), _dt(q), B, Hh, d, eps, _ptr(Hst), _ptr(s), _ptr(o),
        _ptr(workspace), workspace.numel(), _stream(stream)))


def sre_score_topk(Hst, s, kc, vc, pos, keep: int, eps: float = 1e-6, merge: bool = False,
                   Hst_mut=None, s_mut=None, scores: bool = True, stream=None):
    """SRE of candidates kc, vc [B, H, n, d] and top-k. Returns (scores, keep_idx)."""
    _dev(Hst, s, kc, vc, pos)
    B, Hh, n, d = kc.shape
    m = min(keep, n)
    sc = torch.empty(B, Hh, n, dtype=torch.float32, device=kc.device) if scores else None
    ki = torch.empty(B, Hh, max(m, 1), dtype=torch.int32, device=kc.device)
    L = lib()
    ws = _workspace(L.lola_sre_workspace_bytes(B, Hh, d, n), kc.device)
    if merge and Hst_mut is None:
        Hst_mut, s_mut = Hst, s
    _check("lola_sre_score_topk", L.lola_sre_score_topk(
        _ptr(Hst), _ptr(s), _ptr(kc), _ptr(vc), _ptr(pos), _dt(kc), B, Hh, d, n, keep, eps,
        int(merge), _ptr(sc), _ptr(ki), _ptr(Hst_mut), _ptr(s_mut), _ptr(ws), ws.numel(),
        _stream(stream)))
    return sc, ki[..., :m]


def hybrid_readout(q, k, v, seg0: int, nq: int, w0: int, ck, cv, nc: int, Hst, s,
                   eps: float = 1e-6, tau: float | None = None, o=None, stream=None):
    """Hybrid window + cache + state readout of rows seg0..seg0+nq-1. Returns o."""
    _dev(q, k, v, ck, cv, Hst, s)
    B, Hh, T, d = q.shape
    cap = ck.shape[2]
    tau = d ** -0.5 if tau is None else tau
    if o is None:
        o = torch.zeros(B, Hh, T, d, dtype=torch.float32, device=q.device)
    L = lib()
    ws = _workspace(L.lola_readout_workspace_bytes(B, Hh, d, nq), q.device)
    _check("lola_hybrid_readout", L.lola_hybrid_readout(
        _ptr(q), _ptr(k), _ptr(v), _dt(q), B, Hh, T, d, seg0, nq, w0, _ptr(ck), _ptr(cv), nc,
        cap, _ptr(Hst), _ptr(s), eps, tau, _ptr(o), _ptr(ws), ws.numel(), _stream(stream)))
    return o


def lola_fused_applies(dtype, d: int, window: int, cache: int) -> bool:
    """True when the one-launch (fused) schedule takes these sizes."""
    return bool(lib().lola_prefill_fused_applies(_DTYPE[dtype], d, window, cache))


def lola_prefill(q, k, v, window: int, cache: int, eps: float = 1e-6, tau: float | None = None,
                 Hst=None, s=None, kept: bool = False, o=None, workspace=None, stream=None,
                 run: str = "auto"):
    """The LoLA schedule over q, k, v [B, H, T, d]. Returns (o, H, s, kept_pos or None).
    ``run``: "fused" (one launch), "segments" (launches per segment) or "auto"."""
    _dev(q, k, v, Hst, s)
    B, Hh, T, d = q.shape
    D = packed_dim(d)
    tau = d ** -0.5 if tau is None else tau
    dev = q.device
    if o is None:
        o = torch.empty(B, Hh, T, d, dtype=torch.float32, device=dev)
    if Hst is None:
        Hst = torch.zeros(B, Hh, D, d, dtype=torch.float32, device=dev)
        s = torch.zeros(B, Hh, D, dtype=torch.float32, device=dev)
    kp = None
    if kept and T // window > 1:
        kp = torch.empty(T // window - 1, B, Hh, max(cache, 1), dtype=torch.int32, device=dev)
    L = lib()
    if workspace is None:
        workspace = _workspace(L.lola_prefill_workspace_bytes(B, Hh, T, d, window, cache), dev)
    _check("lola_prefill_ex", L.lola_prefill_ex(
        _ptr(q), _ptr(k), _ptr(v), _dt(q), B, Hh, T, d, window, cache, eps, tau, _ptr(o),
        _ptr(Hst), _ptr(s), _ptr(kp), _ptr(workspace), workspace.numel(), _stream(stream),
        LOLA_RUNS[run]))
    return o, Hst, s, (None if kp is None else kp[..., :cache])


def lola_prefill_workspace_bytes(B, H, T, d, window, cache) -> int:
    return int(lib().lola_prefill_workspace_bytes(B, H, T, d, window, cache))
