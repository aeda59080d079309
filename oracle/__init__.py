"""fp64 CPU oracle for causal kernelized linear attention (rank-one PSD feature)
and the LoLA self-recall-error sparse cache.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. The CUDA product path never imports it and shares no code with it.

The arithmetic lives in ``kata_oracle.c`` (plain C, fp64, one head at a time);
this module only converts arrays to contiguous fp64, loops over the LoLA
schedule in the order the LoLA page states it, and returns NumPy arrays.

Sources, by page title and section:
  "Kernelized Linear Attention: Breaking the Capacity Wall with Symmetric
  Cones" s1 (recurrent fixed-size state), s2.1 (output gate), s2.2 (psi(u) =
  u u^T), s2.3 (exact chunked state form); "LoLA: Low-Rank Linear Attention
  with Sparse Caching", Methodology 1-3, "Self-Recall Error", "Inference
  strategy" 1-4.
"""
from __future__ import annotations

import ctypes as C
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_LIB_PATH = _HERE / "liboracle.so"
_lib = None

_dp = C.POINTER(C.c_double)
_ip = C.POINTER(C.c_int)
_lp = C.POINTER(C.c_long)


def _load():
    global _lib
    if _lib is not None:
        return _lib
    src = _HERE / "kata_oracle.c"
    if not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < src.stat().st_mtime:
        from .build import build
        build()
    lib = C.CDLL(str(_LIB_PATH))
    lib.oracle_threads.restype = C.c_int
    lib.oracle_threads.argtypes = []
    lib.oracle_set_threads.argtypes = [C.c_int]
    lib.oracle_packed_dim.restype = C.c_long
    lib.oracle_packed_dim.argtypes = [C.c_int]
    lib.oracle_packed_index.restype = C.c_long
    lib.oracle_packed_index.argtypes = [C.c_int, C.c_int, C.c_int]
    lib.oracle_phi.argtypes = [_dp, C.c_int, _dp]
    lib.oracle_quadratic_heads.argtypes = [C.c_int, _dp, _dp, _dp, C.c_long, C.c_int,
                                           C.c_int, C.c_double, _lp, C.c_long, _dp]
    lib.oracle_recurrent_heads.argtypes = [C.c_int, _dp, _dp, _dp, C.c_long, C.c_int, C.c_int,
                                           C.c_double, _dp, _dp, _dp]
    lib.oracle_sre_heads.argtypes = [C.c_int, _dp, _dp, _dp, _dp, C.c_int, C.c_int, C.c_int,
                                     C.c_double, _dp]
    lib.oracle_topk.restype = C.c_int
    lib.oracle_topk.argtypes = [_dp, _ip, C.c_int, C.c_int, _ip]
    lib.oracle_merge_heads.argtypes = [C.c_int, _dp, _dp, _dp, _dp, C.c_int, _ip, C.c_int,
                                       C.c_int, C.c_int]
    lib.oracle_hybrid_segment_heads.argtypes = [C.c_int, _dp, _dp, _dp, C.c_long, C.c_int,
                                                C.c_int, C.c_double, C.c_double, C.c_long,
                                                C.c_long, C.c_int, _dp, _dp, C.c_int, C.c_int,
                                                _dp, _dp, _dp]
    lib.oracle_feature_dim.restype = C.c_long
    lib.oracle_feature_dim.argtypes = [C.c_int, C.c_int, C.c_int]
    lib.oracle_phi_feature.argtypes = [_dp, C.c_int, C.c_int, C.c_int, _dp]
    lib.oracle_kernel_feature.restype = C.c_double
    lib.oracle_kernel_feature.argtypes = [_dp, _dp, C.c_int, C.c_int, C.c_int]
    lib.oracle_quadratic_feature_heads.argtypes = [C.c_int, _dp, _dp, _dp, C.c_long, C.c_int,
                                                   C.c_int, C.c_double, C.c_int, C.c_int, _dp]
    lib.oracle_recurrent_feature_heads.argtypes = [C.c_int, _dp, _dp, _dp, C.c_long, C.c_int,
                                                   C.c_int, C.c_double, C.c_int, C.c_int, _dp,
                                                   _dp, _dp]
    _lib = lib
    return lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor: read the stored values exactly
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: np.ndarray):
    if a is None:
        return None
    if a.dtype == np.float64:
        return a.ctypes.data_as(_dp)
    if a.dtype == np.int32:
        return a.ctypes.data_as(_ip)
    if a.dtype == np.int64:
        return a.ctypes.data_as(_lp)
    raise TypeError(a.dtype)


def set_threads(n: int) -> None:
    """Thread count for the OpenMP loops over heads."""
    _load().oracle_set_threads(int(n))


def threads() -> int:
    """Threads the OpenMP loops over heads use now."""
    return int(_load().oracle_threads())


def packed_dim(d: int) -> int:
    """D = d(d+1)/2."""
    return int(_load().oracle_packed_dim(d))


def packed_index(d: int, a: int, b: int) -> int:
    return int(_load().oracle_packed_index(d, a, b))


def phi(x) -> np.ndarray:
    """Packed rank-one PSD feature of every row of x [..., d] -> [..., D]."""
    x = _f64(x)
    d = x.shape[-1]
    D = packed_dim(d)
    rows = x.reshape(-1, d)
    out = np.empty((rows.shape[0], D))
    lib = _load()
    for i in range(rows.shape[0]):
        r = np.ascontiguousarray(rows[i])
        o = np.empty(D)
        lib.oracle_phi(_ptr(r), d, _ptr(o))
        out[i] = o
    return out.reshape(x.shape[:-1] + (D,))


def quadratic(q, k, v, eps: float, rows=None) -> np.ndarray:
    """Quadratic form o_i = sum_{j<=i}(q_i.k_j)^2 v_j / (sum_{j<=i}(q_i.k_j)^2 + eps).

    q, k [..., T, d], v [..., T, dv]. ``rows`` selects output rows (shared by
    all heads); the result is [..., len(rows) or T, dv].
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    lead = q.shape[:-2]
    T, d = q.shape[-2:]
    dv = v.shape[-1]
    nh = int(np.prod(lead)) if lead else 1
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = T if r is None else len(r)
    o = np.empty((nh, n, dv))
    _load().oracle_quadratic_heads(nh, _ptr(q), _ptr(k), _ptr(v), T, d, dv, eps, _ptr(r),
                                   0 if r is None else len(r), _ptr(o))
    return o.reshape(lead + (n, dv))


def recurrent(q, k, v, eps: float, H0=None, s0=None, readout: bool = True):
    """Literal recurrent form. Returns (o or None, H [..., D, dv], s [..., D])."""
    k, v = _f64(k), _f64(v)
    lead = k.shape[:-2]
    T, d = k.shape[-2:]
    dv = v.shape[-1]
    D = packed_dim(d)
    nh = int(np.prod(lead)) if lead else 1
    Hst = np.zeros((nh, D, dv)) if H0 is None else _f64(H0).reshape(nh, D, dv).copy()
    s = np.zeros((nh, D)) if s0 is None else _f64(s0).reshape(nh, D).copy()
    qq = _f64(q) if readout else None
    o = np.empty((nh, T, dv)) if readout else None
    _load().oracle_recurrent_heads(nh, _ptr(qq), _ptr(k), _ptr(v), T, d, dv, eps, _ptr(Hst),
                                   _ptr(s), _ptr(o))
    return (None if o is None else o.reshape(lead + (T, dv)),
            Hst.reshape(lead + (D, dv)), s.reshape(lead + (D,)))


# Multi-factor features ("Kernelized Linear Attention ...", s2.3 "Variants",
# reading R13 in kata_oracle.c): the head vector in g sub-vectors of d/g values;
# Mg keeps the g rank-one PSD factors apart, Sigma-g sums them.
FEATURES = {"m1": 0, "mg": 1, "sigmag": 2}


def feature_dim(d: int, feature: str, g: int) -> int:
    """Packed feature dimension of a variant (0: invalid)."""
    return int(_load().oracle_feature_dim(d, FEATURES[feature], g))


def phi_feature(x, feature: str, g: int) -> np.ndarray:
    """Packed feature psi of every row of x [..., d] -> [..., feature_dim]."""
    x = _f64(x)
    d = x.shape[-1]
    Df = feature_dim(d, feature, g)
    assert Df > 0
    rows = x.reshape(-1, d)
    out = np.empty((rows.shape[0], Df))
    lib = _load()
    for i in range(rows.shape[0]):
        r = np.ascontiguousarray(rows[i])
        o = np.empty(Df)
        lib.oracle_phi_feature(_ptr(r), d, FEATURES[feature], g, _ptr(o))
        out[i] = o
    return out.reshape(x.shape[:-1] + (Df,))


def kernel_feature(q, k, feature: str, g: int) -> float:
    """kappa(q, k) = <psi(q), psi(k)> from the sub-vectors' dot products."""
    q, k = _f64(q).ravel(), _f64(k).ravel()
    return float(_load().oracle_kernel_feature(_ptr(q), _ptr(k), q.shape[0], FEATURES[feature],
                                               g))


def quadratic_feature(q, k, v, eps: float, feature: str, g: int) -> np.ndarray:
    """o_i = sum_{j<=i} kappa(q_i,k_j) v_j / (sum_{j<=i} kappa(q_i,k_j) + eps) for [..., T, d]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    lead = q.shape[:-2]
    T, d = q.shape[-2:]
    dv = v.shape[-1]
    nh = int(np.prod(lead)) if lead else 1
    assert feature_dim(d, feature, g) > 0
    o = np.empty((nh, T, dv))
    _load().oracle_quadratic_feature_heads(nh, _ptr(q), _ptr(k), _ptr(v), T, d, dv, eps,
                                           FEATURES[feature], g, _ptr(o))
    return o.reshape(lead + (T, dv))


def recurrent_feature(q, k, v, eps: float, feature: str, g: int, H0=None, s0=None,
                      readout: bool = True):
    """Literal recurrent form with a variant's feature. Returns (o or None, H, s)."""
    k, v = _f64(k), _f64(v)
    lead = k.shape[:-2]
    T, d = k.shape[-2:]
    dv = v.shape[-1]
    Df = feature_dim(d, feature, g)
    assert Df > 0
    nh = int(np.prod(lead)) if lead else 1
    Hst = np.zeros((nh, Df, dv)) if H0 is None else _f64(H0).reshape(nh, Df, dv).copy()
    s = np.zeros((nh, Df)) if s0 is None else _f64(s0).reshape(nh, Df).copy()
    qq = _f64(q) if readout else None
    o = np.empty((nh, T, dv)) if readout else None
    _load().oracle_recurrent_feature_heads(nh, _ptr(qq), _ptr(k), _ptr(v), T, d, dv, eps,
                                           FEATURES[feature], g, _ptr(Hst), _ptr(s), _ptr(o))
    return (None if o is None else o.reshape(lead + (T, dv)),
            Hst.reshape(lead + (Df, dv)), s.reshape(lead + (Df,)))


def decode_feature(H0, s0, q, k, v, eps: float, feature: str, g: int):
    """Decode steps with a variant's feature: q, k, v [steps, B, H, d]."""
    q, k, v = (np.moveaxis(_f64(x), 0, -2) for x in (q, k, v))
    o, Hst, s = recurrent_feature(q, k, v, eps, feature, g, H0=H0, s0=s0)
    return np.moveaxis(o, -2, 0), Hst, s


def decode(H0, s0, q, k, v, eps: float):
    """Decode steps from state (H0, s0): q, k, v [steps, B, H, d].

    Each step updates the state with k, v and then reads out q (update first).
    Returns (o [steps, B, H, dv], H, s).
    """
    q, k, v = (np.moveaxis(_f64(x), 0, -2) for x in (q, k, v))
    o, Hst, s = recurrent(q, k, v, eps, H0=H0, s0=s0)
    return np.moveaxis(o, -2, 0), Hst, s


def sre(Hst, s, kc, vc, eps: float) -> np.ndarray:
    """SRE_j = ||phi(k_j)^T H / (phi(k_j)^T s + eps) - v_j||^2 for kc [..., n, d]."""
    kc, vc = _f64(kc), _f64(vc)
    lead = kc.shape[:-2]
    n, d = kc.shape[-2:]
    dv = vc.shape[-1]
    D = packed_dim(d)
    nh = int(np.prod(lead)) if lead else 1
    Hst = _f64(Hst).reshape(nh, D, dv)
    s = _f64(s).reshape(nh, D)
    out = np.empty((nh, n))
    _load().oracle_sre_heads(nh, _ptr(Hst), _ptr(s), _ptr(kc), _ptr(vc), n, d, dv, eps,
                             _ptr(out))
    return out.reshape(lead + (n,))


def topk(scores, pos, keep: int) -> np.ndarray:
    """Kept candidate slots [..., min(keep, n)], ascending position.

    Order: higher SRE first; an exact tie goes to the smaller position.
    """
    sc = _f64(scores)
    p = np.ascontiguousarray(np.asarray(pos), dtype=np.int32)
    lead = sc.shape[:-1]
    n = sc.shape[-1]
    m = min(keep, n)
    sc2, p2 = sc.reshape(-1, n), p.reshape(-1, n)
    out = np.empty((sc2.shape[0], m), dtype=np.int32)
    lib = _load()
    for h in range(sc2.shape[0]):
        a = np.ascontiguousarray(sc2[h])
        b = np.ascontiguousarray(p2[h])
        o = np.empty(max(m, 1), dtype=np.int32)
        got = lib.oracle_topk(_ptr(a), _ptr(b), n, keep, _ptr(o))
        assert got == m
        out[h] = o[:m]
    return out.reshape(lead + (m,))


def merge(Hst: np.ndarray, s: np.ndarray, kc, vc, keep_idx) -> None:
    """In place: add phi(k_j) v_j^T and phi(k_j) for every candidate not kept."""
    kc, vc = _f64(kc), _f64(vc)
    lead = kc.shape[:-2]
    n, d = kc.shape[-2:]
    dv = vc.shape[-1]
    nh = int(np.prod(lead)) if lead else 1
    ki = np.ascontiguousarray(np.asarray(keep_idx), dtype=np.int32).reshape(nh, -1)
    assert Hst.dtype == np.float64 and Hst.flags.c_contiguous
    assert s.dtype == np.float64 and s.flags.c_contiguous
    _load().oracle_merge_heads(nh, _ptr(Hst), _ptr(s), _ptr(kc), _ptr(vc), n, _ptr(ki),
                               ki.shape[1], d, dv)


def lola(q, k, v, window: int, cache: int, eps: float, tau: float | None = None,
         adopt=None, segments: int | None = None):
    """The LoLA schedule over whole sequences q, k, v [B, H, T, d] (reading R5).

    Segments of ``window`` tokens. Query i of segment g reads out against the
    window pairs at positions [max(0, window*(g-1)), i], the sparse-cache pairs
    and the linear state (H, s). At the end of every segment g >= 1, segment
    g-1 leaves the window; its pairs and the cached pairs are the candidates,
    scored by SRE against the current (H, s); the ``cache`` highest stay, the
    others are merged into (H, s).

    ``adopt(u, cand_pos, scores, keep_idx)`` may return another kept set (same
    shape, candidate slots) for update u; the schedule then continues from it.
    ``segments`` stops after that many segments (a bounded sample).

    Returns dict(o [B,H,T,dv], H, s, kept_pos: list of [B,H,m] arrays per update).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hh, T, d = q.shape
    dv = v.shape[-1]
    D = packed_dim(d)
    nh = B * Hh
    tau = d ** -0.5 if tau is None else tau
    U = window
    G = (T + U - 1) // U if segments is None else segments
    qf, kf, vf = (x.reshape(nh, T, -1) for x in (q, k, v))
    Hst = np.zeros((nh, D, dv))
    s = np.zeros((nh, D))
    o = np.zeros((nh, T, dv))
    cache_pos = np.zeros((nh, 0), dtype=np.int64)
    lib = _load()
    kept_hist = []
    for g in range(G):
        seg0 = g * U
        nq = min(U, T - seg0)
        w0 = max(0, U * (g - 1))
        nc = cache_pos.shape[1]
        ck = np.ascontiguousarray(np.take_along_axis(kf, cache_pos[:, :, None], axis=1)) \
            if nc else np.zeros((nh, 1, d))
        cv = np.ascontiguousarray(np.take_along_axis(vf, cache_pos[:, :, None], axis=1)) \
            if nc else np.zeros((nh, 1, dv))
        lib.oracle_hybrid_segment_heads(nh, _ptr(qf), _ptr(kf), _ptr(vf), T, d, dv, eps, tau,
                                        w0, seg0, nq, _ptr(ck), _ptr(cv), nc, max(nc, 1),
                                        _ptr(Hst), _ptr(s), _ptr(o))
        if g < 1:
            continue
        ev = np.arange(U * (g - 1), U * g, dtype=np.int64)
        cand = np.concatenate([cache_pos, np.broadcast_to(ev, (nh, U))], axis=1)
        kc = np.ascontiguousarray(np.take_along_axis(kf, cand[:, :, None], axis=1))
        vc = np.ascontiguousarray(np.take_along_axis(vf, cand[:, :, None], axis=1))
        sc = sre(Hst, s, kc, vc, eps)
        keep_idx = topk(sc, cand.astype(np.int32), cache)
        if adopt is not None:
            alt = adopt(g - 1, cand.reshape(B, Hh, -1), sc.reshape(B, Hh, -1),
                        keep_idx.reshape(B, Hh, -1))
            if alt is not None:
                keep_idx = np.ascontiguousarray(np.asarray(alt), dtype=np.int32).reshape(nh, -1)
        merge(Hst, s, kc, vc, keep_idx)
        cache_pos = np.take_along_axis(cand, keep_idx.astype(np.int64), axis=1)
        kept_hist.append(cache_pos.reshape(B, Hh, -1).copy())
    return dict(o=o.reshape(B, Hh, T, dv), H=Hst.reshape(B, Hh, D, dv), s=s.reshape(B, Hh, D),
                kept_pos=kept_hist)
