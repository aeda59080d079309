"""Pins for the fp64 oracle: closed forms, invariants, exact-rational brute force,
reductions to library routines and hand-worked fixtures. CPU only.

Each check is chosen so that a plausible slip in the oracle (a dropped sqrt(2),
an exclusive instead of inclusive causal sum, eps in the wrong place, a
transposed index, a wrong tie rule, an off-by-one in the LoLA schedule) fails
at least one of them.
"""
import json
from fractions import Fraction
from pathlib import Path

import numpy as np
import pytest
import torch

import oracle

GOLDEN = Path(__file__).resolve().parent / "golden"


def rel(a, b):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ------------------------------------------------------------------ phi -----

@pytest.mark.parametrize("d", [1, 2, 3, 7, 16, 32, 64])
def test_phi_dimension_and_bijective_index(d):
    D = oracle.packed_dim(d)
    assert D == d * (d + 1) // 2
    idx = sorted(oracle.packed_index(d, a, b) for a in range(d) for b in range(a, d))
    assert idx == list(range(D))


@pytest.mark.parametrize("d", [2, 5, 16, 64])
def test_phi_frobenius_identity(d):
    """<phi(x), phi(y)> = <x x^T, y y^T>_F = (x.y)^2 and ||phi(x)||^2 = ||x||^4."""
    rng = np.random.default_rng(d)
    x = rng.standard_normal((50, d))
    y = rng.standard_normal((50, d))
    px, py = oracle.phi(x), oracle.phi(y)
    lhs = np.sum(px * py, axis=-1)
    rhs = np.sum(x * y, axis=-1) ** 2
    scale = np.sum(x * x, -1) * np.sum(y * y, -1)  # rounding error scales with this
    assert np.max(np.abs(lhs - rhs) / scale) < 1e-13
    assert np.allclose(np.sum(px * px, -1), np.sum(x * x, -1) ** 2, rtol=1e-14, atol=0)


@pytest.mark.parametrize("d", [3, 8])
def test_phi_unpacks_to_outer_product(d):
    """Unpacking the triangle (dividing off-diagonals by sqrt 2) gives np.outer(x, x)."""
    x = np.random.default_rng(1).standard_normal(d)
    p = oracle.phi(x[None])[0]
    M = np.zeros((d, d))
    for a in range(d):
        for b in range(a, d):
            val = p[oracle.packed_index(d, a, b)]
            if a != b:
                val /= np.sqrt(2.0)
            M[a, b] = M[b, a] = val
    assert np.allclose(M, np.outer(x, x), rtol=1e-15, atol=1e-15)


# ----------------------------------------------------- quadratic vs rec -----

@pytest.mark.parametrize("d,dv,T", [(1, 1, 9), (4, 3, 33), (16, 16, 70), (32, 8, 41)])
def test_quadratic_equals_recurrent(d, dv, T):
    rng = np.random.default_rng(d * 100 + T)
    q = rng.standard_normal((2, 3, T, d))
    k = rng.standard_normal((2, 3, T, d))
    v = rng.standard_normal((2, 3, T, dv))
    oq = oracle.quadratic(q, k, v, 1e-6)
    orc, _, _ = oracle.recurrent(q, k, v, 1e-6)
    assert rel(orc, oq) < 1e-12


def test_quadratic_row_subset_matches_full():
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((2, 50, 4)) for _ in range(3))
    rows = np.array([0, 7, 49])
    assert np.array_equal(oracle.quadratic(q, k, v, 1e-6, rows=rows),
                          oracle.quadratic(q, k, v, 1e-6)[:, rows])


def _exact_quadratic(q, k, v, eps):
    """Brute force in exact rationals: o_i = sum_{j<=i} w_ij v_j / (sum w_ij + eps)."""
    T = len(q)
    out = []
    for i in range(T):
        num = [Fraction(0)] * len(v[0])
        den = Fraction(0)
        for j in range(i + 1):
            w = sum(Fraction(a) * Fraction(b) for a, b in zip(q[i], k[j])) ** 2
            den += w
            num = [n + w * Fraction(x) for n, x in zip(num, v[j])]
        out.append([n / (den + eps) for n in num])
    return out


@pytest.mark.parametrize("d,T", [(1, 16), (2, 12), (3, 9), (4, 16)])
def test_exact_rational_brute_force(d, T):
    rng = np.random.default_rng(10 * d + T)
    q = rng.integers(-3, 4, size=(T, d))
    k = rng.integers(-3, 4, size=(T, d))
    v = rng.integers(-5, 6, size=(T, 2))
    eps = Fraction(1, 10 ** 6)
    exact = _exact_quadratic(q.tolist(), k.tolist(), v.tolist(), eps)
    ex = np.array([[float(x) for x in row] for row in exact])
    oq = oracle.quadratic(q[None], k[None], v[None], 1e-6)[0]
    orc, _, _ = oracle.recurrent(q[None], k[None], v[None], 1e-6)
    assert np.allclose(oq, ex, rtol=1e-13, atol=1e-13)
    assert np.allclose(orc[0], ex, rtol=1e-12, atol=1e-12)


def test_golden_worked_examples():
    spec = json.loads((GOLDEN / "quadratic_worked_d2.json").read_text())
    for case in spec["cases"]:
        q, k, v = (np.array(case[n], dtype=np.float64)[None] for n in "qkv")
        want = np.array(case["o"])
        for got in (oracle.quadratic(q, k, v, case["eps"])[0],
                    oracle.recurrent(q, k, v, case["eps"])[0][0]):
            assert np.allclose(got, want, rtol=1e-12, atol=1e-12), case["name"]


# ------------------------------------------------------ closed forms --------

def test_single_token_closed_form():
    rng = np.random.default_rng(4)
    for _ in range(5):
        q, k, v = rng.standard_normal(6), rng.standard_normal(6), rng.standard_normal(6)
        a = float(q @ k) ** 2
        want = a * v / (a + 1e-6)
        for got in (oracle.quadratic(q[None, None], k[None, None], v[None, None], 1e-6),
                    oracle.recurrent(q[None, None], k[None, None], v[None, None], 1e-6)[0]):
            assert np.allclose(got.reshape(-1), want, rtol=1e-14, atol=0)


def test_orthogonal_keys_recall_exactly():
    """k_j = e_j; q_i = k_m (m <= i): only (k_m.k_m)^2 = 1 survives -> v_m/(1+eps)."""
    T = d = 12
    rng = np.random.default_rng(5)
    k = np.eye(d)[:T]
    m = np.array([rng.integers(0, i + 1) for i in range(T)])
    q = k[m]
    v = rng.standard_normal((T, 5))
    want = v[m] / (1 + 1e-6)
    assert np.allclose(oracle.quadratic(q[None], k[None], v[None], 1e-6)[0], want, rtol=1e-15)
    assert np.allclose(oracle.recurrent(q[None], k[None], v[None], 1e-6)[0][0], want,
                       rtol=1e-14)


def test_identical_keys_give_scaled_running_mean():
    """All k_j = k: o_i = mean(v_0..v_i) * (i+1)w / ((i+1)w + eps), w = (q_i.k)^2.

    An exclusive causal sum (j < i) or a missing eps would both fail this.
    """
    T, d = 20, 4
    rng = np.random.default_rng(6)
    k = np.tile(rng.standard_normal(d), (T, 1))
    q = rng.standard_normal((T, d)) * 1e-3
    v = rng.standard_normal((T, 3))
    w = (q @ k[0]) ** 2
    n = np.arange(1, T + 1)[:, None]
    want = np.cumsum(v, 0) / n * (n * w[:, None]) / (n * w[:, None] + 1e-6)
    assert np.allclose(oracle.quadratic(q[None], k[None], v[None], 1e-6)[0], want, rtol=1e-12)
    assert np.allclose(oracle.recurrent(q[None], k[None], v[None], 1e-6)[0][0], want,
                       rtol=1e-11)


def test_convex_output_gate():
    """At eps=0, o_i = g_i r_i + (1 - g_i) v_i (output gating, KATA s2.1).

    r_i is the readout of q_i over the earlier pairs alone and
    g_i = sum_{j<i} w_ij / sum_{j<=i} w_ij; each o_i lies in the convex hull
    of v_0..v_i.
    """
    T, d = 30, 5
    rng = np.random.default_rng(7)
    q, k, v = rng.standard_normal((T, d)), rng.standard_normal((T, d)), rng.standard_normal((T, 4))
    o = oracle.recurrent(q[None], k[None], v[None], 0.0)[0][0]
    for i in range(1, T):
        kk = np.vstack([k[:i], np.zeros(d)])  # zero key at position i adds no weight
        vv = np.vstack([v[:i], np.zeros(4)])
        qq = np.tile(q[i], (i + 1, 1))
        r = oracle.quadratic(qq[None], kk[None], vv[None], 0.0)[0][i]
        w = (k[: i + 1] @ q[i]) ** 2
        g = w[:i].sum() / w.sum()
        assert np.allclose(o[i], g * r + (1 - g) * v[i], rtol=1e-10, atol=1e-12)
        assert np.all(np.abs(o[i]) <= np.abs(v[: i + 1]).max(0) + 1e-12)


def test_scale_invariance_without_eps():
    rng = np.random.default_rng(8)
    q, k, v = (rng.standard_normal((1, 25, 6)) for _ in range(3))
    base = oracle.quadratic(q, k, v, 0.0)
    assert rel(oracle.quadratic(3.5 * q, k, v, 0.0), base) < 1e-13
    assert rel(oracle.quadratic(q, -0.25 * k, v, 0.0), base) < 1e-13
    assert rel(oracle.recurrent(q, 2.0 * k, v, 0.0)[0], base) < 1e-12


def test_causality_and_linearity_in_v():
    rng = np.random.default_rng(9)
    q, k, v = (rng.standard_normal((1, 40, 4)) for _ in range(3))
    o = oracle.recurrent(q, k, v, 1e-6)[0]
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[:, 25:] += 1.0
    k2[:, 25:] -= 2.0
    v2[:, 25:] *= 3.0
    o2 = oracle.recurrent(q2, k2, v2, 1e-6)[0]
    assert np.array_equal(o[:, :25], o2[:, :25])
    va, vb = rng.standard_normal((2, 1, 40, 4))
    oa = oracle.quadratic(q, k, va, 1e-6)
    ob = oracle.quadratic(q, k, vb, 1e-6)
    assert rel(oracle.quadratic(q, k, va + 2 * vb, 1e-6), oa + 2 * ob) < 1e-13


def test_head_permutation_equivariance():
    rng = np.random.default_rng(10)
    q, k, v = (rng.standard_normal((6, 17, 3)) for _ in range(3))
    perm = rng.permutation(6)
    o = oracle.recurrent(q, k, v, 1e-6)[0]
    assert np.array_equal(oracle.recurrent(q[perm], k[perm], v[perm], 1e-6)[0], o[perm])


# ------------------------------------------------------------ decode -------

def test_decode_continues_recurrent_and_quadratic():
    """prefill(T0) state then decode steps T0..T == the whole sequence."""
    rng = np.random.default_rng(11)
    B, H, T, T0, d = 2, 2, 24, 10, 4
    q, k, v = (rng.standard_normal((B, H, T, d)) for _ in range(3))
    _, H0, s0 = oracle.recurrent(q[:, :, :T0], k[:, :, :T0], v[:, :, :T0], 1e-6,
                                 readout=False)
    steps = lambda x: np.moveaxis(x[:, :, T0:], 2, 0)  # noqa: E731
    od, Hd, sd = oracle.decode(H0, s0, steps(q), steps(k), steps(v), 1e-6)
    full = oracle.quadratic(q, k, v, 1e-6)
    assert rel(od, steps(full)) < 1e-12
    _, Hf, sf = oracle.recurrent(q, k, v, 1e-6)
    assert rel(Hd, Hf) < 1e-13 and rel(sd, sf) < 1e-13


def test_normaliser_equals_sum_of_squared_dots():
    """phi(q)^T s = sum_j (q.k_j)^2 >= 0, checked against numpy's matmul."""
    rng = np.random.default_rng(12)
    k = rng.standard_normal((1, 60, 7))
    _, _, s = oracle.recurrent(None, k, np.zeros((1, 60, 1)), 0.0, readout=False)
    qs = rng.standard_normal((10, 7))
    den = oracle.phi(qs) @ s[0]
    assert np.all(den >= 0)
    assert np.allclose(den, ((qs @ k[0].T) ** 2).sum(1), rtol=1e-12)


# ------------------------------------------------------------- SRE ---------

def _state_from_pairs(kk, vv):
    _, Hs, s = oracle.recurrent(None, kk[None], vv[None], 0.0, readout=False)
    return Hs, s


def test_sre_golden():
    spec = json.loads((GOLDEN / "sre_worked_d2.json").read_text())
    Hs, s = _state_from_pairs(np.array(spec["stored"]["k"], float),
                              np.array(spec["stored"]["v"], float))
    kc = np.array([c["k"] for c in spec["cases"]], float)[None]
    vc = np.array([c["v"] for c in spec["cases"]], float)[None]
    got = oracle.sre(Hs, s, kc, vc, spec["eps"])[0]
    assert np.allclose(got, [c["sre"] for c in spec["cases"]], rtol=1e-13, atol=1e-13)


def test_sre_closed_forms():
    rng = np.random.default_rng(13)
    d, eps = 8, 1e-3
    kc, vc = rng.standard_normal((1, 5, d)), rng.standard_normal((1, 5, d))
    D = oracle.packed_dim(d)
    # empty state: prediction 0/(0+eps) = 0 -> ||v||^2
    assert np.allclose(oracle.sre(np.zeros((1, D, d)), np.zeros((1, D)), kc, vc, eps)[0],
                       (vc[0] ** 2).sum(1), rtol=1e-15)
    # single stored pair scored on itself: ||v||^2 (eps / (||k||^4 + eps))^2
    for j in range(5):
        Hs, s = _state_from_pairs(kc[0, j:j + 1], vc[0, j:j + 1])
        got = oracle.sre(Hs, s, kc[:, j:j + 1], vc[:, j:j + 1], eps)[0, 0]
        n4 = float(kc[0, j] @ kc[0, j]) ** 2
        assert np.isclose(got, (vc[0, j] ** 2).sum() * (eps / (n4 + eps)) ** 2, rtol=1e-10)
    # mutually orthogonal stored keys: each pair's SRE is its single-pair value
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    kk = Q.T[:6] * rng.uniform(0.5, 2.0, size=(6, 1))
    vv = rng.standard_normal((6, d))
    Hs, s = _state_from_pairs(kk, vv)
    got = oracle.sre(Hs, s, kk[None], vv[None], eps)[0]
    n4 = (kk ** 2).sum(1) ** 2
    assert np.allclose(got, (vv ** 2).sum(1) * (eps / (n4 + eps)) ** 2, rtol=1e-6)


def test_sre_matches_quadratic_readout():
    """SRE_j = ||o - v_j||^2 where o is the quadratic-form readout of query k_j
    over the stored pairs (a zero key at the query position adds no weight)."""
    rng = np.random.default_rng(14)
    m, d, eps = 15, 4, 1e-6
    kk, vv = rng.standard_normal((m, d)), rng.standard_normal((m, 3))
    Hs, s = _state_from_pairs(kk, vv)
    kc, vc = rng.standard_normal((1, 6, d)), rng.standard_normal((1, 6, 3))
    got = oracle.sre(Hs, s, kc, vc, eps)[0]
    for j in range(6):
        K = np.vstack([kk, np.zeros(d)])
        V = np.vstack([vv, np.zeros(3)])
        Q = np.tile(kc[0, j], (m + 1, 1))
        pred = oracle.quadratic(Q[None], K[None], V[None], eps)[0, m]
        assert np.isclose(got[j], ((pred - vc[0, j]) ** 2).sum(), rtol=1e-11)


# ------------------------------------------------------------ top-k --------

@pytest.mark.parametrize("seed", range(6))
def test_topk_against_sorted(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 9))
    keep = int(rng.integers(0, 10))
    sc = rng.integers(0, 3, size=n).astype(float)  # many exact ties on purpose
    pos = rng.permutation(50)[:n].astype(np.int32)
    got = oracle.topk(sc[None], pos[None], keep)[0]
    order = sorted(range(n), key=lambda j: (-sc[j], pos[j]))
    want = sorted(order[:min(keep, n)], key=lambda j: pos[j])
    assert got.tolist() == want
    kept = set(got.tolist())
    for j in kept:
        for i in set(range(n)) - kept:
            assert sc[j] > sc[i] or (sc[j] == sc[i] and pos[j] < pos[i])


# ------------------------------------------------------------ merge --------

def test_merge_all_equals_recurrent_state_and_none_is_identity():
    rng = np.random.default_rng(15)
    d, n = 5, 9
    kc, vc = rng.standard_normal((2, n, d)), rng.standard_normal((2, n, d))
    D = oracle.packed_dim(d)
    Hs, s = np.zeros((2, D, d)), np.zeros((2, D))
    oracle.merge(Hs, s, kc, vc, np.zeros((2, 0), np.int32))
    _, Hr, sr = oracle.recurrent(None, kc, vc, 0.0, readout=False)
    assert rel(Hs, Hr) < 1e-14 and rel(s, sr) < 1e-14
    H2, s2 = Hs.copy(), s.copy()
    oracle.merge(H2, s2, kc, vc, np.tile(np.arange(n, dtype=np.int32), (2, 1)))
    assert np.array_equal(H2, Hs) and np.array_equal(s2, s)


# ------------------------------------------------------------- LoLA --------

def test_lola_without_merges_is_causal_softmax_attention():
    """Cache capacity >= T: nothing is ever merged, so every earlier pair is in
    the window or the cache and, at eps=0, the hybrid readout is causal softmax
    attention with scale 1/sqrt(d) (torch's reference SDPA in fp64)."""
    rng = np.random.default_rng(16)
    B, H, T, d, U = 1, 2, 48, 8, 4
    q, k, v = (rng.standard_normal((B, H, T, d)) for _ in range(3))
    res = oracle.lola(q, k, v, window=U, cache=T, eps=0.0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=True)
    assert rel(res["o"], ref.numpy()) < 1e-12
    assert np.all(res["H"] == 0) and np.all(res["s"] == 0)


def test_lola_orthogonal_keys_trace():
    """Hand-traced schedule: k_t = e_t, so a candidate's prediction from the
    state is 0 and its SRE is ||v||^2. The cache then always holds the `cache`
    largest-norm values among all evicted tokens (ties: earlier position), the
    first merge happens at the third update, and the final state holds exactly
    the evicted pairs that were dropped."""
    T = d = 24
    U, lam = 4, 3
    rng = np.random.default_rng(17)
    k = np.eye(d)[None, None]
    v = rng.standard_normal((1, 1, T, 3))
    norms = (v[0, 0] ** 2).sum(1)
    norms[5] = norms[2]  # an exact tie, decided by position
    v[0, 0, 5] = v[0, 0, 2]
    q = rng.standard_normal((1, 1, T, d))
    res = oracle.lola(q, k, v, window=U, cache=lam, eps=1e-6)
    G = T // U
    assert len(res["kept_pos"]) == G - 1
    for u, kept in enumerate(res["kept_pos"]):
        evicted = np.arange(0, U * (u + 1))
        order = sorted(evicted, key=lambda j: (-norms[j], j))
        want = sorted(order[:lam])
        assert kept[0, 0].tolist() == want, u
    dropped = sorted(set(range(U * (G - 1))) - set(res["kept_pos"][-1][0, 0].tolist()))
    _, Hr, sr = oracle.recurrent(None, k[:, :, dropped], v[:, :, dropped], 0.0, readout=False)
    assert rel(res["H"], Hr) < 1e-14 and rel(res["s"], sr) < 1e-14


def test_lola_no_cache_state_is_evicted_prefix():
    """Cache capacity 0: every evicted pair is merged at once, so after the
    schedule the state equals the recurrent state over all evicted tokens, and
    a query's readout splits into window-softmax and linear-state terms."""
    rng = np.random.default_rng(18)
    B, H, T, d, U = 1, 1, 32, 4, 8
    q, k, v = (rng.standard_normal((B, H, T, d)) for _ in range(3))
    res = oracle.lola(q, k, v, window=U, cache=0, eps=1e-6)
    G = T // U
    _, Hr, sr = oracle.recurrent(None, k[:, :, :U * (G - 1)], v[:, :, :U * (G - 1)], 0.0,
                                 readout=False)
    assert rel(res["H"], Hr) < 1e-13 and rel(res["s"], sr) < 1e-13
    i = 27  # segment 3: window [16, 27], state over tokens [0, 16)
    _, Hi, si = oracle.recurrent(None, k[:, :, :16], v[:, :, :16], 0.0, readout=False)
    w = np.exp(k[0, 0, 16:i + 1] @ q[0, 0, i] / np.sqrt(d))
    pq = oracle.phi(q[0, 0, i][None])[0]
    num = w @ v[0, 0, 16:i + 1] + pq @ Hi[0, 0]
    den = w.sum() + pq @ si[0, 0] + 1e-6
    assert np.allclose(res["o"][0, 0, i], num / den, rtol=1e-12)


# ---------------------------------------------- multi-factor features -----
# KATA page s2.3 "Variants" (KATA-Mg: several PSD factors; KATA-Sigma-g: summed
# PSD factors), reading R13: the head vector in g sub-vectors of p = d/g values.

VARIANTS = [("mg", 2), ("mg", 4), ("sigmag", 2), ("sigmag", 4), ("mg", 1), ("sigmag", 1)]


@pytest.mark.parametrize("feature,g", VARIANTS)
def test_feature_dimension(feature, g):
    d = 16
    p = d // g
    want = g * p * (p + 1) // 2 if feature == "mg" else p * (p + 1) // 2
    assert oracle.feature_dim(d, feature, g) == want
    assert oracle.feature_dim(16, "mg", 3) == 0  # g must divide d
    assert oracle.feature_dim(16, "m1", 2) == 0


def test_one_factor_is_the_rank_one_feature():
    """g = 1: both variants are psi(u) = u u^T, i.e. M1 (pinned above)."""
    x = np.random.default_rng(5).standard_normal((7, 16))
    for feature in ("mg", "sigmag", "m1"):
        assert np.array_equal(oracle.phi_feature(x, feature, 1), oracle.phi(x))


@pytest.mark.parametrize("g", [2, 4, 8])
def test_factor_features_built_from_the_rank_one_feature(g):
    """Mg's feature is the pinned M1 feature of each sub-vector, in order;
    Sigma-g's is their sum (independent of the oracle's own loops)."""
    d = 16
    p = d // g
    x = np.random.default_rng(g).standard_normal((5, d))
    parts = [oracle.phi(x[:, r * p:(r + 1) * p]) for r in range(g)]
    assert np.allclose(oracle.phi_feature(x, "mg", g), np.concatenate(parts, axis=1),
                       rtol=1e-15, atol=1e-15)
    assert np.allclose(oracle.phi_feature(x, "sigmag", g), np.sum(parts, axis=0),
                       rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("feature,g", VARIANTS)
def test_feature_inner_product_is_the_kernel(feature, g):
    """<psi(x), psi(y)> (feature map) equals kappa(x, y) (sub-vector dot products)."""
    rng = np.random.default_rng(17 + g)
    for _ in range(20):
        x, y = rng.standard_normal(16), rng.standard_normal(16)
        lhs = float(oracle.phi_feature(x[None], feature, g)[0] @
                    oracle.phi_feature(y[None], feature, g)[0])
        rhs = oracle.kernel_feature(x, y, feature, g)
        assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(rhs))
        assert rhs >= 0.0  # PSD factors: non-negative weights


def test_factor_kernels_distinguish_kept_apart_from_summed():
    """A query living in factor 1 and a key living in factor 2: Mg has no
    cross-factor term (weight 0), Sigma-g does ((q_1.k_2)^2); within one factor
    both reduce to M1 on that sub-vector."""
    d, g, p = 8, 2, 4
    rng = np.random.default_rng(2)
    a, b = rng.standard_normal(p), rng.standard_normal(p)
    q = np.concatenate([a, np.zeros(p)])
    k_other = np.concatenate([np.zeros(p), b])
    k_same = np.concatenate([b, np.zeros(p)])
    assert oracle.kernel_feature(q, k_other, "mg", g) == 0.0
    assert np.isclose(oracle.kernel_feature(q, k_other, "sigmag", g), float(a @ b) ** 2,
                      rtol=1e-14)
    for feature in ("mg", "sigmag"):
        assert np.isclose(oracle.kernel_feature(q, k_same, feature, g), float(a @ b) ** 2,
                          rtol=1e-14)
    # Mg of a full vector is the sum of M1 kernels of the sub-vectors
    x, y = rng.standard_normal(d), rng.standard_normal(d)
    m1 = sum(oracle.kernel_feature(x[r * p:(r + 1) * p], y[r * p:(r + 1) * p], "m1", 1)
             for r in range(g))
    assert np.isclose(oracle.kernel_feature(x, y, "mg", g), m1, rtol=1e-14)


@pytest.mark.parametrize("feature,g", VARIANTS)
def test_feature_quadratic_equals_recurrent(feature, g):
    rng = np.random.default_rng(23 * g)
    T, d, dv = 37, 16, 5
    q, k, v = (rng.standard_normal((2, T, d)), rng.standard_normal((2, T, d)),
               rng.standard_normal((2, T, dv)))
    oq = oracle.quadratic_feature(q, k, v, 1e-6, feature, g)
    orc, H, s = oracle.recurrent_feature(q, k, v, 1e-6, feature, g)
    assert rel(orc, oq) < 1e-12
    # the state is the sum of the key features (normaliser) and their v-outer products
    pk = oracle.phi_feature(k, feature, g)
    assert np.allclose(s, pk.sum(axis=1), rtol=1e-12, atol=1e-12)
    assert np.allclose(H, np.einsum("htr,hte->hre", pk, v), rtol=1e-12, atol=1e-12)


def _exact_factor_quadratic(q, k, v, eps, feature, g):
    """Exact rationals: kappa from sub-vector dot products, inclusive causal sum."""
    d = len(q[0])
    p = d // g
    out = []
    for i in range(len(q)):
        num = [Fraction(0)] * len(v[0])
        den = Fraction(0)
        for j in range(i + 1):
            w = Fraction(0)
            for r in range(g):
                for t in range(g):
                    if feature == "mg" and t != r:
                        continue
                    w += sum(Fraction(q[i][r * p + a]) * Fraction(k[j][t * p + a])
                             for a in range(p)) ** 2
            den += w
            num = [n + w * Fraction(x) for n, x in zip(num, v[j])]
        out.append([float(n / (den + eps)) for n in num])
    return np.array(out)


@pytest.mark.parametrize("feature,g", [("mg", 2), ("sigmag", 2), ("sigmag", 3)])
def test_feature_exact_rational_brute_force(feature, g):
    d = 6
    rng = np.random.default_rng(41 + g)
    T = 9
    q = rng.integers(-3, 4, (T, d))
    k = rng.integers(-3, 4, (T, d))
    v = rng.integers(-5, 6, (T, 2))
    eps = Fraction(1, 10 ** 6)
    exact = _exact_factor_quadratic(q.tolist(), k.tolist(), v.tolist(), eps, feature, g)
    for got in (oracle.quadratic_feature(q, k, v, 1e-6, feature, g),
                oracle.recurrent_feature(q, k, v, 1e-6, feature, g)[0]):
        assert np.allclose(got, exact, rtol=1e-12, atol=1e-12)


def test_feature_decode_continues_recurrent():
    rng = np.random.default_rng(9)
    T0, T1, d = 20, 6, 16
    q, k, v = (rng.standard_normal((3, T0 + T1, d)) for _ in range(3))
    for feature, g in (("mg", 4), ("sigmag", 2)):
        full, Hf, sf = oracle.recurrent_feature(q, k, v, 1e-6, feature, g)
        _, H0, s0 = oracle.recurrent_feature(None, k[:, :T0], v[:, :T0], 1e-6, feature, g,
                                             readout=False)
        od, Hd, sd = oracle.decode_feature(H0, s0, *(np.moveaxis(x[:, T0:], 1, 0)
                                                     for x in (q, k, v)), 1e-6, feature, g)
        assert rel(np.moveaxis(od, 0, 1), full[:, T0:]) < 1e-12
        assert rel(Hd, Hf) < 1e-12 and rel(sd, sf) < 1e-12
