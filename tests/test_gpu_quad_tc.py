"""The tcgen05 quadratic form (kata_prefill_ex, KATA_FORM_QUADRATIC, and the
output-only calls kata_prefill routes to it) against the fp64 oracle's
plain definition o_i = sum_{j<=i} (q_i.k_j)^2 v_j / (sum_{j<=i} (q_i.k_j)^2 + eps),
and the final state that the state pass computes beside it (GPU)."""
import numpy as np
import pytest
import torch

import kernelized_linear_attention_chunked_b200 as kata
import oracle
from _util import cuda, rel_l2, tol
from kernelized_linear_attention_chunked_b200.inputs import WORKLOADS, prefill_inputs

pytestmark = pytest.mark.gpu

BF16 = torch.bfloat16


def quad(q, k, v, eps=1e-6):
    o, _, _ = kata.prefill(*cuda(q, k, v), chunk=64, eps=eps, state=False, form="quadratic")
    kata.sync_status()
    return o


# (d, T): one tile (the diagonal only), three and eight tiles (two-stage K/V
# ring wraps), both head dims
SHAPES = [(32, 128), (32, 384), (32, 1024), (64, 128), (64, 640), (64, 1024)]


@pytest.mark.parametrize("d,T", SHAPES)
def test_matches_the_oracle(d, T):
    q, k, v = prefill_inputs(1, 3, T, d, dtype="bf16", seed=d * 7 + T)
    o = quad(q, k, v)
    assert rel_l2(o, oracle.quadratic(q, k, v, 1e-6)) < tol("bf16")


@pytest.mark.parametrize("d", [32, 64])
def test_same_result_as_the_chunked_form(d):
    q, k, v = prefill_inputs(2, 2, 768, d, dtype="bf16", seed=40 + d)
    oq = quad(q, k, v)
    oc, _, _ = kata.prefill(*cuda(q, k, v), chunk=64, state=False, form="chunked")
    kata.sync_status()
    ref = oracle.quadratic(q, k, v, 1e-6)
    assert rel_l2(oq, ref) < tol("bf16") and rel_l2(oc, ref) < tol("bf16")
    # the two forms round differently but agree far inside the tolerance
    assert rel_l2(oq, oc.double().cpu().numpy()) < tol("bf16")


def test_many_heads_and_tiles():
    # grid 160 heads x 2 tiles: more CTAs than two waves of the SMs
    q, k, v = prefill_inputs(8, 20, 256, 32, dtype="bf16", seed=9)
    o = quad(q, k, v)
    assert rel_l2(o, oracle.quadratic(q, k, v, 1e-6)) < tol("bf16")


def test_causality_bit_exact():
    q, k, v = prefill_inputs(1, 2, 512, 64, dtype="bf16", seed=13)
    o0 = quad(q, k, v)
    t = 300
    k2, v2 = k.clone(), v.clone()
    k2[:, :, t] = 1.5 * k2[:, :, t]
    v2[:, :, t] = 2 * v2[:, :, t]
    o1 = quad(q, k2, v2)
    assert torch.equal(o0[:, :, :t], o1[:, :, :t])
    assert not torch.equal(o0[:, :, t:], o1[:, :, t:])


def test_first_token_and_eps():
    # o_0 = a v_0 / (a + eps) with a = (q_0.k_0)^2; a large eps shrinks every row
    q, k, v = prefill_inputs(1, 1, 128, 32, dtype="bf16", seed=21)
    for eps in (1e-6, 0.5):
        o = quad(q, k, v, eps)
        assert rel_l2(o, oracle.quadratic(q, k, v, eps)) < tol("bf16")
        a = float((q[0, 0, 0].double() @ k[0, 0, 0].double()) ** 2)
        want = a * v[0, 0, 0].double().numpy() / (a + eps)
        assert rel_l2(o[0, 0, 0], want) < tol("bf16")


def test_auto_form_routes_output_only_calls():
    B, H, T, d = 1, 2, 256, 32
    assert kata.prefill_auto_form(B, H, T, d, 64, BF16) == "quadratic"
    q, k, v = prefill_inputs(B, H, T, d, dtype="bf16", seed=31)
    n0 = kata.launch_count()
    o, _, _ = kata.prefill(*cuda(q, k, v), chunk=64, state=False)
    kata.sync_status()
    assert kata.launch_count() - n0 == 1  # one kernel: the quadratic form
    assert rel_l2(o, oracle.quadratic(q, k, v, 1e-6)) < tol("bf16")
    # with the final state requested kata_prefill takes the chunked form (the
    # state kernel and the readout kernel)
    assert kata.prefill_auto_form(B, H, T, d, 64, BF16, with_state=True) == "chunked"
    n0 = kata.launch_count()
    kata.prefill(*cuda(q, k, v), chunk=64)
    kata.sync_status()
    assert kata.launch_count() - n0 == 2


# output and final state together: o by the quadratic form on the caller's
# stream, (H, s) by the state pass on the side stream, joined back
@pytest.mark.parametrize("d,T", [(32, 128), (32, 1024), (64, 640), (64, 2048)])
def test_output_and_final_state(d, T):
    q, k, v = prefill_inputs(2, 3, T, d, dtype="bf16", seed=50 + d + T)
    o, H, s = kata.prefill(*cuda(q, k, v), chunk=64, form="quadratic")
    kata.sync_status()
    ro, rH, rs = oracle.recurrent(q, k, v, 1e-6)
    assert rel_l2(o, ro) < tol("bf16")
    assert rel_l2(H, rH) < tol("bf16")
    assert rel_l2(s, rs) < tol("bf16")
    # the same state as the chunked form computes (its passes sum the same
    # fp32 terms, in another order when the sequence is split into segments)
    _, H2, s2 = kata.prefill(*cuda(q, k, v), chunk=64, form="chunked")
    kata.sync_status()
    assert rel_l2(H, H2.double().cpu().numpy()) < 1e-5
    assert rel_l2(s, s2.double().cpu().numpy()) < 1e-5


def test_final_state_is_joined_back_to_the_callers_stream():
    # a kernel queued on the caller's stream right after the call must see the
    # final state: read it on that stream before any host synchronisation
    q, k, v = cuda(*prefill_inputs(1, 4, 1024, 64, dtype="bf16", seed=8))
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        o, H, s = kata.prefill(q, k, v, chunk=64, form="quadratic", stream=stream)
        snapshot = H.clone()  # enqueued on `stream` after the call
    stream.synchronize()
    kata.sync_status()
    assert torch.equal(snapshot, H)
    _, rH, _ = oracle.recurrent(q.cpu(), k.cpu(), v.cpu(), 1e-6, readout=False)
    assert rel_l2(snapshot, rH) < tol("bf16")


def test_quadratic_form_rejects_what_it_cannot_take():
    q, k, v = cuda(*prefill_inputs(1, 1, 128, 32, dtype="bf16", seed=1))
    D = 32 * 33 // 2
    H0 = torch.zeros(1, 1, D, 32, device="cuda")
    s0 = torch.zeros(1, 1, D, device="cuda")
    with pytest.raises(kata.KataError):  # an initial state
        kata.prefill(q, k, v, chunk=64, H_in=H0, s_in=s0, form="quadratic")
    with pytest.raises(kata.KataError):  # no output
        kata.prefill(q, k, v, chunk=64, output=False, form="quadratic")
    with pytest.raises(kata.KataError):  # fp32 inputs
        kata.prefill(q.float(), k.float(), v.float(), chunk=64, state=False, form="quadratic")


def test_full_size_headline_config():
    # B4 H8 T2048 d32 output-only, as the headline step runs it; sampled rows
    # of every head against the oracle, computed row by row
    w = WORKLOADS["prefill_b4_h8_t2048_d32"]
    assert kata.prefill_auto_form(w.B, w.H, w.T, w.d, w.chunk, BF16) == "quadratic"
    q, k, v = prefill_inputs(w.B, w.H, w.T, w.d, dtype=w.dtype, seed=w.seed, recipe=w.recipe)
    o, _, _ = kata.prefill(*cuda(q, k, v), chunk=w.chunk, eps=w.eps, state=False)
    kata.sync_status()
    rows = np.unique(np.array([0, 1, 63, 64, 127, 128, 129, 700, 1029, 1535, 2046, 2047]))
    ref = oracle.quadratic(q, k, v, w.eps, rows=rows)
    assert rel_l2(o[:, :, rows], ref) < tol(w.dtype)
    assert torch.isfinite(o).all()
