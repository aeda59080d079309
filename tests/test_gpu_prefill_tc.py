"""The tcgen05 prefill path (state kernel + readout kernel) against the fp64
oracle, over the shapes that change its schedule: the number of 128-token
chunks per snapshot interval (1, 2 or 4), odd chunk counts, a single chunk,
continuation from an initial state, and state-only calls (GPU)."""
import pytest
import torch

import kernelized_linear_attention_chunked_b200 as kata
import oracle
from _util import cuda, rel_l2, tol
from kernelized_linear_attention_chunked_b200.inputs import prefill_inputs

pytestmark = pytest.mark.gpu

BF16 = torch.bfloat16


def run(q, k, v, **kw):
    # the chunked form (kata_prefill would compute o by the quadratic form at
    # these sizes when no initial state is given)
    out = kata.prefill(*cuda(q, k, v), chunk=64, form="chunked", **kw)
    kata.sync_status()
    return out


def test_tensor_core_path_is_taken():
    for d in (32, 64):
        assert kata.prefill_uses_tensor_cores(2, 3, 1024, d, 64, BF16)
    # T not a multiple of 128, d = 16 or fp32 inputs take the CUDA-core path
    assert not kata.prefill_uses_tensor_cores(1, 1, 192, 32, 64, BF16)
    assert not kata.prefill_uses_tensor_cores(1, 1, 256, 16, 64, BF16)
    assert not kata.prefill_uses_tensor_cores(1, 1, 256, 32, 64, torch.float32)


# (d, T): 1, 3, 8 chunks at d = 32 (1 or 2 chunks per interval); 5, 6, 8 chunks
# at d = 64 (1, 2, 4 chunks per interval)
SHAPES = [(32, 128), (32, 384), (32, 1024), (64, 640), (64, 768), (64, 1024)]


@pytest.mark.parametrize("d,T", SHAPES)
def test_output_and_state(d, T):
    q, k, v = prefill_inputs(1, 3, T, d, dtype="bf16", seed=d * 1000 + T)
    assert kata.prefill_uses_tensor_cores(1, 3, T, d, 64, BF16)
    o, H, s = run(q, k, v)
    ro, rH, rs = oracle.recurrent(q, k, v, 1e-6)
    assert rel_l2(o, ro) < tol("bf16")
    assert rel_l2(H, rH) < tol("bf16")
    assert rel_l2(s, rs) < tol("bf16")
    # state only: no output; the sequence may be split into segments whose
    # partial states are summed, so only the rounding order differs
    none, H2, s2 = run(q, k, v, output=False)
    assert none is None
    assert rel_l2(H2, H.double().cpu().numpy()) < 1e-5
    assert rel_l2(s2, s.double().cpu().numpy()) < 1e-5
    assert rel_l2(H2, rH) < tol("bf16") and rel_l2(s2, rs) < tol("bf16")


@pytest.mark.parametrize("d,T", [(32, 512), (64, 1024), (64, 768)])
def test_continue_from_initial_state_in_place(d, T):
    q, k, v = prefill_inputs(2, 2, T, d, dtype="bf16", seed=77 + d)
    h = T // 2
    first = [x[:, :, :h].contiguous() for x in (q, k, v)]
    second = [x[:, :, h:].contiguous() for x in (q, k, v)]
    _, H1, s1 = run(*first)
    # H_out aliases H_in: every CTA reads and writes only its own feature rows
    o2, H2, s2 = run(*second, H_in=H1, s_in=s1, H_out=H1, s_out=s1)
    ro, rH, rs = oracle.recurrent(q, k, v, 1e-6)
    assert rel_l2(o2, ro[:, :, h:]) < tol("bf16")
    assert rel_l2(H2, rH) < tol("bf16")
    assert rel_l2(s2, rs) < tol("bf16")


def test_many_heads_grid():
    # more heads than SMs: the readout grid is 1 x 160, the state grid 5 x 160
    q, k, v = prefill_inputs(8, 20, 128, 32, dtype="bf16", seed=5)
    o, H, s = run(q, k, v)
    ro, rH, rs = oracle.recurrent(q, k, v, 1e-6)
    assert rel_l2(o, ro) < tol("bf16")
    assert rel_l2(H, rH) < tol("bf16")


def test_causality_of_the_tensor_core_path():
    # perturbing token t must leave every output before t unchanged (bit for bit)
    q, k, v = prefill_inputs(1, 2, 512, 64, dtype="bf16", seed=3)
    o0, _, _ = run(q, k, v)
    t = 300
    k2, v2 = k.clone(), v.clone()
    k2[:, :, t] = 1.5 * k2[:, :, t]
    v2[:, :, t] = 2 * v2[:, :, t]
    o1, _, _ = run(q, k2, v2)
    assert torch.equal(o0[:, :, :t], o1[:, :, :t])
    assert not torch.equal(o0[:, :, t:], o1[:, :, t:])


# final state only, over few heads: the state pass splits the sequence into
# segments (grid z) and sums their partial states; with an initial state (the
# first segment starts from it) and H_out aliasing H_in
@pytest.mark.parametrize("d,T,H", [(32, 1024, 1), (32, 2048, 3), (64, 1024, 2), (64, 640, 1)])
def test_segmented_state_pass(d, T, H):
    q, k, v = prefill_inputs(1, H, T, d, dtype="bf16", seed=90 + d + T + H)
    n0 = kata.launch_count()
    none, Hs, ss = run(q, k, v, output=False)
    assert none is None
    assert kata.launch_count() - n0 == 3  # state pass + the two sums
    _, rH, rs = oracle.recurrent(q, k, v, 1e-6, readout=False)
    assert rel_l2(Hs, rH) < tol("bf16") and rel_l2(ss, rs) < tol("bf16")
    # continue from it in place, state only again
    q2, k2, v2 = prefill_inputs(1, H, T, d, dtype="bf16", seed=91 + d + T + H)
    _, Hc, sc = run(q2, k2, v2, output=False, H_in=Hs, s_in=ss, H_out=Hs, s_out=ss)
    qq, kk, vv = (torch.cat(x, dim=2) for x in ((q, q2), (k, k2), (v, v2)))
    _, rH2, rs2 = oracle.recurrent(qq, kk, vv, 1e-6, readout=False)
    assert rel_l2(Hc, rH2) < tol("bf16") and rel_l2(sc, rs2) < tol("bf16")
