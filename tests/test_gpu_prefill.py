"""kata_prefill against the fp64 oracle on the same seeded inputs (GPU)."""
import numpy as np
import pytest
import torch

import kernelized_linear_attention_chunked_b200 as kata
import oracle
from _util import cuda, rel_l2, tol
from kernelized_linear_attention_chunked_b200.inputs import WORKLOADS, prefill_inputs

pytestmark = pytest.mark.gpu


def run(q, k, v, chunk, eps=1e-6, **kw):
    o, H, s = kata.prefill(*cuda(q, k, v), chunk=chunk, eps=eps, **kw)
    kata.sync_status()
    return o, H, s


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [16, 32, 64])
@pytest.mark.parametrize("chunk", [16, 64, 128])
def test_small_all_shapes(dtype, d, chunk):
    # several chunks, packed dimension ragged against every tile size, odd head count
    q, k, v = prefill_inputs(1, 3, 256, d, dtype=dtype, seed=d + chunk)
    o, H, s = run(q, k, v, chunk)
    ro, rH, rs = oracle.recurrent(q, k, v, 1e-6)
    assert rel_l2(o, ro) < tol(dtype)
    assert rel_l2(H, rH) < tol(dtype)
    assert rel_l2(s, rs) < tol(dtype)


def test_pr1_reference_config_fp32():
    w = WORKLOADS["pr1_ref_t256_d16"]
    q, k, v = prefill_inputs(w.B, w.H, w.T, w.d, dtype=w.dtype, seed=w.seed, recipe=w.recipe)
    o, H, s = run(q, k, v, w.chunk, eps=w.eps)
    ref = oracle.quadratic(q, k, v, w.eps)
    err = rel_l2(o, ref)
    assert err < 1e-4, err
    _, rH, rs = oracle.recurrent(q, k, v, w.eps, readout=False)
    assert rel_l2(H, rH) < 1e-5 and rel_l2(s, rs) < 1e-5


def test_chunk_size_invariance_and_determinism():
    # fp32 inputs take the CUDA-core path, where the chunk length sets the
    # schedule (how many tokens go through the intra-chunk quadratic form
    # before the state absorbs them): every chunk length gives the same output
    # and state up to fp32 reordering, and a repeated call is bit-identical
    q, k, v = prefill_inputs(2, 2, 512, 32, dtype="f32", seed=7)
    runs = [run(q, k, v, c) for c in (16, 32, 64)]
    ref = oracle.quadratic(q, k, v, 1e-6)
    for o, H, s in runs:
        assert rel_l2(o, ref) < 1e-5
        assert rel_l2(H, runs[0][1].cpu().double().numpy()) < 1e-6
    again = run(q, k, v, 32)
    assert torch.equal(again[0], runs[1][0]) and torch.equal(again[1], runs[1][1])


def test_tensor_core_path_ignores_chunk():
    # bf16 d = 32/64 inputs take the tensor-core path, whose chunk is its
    # 128-token tile whatever the caller asks: results are bit-identical
    q, k, v = prefill_inputs(1, 2, 384, 32, dtype="bf16", seed=8)
    outs = [run(q, k, v, c) for c in (16, 64, 128)]
    for o, H, s in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(H, outs[0][1])


def test_initial_state_continues_and_aliasing():
    q, k, v = prefill_inputs(1, 2, 384, 32, dtype="f32", seed=9)
    o1, H1, s1 = run(q[:, :, :128], k[:, :, :128], v[:, :, :128], 64)
    # continue in place: H_out aliases H_in
    o2, H2, s2 = run(q[:, :, 128:].contiguous(), k[:, :, 128:].contiguous(),
                     v[:, :, 128:].contiguous(), 64, H_in=H1, s_in=s1, H_out=H1, s_out=s1)
    full = oracle.quadratic(q, k, v, 1e-6)
    assert rel_l2(torch.cat([o1, o2], dim=2), full) < 1e-4
    _, rH, rs = oracle.recurrent(q, k, v, 1e-6, readout=False)
    assert rel_l2(H1, rH) < 1e-5 and rel_l2(s1, rs) < 1e-5


def test_minimal_and_state_only():
    q, k, v = prefill_inputs(1, 1, 16, 16, dtype="f32", seed=11)
    o, H, s = run(q, k, v, 16)
    assert rel_l2(o, oracle.quadratic(q, k, v, 1e-6)) < 1e-4
    none, H2, s2 = run(q, k, v, 16, output=False)
    assert none is None and torch.equal(H2, H) and torch.equal(s2, s)


def _sampled_rows(T):
    return np.unique(np.array([0, 1, 63, 64, 127, 128, 129, T // 3, T // 2 + 5, T - 2, T - 1]))


@pytest.mark.parametrize("name", ["prefill_b4_h8_t2048_d32", "long_prefill_b2_h16_t16384_d64"])
def test_full_size_configs(name):
    w = WORKLOADS[name]
    q, k, v = prefill_inputs(w.B, w.H, w.T, w.d, dtype=w.dtype, seed=w.seed, recipe=w.recipe)
    o, H, s = run(q, k, v, w.chunk, eps=w.eps)
    rows = _sampled_rows(w.T)
    ref = oracle.quadratic(q, k, v, w.eps, rows=rows)
    assert rel_l2(o[:, :, rows], ref) < tol(w.dtype)
    # final state probed with random queries: the readout of a probe x from the
    # GPU state must equal the oracle's readout of x after the whole sequence
    x = torch.from_numpy(np.random.default_rng(0).standard_normal((w.B, w.H, 3, w.d)))
    px = oracle.phi(x)  # [B, H, 3, D]
    Hg, sg = H.cpu().double().numpy(), s.cpu().double().numpy()
    got = np.einsum("bhpr,bhre->bhpe", px, Hg) / (np.einsum("bhpr,bhr->bhp", px, sg)[..., None] + w.eps)
    for p in range(3):
        qq = q.double().clone()
        qq[:, :, -1] = x[:, :, p]
        want = oracle.quadratic(qq, k, v, w.eps, rows=[w.T - 1])[:, :, 0]
        assert rel_l2(got[:, :, p], want) < tol(w.dtype)
