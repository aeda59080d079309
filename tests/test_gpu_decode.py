"""kata_decode_step against the fp64 oracle from the same fp32 starting state (GPU)."""
import numpy as np
import pytest
import torch

import kernelized_linear_attention_chunked_b200 as kata
import oracle
from _util import REL_F32, cuda, rel_l2
from kernelized_linear_attention_chunked_b200.inputs import decode_inputs

pytestmark = pytest.mark.gpu


def start_state(kp, vp):
    """Prefix state built by the oracle in fp64, then rounded to fp32 (the
    stored state format); the GPU and the oracle both continue from it."""
    _, H0, s0 = oracle.recurrent(None, kp, vp, 0.0, readout=False)
    return torch.from_numpy(H0).float(), torch.from_numpy(s0).float()


def decode_parity(B, H, d, prefix, steps, dtype, seed):
    kp, vp, q, k, v = decode_inputs(B, H, d, prefix, steps, dtype=dtype, seed=seed)
    H0, s0 = start_state(kp, vp)
    Hg, sg = cuda(H0.clone(), s0.clone())
    outs = []
    for t in range(steps):
        outs.append(kata.decode_step(*cuda(q[t], k[t], v[t]), Hg, sg, eps=1e-6))
    kata.sync_status()
    ro, rH, rs = oracle.decode(H0, s0, q, k, v, 1e-6)
    # arithmetic is fp32 for both input dtypes: hold both to the fp32 bar
    assert rel_l2(torch.stack(outs), ro) < REL_F32
    assert rel_l2(Hg, rH) < 1e-5 and rel_l2(sg, rs) < 1e-5


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [16, 32, 64])
def test_small(dtype, d):
    decode_parity(2, 3, d, prefix=40, steps=12, dtype=dtype, seed=d)


def test_config_prefix_on_two_heads():
    # the full 4096-token seeded prefix of the decode workload, on 2 heads
    decode_parity(1, 2, 64, prefix=4096, steps=8, dtype="bf16", seed=3)


def test_full_launch_shape():
    # the benchmark's launch shape (B=64, H=16, d=64) with a short prefix
    decode_parity(64, 16, 64, prefix=16, steps=3, dtype="bf16", seed=13)


def test_zero_state_first_step_closed_form():
    # from an empty state one step gives o = a v / (a + eps), a = (q.k)^2
    B, H, d = 2, 2, 32
    _, _, q, k, v = decode_inputs(B, H, d, 1, 1, dtype="f32", seed=21)
    D = d * (d + 1) // 2
    Hg = torch.zeros(B, H, D, d, device="cuda")
    sg = torch.zeros(B, H, D, device="cuda")
    o = kata.decode_step(*cuda(q[0], k[0], v[0]), Hg, sg, eps=1e-6).cpu().double()
    a = (q[0].double() * k[0].double()).sum(-1, keepdim=True) ** 2
    want = a * v[0].double() / (a + 1e-6)
    assert rel_l2(o, want.numpy()) < 1e-5


def test_deterministic():
    _, _, q, k, v = decode_inputs(4, 4, 64, 1, 1, dtype="bf16", seed=22)
    D = 2080
    H0 = torch.randn(4, 4, D, 64, generator=torch.Generator().manual_seed(0))
    s0 = torch.rand(4, 4, D, generator=torch.Generator().manual_seed(1))
    res = []
    for _ in range(2):
        Hg, sg = cuda(H0.clone(), s0.clone())
        res.append((kata.decode_step(*cuda(q[0], k[0], v[0]), Hg, sg), Hg, sg))
    assert all(torch.equal(a, b) for a, b in zip(res[0], res[1]))
    np.testing.assert_array_equal(res[0][2].cpu().numpy(), res[1][2].cpu().numpy())
