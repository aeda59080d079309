"""The multi-factor features of the KATA page's s2.3 "Variants" (KATA-Mg,
several PSD factors; KATA-Sigma-g, summed PSD factors; reading R13: the head
vector in g sub-vectors) on the GPU, against the fp64 oracle's recurrent and
quadratic forms of the same feature (GPU)."""
import pytest
import torch

import kernelized_linear_attention_chunked_b200 as kata
import oracle
from _util import REL_F32, cuda, rel_l2
from kernelized_linear_attention_chunked_b200.inputs import decode_inputs, prefill_inputs

pytestmark = pytest.mark.gpu

CASES = [(64, "mg", 2), (64, "sigmag", 2), (64, "mg", 8), (64, "sigmag", 4),
         (32, "mg", 4), (32, "sigmag", 2), (16, "sigmag", 2)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d,feature,g", CASES)
def test_prefill_feature_matches_the_oracle(dtype, d, feature, g):
    q, k, v = prefill_inputs(2, 2, 320, d, dtype=dtype, seed=d + g + len(feature))
    o, H, s = kata.prefill_feature(*cuda(q, k, v), feature, g, chunk=64)
    kata.sync_status()
    ro, rH, rs = oracle.recurrent_feature(q, k, v, 1e-6, feature, g)
    # fp32 arithmetic on the stored values: the fp32 bar for both input types
    assert rel_l2(o, ro) < REL_F32
    assert rel_l2(H, rH) < REL_F32 and rel_l2(s, rs) < REL_F32
    assert rel_l2(o, oracle.quadratic_feature(q, k, v, 1e-6, feature, g)) < REL_F32


@pytest.mark.parametrize("d,feature,g", CASES)
def test_decode_feature_continues_the_prefill(d, feature, g):
    # prefill 128 tokens, then 8 decode steps from the GPU state, against the
    # oracle's recurrent form over all 136 tokens
    T0, steps = 128, 8
    q, k, v = prefill_inputs(1, 3, T0 + steps, d, dtype="bf16", seed=60 + d + g)
    _, H, s = kata.prefill_feature(*cuda(q[:, :, :T0].contiguous(), k[:, :, :T0].contiguous(),
                                         v[:, :, :T0].contiguous()), feature, g, output=False)
    outs = []
    for t in range(T0, T0 + steps):
        outs.append(kata.decode_step_feature(*cuda(q[:, :, t].contiguous(),
                                                   k[:, :, t].contiguous(),
                                                   v[:, :, t].contiguous()), H, s, feature, g))
    kata.sync_status()
    ro, rH, rs = oracle.recurrent_feature(q, k, v, 1e-6, feature, g)
    assert rel_l2(torch.stack(outs, dim=2), ro[:, :, T0:]) < REL_F32
    assert rel_l2(H, rH) < REL_F32 and rel_l2(s, rs) < REL_F32


def test_decode_feature_full_launch_shape():
    # the decode workload's launch shape (B64 H16 d64) with the Sigma-2 and
    # M8 features, from the oracle's fp32 prefix state
    for feature, g in (("sigmag", 2), ("mg", 8)):
        kp, vp, q, k, v = decode_inputs(64, 16, 64, 16, 3, dtype="bf16", seed=31 + g)
        _, H0, s0 = oracle.recurrent_feature(None, kp, vp, 0.0, feature, g, readout=False)
        H0, s0 = torch.from_numpy(H0).float(), torch.from_numpy(s0).float()
        Hg, sg = cuda(H0.clone(), s0.clone())
        outs = [kata.decode_step_feature(*cuda(q[t], k[t], v[t]), Hg, sg, feature, g)
                for t in range(3)]
        kata.sync_status()
        ro, rH, rs = oracle.decode_feature(H0, s0, q, k, v, 1e-6, feature, g)
        assert rel_l2(torch.stack(outs), ro) < REL_F32
        assert rel_l2(Hg, rH) < 1e-5 and rel_l2(sg, rs) < 1e-5


def test_rank_one_feature_is_kata_prefill():
    q, k, v = cuda(*prefill_inputs(1, 2, 256, 32, dtype="bf16", seed=3))
    a = kata.prefill_feature(q, k, v, "rank1", 1)
    b = kata.prefill(q, k, v, chunk=64)
    kata.sync_status()
    assert all(torch.equal(x, y) for x, y in zip(a, b))
