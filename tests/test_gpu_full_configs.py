"""Parity at the workloads' own sizes, in the launch configuration the
benchmark times, against the fp64 oracle (GPU).

* prefill B4 H8 T2048 d32 and long prefill B2 H16 T16384 d64: every output row
  of every head, in the quadratic and the chunked form, plus the final state,
  against the oracle's literal recurrent form ("Kernelized Linear Attention:
  Breaking the Capacity Wall with Symmetric Cones", s2.3: the chunked state
  form is exact, so it must reproduce the recurrence).
* decode B64 H16 d64: all 256 steps at the full launch shape; 16 heads spread
  over the batch start from the oracle's fp32 prefix state and are compared
  with the oracle at every step and in their final state.
"""
import numpy as np
import pytest
import torch

import kernelized_linear_attention_chunked_b200 as kata
import oracle
from _util import REL_F32, cuda, rel_l2, tol
from kernelized_linear_attention_chunked_b200.inputs import WORKLOADS, decode_inputs, prefill_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def references():
    """Inputs and the oracle's recurrent form (o for every row, final state)
    of both prefill workloads, computed once."""
    out = {}
    for name in ("prefill_b4_h8_t2048_d32", "long_prefill_b2_h16_t16384_d64"):
        w = WORKLOADS[name]
        q, k, v = prefill_inputs(w.B, w.H, w.T, w.d, dtype=w.dtype, seed=w.seed, recipe=w.recipe)
        out[name] = (w, (q, k, v), oracle.recurrent(q, k, v, w.eps))
    return out


@pytest.mark.parametrize("name", ["prefill_b4_h8_t2048_d32", "long_prefill_b2_h16_t16384_d64"])
@pytest.mark.parametrize("form", ["auto", "quadratic", "chunked"])
def test_every_row_output_only(references, name, form):
    w, (q, k, v), (ro, _, _) = references[name]
    o, _, _ = kata.prefill(*cuda(q, k, v), chunk=w.chunk, eps=w.eps, state=False, form=form)
    kata.sync_status()
    assert torch.isfinite(o).all()
    assert rel_l2(o, ro) < tol(w.dtype)
    # every head on its own, not only the whole tensor
    og = o.cpu().double().numpy()
    for b in range(w.B):
        for h in range(w.H):
            assert rel_l2(og[b, h], ro[b, h]) < tol(w.dtype), (b, h)


@pytest.mark.parametrize("name", ["prefill_b4_h8_t2048_d32", "long_prefill_b2_h16_t16384_d64"])
def test_every_row_with_final_state(references, name):
    # the call a prefill that hands its state to decode makes: o and (H, s)
    w, (q, k, v), (ro, rH, rs) = references[name]
    o, H, s = kata.prefill(*cuda(q, k, v), chunk=w.chunk, eps=w.eps)
    kata.sync_status()
    assert rel_l2(o, ro) < tol(w.dtype)
    assert rel_l2(H, rH) < tol(w.dtype) and rel_l2(s, rs) < tol(w.dtype)
    # the state alone (final-state-only call: the sequence split into segments)
    none, H2, s2 = kata.prefill(*cuda(q, k, v), chunk=w.chunk, eps=w.eps, output=False)
    kata.sync_status()
    assert none is None
    assert rel_l2(H2, rH) < tol(w.dtype) and rel_l2(s2, rs) < tol(w.dtype)


def test_decode_all_steps_full_launch_shape():
    w = WORKLOADS["decode_b64_h16_d64"]
    kp, vp, q, k, v = decode_inputs(w.B, w.H, w.d, w.prefix, w.steps, dtype=w.dtype, seed=w.seed)
    D = w.D
    dev = torch.device("cuda")
    # heads checked against the oracle: 16 spread over batch and head index
    picks = [(b, (5 * b) % w.H) for b in range(0, w.B, 4)]
    bi = torch.tensor([p[0] for p in picks])
    hi = torch.tensor([p[1] for p in picks])
    # every head's prefix state written in by decode steps on the GPU (outputs
    # discarded), then the checked heads' state replaced by the oracle's fp32
    # prefix state, so their parity does not depend on the prefix path
    Hst = torch.zeros(w.B, w.H, D, w.d, device=dev)
    s = torch.zeros(w.B, w.H, D, device=dev)
    o = torch.empty(w.B, w.H, w.d, device=dev)
    kpd = kp.to(dev).permute(2, 0, 1, 3).contiguous()
    vpd = vp.to(dev).permute(2, 0, 1, 3).contiguous()
    for t in range(w.prefix):
        kata.decode_step(kpd[t], kpd[t], vpd[t], Hst, s, eps=w.eps, o=o)
    del kpd, vpd
    _, H0, s0 = oracle.recurrent(None, kp[bi, hi], vp[bi, hi], 0.0, readout=False)
    H0, s0 = torch.from_numpy(H0).float(), torch.from_numpy(s0).float()
    Hst[bi, hi] = H0.to(dev)
    s[bi, hi] = s0.to(dev)
    qd, kd, vd = cuda(q, k, v)
    outs = []
    for t in range(w.steps):
        kata.decode_step(qd[t], kd[t], vd[t], Hst, s, eps=w.eps, o=o)
        outs.append(o[bi, hi].clone())
    kata.sync_status()
    assert torch.isfinite(o).all()
    ro, rH, rs = oracle.decode(H0, s0, q[:, bi, hi], k[:, bi, hi], v[:, bi, hi], w.eps)
    got = torch.stack(outs)  # [steps, picks, d]
    # fp32 arithmetic: the fp32 bar, at every step
    for t in (0, 1, 63, 127, 200, w.steps - 1):
        assert rel_l2(got[t], ro[t]) < REL_F32, t
    assert rel_l2(got, ro) < REL_F32
    assert rel_l2(Hst[bi, hi], rH) < 1e-5 and rel_l2(s[bi, hi], rs) < 1e-5
