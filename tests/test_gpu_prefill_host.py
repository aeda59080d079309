"""kata_prefill_host (host q, k, v in, host o out, the heads in pieces over
two streams) against the device-buffer call and the fp64 oracle, through the
C ABI ("Kernelized Linear Attention: Breaking the Capacity Wall with Symmetric
Cones", s2.2 and s2.3: the quadratic and the chunked form of the same causal
attention)."""
import pytest
import torch

import kernelized_linear_attention_chunked_b200 as kata
import oracle
from _util import cuda, rel_l2, tol
from kernelized_linear_attention_chunked_b200.inputs import prefill_inputs

pytestmark = pytest.mark.gpu


def _host_call(q, k, v, chunk, eps):
    B, H, T, d = q.shape
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    oh = torch.full((B, H, T, d), float("nan")).pin_memory()
    ws = torch.empty(kata.prefill_host_workspace_bytes(B, H, T, d, chunk, q.dtype),
                     dtype=torch.uint8, device="cuda")
    kata.prefill_host(qh, kh, vh, chunk, eps, oh, ws)
    torch.cuda.synchronize()
    kata.sync_status()
    return oh


@pytest.mark.parametrize("B,H,T,d,dtype", [
    (4, 8, 2048, 32, "bf16"),   # quadratic form, two pieces of sixteen heads
    (1, 3, 256, 16, "f32"),     # CUDA-core form, pieces of one and two heads
    (1, 5, 512, 64, "bf16"),    # quadratic form, pieces of two and three heads
    (1, 1, 256, 32, "bf16"),    # one head: one piece
])
def test_host_call_equals_device_call(B, H, T, d, dtype):
    q, k, v = prefill_inputs(B, H, T, d, dtype=dtype, seed=11)
    oh = _host_call(q, k, v, 64, 1e-6)
    od, _, _ = kata.prefill(*cuda(q, k, v), chunk=64, eps=1e-6, state=False)
    kata.sync_status()
    # per head the same kernels run on the same inputs
    assert torch.equal(oh, od.cpu())
    ro, _, _ = oracle.recurrent(q, k, v, 1e-6)
    assert rel_l2(oh, ro) < tol(dtype)


def test_host_call_chunked_form():
    # T past the quadratic form's crossover: the chunked form, pieces of 2 and 3 heads
    B, H, T, d = 1, 5, 8192, 32
    assert kata.prefill_auto_form(B, H, T, d, 64, torch.bfloat16) == "chunked"
    q, k, v = prefill_inputs(B, H, T, d, dtype="bf16", seed=12)
    oh = _host_call(q, k, v, 64, 1e-6)
    od, _, _ = kata.prefill(*cuda(q, k, v), chunk=64, eps=1e-6, state=False)
    kata.sync_status()
    assert torch.isfinite(oh).all()
    assert rel_l2(oh, od.cpu().double().numpy()) < 1e-5
    ro, _, _ = oracle.recurrent(q, k, v, 1e-6)
    assert rel_l2(oh, ro) < tol("bf16")


def test_host_call_repeated_with_device_work_between():
    # the caller's stream waits for the second stream: work queued after the
    # call sees the complete output
    B, H, T, d = 2, 4, 1024, 32
    q, k, v = prefill_inputs(B, H, T, d, dtype="bf16", seed=13)
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    ws = torch.empty(kata.prefill_host_workspace_bytes(B, H, T, d, 64, torch.bfloat16),
                     dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        oh = torch.empty(B, H, T, d).pin_memory()
        kata.prefill_host(qh, kh, vh, 64, 1e-6, oh, ws)
        dev = oh.to("cuda", non_blocking=True)  # queued after the call on the same stream
        outs.append(dev)
    torch.cuda.synchronize()
    kata.sync_status()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
