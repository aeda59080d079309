"""Failure detection on the GPU without a GPU fault: a bounded device wait that
runs out is reported as KATA_ERR_TIMEOUT with its site code, the kernel tears
down through its error path (its copies and MMAs drained, its tensor memory
freed), and the context stays usable: the next calls are parity-green."""
import pytest
import torch

import kernelized_linear_attention_chunked_b200 as kata
import oracle
from _util import cuda, rel_l2, tol
from kernelized_linear_attention_chunked_b200.inputs import prefill_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [32, 64])
def test_forced_timeout_is_reported_and_the_context_stays_usable(d):
    q, k, v = prefill_inputs(1, 2, 384, d, dtype="bf16", seed=71 + d)
    qg, kg, vg = cuda(q, k, v)
    kata.sync_status()  # nothing pending from earlier calls
    # a wait that nothing completes, given up after 4096 polls (milliseconds)
    kata.test_forced_timeout(qg, kg, vg, polls=4096)
    with pytest.raises(kata.KataError) as info:
        kata.sync_status()
    msg = str(info.value)
    assert "KATA_ERR_TIMEOUT" in msg and "0x6FF" in msg, msg
    # the report was read and cleared; the device and the library still work
    kata.sync_status()
    ref = oracle.quadratic(q, k, v, 1e-6)
    for form in ("quadratic", "chunked"):
        o, _, _ = kata.prefill(qg, kg, vg, chunk=64, state=False, form=form)
        kata.sync_status()
        assert rel_l2(o, ref) < tol("bf16"), form


def test_a_stale_report_does_not_stop_later_calls():
    # a timeout that nobody has read yet must not make later launches give up
    # early: they compute correct outputs, and the old report is still there
    q, k, v = prefill_inputs(1, 1, 256, 32, dtype="bf16", seed=5)
    qg, kg, vg = cuda(q, k, v)
    kata.sync_status()
    kata.test_forced_timeout(qg, kg, vg, polls=1024)
    torch.cuda.synchronize()
    o, _, _ = kata.prefill(qg, kg, vg, chunk=64, state=False, form="chunked")
    torch.cuda.synchronize()
    assert rel_l2(o, oracle.quadratic(q, k, v, 1e-6)) < tol("bf16")
    with pytest.raises(kata.KataError):
        kata.sync_status()
    kata.sync_status()
