"""The split of the sequence across CTAs and across ranks (the KATA page's s2.3:
the state propagates across blocks as a prefix sum) against the fp64 oracle
(GPU).

* Scan mode of the chunked prefill: with few heads the sequence is split into
  segments; a first pass computes each segment's state, an exclusive prefix
  gives each segment its carry, and a second pass writes the snapshots from
  the carries.
* kata_state_prefix: exclusive prefix sums over parts' states.
* Context-parallel prefill: two ranks (processes sharing this GPU, gloo for the
  one exchange; their kernels never wait on each other) each own half the
  sequence.
"""
import socket
import sys
from pathlib import Path

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import kernelized_linear_attention_chunked_b200 as kata
import oracle
from _util import cuda, rel_l2, tol
from kernelized_linear_attention_chunked_b200.inputs import prefill_inputs

sys.path.insert(0, str(Path(__file__).resolve().parent))
import _ranks  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,T,d", [(1, 2, 4096, 64), (1, 1, 8192, 32), (1, 3, 2304, 64)])
def test_scan_mode_matches_the_oracle(B, H, T, d):
    # few heads: the (tile, head) CTAs leave SMs idle, so the sequence splits
    q, k, v = prefill_inputs(B, H, T, d, dtype="bf16", seed=T + d)
    o, Hs, ss = kata.prefill(*cuda(q, k, v), chunk=128, form="chunked")
    kata.sync_status()
    ro, rH, rs = oracle.recurrent(q, k, v, 1e-6)
    assert rel_l2(o, ro) < tol("bf16")
    assert rel_l2(Hs, rH) < tol("bf16") and rel_l2(ss, rs) < tol("bf16")


def test_scan_mode_continues_from_a_state():
    q, k, v = prefill_inputs(1, 2, 4096, 64, dtype="bf16", seed=5)
    qa, ka, va = (x[:, :, :1024].contiguous() for x in (q, k, v))
    qb, kb, vb = (x[:, :, 1024:].contiguous() for x in (q, k, v))
    _, H1, s1 = kata.prefill(*cuda(qa, ka, va), chunk=128, output=False)
    o2, H2, s2 = kata.prefill(*cuda(qb, kb, vb), chunk=128, H_in=H1, s_in=s1, form="chunked")
    # H_out aliasing H_in: the call keeps one sequential pass
    Hc, sc = H1.clone(), s1.clone()
    o3, H3, s3 = kata.prefill(*cuda(qb, kb, vb), chunk=128, H_in=Hc, s_in=sc, H_out=Hc, s_out=sc,
                              form="chunked")
    kata.sync_status()
    ro, rH, rs = oracle.recurrent(q, k, v, 1e-6)
    assert H3.data_ptr() == Hc.data_ptr()
    assert rel_l2(Hc, rH) < tol("bf16") and rel_l2(sc, rs) < tol("bf16")
    assert rel_l2(o2, ro[:, :, 1024:]) < tol("bf16")
    assert rel_l2(H2, rH) < tol("bf16") and rel_l2(s2, rs) < tol("bf16")
    assert rel_l2(o3, ro[:, :, 1024:]) < tol("bf16")


def test_state_prefix_is_the_exclusive_sum():
    n, B, H, d = 5, 2, 3, 32
    D = d * (d + 1) // 2
    g = torch.Generator().manual_seed(0)
    Hp = torch.randn(n, B, H, D, d, generator=g)
    sp = torch.rand(n, B, H, D, generator=g)
    Ho, so = kata.state_prefix(*cuda(Hp, sp))
    kata.sync_status()
    Hw = np.concatenate([np.zeros((1,) + Hp.shape[1:]), np.cumsum(Hp.double().numpy(), 0)[:-1]])
    sw = np.concatenate([np.zeros((1,) + sp.shape[1:]), np.cumsum(sp.double().numpy(), 0)[:-1]])
    assert rel_l2(Ho[1:], Hw[1:]) < 1e-6 and rel_l2(so[1:], sw[1:]) < 1e-6
    assert torch.count_nonzero(Ho[0]) == 0 and torch.count_nonzero(so[0]) == 0


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("d,T", [(64, 2048), (32, 4096)])
def test_context_parallel_two_ranks(d, T):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ranks.cp_rank_main, args=(r, 2, port, queue, d, T))
             for r in range(2)]
    for p in procs:
        p.start()
    results = sorted((queue.get(timeout=300) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v = prefill_inputs(1, 2, T, d, dtype="bf16", seed=77)
    ro, rH, rs = oracle.recurrent(q, k, v, 1e-6)
    o = torch.cat([results[0][1], results[1][1]], dim=2)
    assert rel_l2(o, ro) < tol("bf16")
    assert rel_l2(results[1][2], rH) < tol("bf16") and rel_l2(results[1][3], rs) < tol("bf16")
    # rank 0's state is the state after the first half
    _, rH0, _ = oracle.recurrent(q[:, :, :T // 2], k[:, :, :T // 2], v[:, :, :T // 2], 1e-6,
                                 readout=False)
    assert rel_l2(results[0][2], rH0) < tol("bf16")
