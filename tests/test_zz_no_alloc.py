"""lola_sre_score_topk_noalloc: the SRE + top-k + merge entry point that takes no
workspace (its scratch is a fixed device array inside the library, for callers
that cannot allocate device memory while scoring). Called through the C ABI and
compared with lola_sre_score_topk on two calls in a row.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import kernelized_linear_attention_chunked_b200 as kata
from _util import REL_F32, rel_l2
from kernelized_linear_attention_chunked_b200.inputs import candidate_inputs

pytestmark = pytest.mark.gpu


def _p(t):
    return C.c_void_p(t.data_ptr()) if t is not None else None


def _state(B, H, d, seed):
    # any fp32 state will do for comparing the two entry points
    g = torch.Generator().manual_seed(seed)
    D = d * (d + 1) // 2
    Hs = torch.randn(B, H, D, d, generator=g) * 0.05
    s = torch.rand(B, H, D, generator=g)
    return Hs.cuda(), s.cuda()


def _reference(Hs, s, kc, vc, pos, keep, eps):
    Hm, sm = Hs.clone(), s.clone()
    sc, ki = kata.sre_score_topk(Hs, s, kc, vc, pos, keep=keep, eps=eps, merge=True,
                                 Hst_mut=Hm, s_mut=sm)
    return sc, ki, Hm, sm


def _noalloc(Hs, s, kc, vc, pos, keep, eps):
    B, H, n, d = kc.shape
    m = min(keep, n)
    sc = torch.empty(B, H, n, device="cuda")
    ki = torch.empty(B, H, max(m, 1), dtype=torch.int32, device="cuda")
    Hm, sm = Hs.clone(), s.clone()
    st = kata.lib().lola_sre_score_topk_noalloc(
        _p(Hs), _p(s), _p(kc), _p(vc), _p(pos), 1 if kc.dtype == torch.bfloat16 else 0, B, H,
        d, n, keep, eps, 1, _p(sc), _p(ki), _p(Hm), _p(sm),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, kata.lib().kata_last_error()
    kata.sync_status()
    return sc, ki[..., :m], Hm, sm


@pytest.mark.parametrize("B,H,d,n,keep,dtype", [
    (2, 8, 64, 192, 128, "bf16"),   # the LoLA workload's per-update shape
    (1, 3, 32, 70, 25, "f32"),
])
def test_noalloc_matches_workspace_entry_point_twice(B, H, d, n, keep, dtype):
    for call in range(2):  # two calls in a row share the fixed scratch
        Hs, s = _state(B, H, d, seed=10 * call + d)
        kc, vc, pos = (x.cuda() for x in candidate_inputs(B, H, n, d, dtype=dtype,
                                                          seed=20 * call + n))
        want = _reference(Hs, s, kc, vc, pos, keep, 1e-6)
        got = _noalloc(Hs, s, kc, vc, pos, keep, 1e-6)
        assert rel_l2(got[0], want[0].cpu().double().numpy()) < REL_F32
        assert np.array_equal(got[1].cpu().numpy(), want[1].cpu().numpy())
        assert rel_l2(got[2], want[2].cpu().double().numpy()) < REL_F32
        assert rel_l2(got[3], want[3].cpu().double().numpy()) < REL_F32


def test_noalloc_rejects_sizes_beyond_its_scratch():
    B, H, d, n = 4, 16, 64, 192  # 64 heads need more than the fixed 8 MiB
    D = d * (d + 1) // 2
    Hs = torch.zeros(B, H, D, d, device="cuda")
    s = torch.zeros(B, H, D, device="cuda")
    kc, vc, pos = (x.cuda() for x in candidate_inputs(B, H, n, d, dtype="bf16", seed=1))
    ki = torch.empty(B, H, 128, dtype=torch.int32, device="cuda")
    st = kata.lib().lola_sre_score_topk_noalloc(
        _p(Hs), _p(s), _p(kc), _p(vc), _p(pos), 1, B, H, d, n, 128, 1e-6, 0, None, _p(ki),
        None, None, C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 5  # KATA_ERR_WORKSPACE
    assert b"fixed scratch" in kata.lib().kata_last_error()
