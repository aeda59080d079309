"""LoLA pieces against the fp64 oracle (GPU): SRE scores, top-k retention,
merge, hybrid readout and the whole segment schedule."""
import numpy as np
import pytest
import torch

import kernelized_linear_attention_chunked_b200 as kata
import oracle
from _util import REL_F32, allowed_swap, cuda, rel_l2, tol
from kernelized_linear_attention_chunked_b200.inputs import (
    WORKLOADS, candidate_inputs, prefill_inputs, recall_inputs, state_inputs)

pytestmark = pytest.mark.gpu


def oracle_state(B, H, d, tokens, seed):
    ks, vs = state_inputs(B, H, d, tokens, seed=seed)
    _, H0, s0 = oracle.recurrent(None, ks, vs, 0.0, readout=False)
    return torch.from_numpy(H0).float(), torch.from_numpy(s0).float()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d,n,keep", [(16, 40, 25), (64, 192, 128), (32, 70, 200), (64, 130, 0),
                                        (64, 5, 2), (32, 17, 3), (64, 256, 100)])
def test_sre_topk_merge(dtype, d, n, keep):
    B, H = 2, 3
    H0, s0 = oracle_state(B, H, d, 300, seed=d)
    kc, vc, pos = candidate_inputs(B, H, n, d, dtype=dtype, seed=n)
    Hg, sg = cuda(H0.clone(), s0.clone())
    sc, ki = kata.sre_score_topk(Hg, sg, *cuda(kc, vc, pos), keep=keep, eps=1e-6, merge=True)
    kata.sync_status()
    rsc = oracle.sre(H0, s0, kc, vc, 1e-6)
    assert rel_l2(sc, rsc) < REL_F32
    rki = oracle.topk(rsc, pos.numpy(), keep)
    m = min(keep, n)
    ki = ki.cpu().numpy()
    for b in range(B):
        for h in range(H):
            assert allowed_swap(rsc[b, h], ki[b, h], rki[b, h], m)
            assert np.all(np.diff(pos.numpy()[b, h][ki[b, h]]) > 0)  # ascending position
    Hr, sr = H0.double().numpy().copy(), s0.double().numpy().copy()
    oracle.merge(Hr, sr, kc, vc, ki)
    assert rel_l2(Hg, Hr) < 1e-5 and rel_l2(sg, sr) < 1e-5


@pytest.mark.parametrize("d,n,keep", [(32, 130, 64), (64, 130, 64), (64, 192, 128), (64, 256, 0)])
def test_sre_topk_merge_many_heads(d, n, keep):
    # 320 heads: more CTAs than SMs on either path (several per SM over the
    # launch), and enough (head, slice) pairs for the partial-sum path
    B, H = 8, 40
    H0, s0 = oracle_state(B, H, d, 100, seed=d + 1)
    kc, vc, pos = candidate_inputs(B, H, n, d, dtype="bf16", seed=n + d)
    Hg, sg = cuda(H0.clone(), s0.clone())
    sc, ki = kata.sre_score_topk(Hg, sg, *cuda(kc, vc, pos), keep=keep, eps=1e-6, merge=True)
    kata.sync_status()
    rsc = oracle.sre(H0, s0, kc, vc, 1e-6)
    assert rel_l2(sc, rsc) < REL_F32
    rki = oracle.topk(rsc, pos.numpy(), keep)
    ki = ki.cpu().numpy()
    for b in range(B):
        for h in range(H):
            assert allowed_swap(rsc[b, h], ki[b, h], rki[b, h], keep)
    Hr, sr = H0.double().numpy().copy(), s0.double().numpy().copy()
    oracle.merge(Hr, sr, kc, vc, ki)
    assert rel_l2(Hg, Hr) < 1e-5 and rel_l2(sg, sr) < 1e-5


def test_sre_merge_out_of_place():
    # the merged state goes to separate buffers; the input state is untouched
    B, H, n, d, keep = 2, 5, 100, 64, 40
    H0, s0 = oracle_state(B, H, d, 200, seed=9)
    kc, vc, pos = candidate_inputs(B, H, n, d, dtype="bf16", seed=10)
    Hg, sg = cuda(H0.clone(), s0.clone())
    Ho, so = torch.full_like(Hg, float("nan")), torch.full_like(sg, float("nan"))
    _, ki = kata.sre_score_topk(Hg, sg, *cuda(kc, vc, pos), keep=keep, merge=True,
                                Hst_mut=Ho, s_mut=so)
    kata.sync_status()
    assert torch.equal(Hg.cpu(), H0) and torch.equal(sg.cpu(), s0)
    Hr, sr = H0.double().numpy().copy(), s0.double().numpy().copy()
    oracle.merge(Hr, sr, kc, vc, ki.cpu().numpy())
    assert rel_l2(Ho, Hr) < 1e-5 and rel_l2(so, sr) < 1e-5


def test_sre_ties_go_to_smaller_position():
    B, H, n, d = 1, 2, 40, 32
    H0, s0 = oracle_state(B, H, d, 100, seed=1)
    kc, vc, pos = candidate_inputs(B, H, n, d, dtype="bf16", seed=3, ties=True)
    sc, ki = kata.sre_score_topk(*cuda(H0, s0, kc, vc, pos), keep=15, merge=False)
    sc = sc.cpu().numpy()
    assert np.array_equal(sc[..., 0::2], sc[..., 1::2])  # constructed exact ties
    rki = oracle.topk(oracle.sre(H0, s0, kc, vc, 1e-6), pos.numpy(), 15)
    assert np.array_equal(ki.cpu().numpy(), rki)


def test_sre_empty_state_closed_form():
    B, H, n, d = 1, 1, 64, 64
    D = d * (d + 1) // 2
    kc, vc, pos = candidate_inputs(B, H, n, d, dtype="f32", seed=4)
    sc, _ = kata.sre_score_topk(torch.zeros(B, H, D, d, device="cuda"),
                                torch.zeros(B, H, D, device="cuda"), *cuda(kc, vc, pos), keep=8)
    assert rel_l2(sc, (vc.double() ** 2).sum(-1).numpy()) < 1e-6


def test_hybrid_readout_segment():
    B, H, T, d = 1, 3, 512, 64
    q, k, v = recall_inputs(B, H, T, d, dtype="bf16", seed=5)
    H0, s0 = oracle_state(B, H, d, 200, seed=6)
    cap, nc = 160, 100
    ck, cv, _ = candidate_inputs(B, H, cap, d, dtype="bf16", seed=7)
    seg0, nq, w0 = 256, 64, 192
    o = kata.hybrid_readout(*cuda(q, k, v), seg0, nq, w0, *cuda(ck, cv), nc, *cuda(H0, s0),
                            eps=1e-6)
    kata.sync_status()
    want = np.zeros((B, H, T, d))
    nh = B * H
    qq, kk, vv = (x.double().numpy().reshape(nh, T, d) for x in (q, k, v))
    cks = np.ascontiguousarray(ck.double().numpy().reshape(nh, cap, d))
    cvs = np.ascontiguousarray(cv.double().numpy().reshape(nh, cap, d))
    Hh = H0.double().numpy().reshape(nh, -1, d)
    sh = s0.double().numpy().reshape(nh, -1)
    oo = want.reshape(nh, T, d)
    L = oracle._load()
    p = oracle._ptr
    L.oracle_hybrid_segment_heads(nh, p(qq), p(kk), p(vv), T, d, d, 1e-6, d ** -0.5, w0, seg0,
                                  nq, p(cks), p(cvs), nc, cap, p(Hh), p(sh), p(oo))
    assert rel_l2(o[:, :, seg0:seg0 + nq], want[:, :, seg0:seg0 + nq]) < REL_F32


def lola_parity(q, k, v, window, cache, segments=None, run="auto"):
    B, H, T, d = q.shape
    o, Hg, sg, kept = kata.lola_prefill(*cuda(q, k, v), window=window, cache=cache, eps=1e-6,
                                        kept=True, run=run)
    kata.sync_status()
    kept = kept.cpu().numpy()
    adopted = []

    def adopt(u, cand, scores, keep_idx):
        m = keep_idx.shape[-1]
        alt = np.empty_like(keep_idx)
        for b in range(B):
            for h in range(H):
                gpu_pos = kept[u, b, h, :m]
                slot = {int(p_): i for i, p_ in enumerate(cand[b, h])}
                assert all(int(p_) in slot for p_ in gpu_pos), (u, b, h)
                g = np.array(sorted(slot[int(p_)] for p_ in gpu_pos), dtype=np.int32)
                assert allowed_swap(scores[b, h], g, keep_idx[b, h], m), (u, b, h)
                if set(g.tolist()) != set(keep_idx[b, h].tolist()):
                    adopted.append((u, b, h))
                alt[b, h] = g
        return alt

    res = oracle.lola(q, k, v, window=window, cache=cache, eps=1e-6, adopt=adopt,
                      segments=segments)
    n = T if segments is None else segments * window
    assert rel_l2(o[:, :, :n], res["o"][:, :, :n]) < tol("bf16" if q.dtype == torch.bfloat16 else "f32")
    if segments is None:
        assert rel_l2(Hg, res["H"]) < 1e-4 and rel_l2(sg, res["s"]) < 1e-4
    return o, res, adopted


@pytest.mark.parametrize("run", ["segments", "fused"])
def test_lola_schedule_small(run):
    q, k, v = recall_inputs(1, 2, 1024, 64, dtype="bf16", seed=8)
    o, res, _ = lola_parity(q, k, v, window=64, cache=128, run=run)
    assert rel_l2(o, res["o"]) < 1e-4


@pytest.mark.parametrize("run", ["segments", "fused"])
def test_lola_schedule_small_d16_fp32(run):
    q, k, v = prefill_inputs(2, 1, 256, 16, dtype="f32", seed=9)
    lola_parity(q, k, v, window=16, cache=24, run=run)


# the one-launch schedule across its size range: every head dim, both input
# types, segments of 8 to 64 tokens, caches that fill up late or never, the
# largest window + cache it takes
@pytest.mark.parametrize("d,dtype,window,cache,T", [
    (16, "bf16", 8, 8, 128),
    (32, "f32", 32, 40, 512),
    (32, "bf16", 64, 96, 768),
    (64, "bf16", 16, 200, 512),
    (64, "bf16", 64, 128, 640),
    (64, "bf16", 56, 16, 448),
])
def test_fused_schedule_sizes(d, dtype, window, cache, T):
    assert kata.lola_fused_applies(torch.float32 if dtype == "f32" else torch.bfloat16, d,
                                   window, cache)
    q, k, v = recall_inputs(2, 3, T, d, dtype=dtype, seed=d + window + cache)
    o, res, _ = lola_parity(q, k, v, window=window, cache=cache, run="fused")
    assert rel_l2(o, res["o"]) < 1e-4


@pytest.mark.parametrize("run", ["fused6", "fused7", "fused8"])
def test_fused_schedule_every_cluster_size(run):
    # the rows of the state split over 6 to 8 CTAs (uneven slices for 6 and 7),
    # the queries of a segment dealt out to the CTAs in turn
    q, k, v = recall_inputs(1, 3, 768, 64, dtype="bf16", seed=33)
    o, res, _ = lola_parity(q, k, v, window=64, cache=128, run=run)
    assert rel_l2(o, res["o"]) < 1e-4


def test_fused_and_segmented_runs_agree():
    q, k, v = cuda(*recall_inputs(2, 2, 2048, 64, dtype="bf16", seed=12))
    a = kata.lola_prefill(q, k, v, window=64, cache=128, kept=True, run="fused")
    b = kata.lola_prefill(q, k, v, window=64, cache=128, kept=True, run="segments")
    kata.sync_status()
    assert rel_l2(a[0], b[0].double().cpu().numpy()) < 1e-5
    assert rel_l2(a[1], b[1].double().cpu().numpy()) < 1e-5
    assert (a[3] != b[3]).float().mean().item() < 0.01  # kept sets: near-ties only
    # the fused run is deterministic, bit for bit
    c = kata.lola_prefill(q, k, v, window=64, cache=128, kept=True, run="fused")
    kata.sync_status()
    assert all(torch.equal(x, y) for x, y in zip(a, c))


def test_fused_continues_from_a_given_state():
    # the schedule over two halves, the second starting from the first's state
    # and cache-free, equals that same two-call sequence run by the segment
    # kernels (the oracle starts from a zero state, so compare the two paths)
    q, k, v = cuda(*recall_inputs(1, 2, 512, 32, dtype="bf16", seed=14))
    outs = {}
    for run in ("fused", "segments"):
        o1, H1, s1, _ = kata.lola_prefill(q[:, :, :256].contiguous(), k[:, :, :256].contiguous(),
                                          v[:, :, :256].contiguous(), window=32, cache=64,
                                          run=run)
        o2, H2, s2, _ = kata.lola_prefill(q[:, :, 256:].contiguous(), k[:, :, 256:].contiguous(),
                                          v[:, :, 256:].contiguous(), window=32, cache=64,
                                          Hst=H1, s=s1, run=run)
        kata.sync_status()
        outs[run] = (o1, o2, H2, s2)
    for a, b in zip(outs["fused"], outs["segments"]):
        assert rel_l2(a, b.double().cpu().numpy()) < 1e-4


def test_lola_config_full_schedule():
    # the LoLA workload at its own size: all 128 segments of all 16 heads, every
    # one of the 127 kept sets (tie rule, lock-step adoption), every output row
    # and the final state
    w = WORKLOADS["lola_b2_h8_t8192_d64"]
    q, k, v = recall_inputs(w.B, w.H, w.T, w.d, dtype=w.dtype, seed=w.seed)
    o, res, adopted = lola_parity(q, k, v, window=w.window, cache=w.cache)
    assert len(res["kept_pos"]) == w.T // w.window - 1
    # fp32 arithmetic on the stored bf16 values: far inside the bf16 bar
    assert rel_l2(o, res["o"]) < 1e-4
    assert len(adopted) <= 2 * w.B * w.H  # divergences only at near-ties


def hybrid_reference(q, k, v, seg0, nq, w0, ck, cv, nc, H0, s0, tau):
    B, H, T, d = q.shape
    cap = ck.shape[2]
    want = np.zeros((B, H, T, d))
    nh = B * H
    qq, kk, vv = (x.double().numpy().reshape(nh, T, d) for x in (q, k, v))
    cks = np.ascontiguousarray(ck.double().numpy().reshape(nh, cap, d))
    cvs = np.ascontiguousarray(cv.double().numpy().reshape(nh, cap, d))
    Hh = np.ascontiguousarray(H0.double().numpy().reshape(nh, -1, d))
    sh = np.ascontiguousarray(s0.double().numpy().reshape(nh, -1))
    oo = want.reshape(nh, T, d)
    L = oracle._load()
    p = oracle._ptr
    L.oracle_hybrid_segment_heads(nh, p(qq), p(kk), p(vv), T, d, d, 1e-6, tau, w0, seg0, nq,
                                  p(cks), p(cvs), nc, cap, p(Hh), p(sh), p(oo))
    return want[:, :, seg0:seg0 + nq]


@pytest.mark.parametrize("scale", [12.0, 40.0])
def test_hybrid_readout_large_logits(scale):
    # tau q.k up to scale^2 / 8 (18 and 200): past fp32's exp range (88) at the
    # larger scale; the kernel's max shift keeps the quotient finite and exact
    B, H, T, d = 1, 2, 256, 64
    q, k, v = recall_inputs(B, H, T, d, dtype="f32", seed=15)
    q, k = q * scale, k * scale
    H0, s0 = oracle_state(B, H, d, 100, seed=16)
    ck, cv, _ = candidate_inputs(B, H, 32, d, dtype="f32", seed=17)
    seg0, nq, w0 = 128, 64, 64
    o = kata.hybrid_readout(*cuda(q, k, v), seg0, nq, w0, *cuda(ck, cv), 32, *cuda(H0, s0),
                            eps=1e-6)
    kata.sync_status()
    got = o[:, :, seg0:seg0 + nq]
    assert torch.isfinite(got).all()
    want = hybrid_reference(q, k, v, seg0, nq, w0, ck, cv, 32, H0, s0, d ** -0.5)
    assert np.isfinite(want).all()
    assert rel_l2(got, want) < REL_F32
