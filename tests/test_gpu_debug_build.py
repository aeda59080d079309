"""The debug library (device-side bounds checks, KATA_DEBUG=1) on the GPU:
every entry point runs clean on tiny shapes against the fp64 oracle, a checked
access past the end of an array is reported as KATA_ERR_BOUNDS instead of a
fault, and the context stays usable afterwards. Runs in a child process, which
loads libkata_debug.so in place of libkata.so."""
import os
import subprocess
import sys
from pathlib import Path

import pytest

pytestmark = pytest.mark.gpu

ROOT = Path(__file__).resolve().parent.parent

SCRIPT = r'''
import sys
sys.path.insert(0, ROOT); sys.path.insert(0, ROOT + "/tests")
import numpy as np, torch
import kernelized_linear_attention_chunked_b200 as kata
import oracle
from _util import rel_l2
from kernelized_linear_attention_chunked_b200.inputs import (
    candidate_inputs, prefill_inputs, state_inputs)

assert kata.debug_build()
dev = torch.device("cuda", 0)
cu = lambda *xs: [x.to(dev) for x in xs]

# prefill, fp32 (CUDA cores) and bf16 (tensor cores), tiny shapes
for dtype, T, d, chunk in (("f32", 16, 16, 16), ("bf16", 128, 32, 64)):
    q, k, v = prefill_inputs(1, 2, T, d, dtype=dtype, seed=T + d)
    o, H, s = kata.prefill(*cu(q, k, v), chunk=chunk)
    kata.sync_status()
    ro, rH, rs = oracle.recurrent(q, k, v, 1e-6)
    assert rel_l2(o, ro) < 2e-2 and rel_l2(H, rH) < 2e-2, (dtype, T, d)

# decode step
q, k, v = prefill_inputs(1, 2, 1, 16, dtype="f32", seed=3)
D = 16 * 17 // 2
Hs, ss = torch.zeros(1, 2, D, 16, device=dev), torch.zeros(1, 2, D, device=dev)
od = kata.decode_step(*cu(q[:, :, 0], k[:, :, 0], v[:, :, 0]), Hs, ss)
kata.sync_status()

# SRE + top-k + merge: fp32 (partial-sum path) and bf16 d = 32 (tensor cores)
for dtype, d, n, keep in (("f32", 16, 12, 5), ("bf16", 32, 40, 24)):
    ks, vs = state_inputs(1, 2, d, 40, seed=d)
    _, H0, s0 = oracle.recurrent(None, ks, vs, 0.0, readout=False)
    H0, s0 = torch.from_numpy(H0).float(), torch.from_numpy(s0).float()
    kc, vc, pos = candidate_inputs(1, 2, n, d, dtype=dtype, seed=n)
    Hg, sg = cu(H0.clone(), s0.clone())
    sc, ki = kata.sre_score_topk(Hg, sg, *cu(kc, vc, pos), keep=keep, merge=True)
    kata.sync_status()
    assert rel_l2(sc, oracle.sre(H0, s0, kc, vc, 1e-6)) < 1e-4, (dtype, d)

# the LoLA schedule, fused and in segments, tiny (normal draws: no near-ties)
q, k, v = prefill_inputs(1, 2, 256, 16, dtype="f32", seed=5)
ref = oracle.lola(q, k, v, window=32, cache=32, eps=1e-6)
for run in ("auto", "segments"):
    o = kata.lola_prefill(*cu(q, k, v), window=32, cache=32, run=run)[0]
    kata.sync_status()
    assert rel_l2(o, ref["o"]) < 1e-3, run

# a checked access past the end of an array: reported, not a fault
kata.test_bounds_check()
try:
    kata.sync_status()
    raise SystemExit("the failed bounds check was not reported")
except kata.KataError as e:
    assert "KATA_ERR_BOUNDS" in str(e) and "0xB001" in str(e), str(e)

# and the context is still usable
o2, _, _ = kata.prefill(*cu(*prefill_inputs(1, 1, 16, 16, dtype="f32", seed=9)), chunk=16)
kata.sync_status()
print("ok")
'''


def test_debug_library_end_to_end():
    lib = ROOT / "kernelized_linear_attention_chunked_b200" / "libkata_debug.so"
    assert lib.exists(), "libkata_debug.so is built by __graft_entry__.build()"
    env = dict(os.environ, KATA_DEBUG="1")
    r = subprocess.run([sys.executable, "-c", f"ROOT = {str(ROOT)!r}\n" + SCRIPT], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-2000:], r.stderr[-4000:])
    assert r.stdout.strip().endswith("ok")
