"""Calls queued back to back on one stream, with no synchronisation between them, give
bit for bit what each gives alone.  Inside a multi-kernel prefill call each launch after
the first may be scheduled while its predecessor drains (programmatic stream
serialization); this checks that no kernel reads its inputs, or overwrites memory a
previous kernel still reads (outputs, the library's pooled workspace), before that
predecessor has finished.  Alternating two input sets makes any early access show up as
a wrong result.  Cases: the fp32 SIMT prep and walk, few chains (AUTO's two-kernel form
with the segmented walk and prefix, then the guarded fused kernel), and packed sequences
(the chunk-offset scan first; with many chains, the fused kernel on tickets).  Runs in a
child process without KDA_DEBUG, whose per-call synchronisation would hide any overlap."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, torch
sys.path.insert(0, ROOT)
import workloads as W
import gated_delta_rule_75_b200 as kda

torch.cuda.set_device(0)
cases = [
    dict(B=1, T=300, H=2, dk=64, dv=64, io_dtype="f32"),
    dict(B=1, T=2048, H=4, dk=128, dv=128, io_dtype="bf16"),
    dict(H=8, dk=128, dv=128, io_dtype="bf16", lengths=[700, 1, 0, 260, 1500, 64]),
    dict(H=24, dk=128, dv=128, io_dtype="bf16", lengths=[300, 0, 130, 64, 1, 250]),
]
for ci, kw in enumerate(cases):
    sets = []
    for s in range(2):
        cfg = W.small_prefill(seed=90 + 10 * ci + s, h0_std=0.02, **kw)
        inp = W.make_prefill(cfg, "cuda")
        call = (inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["scale"])
        opts = dict(h0=inp["h0"], cu_seqlens=inp["cu_seqlens"])
        ref = kda.chunk_fwd(*call, **opts)
        torch.cuda.synchronize()
        sets.append((call, opts, ref))
    out = [torch.empty_like(sets[0][2][0]) for _ in range(2)]
    hT = [torch.empty_like(sets[0][2][1]) for _ in range(2)]
    got = []
    for i in range(16):
        call, opts, _ = sets[i % 2]
        kda.chunk_fwd(*call, out=out[(i // 2) % 2], hT=hT[(i // 2) % 2], **opts)
        got.append((out[(i // 2) % 2].clone(), hT[(i // 2) % 2].clone()))
    torch.cuda.synchronize()
    for i, (o, h) in enumerate(got):
        ro, rh = sets[i % 2][2]
        assert torch.equal(o, ro) and torch.equal(h, rh), "case %d call %d differs" % (ci, i)
print("order ok")
"""


def test_back_to_back_calls_match_isolated_calls(cuda_ok):
    from gated_delta_rule_75_b200 import build
    build.build()
    env = dict(os.environ)
    env.pop("KDA_DEBUG", None)
    r = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + CHILD], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "order ok" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
