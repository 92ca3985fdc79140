"""The library's prefill and decode calls captured in CUDA graphs (stream-ordered
workspace from the library's pool becomes graph allocation nodes): replays give
bit-for-bit the eager results -- for a fixed-length batch, packed sequences
(chains handed out by tickets) and few chains (AUTO's guarded two-kernel form).  Runs in a child process without KDA_DEBUG, whose
synchronising checks cannot be captured."""
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
# prefill: eager, then captured and replayed on fresh outputs
cfg = W.small_prefill(B=2, T=300, H=3, dk=128, dv=128, io_dtype="bf16", seed=70, h0_std=0.02)
inp = W.make_prefill(cfg, "cuda")
args = (inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["scale"])
ref_out, ref_hT = kda.chunk_fwd(*args, h0=inp["h0"])
out = torch.empty_like(ref_out); hT = torch.empty_like(ref_hT)
side = torch.cuda.Stream()
side.wait_stream(torch.cuda.current_stream())
with torch.cuda.stream(side):
    kda.chunk_fwd(*args, h0=inp["h0"], out=out, hT=hT)
torch.cuda.current_stream().wait_stream(side)
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g):
    kda.chunk_fwd(*args, h0=inp["h0"], out=out, hT=hT)
out.zero_(); hT.zero_()
g.replay(); g.replay()
torch.cuda.synchronize()
assert torch.equal(out, ref_out) and torch.equal(hT, ref_hT), "prefill replay differs"

# packed sequences (the fused kernel hands chains out by tickets: the counter is zeroed inside
# the graph) and few chains (AUTO's two-kernel form with its decay-range flag, then the fused
# kernel returning at once): replays match the eager calls bit for bit
for cfg in (W.small_prefill(H=24, dk=128, dv=128, io_dtype="bf16", seed=72, h0_std=0.02,
                            lengths=[300, 0, 130, 64, 1, 250]),
            W.small_prefill(B=1, T=700, H=2, dk=128, dv=128, io_dtype="bf16", seed=73, h0_std=0.02)):
    inp = W.make_prefill(cfg, "cuda")
    args = (inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["scale"])
    kw = dict(h0=inp["h0"], cu_seqlens=inp["cu_seqlens"])
    ref_out, ref_hT = kda.chunk_fwd(*args, **kw)
    out = torch.empty_like(ref_out); hT = torch.empty_like(ref_hT)
    with torch.cuda.stream(side):
        kda.chunk_fwd(*args, out=out, hT=hT, **kw)
    torch.cuda.current_stream().wait_stream(side)
    g3 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g3):
        kda.chunk_fwd(*args, out=out, hT=hT, **kw)
    out.zero_(); hT.zero_()
    g3.replay(); g3.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(hT, ref_hT), "replay differs: " + cfg.name
    del g3

# decode: 5 chained steps captured once
dcfg = W.DecodeConfig("graph", N=8, H=4, dk=128, dv=128, steps=5, seed=71)
gen = W.decode_generator(dcfg, "cuda")
S0 = W.make_decode_state(dcfg, gen, "cuda")
xs = [W.make_decode_step(dcfg, gen, "cuda") for _ in range(dcfg.steps)]
o = torch.empty((dcfg.N, dcfg.H, dcfg.dv), dtype=torch.bfloat16, device="cuda")
def loop(S):
    outs = []
    for x in xs:
        kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S, 0.088, out=o)
        outs.append(o.clone())
    return outs
S_e = S0.clone(); ref = loop(S_e)
S_g = S0.clone()
with torch.cuda.stream(side):
    loop(S_g.clone())
torch.cuda.current_stream().wait_stream(side)
g2 = torch.cuda.CUDAGraph()
with torch.cuda.graph(g2):
    got = loop(S_g)
S_g.copy_(S0)
g2.replay()
torch.cuda.synchronize()
assert all(torch.equal(a, b) for a, b in zip(got, ref)) and torch.equal(S_g, S_e), "decode replay differs"
print("graphs ok")
"""


def test_prefill_and_decode_in_cuda_graphs(cuda_ok):
    from gated_delta_rule_75_b200 import build
    build.build()
    env = dict(os.environ)
    env.pop("KDA_DEBUG", None)
    r = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + CHILD], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "graphs ok" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
