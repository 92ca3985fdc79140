"""The library's device error word read through kda_get_error, in a child process
without KDA_DEBUG (so no call synchronises or returns a device-side status): a
prefill on well-formed input leaves the word clear and matches the fp64 oracle on
this non-synchronising path; a bounded wait that gives up (the self-test kernel,
reporting into the library's word) leaves its two timeout bits; a malformed
cu_seqlens array and a decode slot out of range leave bit 0, while the calls
themselves return KDA_OK; each take clears the word, and bits left in it change
nothing a later call computes.  Nothing here faults or hangs: the waits are the
bounded ones, and malformed offsets are clamped on the device."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import os, sys, torch
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))
assert "KDA_DEBUG" not in os.environ
import workloads as W
import gated_delta_rule_75_b200 as kda
from kda_testutil import TOL, oracle_prefill, rel

torch.cuda.set_device(0)
kda.get_error()                                   # start from a clear word

# 1. parity on the non-synchronising path, fused tensor-core and SIMT
for impl, io in (("auto", "bf16"), ("simt", "f32")):
    cfg = W.small_prefill(B=1, T=0, H=3, dk=128, dv=128, io_dtype=io, seed=31, h0_std=0.02,
                          lengths=[200, 1, 77, 0, 130])
    inp = W.make_prefill(cfg, "cuda")
    out, hT = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["scale"], h0=inp["h0"], cu_seqlens=inp["cu_seqlens"], impl=impl)
    torch.cuda.synchronize()
    ro, rh = oracle_prefill(inp)
    eo, eh = rel(out, ro), rel(hT, rh)
    print(impl, "rel", eo, eh)
    assert eo <= TOL[io] and eh <= TOL[io], (impl, eo, eh)
    assert kda.get_error() == 0

# 2. a bounded wait that gives up reports bits 1 and 2 into the library's word
st, _ = kda.debug_bounded_wait(3, to_library_word=True)
assert st == 0, st
w = kda.get_error()
print("wait word", hex(w))
assert w == 0x6, hex(w)
assert kda.get_error() == 0                       # the take cleared it

# 3. malformed cu_seqlens (decreasing, and not ending at T): the call returns KDA_OK,
#    the word has bit 0
cfg = W.small_prefill(B=1, T=0, H=2, dk=128, dv=128, io_dtype="bf16", seed=32,
                      lengths=[100, 60, 40])
inp = W.make_prefill(cfg, "cuda")
for bad in ([0, 120, 90, 200], [0, 100, 160, 150]):
    cu = torch.tensor(bad, dtype=torch.int32, device="cuda")
    for impl in ("auto", "simt", "tensorcore_chain"):
        kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                      inp["scale"], cu_seqlens=cu, impl=impl)
        w = kda.get_error()
        assert w == 1, (bad, impl, hex(w))

# 4. a decode slot out of range: bit 0, other rows still updated
dcfg = W.DecodeConfig("err", N=4, H=2, dk=128, dv=128, steps=1, seed=33)
gen = W.decode_generator(dcfg, "cuda")
pool = torch.zeros((3, 2, 128, 128), dtype=torch.float32, device="cuda")
x = W.make_decode_step(dcfg, gen, "cuda")
slots = torch.tensor([0, 7, -1, 2], dtype=torch.int32, device="cuda")
kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, 0.088, slots=slots)
w = kda.get_error()
assert w == 1, hex(w)
assert pool[0].abs().sum() > 0 and pool[2].abs().sum() > 0 and pool[1].abs().sum() == 0

# 5. bits left in the word change nothing later calls compute
kda.debug_bounded_wait(2, to_library_word=True)
cfg = W.small_prefill(B=2, T=130, H=2, dk=128, dv=128, io_dtype="bf16", seed=34, h0_std=0.02)
inp = W.make_prefill(cfg, "cuda")
out, hT = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                        inp["scale"], h0=inp["h0"])
torch.cuda.synchronize()
ro, rh = oracle_prefill(inp)
assert rel(out, ro) <= TOL["bf16"] and rel(hT, rh) <= TOL["bf16"]
assert kda.get_error() == 0x6
print("error word ok")
"""


def test_error_word_without_debug_mode(cuda_ok):
    from gated_delta_rule_75_b200 import build
    build.build()
    env = dict(os.environ)
    env.pop("KDA_DEBUG", None)
    r = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + CHILD], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "error word ok" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
