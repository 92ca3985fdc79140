"""Recall after a long prefill (the pages' regression case for serving: a value
written early must come back after a long context, also when the prefill is
split across calls through a pooled state).  Token 0 writes (k0 = e_0, v0) with
beta = 1; channel 0 never decays and every later key is orthogonal to e_0, so the
state's row 0 holds v0 exactly and the last query q = e_0 (scale 1) must read
v0 -- bit for bit, since v0 is a bf16 value and nothing rounds it."""
import numpy as np
import pytest
import torch

import oracle
from kda_testutil import host, rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda(cuda_ok):
    from gated_delta_rule_75_b200 import build
    build.build()
    import gated_delta_rule_75_b200 as kda
    return kda


def _needle(T, H, d, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn((1, T, H, d), generator=g)
    k[..., 0] = 0.0
    k /= k.norm(dim=-1, keepdim=True)
    k[0, 0] = 0.0
    k[0, 0, :, 0] = 1.0                                  # k0 = e_0
    q = torch.randn((1, T, H, d), generator=g)
    q /= q.norm(dim=-1, keepdim=True)
    q[0, -1] = 0.0
    q[0, -1, :, 0] = 1.0                                 # the last query asks for k0
    v = torch.randn((1, T, H, d), generator=g)
    la = -torch.nn.functional.softplus(torch.randn((1, T, H, d), generator=g))
    la[..., 0] = 0.0                                     # channel 0 keeps its memory
    beta = torch.sigmoid(torch.randn((1, T, H), generator=g))
    beta[0, 0] = 1.0
    bf = lambda x: x.to(torch.bfloat16).cuda()
    return bf(q), bf(k), bf(v), la.cuda(), beta.cuda()


@pytest.mark.parametrize("impl", ["simt", "tensorcore"])
def test_needle_recalled_after_4096_tokens(kda, impl):
    T, H, d = 4096, 2, 128
    q, k, v, la, beta = _needle(T, H, d, 80)
    out, hT = kda.chunk_fwd(q, k, v, la, beta, 1.0, impl=impl)
    torch.cuda.synchronize()
    torch.testing.assert_close(out[0, -1], v[0, 0], rtol=0, atol=0)
    torch.testing.assert_close(hT[0, :, 0], v[0, 0].float(), rtol=0, atol=0)
    ro, _ = oracle.fwd(host(q), host(k), host(v), host(la), host(beta), 1.0)
    assert rel(out, ro) <= 5e-3


def test_needle_through_chunked_prefill_on_pool_slots(kda):
    """The same context prefilled in three calls (split at 1000 and 2500, off the
    64-token grid) through a state pool, the needle read back at the end."""
    T, H, d = 4096, 2, 128
    q, k, v, la, beta = _needle(T, H, d, 81)
    pool = torch.zeros((3, H, d, d), dtype=torch.float32, device="cuda")
    slots = torch.tensor([2], dtype=torch.int32, device="cuda")
    outs = []
    for a, b in ((0, 1000), (1000, 2500), (2500, T)):
        sl = lambda x: x[:, a:b].contiguous()
        o, _ = kda.chunk_fwd(sl(q), sl(k), sl(v), sl(la), sl(beta), 1.0, state_pool=pool, slots=slots)
        outs.append(o)
    torch.cuda.synchronize()
    out = torch.cat(outs, dim=1)
    torch.testing.assert_close(out[0, -1], v[0, 0], rtol=0, atol=0)
    ro, rh = oracle.fwd(host(q), host(k), host(v), host(la), host(beta), 1.0)
    assert rel(out, ro) <= 5e-3 and rel(pool[2:3], rh) <= 5e-3
