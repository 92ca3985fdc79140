"""Host-side arithmetic that bench.py's roofline numbers rest on (no GPU): the
algorithmic bytes and flops per unit against the layouts the kernels use and the
per-head-token figures stated with the kernel table, the roofline fraction counted
on the path's minimal bytes, the DRAM-traffic table lookup keyed by source hashes,
and the derived fp32 peak."""
import os
import re

import bench
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gated_delta_rule_75_b200", "csrc")


def _constants(fname, names):
    src = open(os.path.join(CSRC, fname)).read()
    out = {}
    for n in names:
        m = re.search(rf"constexpr\s+\w+\s+{n}\s*=\s*(\d+)\s*;", src)
        assert m, n
        out[n] = int(m.group(1))
    return out


def test_operand_image_size_matches_the_kernel_layout():
    """The image the tensor-core prep writes per (chunk, head): -W^T (128 channels x 64
    tokens), Q e^G (64 x 128), [Aqk^T | K e^{G_last - G}] (64 x 192), T' (64 x 64), all
    bf16, then e^{G_last} (128 fp32), padded to a 1 KB multiple for the bulk copy."""
    c = _constants("kda_chunk_tc.cu", ["IMG_W", "IMG_QG", "IMG_B2", "IMG_T", "IMG_GAM", "IMG_BYTES"])
    assert c["IMG_QG"] - c["IMG_W"] == 128 * 64 * 2
    assert c["IMG_B2"] - c["IMG_QG"] == 64 * 128 * 2
    assert c["IMG_T"] - c["IMG_B2"] == 64 * (64 + 128) * 2
    assert c["IMG_GAM"] - c["IMG_T"] == 64 * 64 * 2
    assert c["IMG_GAM"] + 128 * 4 <= c["IMG_BYTES"] < c["IMG_GAM"] + 128 * 4 + 1024
    assert c["IMG_BYTES"] % 1024 == 0
    assert bench.TC_WS_BYTES_PER_CHUNK == c["IMG_BYTES"]


def test_prefill_bytes_per_head_token():
    """Per head-token on the benchmark workload: prep 2068 B (q, k bf16, log_alpha fp32,
    beta in; 66560 / 64 image bytes out), state 1552 B (image and v in, out) plus the
    final states once, SIMT prep 3596 B (q, k, v bf16, log_alpha, beta in; the fp32
    workspace W, Ut, Aqk, Q e^G, K e^{G_last - G}, e^{G_last} out)."""
    cfg = W.BATCHED
    ht = cfg.B * cfg.T * cfg.H
    states = cfg.N * cfg.H * cfg.dk * cfg.dv * 4
    assert bench.kernel_algorithmic_bytes("chunk_prep_tc", cfg) == 2068 * ht
    assert bench.kernel_algorithmic_bytes("chunk_state_tc", cfg) == 1552 * ht + states
    assert bench.kernel_algorithmic_bytes("chunk_prep_simt", cfg) == 3596 * ht
    ws_floats = 64 * (128 + 128 + 64 + 128 + 128) + 128      # one (chunk, head) block
    assert 3596 * 64 == 64 * (2 * 128 * 2 + 128 * 2 + 128 * 4 + 4) + 4 * ws_floats
    # the whole-path minimum used for the tensor fraction: q, k, v, out bf16, log_alpha, beta
    assert bench.BYTES_PER_HEAD_TOKEN == 4 * 128 * 2 + 128 * 4 + 4


def test_fused_kernel_bytes():
    """The fused kernel reads q, k, v (bf16), log_alpha, beta and h0 when given, and
    writes out (bf16) and the final states: 1540 B per head-token plus the states."""
    cfg = W.SINGLE                           # h0 given
    ht = cfg.B * cfg.T * cfg.H
    states = cfg.N * cfg.H * cfg.dk * cfg.dv * 4
    assert bench.kernel_algorithmic_bytes("chunk_fused_tc", cfg) == 1540 * ht + 2 * states
    cfg = W.BATCHED                          # h0 = 0: not read
    ht = cfg.B * cfg.T * cfg.H
    states = cfg.N * cfg.H * cfg.dk * cfg.dv * 4
    assert bench.kernel_algorithmic_bytes("chunk_fused_tc", cfg) == 1540 * ht + states


def test_partial_chunks_count_whole_chunks():
    """Packed sequences: every sequence rounds up to whole 64-token chunks."""
    cfg = W.small_prefill(H=2, dk=128, dv=128, io_dtype="bf16", seed=0, lengths=[1, 64, 65])
    ht = cfg.B * cfg.T * cfg.H
    chunks = (1 + 1 + 2) * cfg.H
    assert bench.kernel_algorithmic_bytes("chunk_prep_tc", cfg) == \
        1028 * ht + chunks * bench.TC_WS_BYTES_PER_CHUNK


def test_decode_bytes_per_head_step():
    """132,612 B: the 128 x 128 fp32 state read and written, q, k, v, out bf16,
    log_alpha fp32 and beta."""
    assert bench.decode_bytes_per_head_step(W.DECODE) == 132612


def test_backward_flops_per_head_token():
    """502,101 flop per head-token over the six backward kernels at d = 128, C = 64."""
    cfg = W.BATCHED
    ks = ["chunk_prep_simt", "chunk_state_simt", "bwd_state", "bwd_dense1", "bwd_dense2", "bwd_param"]
    tot = sum(bench.bwd_kernel_flops(k, cfg) for k in ks) / (cfg.B * cfg.T * cfg.H)
    assert abs(tot - 502101.33) < 1.0
    assert bench.bwd_kernel_flops("not_a_kernel", cfg) == 0.0


def test_fp32_alu_peak():
    assert abs(bench.fp32_alu_peak({"sm_max_mhz": 1965.0}) - 74.44992) < 1e-9
    assert abs(bench.fp32_alu_peak(None) - 74.44992) < 1e-9


def test_traffic_entries_apply_only_to_their_sources(tmp_path):
    """Every entry of the committed traffic table is read back as (read + write) /
    launches x scale while the kernel's source files hash to the entry's prefix,
    else ignored; an entry captured on a smaller case is scaled to the workload."""
    import json
    table = json.load(open(bench.TRAFFIC_PATH))
    for e in table["entries"]:
        got = bench.measured_traffic(e["kernel"], e["workload"])
        if bench.kernel_source_sha(e["kernel"]) == e["source_sha256"]:
            assert got == (e["dram_read_bytes"] + e["dram_write_bytes"]) / e["launches"] * e["scale"]
        else:
            assert got is None
    assert len(table["entries"]) >= 4
    assert bench.measured_traffic("chunk_prep_tc", "no_such_workload") is None
    assert bench.kernel_source_sha("no_such_kernel") is None
    # a scaled entry on the current source of the fused kernel
    sha = bench.kernel_source_sha("chunk_fused_tc")
    fake = tmp_path / "t.json"
    fake.write_text(json.dumps({"entries": [
        {"kernel": "chunk_fused_tc", "workload": "w", "source_sha256": sha, "launches": 2,
         "dram_read_bytes": 300, "dram_write_bytes": 100, "scale": 4.0}]}))
    assert bench.measured_traffic("chunk_fused_tc", "w", path=str(fake)) == 800.0
    assert bench.measured_traffic("chunk_fused_tc", "v", path=str(fake)) is None


PEAKS = {"hbm_gbs": 6548.2, "bf16_tflops": 1642.8, "source": "measured"}


def test_roofline_frac_counts_only_the_path_minimum():
    """roofline.frac = 1540 B x the head-tokens one launch processes / the dominant
    kernel's launch time / the measured HBM copy peak.  Hand recomputation for one
    1.90 ms launch on the B=8, H=32, T=8192 workload: 1540 x 2,097,152 B / 1.90 ms
    = 1699.8 GB/s, 0.2596 of 6548.2 GB/s; for a kernel launched twice per step each
    launch covers half the head-tokens."""
    cfg = W.BATCHED
    r = bench.prefill_roofline("chunk_fused_tc", cfg, 1.90, 1.0, PEAKS)
    assert r["bytes_per_head_token"] == 1540
    assert r["head_tokens_per_launch"] == 8 * 8192 * 32
    assert abs(r["achieved"] - 1540 * 2097152 / 1.90e-3 / 1e9) < 1e-6
    assert abs(r["frac"] - 0.25958231) < 1e-7
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6548.2
    # the kernel's own I/O: q, k, v, log_alpha, beta in, out and the final states out
    io = 8 * 8192 * 32 * 1540 + 8 * 32 * 128 * 128 * 4
    assert r["kernel_io_bytes_per_launch"] == io
    assert abs(r["kernel_io_frac"] - io / 1.90e-3 / 1e9 / 6548.2) < 1e-12
    # a two-kernel prep gets no credit for the operand image it writes (2068 B of
    # kernel I/O per head-token against the path's 1540 B)
    r2 = bench.prefill_roofline("chunk_prep_tc", cfg, 0.95, 2.0, PEAKS)
    assert abs(r2["frac"] - r["frac"]) < 1e-12
    assert abs(r2["kernel_io_frac"] / r2["frac"] - 2068 / 1540) < 1e-12


def test_path_bytes_and_flops_follow_the_shapes():
    """(2dk + 2dv) x I/O bytes + 4 dk + 4 per head-token; 2C(3dk + 2dv) + 6 dk dv flop."""
    assert bench.path_bytes_per_head_token(W.BATCHED) == 1540 == bench.BYTES_PER_HEAD_TOKEN
    assert bench.path_bytes_per_head_token(W.TINY) == 4 * 64 * 4 + 64 * 4 + 4
    assert bench.path_flop_per_head_token(W.BATCHED) == 180224 == bench.FLOP_PER_HEAD_TOKEN
    assert bench.path_flop_per_head_token(W.TINY) == 2 * 64 * 5 * 64 + 6 * 64 * 64


def test_binding_fraction_takes_the_lower_roofline():
    """At 117 flop/B the HBM roofline binds: tokens/s over 6548.2e9 / (32 x 1540)."""
    tps = 65536 / 1.90e-3
    hbm_bound = 6548.2e9 / (32 * 1540)
    assert abs(bench.binding_frac(tps, W.BATCHED, PEAKS) - tps / hbm_bound) < 1e-12
    # with a slow tensor peak the tensor roofline binds instead
    slow = dict(PEAKS, bf16_tflops=100.0)
    tc_bound = 100e12 / (32 * 180224)
    assert abs(bench.binding_frac(tps, W.BATCHED, slow) - tps / tc_bound) < 1e-12
