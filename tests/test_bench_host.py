"""Host-side arithmetic that bench.py's roofline numbers rest on (no GPU): the
algorithmic bytes and flops per unit against the layouts the kernels use and the
per-head-token figures stated with the kernel table, the DRAM-traffic table lookup
keyed by source hashes, and the derived fp32 peak."""
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


def test_traffic_rows_apply_only_to_their_sources():
    """Every row of the committed traffic table is read back as (read + write) /
    launches while the kernel's source files hash to the row's prefix, else ignored."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.md")
    rows = 0
    for line in open(path):
        cells = [c.strip().strip("`") for c in line.strip().strip("|").split("|")]
        if len(cells) < 7 or not cells[3].isdigit():
            continue
        rows += 1
        kname, workload, sha = cells[0], cells[1], cells[2]
        got = bench.measured_traffic(kname, workload)
        if bench.kernel_source_sha(kname) == sha:
            assert got == (float(cells[4]) + float(cells[5])) / float(cells[3])
        else:
            assert got is None
    assert rows >= 4
    assert bench.measured_traffic("chunk_prep_tc", "no_such_workload") is None
    assert bench.kernel_source_sha("no_such_kernel") is None
