"""The benchmark's algorithmic counts (the roofline numerators) against the per-workload totals
worked out from the per-token-head formulas: q, k, v, the gate and beta read and o, u written
in the forward (plus the fp32 states), and every input read and every gradient written in the
backward; flops 6 dk dv + 3 C dk + 2 C dv + C^2/3 per token-head forward, twice that backward."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("cfg,fwd_bytes,total_bytes", (
    # GDN B8 T4096 H8 d128: 262144 token-heads x 2 B x 642 + 64 heads x 64 KiB (S_T)
    ((8, 4096, 8, 128, 128, 64, 1, 2, False), 340_787_200, 888_143_872),
    # KDA B4 T16384 H8 d128 with S0: the gate is per channel (+128 elements a token-head)
    ((4, 16384, 8, 128, 128, 64, 2, 2, True), 810_549_248, None),
    # GDN B1 T32768 H16 d128 (the bench draws du, so the backward reads it)
    ((1, 32768, 16, 128, 128, 64, 1, 2, False), 674_234_368, 1_754_267_648),
    # KDA B8 T4096 H16 d128 with du
    ((8, 4096, 16, 128, 128, 64, 2, 2, False), 814_743_552, 2_175_795_200),
))
def test_bytes(bench, cfg, fwd_bytes, total_bytes):
    B, T, H, dk, dv, C, var, elem, s0 = cfg
    c = bench.alg_counts(B, T, H, dk, dv, C, var, elem, s0=s0)
    assert c["fwd_bytes"] == fwd_bytes
    if total_bytes is not None:
        assert c["fwd_bytes"] + c["bwd_bytes"] == total_bytes


def test_flops_and_du(bench):
    c = bench.alg_counts(8, 4096, 8, 128, 128, 64, 1, 2)
    per = 6 * 128 * 128 + 3 * 64 * 128 + 2 * 64 * 128 + 64 * 64 / 3  # 140.6 k per token-head
    assert abs(c["fwd_flops"] - 8 * 4096 * 8 * per) < 1 and c["bwd_flops"] == 2 * c["fwd_flops"]
    assert abs(c["fwd_flops"] / 1e9 - 36.87) < 0.01
    # no du: the backward reads dv fewer elements per token-head
    d = bench.alg_counts(8, 4096, 8, 128, 128, 64, 1, 2, du=False)
    assert c["bwd_bytes"] - d["bwd_bytes"] == 8 * 4096 * 8 * 2 * 128


def test_gradient_kernel_bytes_leave_out_du(bench):
    """The intra-chunk gradient kernel reads q, k, v, beta, the gate and dO and writes dq, dk, dv,
    dbeta, d log alpha: (4 dk + 3 dv + 2 + 2) elements a token-head for Gated DeltaNet, 471.9 MB at
    the headline shape; du goes to the reverse chain."""
    c = bench.alg_counts(8, 4096, 8, 128, 128, 64, 1, 2)
    assert c["bwd_grad_kernel_bytes"] == 8 * 4096 * 8 * 2 * (4 * 128 + 3 * 128 + 2 + 2) == 471_859_200
    assert c["bwd_io_bytes"] - c["bwd_grad_kernel_bytes"] == 8 * 4096 * 8 * 2 * 128


def test_both_arms_print_the_same_config(bench):
    from gated_delta_rule_107_b200.inputs import WORKLOADS
    w = WORKLOADS[2]
    cfg = bench.workload_config(w, w.B, 1)
    assert cfg["workload"].endswith("fwd+bwd") and cfg["B"] == 8 and cfg["T"] == 4096 and cfg["H"] == 8
    assert set(cfg) == {"workload", "B", "T", "H", "dk", "dv", "chunk", "variant", "io", "l2", "parallelism"}
