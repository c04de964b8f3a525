"""Edge cases and error behaviour of the C ABI on the GPU."""
import ctypes

import pytest
import torch

from gated_delta_rule_107_b200 import binding
from parity_util import compare_fwd, gen, gpu_fwd, oracle_fwd

pytestmark = pytest.mark.gpu


def _args(x, out, u, S, ws, need, B, T, H, dk, dv, var=1, chunk=64, dtype=1):
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    return (p(x["q"]), p(x["k"]), p(x["v"]), p(x["loga"]), p(x["beta"]), p(x["S0"]), p(out), p(u), p(S),
            B, T, H, dk, dv, var, chunk, dtype, p(ws), need, torch.cuda.current_stream().cuda_stream)


def test_empty_sequence_copies_state():
    x = gen("gdn", "bf16", 2, 0, 3, 64, 64, seed=1, s0_std=1.0)
    o, u, S = binding.delta_rule_fwd(x["q"], x["k"], x["v"], x["loga"], x["beta"], x["S0"], variant="gdn")
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(S, x["S0"])
    o, u, S = binding.delta_rule_fwd(x["q"], x["k"], x["v"], x["loga"], x["beta"], None, variant="gdn")
    torch.cuda.synchronize()
    assert torch.count_nonzero(S) == 0
    dS_T = torch.randn(2, 3, 64, 64, device="cuda")
    g = binding.delta_rule_bwd(x["q"], x["k"], x["v"], x["loga"], x["beta"], x["S0"], torch.empty_like(x["v"]),
                               None, dS_T, variant="gdn")
    torch.cuda.synchronize()
    assert torch.equal(g["dS0"], dS_T)


def test_empty_batch_is_noop():
    x = gen("kda", "bf16", 0, 10, 2, 128, 128, seed=1)
    o, u, S = binding.delta_rule_fwd(x["q"], x["k"], x["v"], x["loga"], x["beta"], None, variant="kda")
    torch.cuda.synchronize()
    assert o.numel() == 0


def test_invalid_arguments_return_codes():
    B, T, H, d = 1, 70, 2, 64
    x = gen("gdn", "bf16", B, T, H, d, d, seed=2)
    out = torch.empty_like(x["v"])
    need = binding.workspace_size(B, T, H, d, d, 1, 64, 1, 0)
    ws = torch.empty(need + 256, dtype=torch.uint8, device="cuda")
    ok = _args(x, out, None, None, ws, need, B, T, H, d, d)
    assert binding.fwd_raw(*ok) == binding.DR_OK
    torch.cuda.synchronize()
    bad_cases = {
        "variant": (binding.DR_ERR_ARG, {14: 7}),
        "dtype": (binding.DR_ERR_ARG, {16: 9}),
        "head dim": (binding.DR_ERR_UNSUPPORTED, {12: 96}),
        "chunk": (binding.DR_ERR_UNSUPPORTED, {15: 48}),
        "negative T": (binding.DR_ERR_ARG, {10: -1}),
        "missing q": (binding.DR_ERR_ARG, {0: None}),
        "missing gate": (binding.DR_ERR_ARG, {3: None}),
        "misaligned k": (binding.DR_ERR_ALIGN, {1: x["k"].data_ptr() + 2}),
        "small workspace": (binding.DR_ERR_WORKSPACE, {18: max(need - 1, 0)}) if need else None,
        "misaligned workspace": (binding.DR_ERR_ALIGN, {17: ws.data_ptr() + 16}) if need else None,
    }
    for name, case in bad_cases.items():
        if case is None:
            continue
        code, repl = case
        a = list(ok)
        for i, val in repl.items():
            a[i] = val
        assert binding.fwd_raw(*a) == code, name
    assert binding.strerror(binding.DR_ERR_ALIGN).startswith("misaligned")
    with pytest.raises(ValueError):
        binding.delta_rule_fwd(x["q"][:, ::2], x["k"][:, ::2], x["v"][:, ::2], x["loga"][:, ::2],
                               x["beta"][:, ::2], None, variant="gdn")
    assert binding.sync_status() == binding.DR_OK


def test_outputs_do_not_write_past_their_ends():
    """Guard bands after every output stay untouched (no out-of-bounds stores)."""
    B, T, H, d = 2, 77, 3, 128
    for var in ("deltanet", "gdn", "kda"):
        x = gen(var, "bf16", B, T, H, d, d, seed=3, s0_std=0.1, grads=True)
        pad = 4096
        sentinel = -12288.0  # exactly representable in bf16 and fp32

        def guarded(shape, dtype):
            n = 1
            for s in shape:
                n *= s
            buf = torch.full((n + pad,), sentinel, dtype=dtype, device="cuda")
            return buf, buf[:n].view(shape)

        ob, o = guarded((B, T, H, d), torch.bfloat16)
        ub, u = guarded((B, T, H, d), torch.bfloat16)
        sb, S = guarded((B, H, d, d), torch.float32)
        binding.delta_rule_fwd(x["q"], x["k"], x["v"], x["loga"], x["beta"], x["S0"], variant=var, out=o, u=u,
                               S_T=S)
        bufs = {"o": ob, "u": ub, "S_T": sb}
        grads = {}
        for name, shape, dt in (("dq", (B, T, H, d), torch.bfloat16), ("dk", (B, T, H, d), torch.bfloat16),
                                ("dv", (B, T, H, d), torch.bfloat16), ("dbeta", (B, T, H), torch.bfloat16),
                                ("dS0", (B, H, d, d), torch.float32)):
            bufs[name], grads[name] = guarded(shape, dt)
        if var != "deltanet":
            bufs["dalpha"], grads["dalpha"] = guarded(tuple(x["loga"].shape), torch.bfloat16)
        else:
            grads["dalpha"] = None
        binding.delta_rule_bwd(x["q"], x["k"], x["v"], x["loga"], x["beta"], x["S0"], x["dO"], x["du"], x["dS_T"],
                               variant=var, grads=grads)
        torch.cuda.synchronize()
        for name, buf in bufs.items():
            tail = buf[-pad:].float()
            assert torch.all(tail == sentinel), f"{var}: write past the end of {name}"


def test_split_sequence_state_handoff():
    """Running [0, T1) then [T1, T) from the GPU's own S_T equals one run."""
    x = gen("kda", "f32", 1, 300, 2, 64, 64, seed=4, s0_std=0.1)
    full = gpu_fwd(x, "kda")
    t1 = 131
    a = {k: (v[:, :t1] if (v is not None and k != "S0") else v) for k, v in x.items()}
    b = {k: (v[:, t1:] if (v is not None and k != "S0") else v) for k, v in x.items()}
    ra = gpu_fwd(a, "kda")
    b["S0"] = ra["S_T"]
    rb = gpu_fwd(b, "kda")
    assert torch.allclose(torch.cat([ra["o"], rb["o"]], 1), full["o"], atol=2e-5, rtol=1e-4)
    assert torch.allclose(rb["S_T"], full["S_T"], atol=2e-5, rtol=1e-4)
    compare_fwd(full, oracle_fwd(x, "kda"), "f32")


def test_split_sequence_tensor_core_path():
    """Same hand-off on the bf16 tensor-core forward (offset views as inputs)."""
    x = gen("gdn", "bf16", 2, 333, 2, 128, 128, seed=8, s0_std=0.1)
    full = gpu_fwd(x, "gdn")
    t1 = 192
    a = {k: (v[:, :t1].contiguous() if (v is not None and k != "S0") else v) for k, v in x.items()}
    b = {k: (v[:, t1:].contiguous() if (v is not None and k != "S0") else v) for k, v in x.items()}
    ra = gpu_fwd(a, "gdn")
    b["S0"] = ra["S_T"]
    rb = gpu_fwd(b, "gdn")
    ref = oracle_fwd(x, "gdn")
    from parity_util import rel_err, np64
    assert rel_err(np64(torch.cat([ra["o"], rb["o"]], 1)), ref["o"]) < 2e-2
    assert rel_err(np64(rb["S_T"]), ref["S_T"]) < 2e-2


def test_host_buffer_entry_point():
    x = gen("gdn", "bf16", 1, 100, 2, 128, 128, seed=6)
    h = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in x.items()}
    o, u, S = binding.delta_rule_fwd_host(h["q"], h["k"], h["v"], h["loga"], h["beta"], None, variant="gdn")
    r = gpu_fwd(x, "gdn")
    assert torch.equal(o, r["o"].cpu()) and torch.equal(u, r["u"].cpu()) and torch.equal(S, r["S_T"].cpu())


def test_bounded_wait_runs_out_reports_and_leaves_the_context_usable():
    """A wait that nothing completes gives up after its limit and raises the error word;
    the next call still works."""
    import time
    stream = torch.cuda.current_stream().cuda_stream
    assert binding.selftest_timeout(0, stream) == binding.DR_ERR_ARG
    t0 = time.perf_counter()
    assert binding.selftest_timeout(20000, stream) == binding.DR_OK  # 20 ms
    assert binding.sync_status(stream) == binding.DR_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert binding.sync_status(stream) == binding.DR_OK  # read and cleared
    x = gen("gdn", "bf16", 1, 70, 2, 128, 128, seed=21)
    compare_fwd(gpu_fwd(x, "gdn"), oracle_fwd(x, "gdn"), "bf16", what="after a timed-out wait")
