"""CUDA path vs the fp64 oracle on identical seeded inputs (through the C ABI).

Small cases run the oracle on every (b, h); the full-size workloads run the GPU at
full size (the launch configuration the benchmark times) and the oracle on a
sample of heads (heads are independent, so a head slice is an exact sub-problem).
Bar: max|gpu - oracle| / max|oracle| per output <= 1e-4 (fp32 I/O), <= 2e-2 (bf16).
"""
import pytest
import torch

from gated_delta_rule_107_b200.inputs import WORKLOADS
from parity_util import compare_bwd, compare_fwd, gen, gpu_bwd, gpu_fwd, oracle_bwd, oracle_fwd

pytestmark = pytest.mark.gpu

VARS = ("deltanet", "gdn", "kda")


@pytest.mark.parametrize("variant", VARS)
@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("T", (1, 63, 64, 65, 200))
def test_fwd_small(variant, dtype, T):
    x = gen(variant, dtype, 2, T, 3, 128, 128, seed=100 + T, s0_std=0.1)
    compare_fwd(gpu_fwd(x, variant), oracle_fwd(x, variant), dtype, what=f"{variant} {dtype} T={T}")


@pytest.mark.parametrize("variant", VARS)
@pytest.mark.parametrize("dk,dv", ((64, 64), (64, 128), (128, 64)))
def test_fwd_head_dims(variant, dk, dv):
    x = gen(variant, "bf16", 1, 150, 2, dk, dv, seed=7, s0_std=0.05)
    compare_fwd(gpu_fwd(x, variant), oracle_fwd(x, variant), "bf16", what=f"{variant} dk={dk} dv={dv}")


@pytest.mark.parametrize("variant", VARS)
@pytest.mark.parametrize("chunk", (16, 32, 64))
def test_fwd_chunk_sizes(variant, chunk):
    """The result does not depend on the chunk size (fp32 path, tight bar)."""
    x = gen(variant, "f32", 1, 177, 2, 64, 64, seed=9, s0_std=0.2)
    compare_fwd(gpu_fwd(x, variant, chunk=chunk), oracle_fwd(x, variant), "f32", what=f"{variant} C={chunk}")


@pytest.mark.parametrize("variant", VARS)
@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("T,du", ((1, True), (64, False), (130, True)))
def test_bwd_small(variant, dtype, T, du):
    x = gen(variant, dtype, 2, T, 2, 128, 128, seed=200 + T, s0_std=0.1, grads=True, du=du)
    compare_bwd(gpu_bwd(x, variant), oracle_bwd(x, variant), dtype, variant, what=f"{variant} {dtype} T={T}")


@pytest.mark.parametrize("variant", VARS)
def test_bwd_head_dims_and_chunks(variant):
    x = gen(variant, "f32", 1, 99, 2, 64, 128, seed=31, s0_std=0.1, grads=True)
    ref = oracle_bwd(x, variant)
    for chunk in (16, 64):
        compare_bwd(gpu_bwd(x, variant, chunk=chunk), ref, "f32", variant, what=f"{variant} C={chunk}")


def test_bwd_no_upstream_state_grad():
    x = gen("gdn", "bf16", 1, 100, 2, 128, 128, seed=5, grads=True, du=False)
    x["dS_T"] = None
    compare_bwd(gpu_bwd(x, "gdn"), oracle_bwd(x, "gdn"), "bf16", "gdn", what="no du, no dS_T")


# ---- the workloads at full size ------------------------------------------------------------
def _workload(wid):
    w = WORKLOADS[wid]
    return w, gen(w.variant, w.dtype, w.B, w.T, w.H, w.dk, w.dv, seed=w.seed, s0_std=w.s0_std, grads=w.backward,
                  du=w.du)


def test_workload1_deltanet_fp32_full():
    w, x = _workload(1)
    compare_fwd(gpu_fwd(x, w.variant), oracle_fwd(x, w.variant), w.dtype, what=w.name)


@pytest.mark.parametrize("wid,heads", ((2, [0, 7]), (3, [5])))
def test_forward_workloads_full_size_sampled_heads(wid, heads):
    w, x = _workload(wid)
    got = gpu_fwd(x, w.variant)
    compare_fwd(got, oracle_fwd(x, w.variant, heads=heads), w.dtype, heads=heads, what=w.name)
    for key in ("o", "u", "S_T"):
        assert torch.isfinite(got[key]).all(), f"{w.name} {key} not finite"


def test_workload2_backward_full_size_sampled_heads():
    """The headline step (forward + backward at the workload-2 shape)."""
    w, x = _workload(2)
    x.update({k: v for k, v in gen(w.variant, w.dtype, w.B, w.T, w.H, w.dk, w.dv, seed=w.seed + 50, grads=True,
                                   du=True).items() if k in ("dO", "du", "dS_T")})
    g = gpu_bwd(x, w.variant)
    compare_bwd(g, oracle_bwd(x, w.variant, heads=[3]), w.dtype, w.variant, heads=[3], what=w.name + " bwd")


@pytest.mark.parametrize("wid,heads", ((4, [2]), (5, [11])))
def test_backward_workloads_full_size_sampled_heads(wid, heads):
    w, x = _workload(wid)
    g = gpu_bwd(x, w.variant)
    compare_bwd(g, oracle_bwd(x, w.variant, heads=heads), w.dtype, w.variant, heads=heads, what=w.name)
    for key, t in g.items():
        if t is not None:
            assert torch.isfinite(t).all(), f"{w.name} {key} not finite"


def test_kda_bwd_fast_decay_channels_take_the_direct_form():
    """Channels whose gates fall by 3 nats a token span 192 nats over a 64-token chunk, past what the
    midpoint-split intra-chunk gradient accepts; such chunks take the direct form, while the ragged
    last chunk (2 tokens) takes the split form, in one call (fp32, tight bar)."""
    x = gen("kda", "f32", 1, 130, 2, 128, 128, seed=41, s0_std=0.1, grads=True)
    x["loga"][..., :8] = -3.0
    compare_bwd(gpu_bwd(x, "kda"), oracle_bwd(x, "kda"), "f32", "kda", what="kda fast-decay channels")


# ---- fast-decaying gates on the bf16 tensor-core path --------------------------------------
# The workload distribution log alpha = -softplus(N(-3, 1)) keeps a chunk's cumulative gate
# within a few nats; these cases make some channels (KDA) or heads (Gated DeltaNet) fall by
# 3 nats a token (192 over a chunk), and by 12 (far past the exponent range of one factor).
@pytest.mark.parametrize("dv", (128, 64))
def test_kda_bf16_fast_decay_channels_forward(dv):
    """KDA's pair factors e^{g_r - g_i} on channels falling 3 nats a token: split at each 16-token
    block's first token, every factor stays in range (a split at the chunk midpoint does not)."""
    x = gen("kda", "bf16", 2, 200, 3, 128, dv, seed=43, s0_std=0.1)
    x["loga"][..., :8] = -3.0
    compare_fwd(gpu_fwd(x, "kda"), oracle_fwd(x, "kda"), "bf16", what=f"kda bf16 dv={dv} fast-decay channels")


def test_kda_bf16_fast_decay_channels_backward():
    x = gen("kda", "bf16", 2, 200, 2, 128, 128, seed=44, s0_std=0.1, grads=True)
    x["loga"][..., :8] = -3.0
    compare_bwd(gpu_bwd(x, "kda"), oracle_bwd(x, "kda"), "bf16", "kda", what="kda bf16 fast-decay channels")


@pytest.mark.parametrize("T", (64, 137))
def test_kda_bf16_extreme_decay_takes_exact_in_block_sums(T):
    """Channels falling 12 nats a token fall 180 inside one 16-token block, past what one factor
    can carry: such chunks take their in-block entries from exact per-pair sums (k_kda_diag),
    next to ordinary chunks and a ragged last chunk in the same call."""
    x = gen("kda", "bf16", 2, T, 2, 128, 128, seed=45, s0_std=0.1, grads=True)
    x["loga"][0, :, :, :4] = -12.0  # batch 0 only: batch 1 keeps ordinary chunks
    x["loga"][..., 4:8] = -3.0
    compare_fwd(gpu_fwd(x, "kda"), oracle_fwd(x, "kda"), "bf16", what=f"kda bf16 extreme decay T={T}")
    compare_bwd(gpu_bwd(x, "kda"), oracle_bwd(x, "kda"), "bf16", "kda", what=f"kda bf16 extreme decay T={T}")


@pytest.mark.parametrize("dv", (128, 64))
def test_gdn_bf16_fast_decay_heads(dv):
    """A head whose gate falls 3 nats a token strays more than 80 nats from the chunk midpoint, so
    its chunks take the exact per-pair exponentials of the tensor-core kernels, forward and
    backward; the other heads keep the midpoint split."""
    x = gen("gdn", "bf16", 2, 200, 3, 128, dv, seed=46, s0_std=0.1, grads=True)
    x["loga"][:, :, 0] = -3.0
    compare_fwd(gpu_fwd(x, "gdn"), oracle_fwd(x, "gdn"), "bf16", what=f"gdn bf16 dv={dv} fast-decay head")
    compare_bwd(gpu_bwd(x, "gdn"), oracle_bwd(x, "gdn"), "bf16", "gdn", what=f"gdn bf16 dv={dv} fast-decay head")


# ---- run-to-run determinism ----------------------------------------------------------------
def _bitwise_equal(a, b, what):
    for key in a:
        if a[key] is None:
            continue
        assert torch.equal(a[key], b[key]), f"{what}: {key} differs between two identical calls"


def test_kda_backward_is_deterministic_at_workload5_size():
    """Two identical KDA backward calls at the training workload's size (B8 T4096 H16) return the
    same bits: the library has no atomics in its arithmetic, so any difference is a race."""
    w, x = _workload(5)
    _bitwise_equal(gpu_bwd(x, w.variant), gpu_bwd(x, w.variant), w.name)


@pytest.mark.parametrize("variant", VARS)
def test_cuda_core_backward_is_deterministic(variant):
    """The CUDA-core path (fp32 I/O) at C = 64, where every chunk takes the tiled gradient kernel."""
    x = gen(variant, "f32", 4, 1024, 8, 128, 128, seed=47, s0_std=0.1, grads=True)
    _bitwise_equal(gpu_bwd(x, variant), gpu_bwd(x, variant), f"{variant} f32")
