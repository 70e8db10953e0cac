"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Small cases span several 128-row tiles, several 64-wide K blocks and ragged
tails; full-size workloads run in the launch configuration the bench times
and are checked on sampled rows / columns that the oracle computes one by
one.  Every case feeds both sides the same bf16-rounded tensors.
"""

import numpy as np
import pytest
import torch

import oracle
from factored_weight_norm_b200 import dora as D
from factored_weight_norm_b200 import workloads as wlmod
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _wl(d_out, d_in, r, s=0.5, tokens=64, dtype="bf16", seed=7, w_std=0.02, b_std=0.01, m_noise=1e-3):
    return wlmod.Workload(f"case_{d_out}x{d_in}_r{r}", d_out, d_in, r, s, tokens, dtype, w_std, b_std, m_noise, seed)


def _oracle_norm(W, A, B, s, rows=None):
    W64, A64, B64 = P.f64(W), P.f64(A), P.f64(B)
    if rows is None:
        return oracle.row_norm(W64, A64, B64, s)
    return oracle.row_norm_rows(W64, A64, B64, s, rows)


# ------------------------------------------------------------------- norm
SMALL_NORM = [
    (128, 64, 16),      # one tile, one K block, smallest rank
    (256, 512, 64),
    (300, 520, 48),     # ragged M tile and ragged K block
    (136, 200, 112),    # rank below one box: N-side boxes of r rows, ragged M tile
    (1000, 1000, 128),
    (512, 1024, 384),   # headline rank, two MMA pieces (256 + 128)
    (384, 640, 256),
    (264, 4104, 512),   # full TMEM chunk, K tail of 8
    (384, 640, 768),    # two N chunks of 384
    (200, 328, 272),    # chunk of 272 = 256 + 16 pieces
    (8, 8, 16),         # rank above d_in, 8 rows
]


@pytest.mark.parametrize("shape", SMALL_NORM, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("s", [0.5, -2.0])
def test_norm_bf16_small(shape, s):
    d_out, d_in, r = shape
    wl = _wl(d_out, d_in, r, s=s)
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    n = D.dora_factored_norm(W, A, B, s)
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK
    P.assert_norm_close(n, _oracle_norm(W, A, B, s), torch.bfloat16)


def test_bounded_wait_timeout_is_reported_and_the_context_survives():
    """A bounded wait that runs out (on an mbarrier nothing completes) records
    DORA_ERR_TIMEOUT; the host reads and clears it, and the next call works."""
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK
    D.dora_selftest_timeout(2_000_000)  # about a millisecond
    assert D.dora_device_status() == D.DORA_ERR_TIMEOUT
    assert D.dora_device_status() == D.DORA_OK  # read-and-clear
    wl = _wl(384, 640, 256)
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    n = D.dora_factored_norm(W, A, B, wl.s)
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK
    P.assert_norm_close(n, _oracle_norm(W, A, B, wl.s), torch.bfloat16)


def test_norm_bf16_s_zero_and_b_zero():
    wl = _wl(300, 256, 32)
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    plain = np.linalg.norm(P.f64(W), axis=1)
    P.assert_norm_close(D.dora_factored_norm(W, A, B, 0.0), plain, torch.bfloat16)
    P.assert_norm_close(D.dora_factored_norm(W, A, torch.zeros_like(B), 1.5), plain, torch.bfloat16)


def test_norm_bf16_rank_zero_uses_plain_norm():
    wl = _wl(136, 64, 16)
    W, _, _, _ = wlmod.make_weights(wl, DEV)
    A = torch.empty(0, 64, dtype=torch.bfloat16, device=DEV)
    B = torch.empty(136, 0, dtype=torch.bfloat16, device=DEV)
    n = D.dora_factored_norm(W, A, B, 0.5)
    P.assert_norm_close(n, np.linalg.norm(P.f64(W), axis=1), torch.bfloat16)


def test_norm_bf16_pure_lora_rows():
    """W = 0: n = s ||B_i A||; every term but the Gram one vanishes."""
    wl = _wl(256, 256, 64, s=1.25, b_std=0.05)
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    W = torch.zeros_like(W)
    n = D.dora_factored_norm(W, A, B, wl.s)
    P.assert_norm_close(n, _oracle_norm(W, A, B, wl.s), torch.bfloat16)


def test_norm_bf16_cancellation_is_documented_limit():
    """s B_i A close to -W_i: absolute error ~ eps ||W_i||^2, relative error grows
    as ||W_i||^2 / n_i^2.  Recorded, not held to the 2e-3 bound."""
    wl = _wl(128, 256, 16, s=1.0, b_std=0.02)
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    W2 = (-(B.float() @ A.float()) + 0.05 * W.float()).to(torch.bfloat16)
    n = D.dora_factored_norm(W2, A, B, 1.0)
    ref = _oracle_norm(W2, A, B, 1.0)
    base = np.linalg.norm(P.f64(W2), axis=1)
    rel = np.abs(P.f64(n) - ref) / ref
    # error model: the Gram term is carried as bf16 (s/2) G, so its absolute
    # error is about 2^-9 s^2 B_i G B_i^T ~ 2^-9 ||W_i||^2 here
    bound = 2e-3 * (base / ref) ** 2 + 2e-3
    assert np.all(rel <= bound)


def test_norm_f32_tiny_config():
    wl = wlmod.WORKLOADS["tiny_f32"]
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    n = D.dora_factored_norm(W, A, B, wl.s)
    P.assert_norm_close(n, _oracle_norm(W, A, B, wl.s), torch.float32)


@pytest.mark.parametrize("shape", [(7, 13, 3), (65, 129, 17), (300, 1000, 40)])
def test_norm_f32_any_shape(shape):
    d_out, d_in, r = shape
    wl = _wl(d_out, d_in, r, s=-0.7, dtype="f32")
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    n = D.dora_factored_norm(W, A, B, wl.s)
    P.assert_norm_close(n, _oracle_norm(W, A, B, wl.s), torch.float32)


def test_norm_deterministic():
    wl = _wl(1000, 1000, 128)
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    a = D.dora_factored_norm(W, A, B, 0.5).clone()
    b = D.dora_factored_norm(W, A, B, 0.5).clone()
    assert torch.equal(a, b)


def test_norm_allocates_nothing():
    wl = _wl(1024, 2048, 384)
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    n = torch.empty(wl.d_out, dtype=torch.float32, device=DEV)
    ws = torch.empty(D.dora_factored_norm_workspace_size(wl.d_out, wl.d_in, wl.r), dtype=torch.uint8, device=DEV)
    D.dora_factored_norm(W, A, B, 0.5, n_out=n, workspace=ws)  # first call: module load, descriptors
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    peak0 = torch.cuda.max_memory_allocated()
    for _ in range(3):
        D.dora_factored_norm(W, A, B, 0.5, n_out=n, workspace=ws)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.max_memory_allocated() == peak0
    # O(d_out r + r^2) workspace: no term grows with d_out * d_in
    big = D.dora_factored_norm_workspace_size(8192, 8192, 384)
    assert big < 8192 * 8192 * 2 / 8


# -------------------------------------------------- full-size norm (sampled)
def _sample_rows(d_out, k=384, seed=0):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 129, d_out // 2, d_out - 129, d_out - 128, d_out - 1]
    return np.unique(np.concatenate([[f for f in fixed if 0 <= f < d_out], rng.integers(0, d_out, k)]))


@pytest.mark.parametrize("name", ["bf16_4096_r64", "bf16_8192_r384", "bf16_mlp_up_5120x27648_r384"])
def test_norm_full_size(name):
    wl = wlmod.WORKLOADS[name]
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    n = D.dora_factored_norm(W, A, B, wl.s)
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK
    rows = _sample_rows(wl.d_out)
    P.assert_norm_close(P.f64(n)[rows], _oracle_norm(W, A, B, wl.s, rows), torch.bfloat16)


@pytest.mark.parametrize("wl", wlmod.RANK_SWEEP, ids=lambda w: w.name)
def test_norm_rank_sweep(wl):
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    n = D.dora_factored_norm(W, A, B, wl.s)
    rows = _sample_rows(wl.d_out, k=128)
    P.assert_norm_close(P.f64(n)[rows], _oracle_norm(W, A, B, wl.s, rows), torch.bfloat16)


# --------------------------------------------------------------- compose
def _compose_inputs(wl, tokens=None, near_unity=False):
    W, A, B, m = wlmod.make_weights(wl, DEV)
    _, base, lora = wlmod.make_activations(wl, W, A, B, DEV, tokens=tokens)
    dy = wlmod.make_grad(wl, DEV, tokens=tokens)
    if near_unity:
        m, n = wlmod.make_near_unity_mn(wl, W, DEV)
    else:
        n = torch.linalg.vector_norm(W.float(), dim=1) * (1 + 1e-3 * torch.randn(wl.d_out, device=DEV))
    return base, lora, m.float().contiguous(), n.float().contiguous(), dy


COMPOSE_SHAPES = [(1, 8), (37, 264), (64, 4096), (300, 1000), (129, 2056)]


@pytest.mark.parametrize("shape", COMPOSE_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_compose_fwd_bwd_bf16_small(shape):
    T, d_out = shape
    wl = _wl(d_out, 64, 16, s=0.5, tokens=T)
    base, lora, m, n, dy = _compose_inputs(wl)
    y = D.dora_compose_fwd(base, lora, m, n, wl.s)
    d_base, d_lora, d_m = D.dora_compose_bwd(dy, base, lora, m, n, wl.s)
    torch.cuda.synchronize()
    args = [P.f64(t) for t in (base, lora, m, n)]
    P.assert_act_close(y, oracle.compose_forward(*args, wl.s), "y")
    rb, rl, rm = oracle.compose_backward(P.f64(dy), *args, wl.s)
    P.assert_act_close(d_base, rb, "d_base")
    P.assert_act_close(d_lora, rl, "d_lora")
    P.assert_act_close(d_m, rm, "d_m")


@pytest.mark.parametrize("shape", [(32, 64), (5, 7), (33, 130), (16, 4)], ids=lambda s: "x".join(map(str, s)))
def test_compose_f32(shape):
    T, d_out = shape
    wl = _wl(d_out, 16, 4, s=2.0, tokens=T, dtype="f32")
    base, lora, m, n, dy = _compose_inputs(wl)
    y = D.dora_compose_fwd(base, lora, m, n, wl.s)
    d_base, d_lora, d_m = D.dora_compose_bwd(dy, base, lora, m, n, wl.s)
    args = [P.f64(t) for t in (base, lora, m, n)]
    P.assert_act_close(y, oracle.compose_forward(*args, wl.s), "y")
    rb, rl, rm = oracle.compose_backward(P.f64(dy), *args, wl.s)
    P.assert_act_close(d_base, rb, "d_base")
    P.assert_act_close(d_lora, rl, "d_lora")
    P.assert_act_close(d_m, rm, "d_m")


def test_tiny_f32_config_end_to_end():
    """Config 1: fp32 norm on the GPU, then compose forward and backward."""
    wl = wlmod.WORKLOADS["tiny_f32"]
    W, A, B, m = wlmod.make_weights(wl, DEV)
    _, base, lora = wlmod.make_activations(wl, W, A, B, DEV)
    dy = wlmod.make_grad(wl, DEV)
    n = D.dora_factored_norm(W, A, B, wl.s)
    y = D.dora_compose_fwd(base, lora, m, n, wl.s)
    d_base, d_lora, d_m = D.dora_compose_bwd(dy, base, lora, m, n, wl.s)
    n_ref = _oracle_norm(W, A, B, wl.s)
    P.assert_norm_close(n, n_ref, torch.float32)
    args = [P.f64(base), P.f64(lora), P.f64(m), n_ref]
    P.assert_act_close(y, oracle.compose_forward(*args, wl.s), "y")
    rb, rl, rm = oracle.compose_backward(P.f64(dy), *args, wl.s)
    P.assert_act_close(d_base, rb, "d_base")
    P.assert_act_close(d_lora, rl, "d_lora")
    P.assert_act_close(d_m, rm, "d_m")


def test_compose_empty_tokens():
    d_out = 64
    e = torch.empty(0, d_out, dtype=torch.bfloat16, device=DEV)
    m = torch.ones(d_out, device=DEV)
    n = torch.ones(d_out, device=DEV)
    y = D.dora_compose_fwd(e, e, m, n, 0.5)
    assert y.shape == (0, d_out)
    d_m = torch.full((d_out,), 7.0, device=DEV)
    _, _, d_m = D.dora_compose_bwd(e, e, e, m, n, 0.5, d_m=d_m)
    assert torch.equal(d_m, torch.zeros(d_out, device=DEV))


def test_compose_g_equal_one_invariant():
    wl = _wl(1024, 64, 16, tokens=96)
    base, lora, m, n, _ = _compose_inputs(wl)
    y = D.dora_compose_fwd(base, lora, n, n, wl.s)  # m = n bitwise
    # g = 1, delta = 0: y = base + s*lora (fp32 sum, one bf16 rounding)
    P.assert_act_close(y, P.f64(base) + wl.s * P.f64(lora), "y")


def test_compose_d_lora_is_s_times_d_base():
    wl = _wl(512, 64, 16, tokens=40, s=0.5)
    base, lora, m, n, dy = _compose_inputs(wl)
    d_base, d_lora, _ = D.dora_compose_bwd(dy, base, lora, m, n, 0.5)
    assert torch.equal(d_lora.float(), (0.5 * d_base.float()))


def test_compose_near_unity_headline_shape():
    """g - 1 ~ 1e-4 at d_out = 8192: y - base under the rounding-aware rule."""
    wl = wlmod.TOKEN_SWEEP[0]  # T = 1024, d_out = 8192
    base, lora, m, n, _ = _compose_inputs(wl, near_unity=True)
    g = P.f64(m) / P.f64(n)
    assert 1e-5 < np.median(np.abs(g - 1)) < 1e-3
    y = D.dora_compose_fwd(base, lora, m, n, wl.s)
    rows = np.arange(0, wl.tokens, 7)
    b = P.f64(base)[rows]
    y_exact = oracle.compose_forward(b, P.f64(lora)[rows], P.f64(m), P.f64(n), wl.s)
    P.near_unity_check(P.f64(y)[rows], y_exact, b)


@pytest.mark.parametrize("name", ["bf16_4096_r64", "bf16_8192_r384", "bf16_mlp_up_5120x27648_r384"])
def test_compose_full_size_sampled(name):
    wl = wlmod.WORKLOADS[name]
    base, lora, m, n, dy = _compose_inputs(wl)
    y = D.dora_compose_fwd(base, lora, m, n, wl.s)
    d_base, d_lora, d_m = D.dora_compose_bwd(dy, base, lora, m, n, wl.s)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([[0, wl.tokens - 1], rng.integers(0, wl.tokens, 24)]))
    cols = np.unique(np.concatenate([[0, 7, 8, wl.d_out - 1], rng.integers(0, wl.d_out, 96)]))
    m64, n64 = P.f64(m), P.f64(n)
    b_r, l_r, dy_r = P.f64(base[rows]), P.f64(lora[rows]), P.f64(dy[rows])
    P.assert_act_close(P.f64(y[rows]), oracle.compose_forward(b_r, l_r, m64, n64, wl.s), "y")
    rb, rl, _ = oracle.compose_backward(dy_r, b_r, l_r, m64, n64, wl.s)
    P.assert_act_close(P.f64(d_base[rows]), rb, "d_base")
    P.assert_act_close(P.f64(d_lora[rows]), rl, "d_lora")
    cols_t = torch.as_tensor(cols, device=DEV)
    ref_dm = oracle.compose_backward_columns(
        P.f64(dy[:, cols_t]), P.f64(base[:, cols_t]), P.f64(lora[:, cols_t]), m64[cols], n64[cols], wl.s,
        np.arange(len(cols)),
    )
    P.assert_act_close(P.f64(d_m)[cols], ref_dm, "d_m")


@pytest.mark.parametrize("wl", wlmod.TOKEN_SWEEP[:3], ids=lambda w: w.name)
def test_compose_token_sweep_sampled(wl):
    base, lora, m, n, dy = _compose_inputs(wl, near_unity=True)
    y = D.dora_compose_fwd(base, lora, m, n, wl.s)
    d_base, d_lora, d_m = D.dora_compose_bwd(dy, base, lora, m, n, wl.s)
    rows = np.arange(0, wl.tokens, max(1, wl.tokens // 16))
    args = [P.f64(base[rows]), P.f64(lora[rows]), P.f64(m), P.f64(n)]
    y_exact = oracle.compose_forward(*args, wl.s)
    P.assert_act_close(P.f64(y[rows]), y_exact, "y")
    P.near_unity_check(P.f64(y[rows]), y_exact, args[0])
    cols = np.arange(0, wl.d_out, 97)
    cols_t = torch.as_tensor(cols, device=DEV)
    ref_dm = oracle.compose_backward_columns(
        P.f64(dy[:, cols_t]), P.f64(base[:, cols_t]), P.f64(lora[:, cols_t]), P.f64(m)[cols], P.f64(n)[cols],
        wl.s, np.arange(len(cols)),
    )
    P.assert_act_close(P.f64(d_m)[cols], ref_dm, "d_m")


def test_compose_deterministic_and_no_alloc():
    wl = _wl(2048, 64, 16, tokens=512)
    base, lora, m, n, dy = _compose_inputs(wl)
    ws = torch.empty(D.dora_compose_bwd_workspace_size(512, 2048), dtype=torch.uint8, device=DEV)
    outs = [torch.empty_like(base) for _ in range(3)]
    d_m = torch.empty(2048, device=DEV)
    D.dora_compose_bwd(dy, base, lora, m, n, 0.5, outs[0], outs[1], d_m, ws)
    torch.cuda.synchronize()
    first = d_m.clone()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        D.dora_compose_fwd(base, lora, m, n, 0.5, y=outs[2])
        D.dora_compose_bwd(dy, base, lora, m, n, 0.5, outs[0], outs[1], d_m, ws)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.equal(first, d_m)


# --------------------------------------------------------- end to end
@pytest.mark.parametrize("name", ["bf16_4096_r64"])
def test_norm_then_compose_end_to_end(name):
    """GPU n feeds the GPU compose; y is compared with the oracle's own n."""
    wl = wlmod.WORKLOADS[name].with_(tokens=256)
    W, A, B, m = wlmod.make_weights(wl, DEV)
    _, base, lora = wlmod.make_activations(wl, W, A, B, DEV)
    n = D.dora_factored_norm(W, A, B, wl.s)
    y = D.dora_compose_fwd(base, lora, m, n, wl.s)
    n_ref = _oracle_norm(W, A, B, wl.s)
    y_ref = oracle.compose_forward(P.f64(base), P.f64(lora), P.f64(m), n_ref, wl.s)
    P.assert_act_close(y, y_ref, "y")


def test_device_status_clean_after_suite():
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK


@pytest.mark.parametrize("fill", [0x00, 0xFF, 0x5A])
def test_compose_bwd_ignores_workspace_contents(fill):
    # the column-strip arrival counters carry a per-call tag: whatever the
    # workspace holds on entry, the result is the one a fresh buffer gives
    wl = _wl(1024, 64, 16, s=0.5, tokens=777)
    base, lora, m, n, dy = _compose_inputs(wl)
    clean = torch.zeros(D.dora_compose_bwd_workspace_size(wl.tokens, wl.d_out), dtype=torch.uint8, device=DEV)
    ref = [t.clone() for t in D.dora_compose_bwd(dy, base, lora, m, n, wl.s, workspace=clean)]
    dirty = torch.full_like(clean, fill)
    for _ in range(2):
        got = D.dora_compose_bwd(dy, base, lora, m, n, wl.s, workspace=dirty)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)


@pytest.mark.parametrize("shape", [(256, 1024, 4096), (384, 520, 2048)], ids=lambda s: "x".join(map(str, s)))
def test_norm_bf16_largest_ranks(shape):
    # the largest accepted rank (4096): 8 N chunks of 512, a 32 x 32 tile Gram,
    # rank above d_in
    d_out, d_in, r = shape
    wl = _wl(d_out, d_in, r, s=0.5)
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    n = D.dora_factored_norm(W, A, B, wl.s)
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK
    P.assert_norm_close(n, _oracle_norm(W, A, B, wl.s), torch.bfloat16)
