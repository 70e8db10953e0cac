"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, validates arguments before touching the GPU, and sizes workspaces
without any O(d_out * d_in) term.  No compute call is made here."""

import ctypes
import os
import re
import subprocess

import pytest

from factored_weight_norm_b200 import build as build_mod
from factored_weight_norm_b200 import dora as D

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dora.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return D.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dora_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("dora_factored_norm", "dora_compose_fwd", "dora_compose_bwd"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", D.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (dora_[a-z0-9_]+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    extra = sorted(exported - set(names))
    assert not extra, f"exported but not declared: {extra}"
    assert set(D.SIGNATURES) == set(names)


def test_status_strings(lib):
    for st in range(6):
        assert D.status_string(st).startswith("DORA_")
    assert "unknown" in D.status_string(99)


FAKE = ctypes.c_void_p(0x10000)      # 64 KiB aligned, never dereferenced
MISALIGNED = ctypes.c_void_p(0x10002)


def _norm(lib, W=FAKE, A=FAKE, B=FAKE, d_out=64, d_in=128, r=16, dt=D.DORA_BF16, n=FAKE, ws=FAKE, wsb=1 << 30):
    return lib.dora_factored_norm(W, A, B, d_out, d_in, r, 0.5, dt, n, ws, wsb, None)


def test_norm_argument_errors(lib):
    assert _norm(lib, W=None) == D.DORA_ERR_INVALID_ARG
    assert _norm(lib, n=None) == D.DORA_ERR_INVALID_ARG
    assert _norm(lib, A=None) == D.DORA_ERR_INVALID_ARG
    assert _norm(lib, d_out=-1) == D.DORA_ERR_INVALID_ARG
    assert _norm(lib, r=-3) == D.DORA_ERR_INVALID_ARG
    assert _norm(lib, dt=7) == D.DORA_ERR_UNSUPPORTED
    assert _norm(lib, d_in=100) == D.DORA_ERR_UNSUPPORTED  # bf16 needs d_in % 8 == 0
    assert _norm(lib, r=24) == D.DORA_ERR_UNSUPPORTED      # bf16 needs r % 16 == 0
    assert _norm(lib, r=8192) == D.DORA_ERR_UNSUPPORTED    # beyond the supported rank
    assert _norm(lib, W=MISALIGNED) == D.DORA_ERR_UNSUPPORTED
    assert _norm(lib, ws=None) == D.DORA_ERR_WORKSPACE
    assert _norm(lib, wsb=16) == D.DORA_ERR_WORKSPACE
    assert _norm(lib, ws=MISALIGNED) == D.DORA_ERR_UNSUPPORTED
    assert _norm(lib, d_out=0) == D.DORA_OK  # nothing to do, nothing launched


def test_selftest_timeout_argument_errors(lib):
    # rejected on the host before any device work
    assert lib.dora_selftest_timeout(0, None) == D.DORA_ERR_INVALID_ARG
    assert lib.dora_selftest_timeout(-5, None) == D.DORA_ERR_INVALID_ARG
    assert lib.dora_selftest_timeout(10**12, None) == D.DORA_ERR_INVALID_ARG


def _problems(*specs):
    arr = (D.NormProblem * len(specs))()
    for i, sp in enumerate(specs):
        q = dict(W=FAKE.value, A=FAKE.value, B=FAKE.value, d_out=256, d_in=128, r=16, s=0.5, n_out=FAKE.value)
        q.update(sp)
        arr[i] = D.NormProblem(q["W"], q["A"], q["B"], q["d_out"], q["d_in"], q["r"], q["s"], q["n_out"])
    return arr


def test_batched_argument_errors(lib):
    f, size = lib.dora_factored_norm_batched, lib.dora_factored_norm_batched_workspace_size
    good = _problems({}, {"r": 384, "d_out": 1000})
    need = size(good, 2, D.DORA_BF16)
    assert need > 0
    assert f(None, 0, D.DORA_BF16, None, 0, None) == D.DORA_OK  # nothing to do
    assert f(None, 2, D.DORA_BF16, None, 0, None) == D.DORA_ERR_INVALID_ARG
    assert size(None, -1, D.DORA_BF16) == 0
    assert f(good, 2, 7, FAKE, need, None) == D.DORA_ERR_UNSUPPORTED
    # every module is checked before anything is launched
    assert f(_problems({}, {"d_out": -1}), 2, D.DORA_BF16, FAKE, 1 << 30, None) == D.DORA_ERR_INVALID_ARG
    assert f(_problems({}, {"W": None}), 2, D.DORA_BF16, FAKE, 1 << 30, None) == D.DORA_ERR_INVALID_ARG
    assert f(_problems({"d_in": 100}), 1, D.DORA_BF16, FAKE, 1 << 30, None) == D.DORA_ERR_UNSUPPORTED
    assert f(_problems({"r": 24}), 1, D.DORA_BF16, FAKE, 1 << 30, None) == D.DORA_ERR_UNSUPPORTED
    assert f(good, 2, D.DORA_BF16, None, 0, None) == D.DORA_ERR_WORKSPACE
    assert f(good, 2, D.DORA_BF16, FAKE, need - 1, None) == D.DORA_ERR_WORKSPACE
    assert f(good, 2, D.DORA_BF16, MISALIGNED, need, None) == D.DORA_ERR_UNSUPPORTED


def test_batched_workspace_has_no_dense_term(lib):
    # 64 modules of 8192 x 8192 at r = 384: the table, the work lists and each
    # module's (s/2) G, nothing of size d_out x d_in
    arr = _problems(*[{"d_out": 8192, "d_in": 8192, "r": 384}] * 64)
    need = lib.dora_factored_norm_batched_workspace_size(arr, 64, D.DORA_BF16)
    assert need < 64 * (384 * 384 * 2 + 4096) + (1 << 20)


def test_compose_argument_errors(lib):
    f = lib.dora_compose_fwd
    assert f(None, FAKE, FAKE, FAKE, 0.5, 4, 64, D.DORA_BF16, FAKE, None) == D.DORA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, 0.5, -1, 64, D.DORA_BF16, FAKE, None) == D.DORA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, 0.5, 4, 60, D.DORA_BF16, FAKE, None) == D.DORA_ERR_UNSUPPORTED
    assert f(FAKE, MISALIGNED, FAKE, FAKE, 0.5, 4, 64, D.DORA_BF16, FAKE, None) == D.DORA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, 0.5, 0, 64, D.DORA_BF16, FAKE, None) == D.DORA_OK
    b = lib.dora_compose_bwd
    ws = lib.dora_compose_bwd_workspace_size(4, 64)
    # dy, base, lora, m, n, s, tokens, d_out, dt, d_base, d_lora, d_m, workspace, bytes, stream
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, 0.5, 4, 64, D.DORA_BF16, FAKE, FAKE, FAKE, FAKE, ws, None]
    bad = list(args)
    bad[11] = None  # d_m
    assert b(*bad) == D.DORA_ERR_INVALID_ARG
    bad = list(args)
    bad[13] = ws - 1
    assert b(*bad) == D.DORA_ERR_WORKSPACE
    bad = list(args)
    bad[12] = None
    assert b(*bad) == D.DORA_ERR_WORKSPACE
    bad = list(args)
    bad[7] = 12
    assert b(*bad) == D.DORA_ERR_UNSUPPORTED


def test_compose_bias_argument_errors(lib):
    odd = ctypes.c_void_p(0x10001)
    f = lib.dora_compose_fwd_bias
    # base, lora, bias, m, n, s, tokens, d_out, dt, y, stream
    assert f(None, FAKE, FAKE, FAKE, FAKE, 0.5, 4, 64, D.DORA_BF16, FAKE, None) == D.DORA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, odd, FAKE, FAKE, 0.5, 4, 64, D.DORA_BF16, FAKE, None) == D.DORA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, MISALIGNED, FAKE, FAKE, 0.5, 4, 64, D.DORA_BF16, FAKE, None) == D.DORA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, MISALIGNED, FAKE, FAKE, 0.5, 4, 64, D.DORA_F32, FAKE, None) == D.DORA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 0.5, 0, 64, D.DORA_BF16, FAKE, None) == D.DORA_OK
    b = lib.dora_compose_bwd_bias
    ws = lib.dora_compose_bwd_workspace_size(4, 64)
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.5, 4, 64, D.DORA_BF16, FAKE, FAKE, FAKE, FAKE, ws, None]
    bad = list(args)
    bad[3] = MISALIGNED  # a bf16 bias must be 16-byte aligned
    assert b(*bad) == D.DORA_ERR_UNSUPPORTED
    bad = list(args)
    bad[12] = None  # d_m
    assert b(*bad) == D.DORA_ERR_INVALID_ARG
    na = lib.dora_compose_bwd_noalloc_bias
    assert na(FAKE, FAKE, FAKE, odd, FAKE, FAKE, 0.5, 4, 64, D.DORA_BF16, FAKE, FAKE, FAKE, None) == D.DORA_ERR_UNSUPPORTED
    assert na(FAKE, FAKE, FAKE, None, FAKE, FAKE, 0.5, 4, 64, D.DORA_BF16, FAKE, FAKE, None, None) == D.DORA_ERR_INVALID_ARG


def test_workspace_has_no_dense_term(lib):
    # the dense product B A would be d_out * d_in * 2 bytes; the workspace is
    # O(d_out r + r^2 + SMs * 128)
    for d_out, d_in, r in ((8192, 8192, 384), (27648, 5120, 384), (8192, 8192, 768), (4096, 4096, 64)):
        ws = lib.dora_factored_norm_workspace_size(d_out, d_in, r, D.DORA_BF16)
        assert 0 < ws < d_out * d_in * 2 / 8, (d_out, d_in, r, ws)
        # growing d_in does not grow the workspace
        assert lib.dora_factored_norm_workspace_size(d_out, 4 * d_in, r, D.DORA_BF16) == ws
    ws_bwd = lib.dora_compose_bwd_workspace_size(8192, 8192)
    assert 0 < ws_bwd < 8192 * 8192 * 2 / 16
    assert lib.dora_compose_bwd_workspace_size(65536, 8192) == ws_bwd  # independent of tokens
    assert lib.dora_factored_norm_workspace_size(-1, 8, 16, D.DORA_BF16) == 0


def test_num_sms_without_device(lib):
    import torch

    if not torch.cuda.is_available():
        assert lib.dora_num_sms() == 0


# ------------------------------------------------ stream-K schedule algebra
# A mirror of the norm kernel's schedule: weighted contiguous unit ranges,
# the owner search over them, and the rotated walk of one range.
def _cum(c, early, w_e, w_l):
    return w_e * min(c, early) + w_l * max(0, c - early)


def _start(c, U, G, early, w_e, w_l):
    return U * _cum(c, early, w_e, w_l) // _cum(G, early, w_e, w_l)


def _owner(u, U, G, early, w_e, w_l):
    lo, hi = 0, G - 1
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if _start(mid, U, G, early, w_e, w_l) <= u:
            lo = mid
        else:
            hi = mid - 1
    return lo


def _walk(u0, u1, kb_total):
    """Units of [u0, u1) in walk order with the segment-end flags: from the
    first tile boundary tb on, then [u0, tb)."""
    tb = min(u1, -(-u0 // kb_total) * kb_total)
    order = list(range(tb, u1)) + list(range(u0, tb)) if u0 < tb < u1 else list(range(u0, u1))
    len2 = tb - u0 if u0 < tb < u1 else 0
    out = []
    for i, u in enumerate(order):
        left = len(order) - i
        last = left == 1 or u % kb_total == kb_total - 1 or (len2 > 0 and left == len2 + 1)
        out.append((u, last))
    return out


@pytest.mark.parametrize("U,G,early,w_e,w_l", [(1, 1, 1, 1, 1), (3, 3, 3, 1, 1), (7, 3, 3, 5, 5), (8384, 148, 148, 16, 16),
                                               (134 * 216, 148, 124, 3139, 2900), (10, 7, 5, 16, 0), (8576, 148, 124, 945, 730),
                                               (300, 148, 140, 40, 2)])
def test_stream_k_partition(U, G, early, w_e, w_l):
    """Weighted ranges tile [0, U); the owner search inverts them; the rotated
    walk visits each unit once, in segments of one tile each; a tile's
    segments are the nonempty ranges meeting it; segment slot c + tile is
    unique."""
    ranges = [(_start(c, U, G, early, w_e, w_l), _start(c + 1, U, G, early, w_e, w_l)) for c in range(G)]
    assert ranges[0][0] == 0 and ranges[-1][1] == U
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0 and a0 <= a1
    for c, (a, b) in enumerate(ranges):
        for u in range(a, b):
            assert _owner(u, U, G, early, w_e, w_l) == c
    for kb_total in (1, 3, 134):
        seen = set()
        segs = {}
        for c, (a, b) in enumerate(ranges):
            walk = _walk(a, b, kb_total)
            assert sorted(u for u, _ in walk) == list(range(a, b))
            seg = []
            for u, last in walk:
                seg.append(u)
                if last:
                    tiles = {v // kb_total for v in seg}
                    assert len(tiles) == 1 and seg == list(range(seg[0], seg[-1] + 1))
                    t = tiles.pop()
                    segs[t] = segs.get(t, 0) + 1
                    idx = c + t
                    assert idx not in seen
                    seen.add(idx)
                    seg = []
            assert not seg
        assert max(seen, default=0) < G + (U + kb_total - 1) // kb_total
        for t, n in segs.items():
            o0 = _owner(t * kb_total, U, G, early, w_e, w_l)
            o1 = _owner(min(U, (t + 1) * kb_total) - 1, U, G, early, w_e, w_l)
            assert n == sum(1 for o in range(o0, o1 + 1) if ranges[o][1] > ranges[o][0])


def test_fused_linear_argument_errors(lib):
    f = lib.dora_fused_linear_fwd
    ws = lib.dora_fused_linear_fwd_workspace_size(4, 16)
    assert ws == 256
    assert lib.dora_fused_linear_fwd_workspace_size(8192, 384) == 8192 * 384 * 2
    # x, W, A, B, bias, m, n, s, tokens, d_in, d_out, r, dt, y, workspace, bytes, stream
    args = [FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 0.5, 4, 64, 64, 16, D.DORA_BF16, FAKE, FAKE, ws, None]

    def call(**kw):
        a = list(args)
        names = ["x", "W", "A", "B", "bias", "m", "n", "s", "tokens", "d_in", "d_out", "r", "dt", "y", "ws", "wsb"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return f(*a)

    assert call(dt=D.DORA_F32) == D.DORA_ERR_UNSUPPORTED
    assert call(tokens=-1) == D.DORA_ERR_INVALID_ARG
    assert call(tokens=0) == D.DORA_OK
    assert call(d_out=0) == D.DORA_OK
    assert call(d_in=0) == D.DORA_ERR_UNSUPPORTED
    assert call(x=None) == D.DORA_ERR_INVALID_ARG
    assert call(A=None) == D.DORA_ERR_INVALID_ARG
    assert call(m=None) == D.DORA_ERR_INVALID_ARG
    assert call(d_in=60) == D.DORA_ERR_UNSUPPORTED
    assert call(r=12) == D.DORA_ERR_UNSUPPORTED
    assert call(d_out=20) == D.DORA_ERR_UNSUPPORTED
    assert call(W=MISALIGNED) == D.DORA_ERR_UNSUPPORTED
    assert call(bias=ctypes.c_void_p(0x10001)) == D.DORA_ERR_UNSUPPORTED
    assert call(wsb=ws - 1) == D.DORA_ERR_WORKSPACE
    assert call(ws=None) == D.DORA_ERR_WORKSPACE
    assert call(ws=MISALIGNED) == D.DORA_ERR_UNSUPPORTED


def test_norm_bwd_argument_errors(lib):
    f = lib.dora_factored_norm_bwd
    ws = lib.dora_factored_norm_bwd_workspace_size(64, 128, 16)
    # W, A, B, s, n, d_n, d_out, d_in, r, dt, dA, dB, workspace, bytes, stream
    args = [FAKE, FAKE, FAKE, 0.5, FAKE, FAKE, 64, 128, 16, D.DORA_BF16, FAKE, FAKE, FAKE, ws, None]
    names = ["W", "A", "B", "s", "n", "d_n", "d_out", "d_in", "r", "dt", "dA", "dB", "ws", "wsb"]

    def call(**kw):
        a = list(args)
        for k, v in kw.items():
            a[names.index(k)] = v
        return f(*a)

    assert call(dt=D.DORA_F32) == D.DORA_ERR_UNSUPPORTED
    assert call(r=-1) == D.DORA_ERR_INVALID_ARG
    assert call(r=0) == D.DORA_OK            # empty gradients, nothing launched
    assert call(dA=None) == D.DORA_ERR_INVALID_ARG
    assert call(W=None) == D.DORA_ERR_INVALID_ARG
    assert call(d_n=None) == D.DORA_ERR_INVALID_ARG
    assert call(d_out=60) == D.DORA_ERR_UNSUPPORTED
    assert call(r=12) == D.DORA_ERR_UNSUPPORTED
    assert call(A=MISALIGNED) == D.DORA_ERR_UNSUPPORTED
    assert call(dB=MISALIGNED) == D.DORA_ERR_UNSUPPORTED
    assert call(wsb=ws - 1) == D.DORA_ERR_WORKSPACE
    assert call(ws=None) == D.DORA_ERR_WORKSPACE


def test_norm_bwd_workspace_has_no_dense_term(lib):
    for d_out, d_in, r in ((8192, 8192, 384), (27648, 5120, 384), (4096, 4096, 64)):
        ws = lib.dora_factored_norm_bwd_workspace_size(d_out, d_in, r)
        assert ws < d_out * d_in * 2 // 4  # O(r d_out + r^2): 22.6 MB vs the dense 134 MB at 8192^2, r = 384
        assert lib.dora_factored_norm_bwd_workspace_size(d_out, 2 * d_in, r) == ws  # independent of d_in


def test_norm_sq_and_finish_argument_errors(lib):
    f = lib.dora_factored_norm_sq
    assert f(FAKE, FAKE, FAKE, 64, 128, 16, 0.5, D.DORA_BF16, None, FAKE, 1 << 30, None) == D.DORA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 64, 128, 12, 0.5, D.DORA_BF16, FAKE, FAKE, 1 << 30, None) == D.DORA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 64, 128, 16, 0.5, D.DORA_BF16, FAKE, FAKE, 0, None) == D.DORA_ERR_WORKSPACE
    assert f(FAKE, FAKE, FAKE, 0, 128, 16, 0.5, D.DORA_BF16, FAKE, FAKE, 0, None) == D.DORA_OK
    g = lib.dora_norm_finish
    assert g(None, 8, None) == D.DORA_ERR_INVALID_ARG
    assert g(FAKE, -1, None) == D.DORA_ERR_INVALID_ARG
    assert g(ctypes.c_void_p(0x10002), 8, None) == D.DORA_ERR_UNSUPPORTED
    assert g(None, 0, None) == D.DORA_OK
