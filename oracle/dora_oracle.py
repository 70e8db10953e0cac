"""Plain fp64 CPU oracle for the high-rank DoRA hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code with
the CUDA library (no kernels, headers, helpers or constants); both sides only
consume the same seeded inputs.

What it computes, and where that is defined
-------------------------------------------
Sources are the pages this project was specified from:

* "Scaling DoRA: High-Rank Adaptation via Factored Norms and Fused Kernels"
  (Zelenin & Zhuravlyova, arXiv 2603.22276), Abstract: DoRA's forward pass
  needs the row-wise norm of ``W + sBA``; frameworks materialise the dense
  ``[d_out, d_in]`` product ``BA`` to get it; the magnitude rescaling is then
  composed with the base and LoRA outputs.
* "DoRA: Weight-decomposed low-rank adaptation" (summary page, section
  "Method"): the pretrained weight is split into a magnitude vector and a
  direction matrix normalised per output channel; the low-rank update adapts
  the direction only.

The factored norm of the first page reaches *exactly* (up to rounding order)
the dense row norm, so this oracle is the plain definition written out, not
the factored algorithm:

    W' = W + s * (B @ A)                  dense [d_out, d_in], fp64
    n_i = sqrt(sum_k W'_ik ** 2)          one norm per output channel
    g_i = m_i / n_i
    y[t, i] = g_i * (base[t, i] + s * lora[t, i])     (no bias; see below)

Backward (the norm ``n`` is held constant, see ``compose_backward``) with an
upstream gradient ``dy``:

    d_base = g * dy
    d_lora = s * g * dy
    d_m_i  = sum_t dy[t, i] * (base[t, i] + s * lora[t, i]) / n_i

Two more definitions serve the paths built on top of these:

    linear_forward:  y = b + g * (x W'^T)           the adapted layer itself
    norm_backward:   dV = (d_n / n) V', dB = s dV A^T, dA = s B^T dV
                     (the row norms' gradients into A and B, norm attached)

Layout convention (PyTorch ``nn.Linear``): ``W`` is ``[d_out, d_in]``, ``A``
(lora_A) is ``[r, d_in]``, ``B`` (lora_B) is ``[d_out, r]``; activations are
``[tokens, d_out]`` row-major; ``m``/``n`` are per output channel.  The
"column-wise" norm of the DoRA summary page is written for a ``[d, k]`` weight
whose columns are output channels; in ``[d_out, d_in]`` storage the same norm
is taken along each row.

Readings where the pages are silent (each also listed in the design notes):

* ``n`` is detached in backward (no gradient flows into ``A``/``B`` through
  the norm).  The DoRA summary page ("Statistical analysis" / "Strengths")
  mentions a training-memory modification of the original method; treating
  the norm as a constant is the plainest reading consistent with the three
  outputs the hot path is asked for.
* No epsilon is invented: ``n_i^2`` is used as computed; ``n_i == 0`` gives
  IEEE inf/nan in ``g`` exactly as the definition does.
* Bias: the pages never mention one.  Where the adapted layer has a bias
  ``b``, ``base`` is taken to be the frozen base layer's output ``x W^T + b``
  (what a framework's base layer returns), and the magnitude rescaling acts
  on the weight's product only, as the DoRA summary page's Method defines the
  adapted weight ``m * V / ||V||``:  ``y = b + g * ((base - b) + s * lora)``.
  ``bias=None`` (the default) is ``b = 0``.  The bias is frozen: no gradient
  is returned for it.

Every function takes float64 numpy arrays (callers round bf16 inputs first,
then widen) and returns float64 results.  No blocking, fusion or reordering
beyond what the definition states.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "dense_adapted_weight",
    "row_norm",
    "row_norm_rows",
    "magnitude_scale",
    "compose_forward",
    "compose_backward",
    "compose_backward_columns",
    "linear_forward",
    "norm_backward",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def dense_adapted_weight(W, A, B, s) -> np.ndarray:
    """``W + s * (B @ A)``, the dense ``[d_out, d_in]`` adapted weight.

    Scaling DoRA, Abstract: the product ``BA`` that every surveyed framework
    materialises.  The oracle materialises it on purpose.
    """
    W, A, B = _f64(W), _f64(A), _f64(B)
    return W + float(s) * (B @ A)


def row_norm(W, A, B, s) -> np.ndarray:
    """``n_i = ||W_i + s * B_i A||_2`` for every output channel i.

    Scaling DoRA, Abstract (the norm is taken over each row of W + sBA); DoRA summary
    page, Method (per-output-channel vector norm of the adapted weight).
    """
    Wp = dense_adapted_weight(W, A, B, s)
    return np.sqrt(np.sum(Wp * Wp, axis=1))


def row_norm_rows(W, A, B, s, rows) -> np.ndarray:
    """``row_norm`` restricted to the output channels listed in ``rows``.

    Same definition, evaluated only for a sample of rows so that full-size
    problems can be checked one row at a time.
    """
    rows = np.asarray(rows, dtype=np.int64)
    W_rows = _f64(W)[rows]
    B_rows = _f64(B)[rows]
    return row_norm(W_rows, A, B_rows, s)


def magnitude_scale(m, n) -> np.ndarray:
    """``g = m / n`` (fp64, IEEE semantics for ``n == 0``).

    DoRA summary page, Method: the direction is normalised and rescaled by the
    learned magnitude.
    """
    with np.errstate(divide="ignore", invalid="ignore"):
        return _f64(m) / _f64(n)


def _bias(bias, d_out) -> np.ndarray:
    return np.zeros(d_out) if bias is None else _f64(bias)


def compose_forward(base, lora, m, n, s, bias=None) -> np.ndarray:
    """``y = b + g * ((base - b) + s * lora)`` broadcast over tokens.

    Scaling DoRA, Abstract: the DoRA composition of the base output, the LoRA
    output and the magnitude rescaling.  ``base = x W^T + b`` and
    ``lora = x A^T B^T`` (unscaled) are ``[tokens, d_out]``; ``bias`` is the
    base layer's ``b`` (``None``: no bias), which the rescaling leaves alone.
    """
    base, lora = _f64(base), _f64(lora)
    b = _bias(bias, base.shape[1])
    g = magnitude_scale(m, n)
    return b[None, :] + g[None, :] * ((base - b[None, :]) + float(s) * lora)


def compose_backward(dy, base, lora, m, n, s, bias=None):
    """Gradients of ``y = b + (m / n) * ((base - b) + s * lora)``, ``n`` constant.

    Returns ``(d_base, d_lora, d_m)``:
      d_base = g * dy,  d_lora = s * g * dy,
      d_m_i  = sum_t dy[t, i] * ((base[t, i] - b_i) + s * lora[t, i]) / n_i.
    Chain rule on the forward definition above (Scaling DoRA, Abstract,
    "gradient computation"), with the norm detached and the bias frozen.
    """
    dy, base, lora = _f64(dy), _f64(base), _f64(lora)
    s = float(s)
    b = _bias(bias, base.shape[1])
    g = magnitude_scale(m, n)
    d_base = g[None, :] * dy
    d_lora = s * g[None, :] * dy
    with np.errstate(divide="ignore", invalid="ignore"):
        d_m = np.sum(dy * ((base - b[None, :]) + s * lora), axis=0) / _f64(n)
    return d_base, d_lora, d_m


def compose_backward_columns(dy, base, lora, m, n, s, cols, bias=None) -> np.ndarray:
    """``d_m`` of ``compose_backward`` for the output channels in ``cols``.

    ``dy``/``base``/``lora`` are the full ``[tokens, d_out]`` arrays (or any
    array indexable by column); only the listed columns are reduced.
    """
    cols = np.asarray(cols, dtype=np.int64)
    dy_c = _f64(np.asarray(dy)[:, cols])
    base_c = _f64(np.asarray(base)[:, cols])
    lora_c = _f64(np.asarray(lora)[:, cols])
    b_c = None if bias is None else _f64(bias)[cols]
    _, _, d_m = compose_backward(dy_c, base_c, lora_c, _f64(m)[cols], _f64(n)[cols], s, bias=b_c)
    return d_m


def linear_forward(x, W, A, B, m, n, s, bias=None, cols=None) -> np.ndarray:
    """The adapted layer's output ``y = b + (m / n) * (x W'^T)``, ``W' = W + s B A``.

    DoRA summary page, Method: the adapted weight is the magnitude times the
    per-channel normalised direction ``W' / ||W'||`` (here with the given ``n``
    standing for ``||W'_i||``); the layer applies it to ``x`` ``[tokens, d_in]``
    and adds the frozen bias ``b`` (``None``: no bias).  Scaling DoRA,
    Abstract: this is the output the fused composition produces.  ``cols``
    restricts the result to those output channels (``W'`` is formed densely
    for them only); ``None`` means all.
    """
    x, W, A, B = _f64(x), _f64(W), _f64(A), _f64(B)
    d_out = W.shape[0]
    cols = np.arange(d_out) if cols is None else np.asarray(cols, dtype=np.int64)
    Wp = dense_adapted_weight(W[cols], A, B[cols], s)
    g = magnitude_scale(_f64(m)[cols], _f64(n)[cols])
    b = _bias(bias, d_out)[cols]
    return b[None, :] + g[None, :] * (x @ Wp.T)


def norm_backward(W, A, B, s, n, d_n):
    """Gradients of the row norms ``n_i = ||W_i + s B_i A||`` w.r.t. ``A`` and ``B``.

    For the training variant that keeps the norm attached (Scaling DoRA,
    Abstract, gradients through the norm; the DoRA summary page's Method defines
    the norm of the adapted weight ``V = W + sBA``).  ``d_n`` is the upstream
    gradient of the loss w.r.t. ``n`` (for the DoRA compose it is
    ``-(m / n) * d_m``).  Chain rule on the dense definition: ``dn_i/dV_i =
    V_i / n_i``, so with ``dV = (d_n / n)[:, None] * V``

        dB = s * dV @ A.T        [d_out, r]
        dA = s * B.T @ dV        [r, d_in]

    Returns ``(dA, dB)``; ``W`` gets no gradient (frozen).  ``n`` is taken as
    given (the forward's norms), not recomputed.
    """
    W, A, B = _f64(W), _f64(A), _f64(B)
    s = float(s)
    V = dense_adapted_weight(W, A, B, s)
    with np.errstate(divide="ignore", invalid="ignore"):
        c = _f64(d_n) / _f64(n)
    dV = c[:, None] * V
    return s * (B.T @ dV), s * (dV @ A.T)
