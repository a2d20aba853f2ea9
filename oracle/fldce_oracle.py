"""Float64 CPU oracle of the fused linear diffusion cross-entropy.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check
in ``__graft_entry__.py`` and the CPU-baseline leg of ``bench.py`` may import
or call this module.  The CUDA library and its Python binding never import,
link or call it, and it imports nothing from them: the two sides share no
code.  Inputs arrive as arrays (float64 copies of the exact bf16/fp32 values
the GPU sees) and every step below is plain numpy in float64.

Source of the arithmetic: the page "fused_linear_diffusion_cross_entropy.py"
(the loss module of a block-diffusion LM fine-tune, adapted from
flash-linear-attention / Liger-Kernel).  Section names below are that page's
function names and the numbered comment steps inside ``cross_entropy_kernel``.
The split-vocabulary merge follows the worked example in section 4
("output-layer embedding") of the tensor-parallel tutorial page
(daliqc.cn developer article 673292621566021).

What the method computes is a closed definition, so the oracle writes the
definition out; the fused GPU kernels reach the same numbers up to rounding
order.  For token n with hidden state H[n], target y_n, masking probability
p_n, logit scale s, label smoothing eps, normaliser T and upstream gradient g:

    z[n, v]   = s * <H[n], W[v]>                       (logits, all v < V)
    lse[n]    = log sum_v exp(z[n, v])
    CE[n]     = (1 - eps) (lse[n] - z[n, y_n]) + eps (lse[n] - mean_v z[n, v])
    loss[n]   = CE[n] / (p_n T)            (0 when y_n is ignore_index)
    G[n, v]   = g s (softmax[n, v] - eps/V - (1 - eps) [v = y_n]) / (p_n T)
    dH        = G W,   dW = G^T H,   loss = sum_n loss[n]

With the page's optional bias b, the logits are z = s * (<H[n], W[v]> + b[v])
and db = sum_n G[n, :].

Readings of points the page leaves open or gets inconsistent (each is also
listed with its justification in the design notes of the repository):

* The page divides only the hard-label part of the loss by p_mask but the
  whole gradient; the oracle divides the whole smoothed CE, which is the
  loss whose derivative the page's gradient is (pinned by finite differences).
* ``total``: a value > 0 is used as given ('mean' reduction with an explicit
  normaliser, 'sum' is total = 1); a value <= 0 means the count of tokens
  that carry a loss (the page's ``target.ne(ignore_index).sum()``).
* A target outside [0, V) that is not ignore_index is a caller error: it is
  counted, and the token is treated as ignored (also in the count).
* p_mask of an ignored token is never read.
* The upstream gradient g (``do`` in the page's backward) multiplies every
  gradient; the page applies it after the fact, here it is folded into G.
* argmax (lowest index among equal maxima) is an extra output; the page has
  none.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, brute force, library cross-checks, finite differences and the
tutorial's printed split-softmax values); none is unpinned.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

__all__ = [
    "valid_tokens", "resolve_total", "logits", "logsumexp_rows", "partial_lse",
    "merge_partial_lse", "smoothed_ce", "token_coef", "grad_logits", "fldce",
    "fldce_rows", "fldce_dw_rows", "contract_gradients", "bias_gradient", "OracleResult",
]


def valid_tokens(target: np.ndarray, V: int, ignore_index: int):
    """Tokens that carry a loss, and the count of malformed targets.

    cross_entropy_kernel, step 1: a token whose target equals ignore_index
    contributes nothing and its gradient row is zero.  Targets outside
    [0, V) are not defined by the page (they would index out of bounds);
    they are treated as ignored and counted as errors.
    """
    target = np.asarray(target, dtype=np.int64)
    not_ignored = target != ignore_index
    in_range = (target >= 0) & (target < V)
    valid = not_ignored & in_range
    n_err = int(np.count_nonzero(not_ignored & ~in_range))
    return valid, n_err


def resolve_total(total: float, valid: np.ndarray) -> float:
    """The normaliser T of the 'mean' reduction.

    fused_linear_cross_entropy_forward: T is the number of non-ignored
    targets; an explicit positive value overrides it (T = 1 is 'sum').
    """
    if total > 0:
        return float(total)
    return float(np.count_nonzero(valid))


def logits(H: np.ndarray, W: np.ndarray, logit_scale: float, bias=None) -> np.ndarray:
    """z = s * (H W^T + b) in float64 (F.linear(c_x, weight, bias) of the
    chunk loop, then the scale applied in logsumexp_fwd_kernel and
    cross_entropy_kernel step 5)."""
    z = np.asarray(H, np.float64) @ np.asarray(W, np.float64).T
    if bias is not None:
        z = z + np.asarray(bias, np.float64)[None, :]
    return logit_scale * z


def logsumexp_rows(z: np.ndarray) -> np.ndarray:
    """lse[n] = m + log sum_v exp(z[n, v] - m), m = max_v z[n, v]
    (logsumexp_fwd_kernel's per-block formula applied to the whole row)."""
    m = z.max(axis=1)
    return m + np.log(np.exp(z - m[:, None]).sum(axis=1))


def partial_lse(z: np.ndarray, splits: list) -> tuple:
    """Per-split running statistics (max m_k, sum_k exp(z - m_k)) of each row.

    logsumexp_fwd: the vocabulary is cut into blocks and each block keeps its
    own maximum; ``splits`` lists the block boundaries [0 = b_0 < ... < b_K = V].
    """
    ms, ls = [], []
    for a, b in zip(splits[:-1], splits[1:]):
        blk = z[:, a:b]
        m = blk.max(axis=1)
        ms.append(m)
        ls.append(np.exp(blk - m[:, None]).sum(axis=1))
    return np.stack(ms, axis=1), np.stack(ls, axis=1)


def merge_partial_lse(m_parts: np.ndarray, l_parts: np.ndarray) -> np.ndarray:
    """Merge per-split (max, sum-exp) pairs into the row logsumexp.

    logsumexp_fwd merges its per-block values with a second logsumexp; the
    tutorial's section 4 adds the per-shard softmax denominators.  With the
    maxima kept explicitly: lse = M + log sum_k l_k exp(m_k - M), M = max_k m_k.
    """
    M = m_parts.max(axis=1)
    return M + np.log((l_parts * np.exp(m_parts - M[:, None])).sum(axis=1))


def smoothed_ce(z: np.ndarray, lse: np.ndarray, y: np.ndarray, eps: float) -> np.ndarray:
    """Label-smoothed cross-entropy of each row, before the p_mask division.

    cross_entropy_kernel steps 4 and the label-smoothing block after step 5:
    the smoothed target is q' = (1 - eps) onehot(y) + eps / V, and
    H(q', softmax z) = (1 - eps)(lse - z_y) + eps (lse - mean_v z).
    Rows whose y is out of range must be masked by the caller.
    """
    V = z.shape[1]
    yy = np.clip(y, 0, V - 1)
    z_y = z[np.arange(z.shape[0]), yy]
    return (1.0 - eps) * (lse - z_y) + eps * (lse - z.sum(axis=1) / V)


def token_coef(valid: np.ndarray, p_mask: np.ndarray, T: float) -> np.ndarray:
    """1 / (p_n T) for tokens that carry a loss, exactly 0 otherwise.

    cross_entropy_kernel step 4 divides by p_mask (the diffusion 1/t
    weight) and step 6 by ``total``; an ignored token's p_mask is never
    read (it may be 0 or NaN), so it is selected away, not multiplied.
    """
    p = np.asarray(p_mask, np.float64)
    out = np.zeros(valid.shape[0], np.float64)
    out[valid] = 1.0 / (p[valid] * T)
    return out


def grad_logits(z: np.ndarray, lse: np.ndarray, y: np.ndarray, valid: np.ndarray,
                coef: np.ndarray, logit_scale: float, eps: float,
                grad_out: float) -> np.ndarray:
    """dLoss/d(H W^T) for each row: G = g s (softmax - eps/V - (1 - eps) onehot(y)) * coef.

    cross_entropy_kernel step 5 (softmax minus eps/V, times the scale, over
    p_mask and total), step 6 (the -(1 - eps) correction at the target
    column) and fused_linear_cross_entropy_backward (times ``do``).
    Ignored rows are exactly zero.
    """
    V = z.shape[1]
    G = np.exp(z - lse[:, None]) - eps / V
    rows = np.nonzero(valid)[0]
    G[rows, y[rows]] -= (1.0 - eps)
    G *= (grad_out * logit_scale * coef)[:, None]
    G[~valid] = 0.0
    return G


def contract_gradients(G: np.ndarray, H: np.ndarray, W: np.ndarray):
    """dH = G W and dW = G^T H (the two matmuls after cross_entropy_kernel in
    fused_linear_cross_entropy_forward's chunk loop)."""
    return G @ W, G.T @ H


def bias_gradient(G: np.ndarray) -> np.ndarray:
    """db = sum_n G[n, :] (db += c_logits.sum(0) in the chunk loop)."""
    return G.sum(axis=0)


@dataclass
class OracleResult:
    loss: float
    loss_per_token: np.ndarray   # [N]
    lse: np.ndarray              # [N], every row (ignored ones too)
    argmax: np.ndarray           # [N] int64, lowest index among maxima
    top2_gap: np.ndarray         # [N] z_max - z_second (for tie margins)
    dH: Optional[np.ndarray]     # [N, D] (or rows asked for)
    dW: Optional[np.ndarray]     # [V, D] (or rows asked for)
    total: float
    n_valid: int
    n_err: int
    db: Optional[np.ndarray] = None   # [V] when a bias was given


def _top2_gap(z: np.ndarray) -> np.ndarray:
    if z.shape[1] < 2:
        return np.full(z.shape[0], np.inf)
    part = np.partition(z, z.shape[1] - 2, axis=1)
    return part[:, -1] - part[:, -2]


def fldce(H, W, target, p_mask, *, logit_scale: float = 1.0,
          label_smoothing: float = 0.0, ignore_index: int = -100,
          total: float = 0.0, grad_out: float = 1.0, bias=None) -> OracleResult:
    """The whole method on one batch (fused_linear_cross_entropy_forward with
    the backward scaling), materialising the [N, V] logits in float64.

    Meant for sizes where N*V*8 bytes fits comfortably in host memory.
    """
    H = np.asarray(H, np.float64)
    W = np.asarray(W, np.float64)
    y = np.asarray(target, np.int64)
    N, V = H.shape[0], W.shape[0]
    valid, n_err = valid_tokens(y, V, ignore_index)
    T = resolve_total(total, valid)
    z = logits(H, W, logit_scale, bias)
    lse = logsumexp_rows(z)
    ce = smoothed_ce(z, lse, y, label_smoothing)
    coef = token_coef(valid, p_mask, T)
    loss_tok = np.where(valid, ce * coef, 0.0)
    G = grad_logits(z, lse, y, valid, coef, logit_scale, label_smoothing, grad_out)
    dH, dW = contract_gradients(G, H, W)
    return OracleResult(
        loss=float(loss_tok.sum()), loss_per_token=loss_tok, lse=lse,
        argmax=np.argmax(z, axis=1).astype(np.int64), top2_gap=_top2_gap(z),
        dH=dH, dW=dW, total=T, n_valid=int(valid.sum()), n_err=n_err,
        db=None if bias is None else bias_gradient(G))


def fldce_rows(H, W, target, p_mask, rows, *, total: float, logit_scale: float = 1.0,
               label_smoothing: float = 0.0, ignore_index: int = -100,
               grad_out: float = 1.0, row_block: int = 64, bias=None) -> OracleResult:
    """Per-token outputs (lse, loss_n, argmax, dH row) for selected token rows.

    Each token's row depends only on its own logits, so any row can be
    computed on its own; ``total`` must be the resolved normaliser of the
    whole batch (see :func:`resolve_total`).  dW is not computed here.
    """
    H = np.asarray(H, np.float64)
    W = np.asarray(W, np.float64)
    y_all = np.asarray(target, np.int64)
    rows = np.asarray(rows, np.int64)
    V = W.shape[0]
    lse_o, loss_o, am_o, gap_o, dH_o = [], [], [], [], []
    for a in range(0, rows.shape[0], row_block):
        r = rows[a:a + row_block]
        y = y_all[r]
        valid, _ = valid_tokens(y, V, ignore_index)
        z = logits(H[r], W, logit_scale, bias)
        lse = logsumexp_rows(z)
        ce = smoothed_ce(z, lse, y, label_smoothing)
        coef = token_coef(valid, np.asarray(p_mask)[r], total)
        G = grad_logits(z, lse, y, valid, coef, logit_scale, label_smoothing, grad_out)
        lse_o.append(lse)
        loss_o.append(np.where(valid, ce * coef, 0.0))
        am_o.append(np.argmax(z, axis=1))
        gap_o.append(_top2_gap(z))
        dH_o.append(G @ W)
    valid_all, n_err = valid_tokens(y_all, V, ignore_index)
    loss_tok = np.concatenate(loss_o)
    return OracleResult(
        loss=float(loss_tok.sum()), loss_per_token=loss_tok, lse=np.concatenate(lse_o),
        argmax=np.concatenate(am_o).astype(np.int64), top2_gap=np.concatenate(gap_o),
        dH=np.concatenate(dH_o), dW=None, total=float(total),
        n_valid=int(valid_all.sum()), n_err=n_err)


def fldce_dw_rows(H, W, target, p_mask, vocab_rows, *, total: float,
                  logit_scale: float = 1.0, label_smoothing: float = 0.0,
                  ignore_index: int = -100, grad_out: float = 1.0,
                  row_block: int = 128, bias=None):
    """dW rows for selected vocabulary entries, and lse / loss of every token.

    dW[v] = sum_n G[n, v] H[n] needs every token's lse, so all logits are
    formed (row block by row block); only the selected columns of G are kept.
    Returns (dW_rows [k, D], lse [N], loss_per_token [N]).
    """
    H = np.asarray(H, np.float64)
    W = np.asarray(W, np.float64)
    y_all = np.asarray(target, np.int64)
    vr = np.asarray(vocab_rows, np.int64)
    N, V = H.shape[0], W.shape[0]
    dW = np.zeros((vr.shape[0], H.shape[1]), np.float64)
    lse_all = np.empty(N, np.float64)
    loss_all = np.empty(N, np.float64)
    for a in range(0, N, row_block):
        sl = slice(a, min(N, a + row_block))
        y = y_all[sl]
        valid, _ = valid_tokens(y, V, ignore_index)
        z = logits(H[sl], W, logit_scale, bias)
        lse = logsumexp_rows(z)
        ce = smoothed_ce(z, lse, y, label_smoothing)
        coef = token_coef(valid, np.asarray(p_mask)[sl], total)
        lse_all[sl] = lse
        loss_all[sl] = np.where(valid, ce * coef, 0.0)
        # the selected columns of G, with the target-column correction
        Gs = np.exp(z[:, vr] - lse[:, None]) - label_smoothing / V
        hit = (y[:, None] == vr[None, :]) & valid[:, None]
        Gs = Gs - (1.0 - label_smoothing) * hit
        Gs *= (grad_out * logit_scale * coef)[:, None]
        Gs[~valid] = 0.0
        dW += Gs.T @ H[sl]
    return dW, lse_all, loss_all
