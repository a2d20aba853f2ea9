"""Pins for the float64 oracle, checked against facts that do not come from it.

Each pin is a plain function that raises AssertionError; the tests run them
on the oracle as written, and ``test_mutants_are_caught`` runs all of them on
deliberately broken copies (a dropped term, a wrong sign or index, a swapped
operand) and requires every mutant to fail at least one pin.

Sources of the pinned facts:
* closed forms of the loss at constant logits and of label smoothing
  (cross_entropy_kernel, label-smoothing block, on the page
  "fused_linear_diffusion_cross_entropy.py");
* PyTorch's float64 ``F.cross_entropy`` and autograd (library routines);
* central finite differences of the loss;
* naive triple loops on tiny shapes;
* the split-softmax values printed in section 4 of the tensor-parallel
  tutorial page (tests/golden/split_softmax_tp_tutorial.json).
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle.fldce_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _case(N=24, D=16, V=37, seed=0, ignore_frac=0.4, sigma=0.7):
    rng = np.random.default_rng(seed)
    H = rng.standard_normal((N, D))
    W = sigma * rng.standard_normal((V, D))
    y = rng.integers(0, V, N)
    y[rng.random(N) < ignore_frac] = -100
    p = rng.uniform(0.05, 1.0, N)
    return H, W, y, p


# ----------------------------------------------------------------- pins

def pin_all_zero_logits():
    """P-1: zero logits give lse = log V, CE = log V for any eps, and
    G = g s (1 - eps)(1/V - [v = y]) / (p T)."""
    N, D, V = 9, 5, 11
    H, W, y, p = _case(N, D, V, seed=1)
    for eps, s, g, T in [(0.0, 1.0, 1.0, 0.0), (0.3, 0.7, 2.5, 4.0)]:
        for zero_h in (True, False):
            Hz = np.zeros_like(H) if zero_h else H
            Wz = W if zero_h else np.zeros_like(W)
            r = O.fldce(Hz, Wz, y, p, logit_scale=s, label_smoothing=eps, total=T, grad_out=g)
            valid = y != -100
            Tn = T if T > 0 else valid.sum()
            assert np.allclose(r.lse, math.log(V), rtol=0, atol=1e-13)
            want_tok = np.where(valid, math.log(V) / (p * Tn), 0.0)
            assert np.allclose(r.loss_per_token, want_tok, rtol=1e-13, atol=0)
            assert abs(r.loss - want_tok.sum()) <= 1e-12 * abs(want_tok.sum())
            G = np.zeros((N, V))
            for n in np.nonzero(valid)[0]:
                G[n, :] = g * s * (1 - eps) / V / (p[n] * Tn)
                G[n, y[n]] -= g * s * (1 - eps) / (p[n] * Tn)
            assert np.allclose(r.dH, G @ Wz, rtol=1e-12, atol=1e-14)
            assert np.allclose(r.dW, G.T @ Hz, rtol=1e-12, atol=1e-14)


def pin_label_smoothing_closed_form():
    """P-2: (1 - eps)(lse - z_y) + eps (lse - mean z) equals the smoothed
    target's cross-entropy -sum_v q'_v log softmax_v, and PyTorch's."""
    H, W, y, p = _case(seed=2, ignore_frac=0.0)
    for eps in (0.0, 0.1, 0.5, 1.0):
        z = O.logits(H, W, 0.8)
        lse = O.logsumexp_rows(z)
        got = O.smoothed_ce(z, lse, y, eps)
        V = z.shape[1]
        logsm = np.log(np.exp(z) / np.exp(z).sum(1, keepdims=True))
        q = np.full(z.shape, eps / V)
        q[np.arange(len(y)), y] += 1 - eps
        want = -(q * logsm).sum(1)
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12)
        ref = F.cross_entropy(torch.from_numpy(z), torch.from_numpy(y), reduction="none",
                              label_smoothing=eps).numpy()
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def pin_ignored_tokens():
    """P-3: an ignored token has loss 0 and a zero dH row, whatever its
    p_mask (0 or NaN), and adds nothing to dW."""
    H, W, y, p = _case(seed=3, ignore_frac=0.5)
    ign = y == -100
    p_bad = p.copy()
    p_bad[ign] = np.where(np.arange(ign.sum()) % 2 == 0, 0.0, np.nan)
    r = O.fldce(H, W, y, p_bad, label_smoothing=0.2, logit_scale=1.3, total=10.0)
    assert np.all(r.loss_per_token[ign] == 0.0)
    assert np.all(r.dH[ign] == 0.0)
    assert np.all(np.isfinite(r.dH)) and np.all(np.isfinite(r.dW)) and np.isfinite(r.loss)
    keep = ~ign
    r2 = O.fldce(H[keep], W, y[keep], p[keep], label_smoothing=0.2, logit_scale=1.3, total=10.0)
    assert np.allclose(r.dW, r2.dW, rtol=1e-13, atol=1e-15)
    assert abs(r.loss - r2.loss) <= 1e-13 * abs(r2.loss)
    # the count-of-valid normaliser excludes ignored (and out-of-range) targets
    y3 = y.copy()
    y3[np.nonzero(keep)[0][:2]] = W.shape[0] + 5
    v3, nerr = O.valid_tokens(y3, W.shape[0], -100)
    assert nerr == 2 and O.resolve_total(0.0, v3) == keep.sum() - 2


def pin_plain_ce_matches_torch():
    """P-4: p = 1, T = count, g = 1 is PyTorch's mean cross-entropy with
    ignore_index and label smoothing; its autograd gives dH and dW."""
    H, W, y, _ = _case(seed=4, ignore_frac=0.3)
    for eps, s in [(0.0, 1.0), (0.15, 0.6)]:
        r = O.fldce(H, W, y, np.ones(len(y)), logit_scale=s, label_smoothing=eps, total=0.0)
        Ht = torch.tensor(H, requires_grad=True)
        Wt = torch.tensor(W, requires_grad=True)
        L = F.cross_entropy(s * (Ht @ Wt.T), torch.from_numpy(y), ignore_index=-100,
                            label_smoothing=eps, reduction="mean")
        L.backward()
        assert abs(r.loss - L.item()) <= 1e-12 * abs(L.item())
        assert np.allclose(r.dH, Ht.grad.numpy(), rtol=1e-10, atol=1e-14)
        assert np.allclose(r.dW, Wt.grad.numpy(), rtol=1e-10, atol=1e-14)


def pin_diffusion_weighting_autograd():
    """P-4b: with per-token p_mask, explicit T and grad_out g, the gradients
    are those PyTorch's autograd gives for g * sum_n CE_n / (p_n T)."""
    H, W, y, p = _case(seed=5, ignore_frac=0.4)
    eps, s, T, g = 0.1, 0.5, 7.0, 1.7
    r = O.fldce(H, W, y, p, logit_scale=s, label_smoothing=eps, total=T, grad_out=g)
    Ht = torch.tensor(H, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    yt = torch.from_numpy(y)
    ce = F.cross_entropy(s * (Ht @ Wt.T), yt, ignore_index=-100, label_smoothing=eps,
                         reduction="none")
    w = torch.where(yt != -100, 1.0 / (torch.from_numpy(p) * T), torch.zeros(len(y), dtype=torch.float64))
    L = (ce * w).sum()
    L.backward(torch.tensor(g, dtype=torch.float64))
    assert abs(r.loss - L.item()) <= 1e-12 * abs(L.item())
    assert np.allclose(r.loss_per_token, (ce * w).detach().numpy(), rtol=1e-12, atol=0)
    assert np.allclose(r.dH, Ht.grad.numpy(), rtol=1e-10, atol=1e-14)
    assert np.allclose(r.dW, Wt.grad.numpy(), rtol=1e-10, atol=1e-14)


def pin_finite_differences():
    """P-5: central differences of g * L in float64 match dH and dW."""
    N, D, V = 6, 4, 9
    H, W, y, p = _case(N, D, V, seed=6, ignore_frac=0.3, sigma=1.0)
    kw = dict(logit_scale=0.9, label_smoothing=0.2, total=3.0)
    g = 1.3
    r = O.fldce(H, W, y, p, grad_out=g, **kw)
    h = 1e-6
    rng = np.random.default_rng(0)
    for _ in range(8):
        i, j = rng.integers(0, N), rng.integers(0, D)
        Hp, Hm = H.copy(), H.copy()
        Hp[i, j] += h
        Hm[i, j] -= h
        fd = g * (O.fldce(Hp, W, y, p, **kw).loss - O.fldce(Hm, W, y, p, **kw).loss) / (2 * h)
        assert abs(fd - r.dH[i, j]) <= 1e-6 * max(1.0, abs(r.dH[i, j])), (fd, r.dH[i, j])
        a, b = rng.integers(0, V), rng.integers(0, D)
        Wp, Wm = W.copy(), W.copy()
        Wp[a, b] += h
        Wm[a, b] -= h
        fd = g * (O.fldce(H, Wp, y, p, **kw).loss - O.fldce(H, Wm, y, p, **kw).loss) / (2 * h)
        assert abs(fd - r.dW[a, b]) <= 1e-6 * max(1.0, abs(r.dW[a, b])), (fd, r.dW[a, b])


def pin_brute_force_loops():
    """P-6: logits, softmax and G by naive loops, then dH, dW by triple loops."""
    N, D, V = 5, 3, 7
    H, W, y, p = _case(N, D, V, seed=7, ignore_frac=0.3, sigma=1.0)
    y[0] = 3
    y[1] = -100
    s, eps, T, g = 1.1, 0.25, 2.0, 0.5
    r = O.fldce(H, W, y, p, logit_scale=s, label_smoothing=eps, total=T, grad_out=g)
    loss = 0.0
    G = [[0.0] * V for _ in range(N)]
    for n in range(N):
        z = [s * sum(H[n][d] * W[v][d] for d in range(D)) for v in range(V)]
        mx = max(z)
        den = sum(math.exp(zv - mx) for zv in z)
        logp = [zv - mx - math.log(den) for zv in z]
        if y[n] == -100:
            continue
        q = [eps / V + ((1 - eps) if v == y[n] else 0.0) for v in range(V)]
        ce = -sum(q[v] * logp[v] for v in range(V))
        loss += ce / (p[n] * T)
        assert abs(r.loss_per_token[n] - ce / (p[n] * T)) <= 1e-12 * abs(ce / (p[n] * T))
        assert abs(r.lse[n] - (mx + math.log(den))) <= 1e-12
        for v in range(V):
            G[n][v] = g * s * (math.exp(logp[v]) - q[v]) / (p[n] * T)
    assert abs(r.loss - loss) <= 1e-12 * abs(loss)
    for n in range(N):
        for d in range(D):
            want = sum(G[n][v] * W[v][d] for v in range(V))
            assert abs(r.dH[n, d] - want) <= 1e-12 * max(1.0, abs(want))
    for v in range(V):
        for d in range(D):
            want = sum(G[n][v] * H[n][d] for n in range(N))
            assert abs(r.dW[v, d] - want) <= 1e-12 * max(1.0, abs(want))
    want_am = [max(range(V), key=lambda v: (s * sum(H[n][d] * W[v][d] for d in range(D)), -v))
               for n in range(N)]
    assert list(r.argmax) == want_am


def pin_split_merge():
    """P-7: merging per-split (max, sum-exp) pairs gives the one-shot
    logsumexp for any cut of the vocabulary, and reproduces the printed
    split-softmax probabilities of the tensor-parallel tutorial."""
    rng = np.random.default_rng(8)
    z = 20.0 * rng.standard_normal((7, 50))
    want = np.array([math.log(sum(math.exp(v) for v in row)) for row in z])
    for splits in ([0, 50], [0, 1, 50], [0, 13, 26, 39, 50], list(range(0, 51, 5))):
        m, l = O.partial_lse(z, splits)
        assert np.allclose(O.merge_partial_lse(m, l), want, rtol=1e-13, atol=1e-12)
    with open(os.path.join(GOLDEN, "split_softmax_tp_tutorial.json")) as f:
        gd = json.load(f)
    wt = np.array(gd["words_table"], float)
    pr = np.array(gd["predicts"], float)
    Y = (pr / np.linalg.norm(pr, axis=1, keepdims=True)) @ (
        wt / np.linalg.norm(wt, axis=1, keepdims=True)).T
    m, l = O.partial_lse(Y, gd["shard_bounds"])
    lse = O.merge_partial_lse(m, l)
    prob = np.exp(Y - lse[:, None])
    tol = 0.5 * 10.0 ** (-gd["printed_decimals"]) + 1e-12
    assert np.allclose(prob[0, 0:2], gd["printed_row0_shard0"], rtol=0, atol=tol)
    assert np.allclose(prob[0, 2:4], gd["printed_row0_shard1"], rtol=0, atol=tol)


def pin_row_sum_invariant():
    """P-8: every G row sums to zero, so sum_v dW[v] = 0."""
    H, W, y, p = _case(seed=9)
    r = O.fldce(H, W, y, p, label_smoothing=0.3, logit_scale=2.0, total=5.0, grad_out=3.0)
    assert np.allclose(r.dW.sum(0), 0.0, atol=1e-12 * np.abs(r.dW).max())


def pin_identical_vocab_rows():
    """P-9: identical W rows make every logit of a token equal, so dH = 0,
    lse = z + log V and CE = log V."""
    N, D, V = 8, 6, 13
    H, W, y, p = _case(N, D, V, seed=10, ignore_frac=0.0)
    W[:] = W[0]
    r = O.fldce(H, W, y, p, label_smoothing=0.2, total=0.0)
    z0 = H @ W[0]
    assert np.allclose(r.dH, 0.0, atol=1e-14)
    assert np.allclose(r.lse, z0 + math.log(V), rtol=1e-13, atol=1e-13)
    assert np.allclose(r.loss_per_token * p * N, math.log(V), rtol=1e-12)


def pin_permutation_equivariance():
    """P-10: permuting vocabulary rows with the targets permutes dW and keeps
    the loss and dH; permuting tokens permutes dH and the per-token loss."""
    H, W, y, p = _case(seed=11)
    kw = dict(label_smoothing=0.1, logit_scale=0.7, total=6.0)
    r = O.fldce(H, W, y, p, **kw)
    V = W.shape[0]
    perm = np.random.default_rng(1).permutation(V)
    inv = np.argsort(perm)
    y2 = np.where(y == -100, -100, inv[np.clip(y, 0, V - 1)])
    r2 = O.fldce(H, W[perm], y2, p, **kw)
    assert abs(r.loss - r2.loss) <= 1e-13 * abs(r.loss)
    assert np.allclose(r.dH, r2.dH, rtol=1e-12, atol=1e-15)
    assert np.allclose(r.dW[perm], r2.dW, rtol=1e-12, atol=1e-15)
    tp = np.random.default_rng(2).permutation(H.shape[0])
    r3 = O.fldce(H[tp], W, y[tp], p[tp], **kw)
    assert np.allclose(r.dH[tp], r3.dH, rtol=1e-12, atol=1e-15)
    assert np.allclose(r.loss_per_token[tp], r3.loss_per_token, rtol=1e-13, atol=0)


def pin_sampled_variants():
    """The row-sampled helpers (used at full size) equal the full oracle on
    the rows they return."""
    H, W, y, p = _case(N=40, D=8, V=30, seed=12)
    kw = dict(logit_scale=0.9, label_smoothing=0.1, grad_out=1.5)
    r = O.fldce(H, W, y, p, total=0.0, **kw)
    rows = np.array([0, 3, 17, 39])
    rr = O.fldce_rows(H, W, y, p, rows, total=r.total, row_block=3, **kw)
    assert np.allclose(rr.dH, r.dH[rows], rtol=1e-13, atol=1e-16)
    assert np.allclose(rr.loss_per_token, r.loss_per_token[rows], rtol=1e-13, atol=0)
    assert np.array_equal(rr.argmax, r.argmax[rows])
    vr = np.array([0, 5, 29])
    dW, lse, lt = O.fldce_dw_rows(H, W, y, p, vr, total=r.total, row_block=7, **kw)
    assert np.allclose(dW, r.dW[vr], rtol=1e-12, atol=1e-16)
    assert np.allclose(lse, r.lse, rtol=1e-14)
    assert np.allclose(lt, r.loss_per_token, rtol=1e-13, atol=0)


def pin_bias_autograd_and_fd():
    """Bias: PyTorch float64 autograd of g * sum CE(s F.linear(H, W, b))/(p T)
    gives dH, dW and db; central differences in b agree."""
    H, W, y, p = _case(seed=13, ignore_frac=0.3)
    rng = np.random.default_rng(5)
    b = rng.standard_normal(W.shape[0])
    eps, s_, T, g = 0.15, 0.8, 9.0, 1.3
    r = O.fldce(H, W, y, p, logit_scale=s_, label_smoothing=eps, total=T, grad_out=g, bias=b)
    Ht = torch.tensor(H, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    bt = torch.tensor(b, requires_grad=True)
    yt = torch.from_numpy(y)
    ce = F.cross_entropy(s_ * F.linear(Ht, Wt, bt), yt, ignore_index=-100,
                         label_smoothing=eps, reduction="none")
    w = torch.where(yt != -100, 1.0 / (torch.from_numpy(p) * T), torch.zeros(len(y), dtype=torch.float64))
    L = (ce * w).sum()
    L.backward(torch.tensor(g, dtype=torch.float64))
    assert abs(r.loss - L.item()) <= 1e-12 * abs(L.item())
    assert np.allclose(r.dH, Ht.grad.numpy(), rtol=1e-10, atol=1e-14)
    assert np.allclose(r.dW, Wt.grad.numpy(), rtol=1e-10, atol=1e-14)
    assert np.allclose(r.db, bt.grad.numpy(), rtol=1e-10, atol=1e-14)
    h = 1e-6
    for v in (0, 7, W.shape[0] - 1):
        bp, bm = b.copy(), b.copy()
        bp[v] += h
        bm[v] -= h
        kw = dict(logit_scale=s_, label_smoothing=eps, total=T)
        fd = g * (O.fldce(H, W, y, p, bias=bp, **kw).loss - O.fldce(H, W, y, p, bias=bm, **kw).loss) / (2 * h)
        assert abs(fd - r.db[v]) <= 1e-6 * max(1.0, abs(r.db[v]))
    # zero bias changes nothing
    r0 = O.fldce(H, W, y, p, logit_scale=s_, label_smoothing=eps, total=T, grad_out=g,
                 bias=np.zeros(W.shape[0]))
    r1 = O.fldce(H, W, y, p, logit_scale=s_, label_smoothing=eps, total=T, grad_out=g)
    assert np.allclose(r0.dW, r1.dW, rtol=1e-14, atol=0) and abs(r0.loss - r1.loss) <= 1e-14 * abs(r1.loss)


PINS = [pin_bias_autograd_and_fd, pin_all_zero_logits, pin_label_smoothing_closed_form, pin_ignored_tokens,
        pin_plain_ce_matches_torch, pin_diffusion_weighting_autograd,
        pin_finite_differences, pin_brute_force_loops, pin_split_merge,
        pin_row_sum_invariant, pin_identical_vocab_rows, pin_permutation_equivariance,
        pin_sampled_variants]


@pytest.mark.parametrize("pin", PINS, ids=[f.__name__ for f in PINS])
def test_pin(pin):
    pin()


# ----------------------------------------------------------------- mutants

def _mut_ce_drops_smoothing(z, lse, y, eps):
    V = z.shape[1]
    return (1.0 - eps) * (lse - z[np.arange(z.shape[0]), np.clip(y, 0, V - 1)])


def _mut_ce_mean_not_sum(z, lse, y, eps):
    V = z.shape[1]
    z_y = z[np.arange(z.shape[0]), np.clip(y, 0, V - 1)]
    return (1.0 - eps) * (lse - z_y) + eps * (lse - z.sum(axis=1))


def _wrap_grad(fn):
    orig = O.grad_logits

    def g(z, lse, y, valid, coef, s, eps, go):
        return fn(orig, z, lse, y, valid, coef, s, eps, go)
    return g


MUTANTS = {
    "ce_drops_smoothing_term": ("smoothed_ce", lambda: _mut_ce_drops_smoothing),
    "ce_smoothing_sum_not_mean": ("smoothed_ce", lambda: _mut_ce_mean_not_sum),
    "grad_target_sign_flipped": ("grad_logits", lambda: _wrap_grad(
        lambda o, z, lse, y, valid, coef, s, eps, go:
        o(z, lse, y, valid, coef, s, eps, go) + 2 * (go * s * coef)[:, None] * (1 - eps) *
        (np.arange(z.shape[1])[None, :] == y[:, None]) * valid[:, None])),
    "grad_target_off_by_one": ("grad_logits", lambda: _wrap_grad(
        lambda o, z, lse, y, valid, coef, s, eps, go:
        o(z, lse, np.where(valid, (y + 1) % z.shape[1], y), valid, coef, s, eps, go))),
    "grad_missing_scale": ("grad_logits", lambda: _wrap_grad(
        lambda o, z, lse, y, valid, coef, s, eps, go: o(z, lse, y, valid, coef, 1.0, eps, go))),
    "grad_missing_grad_out": ("grad_logits", lambda: _wrap_grad(
        lambda o, z, lse, y, valid, coef, s, eps, go: o(z, lse, y, valid, coef, s, eps, 1.0))),
    "grad_drops_eps_over_V": ("grad_logits", lambda: _wrap_grad(
        lambda o, z, lse, y, valid, coef, s, eps, go:
        o(z, lse, y, valid, coef, s, eps, go) + (go * s * coef * eps / z.shape[1])[:, None]
        * valid[:, None])),
    "coef_times_p": ("token_coef", lambda: (
        lambda valid, p, T: np.where(valid, np.asarray(p, float) / T, 0.0))),
    "coef_ignores_total": ("token_coef", lambda: (
        lambda valid, p, T: np.where(valid, 1.0 / np.where(valid, np.asarray(p, float), 1.0), 0.0))),
    "lse_no_max_shift_merge": ("merge_partial_lse", lambda: (
        lambda m, l: np.log(l.sum(axis=1)) + m.max(axis=1))),
    "logits_scale_squared": ("logits", lambda: (
        lambda H, W, s, bias=None: s * s * (np.asarray(H, float) @ np.asarray(W, float).T
                                            + (0.0 if bias is None else bias)))),
    "logits_transposed_weight": ("logits", lambda: (
        lambda H, W, s, bias=None: s * (np.asarray(H, float) @ np.asarray(W, float)[::-1].T
                                        + (0.0 if bias is None else bias)))),
    "total_counts_ignored": ("resolve_total", lambda: (
        lambda total, valid: float(total) if total > 0 else float(valid.shape[0]))),
    "valid_ignores_range": ("valid_tokens", lambda: (
        lambda y, V, ii: (np.asarray(y) != ii, 0))),
    "dW_from_shifted_tokens": ("contract_gradients", lambda: (
        lambda G, H, W: (G @ W, G.T @ np.roll(H, 1, axis=0)))),
    "dH_from_reversed_vocab": ("contract_gradients", lambda: (
        lambda G, H, W: (G @ W[::-1], G.T @ H))),
    "bias_ignored_in_logits": ("logits", lambda: (
        lambda H, W, s, bias=None: s * (np.asarray(H, float) @ np.asarray(W, float).T))),
    "bias_outside_scale": ("logits", lambda: (
        lambda H, W, s, bias=None: s * (np.asarray(H, float) @ np.asarray(W, float).T)
        + (0.0 if bias is None else np.asarray(bias, float)[None, :]))),
    "db_mean_not_sum": ("bias_gradient", lambda: (lambda G: G.mean(axis=0))),
    "lse_off_by_log": ("logsumexp_rows", lambda: (
        lambda z: z.max(axis=1) + np.log(np.exp(z - z.max(axis=1)[:, None]).sum(axis=1) + 1.0))),
}


def _run_pins():
    failed = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, IndexError, ValueError, FloatingPointError):
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutants_are_caught(name, monkeypatch):
    attr, make = MUTANTS[name]
    monkeypatch.setattr(O, attr, make())
    failed = _run_pins()
    assert failed, f"mutant {name} passed every pin"
