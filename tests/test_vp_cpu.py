"""The vocabulary-parallel exchange (dp.fwd_bwd_vocab_parallel) on two gloo
ranks on the CPU.  Each rank holds every token and one vocabulary shard; the
per-shard steps are stood in for by float64 arithmetic built on the oracle's
functions (shard logits, per-split statistics, the split merge), so the test
checks the exchange: the gathered statistics merged in rank order, the loss
on every rank, the summed dH and each rank's dW / db rows, against the
oracle on the whole vocabulary."""
import math
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp



class OracleShardKernels:
    def __init__(self, v0, Vt, kw):
        self.v0, self.Vt, self.kw = v0, Vt, kw

    def vp_stats(self, H, W, target, p_mask, bias):
        import oracle.fldce_oracle as O
        s = self.kw["logit_scale"]
        z = O.logits(H.numpy(), W.numpy(), s, None if bias is None else bias.numpy())
        m, l = O.partial_lse(z, [0, z.shape[1]])
        y = target.numpy() - self.v0
        loc = (y >= 0) & (y < z.shape[1])
        zy = np.where(loc, z[np.arange(len(y)), np.clip(y, 0, z.shape[1] - 1)], 0.0)
        st = np.zeros((len(y), 8))
        st[:, 0], st[:, 1], st[:, 2], st[:, 3] = m[:, 0], l[:, 0], zy, z.sum(1)
        st[:, 4] = np.argmax(z, 1) + self.v0
        return torch.from_numpy(st)

    def vp_fwd_bwd(self, H, W, target, p_mask, total, grad_out, bias, all_stats, out):
        import oracle.fldce_oracle as O
        s, eps = self.kw["logit_scale"], self.kw["label_smoothing"]
        A = all_stats.numpy()
        lse = O.merge_partial_lse(A[:, :, 0].T, A[:, :, 1].T)
        zy, sz = A[:, :, 2].sum(0), A[:, :, 3].sum(0)
        y = target.numpy()
        valid, _ = O.valid_tokens(y, self.Vt, -100)
        T = O.resolve_total(total, valid)
        coef = O.token_coef(valid, p_mask.numpy(), T)
        ce = (1 - eps) * (lse - zy) + eps * (lse - sz / self.Vt)
        loss = np.where(valid, ce * coef, 0.0).sum()
        z = O.logits(H.numpy(), W.numpy(), s, None if bias is None else bias.numpy())
        G = np.exp(z - lse[:, None]) - eps / self.Vt
        yl = y - self.v0
        hit = valid & (yl >= 0) & (yl < z.shape[1])
        G[np.nonzero(hit)[0], yl[hit]] -= (1 - eps)
        G *= (grad_out * s * coef)[:, None]
        G[~valid] = 0.0
        res = {"loss": torch.tensor([loss]), "dH": torch.from_numpy(G @ W.numpy()),
               "dW": torch.from_numpy(G.T @ H.numpy())}
        if bias is not None:
            res["db"] = torch.from_numpy(G.sum(0))
        return res


def _case():
    rng = np.random.default_rng(3)
    N, D, V = 30, 8, 41
    H = rng.standard_normal((N, D))
    W = 0.8 * rng.standard_normal((V, D))
    b = rng.standard_normal(V)
    y = rng.integers(0, V, N)
    y[rng.random(N) < 0.4] = -100
    p = rng.uniform(0.05, 1, N)
    return H, W, b, y, p


def _worker(rank, port, outdir, cuts):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from linear_diffusion_cross_b200.dp import fwd_bwd_vocab_parallel
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=len(cuts) - 1)
    try:
        H, W, b, y, p = _case()
        a, e = cuts[rank], cuts[rank + 1]
        k = OracleShardKernels(a, W.shape[0], dict(logit_scale=0.9, label_smoothing=0.1))
        out = fwd_bwd_vocab_parallel(k, torch.from_numpy(H), torch.from_numpy(W[a:e]),
                                     torch.from_numpy(y), torch.from_numpy(p), total=0.0,
                                     grad_out=1.3, bias_shard=torch.from_numpy(b[a:e]))
        np.savez(os.path.join(outdir, f"r{rank}.npz"), loss=out["loss"].numpy(),
                 dH=out["dH"].numpy(), dW=out["dW"].numpy(), db=out["db"].numpy(), a=a, e=e)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts", [(0, 17, 41), (0, 5, 30, 41)])
def test_vocab_parallel_exchange_matches_whole_vocabulary(cuts):
    """Two shards (17 + 24 rows) and three uneven ones (5 + 25 + 11 rows):
    every rank's loss and dH equal the oracle's on the whole vocabulary, and
    its dW and db rows equal the oracle's rows of its shard."""
    import oracle.fldce_oracle as O
    world = len(cuts) - 1
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(port, d, cuts), nprocs=world, join=True,
                           start_method="spawn")
        H, W, b, y, p = _case()
        ref = O.fldce(H, W, y, p, total=0.0, logit_scale=0.9, label_smoothing=0.1,
                      grad_out=1.3, bias=b)
        for r in range(world):
            z = np.load(os.path.join(d, f"r{r}.npz"))
            a, e = int(z["a"]), int(z["e"])
            assert (a, e) == (cuts[r], cuts[r + 1])
            assert math.isclose(float(z["loss"][0]), ref.loss, rel_tol=1e-12)
            assert np.allclose(z["dH"], ref.dH, rtol=1e-11, atol=1e-15)
            assert np.allclose(z["dW"], ref.dW[a:e], rtol=1e-11, atol=1e-15)
            assert np.allclose(z["db"], ref.db[a:e], rtol=1e-11, atol=1e-15)
