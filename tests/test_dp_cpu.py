"""The data-parallel exchange (linear_diffusion_cross_b200.dp) on two gloo
ranks on the CPU.  Each rank holds half the tokens; the per-rank fused step
is stood in for by the float64 oracle on that rank's shard, so the test
checks the exchange itself: the job-wide normaliser, the sums of dW, db and
the loss, and that every rank's dH rows are final.  The composition must
equal the oracle on the whole batch."""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2


class OracleKernels:
    """Per-rank steps computed by the float64 oracle on CPU tensors."""

    def __init__(self, V, kw):
        self.V = V
        self.kw = kw

    def count_valid(self, target):
        import oracle.fldce_oracle as O
        valid, _ = O.valid_tokens(target.numpy(), self.V, self.kw["ignore_index"])
        return torch.tensor([int(valid.sum())], dtype=torch.int32)

    def fwd_bwd(self, H, W, target, p_mask, total, grad_out, count, bias, out):
        import oracle.fldce_oracle as O
        T = total if total > 0 else float(count.item())
        r = O.fldce(H.numpy(), W.numpy(), target.numpy(), p_mask.numpy(), total=T,
                    grad_out=grad_out, bias=None if bias is None else bias.numpy(), **self.kw)
        res = {"loss": torch.tensor([r.loss], dtype=torch.float64),
               "dH": torch.from_numpy(r.dH), "dW": torch.from_numpy(r.dW)}
        if bias is not None:
            res["db"] = torch.from_numpy(r.db)
        return res

    def reduce_weight_grads(self, tensors, group):
        for t in tensors:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)


def _case(seed=0, N=40, D=8, V=30):
    rng = np.random.default_rng(seed)
    H = rng.standard_normal((N, D))
    W = 0.7 * rng.standard_normal((V, D))
    y = rng.integers(0, V, N)
    y[rng.random(N) < 0.4] = -100
    p = rng.uniform(0.05, 1.0, N)
    b = rng.standard_normal(V)
    return H, W, y, p, b


def _worker(rank, port, outdir, total, use_bias):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from linear_diffusion_cross_b200.dp import fwd_bwd_data_parallel
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=WORLD)
    try:
        H, W, y, p, b = _case()
        N = H.shape[0]
        sl = slice(rank * N // WORLD, (rank + 1) * N // WORLD)
        kw = dict(logit_scale=0.9, label_smoothing=0.1, ignore_index=-100)
        k = OracleKernels(W.shape[0], kw)
        out = fwd_bwd_data_parallel(
            k, torch.from_numpy(H[sl]), torch.from_numpy(W), torch.from_numpy(y[sl]),
            torch.from_numpy(p[sl]), total=total, grad_out=1.5,
            bias=torch.from_numpy(b) if use_bias else None)
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), loss=out["loss"].numpy(),
                 dW=out["dW"].numpy(), dH=out["dH"].numpy(),
                 db=out["db"].numpy() if use_bias else np.zeros(1))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("total,use_bias", [(0.0, True), (0.0, False), (11.0, True)])
def test_data_parallel_exchange_matches_whole_batch(total, use_bias):
    import oracle.fldce_oracle as O
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(_free_port(), d, total, use_bias), nprocs=WORLD,
                           join=True, start_method="spawn")
        H, W, y, p, b = _case()
        ref = O.fldce(H, W, y, p, total=total, grad_out=1.5, logit_scale=0.9,
                      label_smoothing=0.1, bias=b if use_bias else None)
        N = H.shape[0]
        for rank in range(WORLD):
            r = np.load(os.path.join(d, f"rank{rank}.npz"))
            assert abs(float(r["loss"][0]) - ref.loss) <= 1e-12 * abs(ref.loss)
            assert np.allclose(r["dW"], ref.dW, rtol=1e-11, atol=1e-15)
            sl = slice(rank * N // WORLD, (rank + 1) * N // WORLD)
            assert np.allclose(r["dH"], ref.dH[sl], rtol=1e-11, atol=1e-15)
            if use_bias:
                assert np.allclose(r["db"], ref.db, rtol=1e-11, atol=1e-15)


def test_accumulating_plan_is_refused():
    """Summing an accumulated dW over ranks every step would add the earlier
    steps once per rank: the data-parallel step refuses such a plan before
    any collective."""
    from types import SimpleNamespace

    from linear_diffusion_cross_b200.dp import fwd_bwd_data_parallel
    kernels = SimpleNamespace(plan=SimpleNamespace(dw_accumulate=True))
    with pytest.raises(ValueError):
        fwd_bwd_data_parallel(kernels, None, None, None, None, total=1.0)


# ------------------------------------------------------------ a rank that leaves
PG_TIMEOUT_S = 5


def _leaver_worker(rank, port, outdir, total):
    """Both ranks run one data-parallel step; then rank 1 leaves (exits
    between steps, with no collective in flight) and rank 0 starts a second
    step.  Rank 0 records whether that step raised, and how long it took."""
    import datetime
    import sys
    import time
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from linear_diffusion_cross_b200.dp import fwd_bwd_data_parallel
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=WORLD, timeout=datetime.timedelta(seconds=PG_TIMEOUT_S))
    H, W, y, p, _ = _case()
    N = H.shape[0]
    sl = slice(rank * N // WORLD, (rank + 1) * N // WORLD)
    k = OracleKernels(W.shape[0], dict(logit_scale=1.0, label_smoothing=0.0, ignore_index=-100))
    args = (k, torch.from_numpy(H[sl]), torch.from_numpy(W), torch.from_numpy(y[sl]),
            torch.from_numpy(p[sl]))
    fwd_bwd_data_parallel(*args, total=total)
    dist.barrier()                       # step 1 is complete on both ranks
    if rank == 1:
        os._exit(0)                      # leaves without tearing down the group
    time.sleep(0.5)                      # the peer is gone before step 2 starts
    t0 = time.monotonic()
    try:
        fwd_bwd_data_parallel(*args, total=total)
        outcome = "completed"
    except Exception as e:              # gloo reports the lost peer or the timeout
        outcome = type(e).__name__ + ": " + str(e).splitlines()[0][:200]
    dt = time.monotonic() - t0
    with open(os.path.join(outdir, "rank0.txt"), "w") as f:
        f.write(f"{dt}\n{outcome}\n")
    os._exit(0)                          # the group is broken: skip its teardown


@pytest.mark.parametrize("total", [0.0, 11.0])
def test_rank_leaving_between_steps_fails_the_next_step(total):
    """The host-side form of failure detection in the data-parallel step: when
    a rank leaves between steps, the surviving rank's next collective ends
    with an error within the process group's timeout instead of hanging.
    (total <= 0 fails on the count's all-reduce before any kernel; an explicit
    total fails after the local step, on the dW reduction.)"""
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_leaver_worker, args=(_free_port(), d, total), nprocs=WORLD,
                           join=True, start_method="spawn")
        with open(os.path.join(d, "rank0.txt")) as f:
            dt, outcome = f.read().splitlines()[:2]
    assert outcome != "completed", "the step completed without its peer"
    assert float(dt) < 6 * PG_TIMEOUT_S, f"took {dt} s to fail: {outcome}"


# ------------------------------------------------------------ uneven shards, three ranks
UNEVEN_CUTS = (0, 7, 7 + 21, 40)     # rank 0: 7 tokens, rank 1: 21, rank 2: 12


def _uneven_worker(rank, port, outdir, total, world):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from linear_diffusion_cross_b200.dp import fwd_bwd_data_parallel
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        H, W, y, p, b = _case(seed=3)
        y = y.copy()
        y[UNEVEN_CUTS[0]:UNEVEN_CUTS[1]] = -100        # rank 0 holds no valid token
        sl = slice(UNEVEN_CUTS[rank], UNEVEN_CUTS[rank + 1])
        kw = dict(logit_scale=1.3, label_smoothing=0.05, ignore_index=-100)
        k = OracleKernels(W.shape[0], kw)
        out = fwd_bwd_data_parallel(
            k, torch.from_numpy(H[sl]), torch.from_numpy(W), torch.from_numpy(y[sl]),
            torch.from_numpy(p[sl]), total=total, grad_out=0.75, bias=torch.from_numpy(b))
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), loss=out["loss"].numpy(),
                 dW=out["dW"].numpy(), dH=out["dH"].numpy(), db=out["db"].numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("total", [0.0, 40.0])
def test_three_uneven_ranks_match_whole_batch(total):
    """Three ranks with 7, 21 and 12 tokens (the first holding no token that
    carries a loss): the job-wide count, the summed dW, db and loss and each
    rank's dH rows equal the oracle on the whole batch."""
    import oracle.fldce_oracle as O
    world = len(UNEVEN_CUTS) - 1
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_uneven_worker, args=(_free_port(), d, total, world), nprocs=world,
                           join=True, start_method="spawn")
        H, W, y, p, b = _case(seed=3)
        y = y.copy()
        y[UNEVEN_CUTS[0]:UNEVEN_CUTS[1]] = -100
        ref = O.fldce(H, W, y, p, total=total, grad_out=0.75, logit_scale=1.3,
                      label_smoothing=0.05, bias=b)
        for rank in range(world):
            r = np.load(os.path.join(d, f"rank{rank}.npz"))
            assert abs(float(r["loss"][0]) - ref.loss) <= 1e-12 * abs(ref.loss)
            assert np.allclose(r["dW"], ref.dW, rtol=1e-11, atol=1e-15)
            assert np.allclose(r["db"], ref.db, rtol=1e-11, atol=1e-15)
            sl = slice(UNEVEN_CUTS[rank], UNEVEN_CUTS[rank + 1])
            assert np.allclose(r["dH"], ref.dH[sl], rtol=1e-11, atol=1e-15)
        assert np.all(np.load(os.path.join(d, "rank0.npz"))["dH"] == 0.0)
