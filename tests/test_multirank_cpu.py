"""The N > 1 path on the CPU: two gloo ranks, each with its own seeded shard of the batch.

Every (b, h) scan is independent, so the only cross-rank quantity is dW0, which sums over the
global batch (W0 is shared over b). Each rank computes its shard's dW0 with the float64 oracle,
the ranks all-reduce it through the same helper bench.py uses, and the result must equal the
oracle's dW0 over the concatenated global batch. The job time is the slowest rank's.
"""

import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

WORLD = 2
SHAPE = dict(B=2, H=2, T=70, d_in=12, d_out=8)
CFG_INDEX = 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shard(rank):
    from token_weight_scans_b200 import inputs, multirank
    return inputs.draw(SHAPE["B"], SHAPE["H"], SHAPE["T"], SHAPE["d_in"], SHAPE["d_out"],
                       dtype="f32", alpha_mode="log_uniform",
                       seed=multirank.rank_seed(CFG_INDEX, rank))


def _oracle_dW0(d):
    import oracle
    d64 = {k: np.asarray(v, dtype=np.float64) for k, v in d.items()}
    return oracle.bwd(d64["x"], d64["g"], d64["eta"], d64["alpha"], d64["W0"], d64["dy"],
                      nthreads=1)["dW0"]


def _worker(rank, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from token_weight_scans_b200 import multirank
        d = _shard(rank)
        dW0 = torch.from_numpy(_oracle_dW0(d))
        multirank.allreduce_dW0(dW0, dist)
        ms = multirank.max_over_ranks(1.5 + rank, dist)
        np.save(os.path.join(out_dir, f"dW0_{rank}.npy"), dW0.numpy())
        np.save(os.path.join(out_dir, f"ms_{rank}.npy"), np.array([ms]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def ran(tmp_path_factory):
    out = tmp_path_factory.mktemp("multirank")
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, str(out))) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0] * WORLD, codes
    return out


def test_shards_are_distinct_draws():
    a, b = _shard(0), _shard(1)
    assert not np.array_equal(a["x"], b["x"])
    assert not np.array_equal(a["dy"], b["dy"])
    # W0 is drawn per shard too; the global batch uses rank 0's (one persistent weight)
    assert a["W0"].shape == (SHAPE["H"], SHAPE["d_out"], SHAPE["d_in"])


def test_allreduced_dW0_equals_global_batch(ran):
    a, b = _shard(0), _shard(1)
    # dW0 = sum_{b,t} u_t x_t^T depends on dy and x only, so the global batch is the
    # concatenation of the shards along b
    glob = {k: np.concatenate([a[k], b[k]], axis=0) for k in ("x", "g", "eta", "alpha", "dy")}
    glob["W0"] = a["W0"]
    ref = _oracle_dW0(glob)
    for r in range(WORLD):
        got = np.load(os.path.join(ran, f"dW0_{r}.npy"))
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    # and it is not just one rank's share
    assert not np.allclose(_oracle_dW0(a), ref)


def test_job_time_is_the_slowest_rank(ran):
    from token_weight_scans_b200 import multirank
    for r in range(WORLD):
        assert float(np.load(os.path.join(ran, f"ms_{r}.npy"))[0]) == 1.5 + (WORLD - 1)
    assert multirank.weak_scaling_value(1000, WORLD, 4, 2.0) == pytest.approx(1000 * 2 * 4 / 2e-3)
    assert multirank.global_batch(8, WORLD) == 16
