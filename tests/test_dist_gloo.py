"""Multi-process host logic of the token-sharded path, on CPU with the gloo backend (2 ranks).

The path shards by tokens; its one exchange is the calibration statistics, combined as an
elementwise MAX / MIN over ranks (RPTQ article, text after Fig. 2: the per-channel range is taken
over the whole calibration set).  These tests check that the combined statistics equal the
statistics of the union of all ranks' tokens, that every rank then derives the same clusters,
and the max / sum helpers the benchmark uses for its slowest-rank timing.
"""
import json
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str) -> None:
    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        import oracle
        from post_activation_quantization_b200 import dist as pdist
        from post_activation_quantization_b200 import synthetic

        res = {"world": list(pdist.world())}
        C, T, seed, g, iters, bits = 256, 48, 11, 8, 10, 4
        m = synthetic.channel_model(C, seed, 0.02, 20.0)
        gamma, beta = synthetic.ln_params(C, seed)
        shards = [oracle._f32(synthetic.activations(T, m, seed + 7919 * r, dtype="bf16", calibration=True))
                  for r in range(world)]
        mx, mn = oracle.minmax_ln(shards[rank], gamma, beta, 1e-5)
        tmx, tmn = torch.from_numpy(mx.copy()), torch.from_numpy(mn.copy())
        pdist.allreduce_minmax(tmx, tmn)
        # statistics of the union of every rank's tokens, computed on this rank alone
        umx, umn = oracle.minmax_ln(np.concatenate(shards, axis=0), gamma, beta, 1e-5)
        res["union_max_equal"] = bool(np.array_equal(tmx.numpy(), umx))
        res["union_min_equal"] = bool(np.array_equal(tmn.numpy(), umn))
        res["own_differs"] = bool(not np.array_equal(mx, umx) or not np.array_equal(mn, umn))
        cal = oracle.calibrate(tmx.numpy(), tmn.numpy(), g, iters, bits)
        key = torch.tensor(np.concatenate([cal["R"].astype(np.int64), cal["zero"].astype(np.int64),
                                           cal["scale"].astype(np.float32).view(np.int32).astype(np.int64)]))
        keys = [torch.empty_like(key) for _ in range(world)]
        dist.all_gather(keys, key)
        res["same_clusters"] = all(bool(torch.equal(keys[0], k)) for k in keys)
        res["max"] = pdist.max_over_ranks(1.5 + rank)
        res["sum"] = pdist.sum_over_ranks(10.0 * (rank + 1))
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_two_rank_calibration_and_timing_helpers(tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, WORLD, port, str(tmp_path))) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a gloo rank did not finish")
        assert p.exitcode == 0
    for r in range(WORLD):
        with open(tmp_path / f"rank{r}.json") as f:
            res = json.load(f)
        assert res["world"] == [r, WORLD, r]
        assert res["union_max_equal"] and res["union_min_equal"]
        assert res["own_differs"]  # the exchange really changed something
        assert res["same_clusters"]
        assert res["max"] == 1.5 + WORLD - 1
        assert res["sum"] == 10.0 * WORLD * (WORLD + 1) / 2


def test_single_process_helpers_are_identity():
    import torch

    from post_activation_quantization_b200 import dist as pdist
    a, b = torch.tensor([1.0, -2.0]), torch.tensor([0.5, -3.0])
    pdist.allreduce_minmax(a, b)
    assert a.tolist() == [1.0, -2.0] and b.tolist() == [0.5, -3.0]
    assert pdist.max_over_ranks(3.25) == 3.25
    assert pdist.sum_over_ranks(7.0) == 7.0


def _rank_dies(rank: int, world: int, port: int, out_dir: str) -> None:
    """Rank 1 leaves before the calibration exchange; rank 0 must get an error, not hang."""
    import datetime
    import time

    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    from post_activation_quantization_b200 import dist as pdist
    if rank == 1:
        os._exit(0)  # the failing rank: gone between steps, nothing of it in flight
    mx, mn = torch.zeros(16), torch.zeros(16)
    t0 = time.time()
    try:
        pdist.allreduce_minmax(mx, mn)
        res = "returned"
    except Exception as e:  # the surviving rank learns of it from the collective
        res = f"raised {type(e).__name__}"
    with open(os.path.join(out_dir, "rank0.txt"), "w") as f:
        f.write(f"{res} {time.time() - t0:.1f}")
    os._exit(0)


def test_a_lost_rank_ends_the_exchange_with_an_error(tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_dies, args=(r, WORLD, port, str(tmp_path))) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank hung after its peer left")
    res = (tmp_path / "rank0.txt").read_text().split()
    assert res[0] == "raised", res
    assert float(res[-1]) < 60.0
