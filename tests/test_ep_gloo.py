"""Expert parallelism over real process groups on the CPU: 2 and 4 gloo ranks
run expert_layer_dual_b200.ep.EPLayer.forward (the host logic of the
expert-parallel layer: per-rank split sizes, the count exchange, the two
all-to-all-v exchanges of rows and of expert outputs, where returned rows
land) with every step on the data computed by the oracle (ep_oracle_ops).
Each rank's output must equal the oracle's whole layer on that rank's tokens
exactly: the expert FFN of a row does not depend on where it runs, and every
sum is taken in the same order."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from expert_layer_dual_b200.configs import MoEConfig

CASES = {
    "bf16": MoEConfig("ep-bf16", T=96, d=256, E=8, k=2, I=128, Is=128, seed=61),
    "fp8": MoEConfig("ep-fp8", T=64, d=256, E=8, k=4, I=128, Is=0, wdtype=1, seed=62),
    "bias": MoEConfig("ep-bias", T=80, d=256, E=16, k=4, I=128, Is=128, zipf_bias=True, seed=63),
}


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _token_ranges(T: int, world: int):
    """Uneven token counts per rank (the last rank may get none)."""
    cuts = [0] + [min(T, (T * (2 * r + 1)) // (2 * world) + r * 3) for r in range(1, world)] + [T]
    return [(cuts[r], max(cuts[r], cuts[r + 1])) for r in range(world)]


def _rank_main(rank, world, port, name, out):
    import oracle
    from ep_oracle_ops import OracleOps
    from expert_layer_dual_b200.ep import EPLayer, TorchExchange
    from expert_layer_dual_b200.inputs import make_layer
    from gpu_util import bits, oracle_layer

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = CASES[name]
        inp = make_layer(cfg)
        lo, hi = _token_ranges(cfg.T, world)[rank]
        x = inp["x"][lo:hi].contiguous()
        layer = EPLayer(cfg, inp, rank, world, ops=OracleOps(cfg, inp, rank, world))
        y = layer.forward(x, TorchExchange()).numpy()
        ref = oracle.forward(oracle_layer(cfg, inp, T=hi - lo), bits(inp["x"][lo:hi]))["y"]
        out[rank] = (hi - lo, bool(np.array_equal(y, ref)), float(np.abs(y - ref).max(initial=0.0)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("name", sorted(CASES))
def test_ep_over_gloo_ranks_equals_the_oracle(name, world):
    import oracle
    oracle.build()                      # once, before the ranks start
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), name, out), nprocs=world,
                       start_method="spawn", join=True)
    res = dict(out)
    assert sorted(res) == list(range(world))
    assert sum(n for n, _, _ in res.values()) == CASES[name].T
    for r, (n, same, err) in res.items():
        assert same, f"rank {r} ({n} tokens): max |y - y_oracle| = {err:.3g}"


def test_split_counts_follow_the_expert_ranges():
    from expert_layer_dual_b200.ep import split_counts
    offsets = [0, 3, 3, 7, 10, 10, 12, 15, 20]      # 8 experts
    assert split_counts(offsets, 2, 8) == [10, 10]
    assert split_counts(offsets, 4, 8) == [3, 7, 2, 8]
    assert split_counts(offsets, 1, 8) == [20]
