"""Host logic of expert_layer_dual_b200.tp_norm.LamportAllReduceNorm over 2 and
3 gloo ranks on the CPU, with a stand-in for the library's peer-memory calls
(the real ones need GPUs): every rank's buffer handle reaches every other
rank, each rank maps exactly the others' buffers in rank order, the call
number advances identically on every rank, and close() unmaps before it
frees.  The kernel itself is tested on a GPU (test_gpu_allreduce_norm.py)."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class FakeLib:
    """Records the calls the layer makes; pointers are rank * 1000 + a counter."""

    def __init__(self, rank):
        self.rank, self.log = rank, []

    def lamport_buffer_bytes(self, G, T_max, d):
        return 3 * G * T_max * d * 2

    def peer_buffer_alloc(self, nbytes):
        self.log.append(("alloc", nbytes))
        return self.rank * 1000 + 1, bytes([self.rank]) * 64

    def lamport_init(self, ptr, nbytes):
        self.log.append(("init", ptr, nbytes))

    def peer_buffer_open(self, handle):
        self.log.append(("open", handle[0]))
        return handle[0] * 1000 + 500

    def allreduce_rmsnorm(self, bufs, rank, call, T_max, x, residual, gamma, eps, out, rout, ws,
                          stream=None):
        self.log.append(("ar", tuple(bufs), rank, call))

    def peer_buffer_close(self, ptr):
        self.log.append(("close", ptr))

    def peer_buffer_free(self, ptr):
        self.log.append(("free", ptr))

    def read_device_status(self, ws):
        return 0


def _rank_main(rank, world, port, out):
    from expert_layer_dual_b200.tp_norm import LamportAllReduceNorm
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lib = FakeLib(rank)
        layer = LamportAllReduceNorm(16, 256, device="cpu", lib=lib)
        x = torch.zeros((4, 256), dtype=torch.bfloat16)
        g = torch.ones(256, dtype=torch.bfloat16)
        for _ in range(3):
            layer(x, None, g, 1e-6)
        layer.close()
        out[rank] = lib.log
    finally:
        dist.destroy_process_group()


def test_lamport_setup_over_gloo_ranks():
    for world in (2, 3):
        out = mp.get_context("spawn").Manager().dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                           start_method="spawn", join=True)
        for rank in range(world):
            log = out[rank]
            own = rank * 1000 + 1
            bufs = tuple(own if r == rank else r * 1000 + 500 for r in range(world))
            assert log[0] == ("alloc", 3 * world * 16 * 256 * 2)
            assert log[1] == ("init", own, 3 * world * 16 * 256 * 2)
            assert [e for e in log if e[0] == "open"] == [("open", r) for r in range(world) if r != rank]
            assert [e for e in log if e[0] == "ar"] == [("ar", bufs, rank, c) for c in range(3)]
            closes = [i for i, e in enumerate(log) if e[0] == "close"]
            assert [log[i][1] for i in closes] == [b for r, b in enumerate(bufs) if r != rank]
            assert log[-1] == ("free", own) and all(i < len(log) - 1 for i in closes)
