"""The fused all-reduce + residual + RMSNorm kernel ("HPC-Ops ...",
HPC-Ops的技術原理, "Fused AllReduce+Norm") with G ranks emulated on one GPU in
one cooperative launch (moe_allreduce_rmsnorm_emulated runs the same kernel
and Lamport protocol the multi-GPU entry point runs, the peers' buffers being
local memory), against the oracle.

Bars: residual_out is one bf16 rounding of an FP32 sum of bf16 values (rtol
2^-8, plus 1e-6 of the row scale for the FP32 sum); out adds FP32 products
and rsqrt (a few ulp of FP32) before its bf16 rounding: rtol 2^-8 + 2e-6 of
the row's maximum.  Every rank computes the same bits."""
import numpy as np
import pytest
import torch

import oracle
from expert_layer_dual_b200.inputs import random_bf16
from gpu_util import bf16_to_f64, bits

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import expert_layer_dual_b200.moe as M

DEV = "cuda"


def _setup(G, T_max, d):
    nbytes = M.lamport_buffer_bytes(G, T_max, d)
    bufs = [torch.empty(nbytes, dtype=torch.uint8, device=DEV) for _ in range(G)]
    for b in bufs:
        M.lamport_init(b, nbytes)
    return bufs


def _run(bufs, call, T_max, xs, res, gamma, eps, ranks=None, timeout_us=2_000_000):
    G = len(bufs)
    n = G if ranks is None else ranks
    T, d = xs[0].shape
    outs = [torch.empty((T, d), dtype=torch.bfloat16, device=DEV) for _ in range(n)]
    routs = [torch.empty((T, d), dtype=torch.bfloat16, device=DEV) for _ in range(n)]
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    M.allreduce_rmsnorm_emulated(bufs, call, T_max, [x.view(torch.uint16) for x in xs],
                                 None if res is None else [res.view(torch.uint16)] * n,
                                 gamma.view(torch.uint16), eps, [o.view(torch.uint16) for o in outs],
                                 [o.view(torch.uint16) for o in routs], ws, ranks=n,
                                 timeout_us=timeout_us)
    return outs, routs, M.read_device_status(ws)


def _check(xs, res, gamma, eps, outs, routs):
    xb = np.stack([bits(x) for x in xs])
    ref_res, ref_out = oracle.allreduce_rmsnorm(xb, None if res is None else bits(res), bits(gamma), eps)
    scale = np.max(np.abs(ref_res), axis=1, keepdims=True)
    got_res = bf16_to_f64(routs[0])
    assert np.all(np.abs(got_res - ref_res) <= 2.0 ** -8 * np.abs(ref_res) + 1e-6 * scale)
    oscale = np.max(np.abs(ref_out), axis=1, keepdims=True)
    got = bf16_to_f64(outs[0])
    assert np.all(np.abs(got - ref_out) <= 2.0 ** -8 * np.abs(ref_out) + 2e-6 * oscale)
    for o, r in zip(outs[1:], routs[1:]):                  # every rank has the same bits
        assert torch.equal(o, outs[0]) and torch.equal(r, routs[0])


@pytest.mark.parametrize("G,T,d", [(1, 5, 256), (2, 64, 4096), (4, 37, 1024), (8, 64, 4096),
                                   (8, 300, 512), (3, 1, 8192)])
def test_allreduce_rmsnorm_emulated_against_oracle(G, T, d):
    xs = [random_bf16((T, d), seed=G * 100 + T, idx=r, std=0.5).to(DEV) for r in range(G)]
    res = random_bf16((T, d), seed=G * 100 + T, idx=40).to(DEV)
    gamma = random_bf16((d,), seed=d, idx=41, std=0.3).to(DEV)
    bufs = _setup(G, T, d)
    outs, routs, status = _run(bufs, 0, T, xs, res, gamma, 1e-6)
    assert status == M.OK
    _check(xs, res, gamma, 1e-6, outs, routs)


def test_allreduce_rmsnorm_cycles_its_buffers_and_leaves_them_empty():
    # seven calls in a row (every slot used at least twice), varying T below T_max,
    # no residual on some calls, inputs holding -0.0 (sent as +0.0: never mistaken
    # for "not arrived"); afterwards every buffer is back to the empty pattern
    G, T_max, d = 4, 48, 768
    bufs = _setup(G, T_max, d)
    gamma = random_bf16((d,), seed=5, idx=42, std=0.3).to(DEV)
    for call in range(7):
        T = [48, 17, 1, 48, 30, 5, 48][call]
        xs = [random_bf16((T, d), seed=call, idx=r).to(DEV) for r in range(G)]
        xs[1][0, :16] = -0.0
        res = None if call % 3 == 1 else random_bf16((T, d), seed=call, idx=43).to(DEV)
        outs, routs, status = _run(bufs, call, T_max, xs, res, gamma, 1e-5)
        assert status == M.OK
        _check(xs, res, gamma, 1e-5, outs, routs)
    torch.cuda.synchronize()
    for b in bufs:
        assert bool((b.view(torch.int16) == -32768).all())


def test_allreduce_rmsnorm_missing_rank_times_out():
    # rank 3 of 4 never sends: the others' bounded waits run out and report a
    # timeout; the context stays usable and re-initialised buffers work again
    G, T, d = 4, 8, 256
    bufs = _setup(G, T, d)
    xs = [random_bf16((T, d), seed=9, idx=r).to(DEV) for r in range(G)]
    gamma = random_bf16((d,), seed=9, idx=44).to(DEV)
    _, _, status = _run(bufs, 0, T, xs, None, gamma, 1e-6, ranks=3, timeout_us=2000)
    assert status == M.DEVICE_TIMEOUT
    bufs = _setup(G, T, d)
    outs, routs, status = _run(bufs, 0, T, xs, None, gamma, 1e-6)
    assert status == M.OK
    _check(xs, None, gamma, 1e-6, outs, routs)
