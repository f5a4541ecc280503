"""Expert parallelism on one GPU: G ranks emulated in one process
(expert_layer_dual_b200.ep.emulate runs every rank's phases through the
library's kernels, the two all-to-all-v exchanges as tensor copies).  Each
rank's output must equal moe_forward on that rank's tokens bit for bit: the
rows reach the same grouped GEMMs (on that rank's experts only), the shared
expert runs on the rank's own tokens, and the combine is the same.  The real
exchange (NCCL) needs several GPUs; its host logic is covered by
test_ep_gloo.py on CPU ranks."""
import pytest
import torch

from expert_layer_dual_b200.configs import MoEConfig
from expert_layer_dual_b200.inputs import make_layer

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import expert_layer_dual_b200.moe as M
    from expert_layer_dual_b200.ep import EPLayer, emulate

DEV = "cuda"

CASES = [
    MoEConfig("ep-bf16", T=300, d=512, E=16, k=4, I=256, Is=256, seed=71),
    # >= 256 rows per expert at the owners: the 256-row gate-up and CTA-pair down
    MoEConfig("ep-many", T=900, d=384, E=8, k=4, I=256, Is=256, seed=72),
    MoEConfig("ep-fp8", T=200, d=512, E=16, k=4, I=256, Is=0, wdtype=1, seed=73),
    MoEConfig("ep-mx", T=200, d=512, E=16, k=4, I=256, Is=256, wdtype=2, seed=74),
    MoEConfig("ep-f8t", T=200, d=512, E=16, k=4, I=256, Is=256, wdtype=3, seed=75),
    MoEConfig("ep-bias", T=256, d=256, E=64, k=8, I=128, Is=128, zipf_bias=True, seed=76),
]


def _chunks(T, G):
    """Uneven token counts per rank, one rank possibly empty."""
    cuts = [0] + [min(T, T * r // G + 7 * r) for r in range(1, G)] + [T]
    return [(cuts[r], max(cuts[r], cuts[r + 1])) for r in range(G)]


@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_ep_emulated_ranks_equal_moe_forward(cfg, G):
    inp = make_layer(cfg)
    full = M.MoELayer(cfg, inp)
    layers = [EPLayer(cfg, inp, r, G, device=DEV) for r in range(G)]
    for layer in layers:   # the per-tensor FP8 layer's static scales belong to the whole layer
        assert layer.ops.full.act_scales == full.act_scales
    xs = [inp["x"][lo:hi].contiguous().to(DEV) for lo, hi in _chunks(cfg.T, G)]
    ys = emulate(layers, xs)
    for r, (x, y) in enumerate(zip(xs, ys)):
        if x.shape[0] == 0:
            assert y.shape[0] == 0
            continue
        ref = full.forward(x)
        assert full.device_status() == M.OK
        assert torch.equal(y, ref), f"rank {r}: {int((y != ref).sum())} elements differ"


def test_ep_dispatch_and_gather_rows():
    # the dispatch packs rows in permuted order with owner-local expert ids; the
    # gather puts rows back by index
    cfg = CASES[0]
    inp = make_layer(cfg)
    full = M.MoELayer(cfg, inp)
    x = inp["x"].to(DEV)
    shape = full.shape(cfg.T)
    ws = torch.empty(M.workspace_bytes(shape), dtype=torch.uint8, device=DEV)
    M.route(shape, full.weights, x.view(torch.uint16), ws)
    v = M.workspace_view(ws, shape)
    El = 4
    rows = torch.empty((cfg.T * cfg.k, cfg.d), dtype=torch.bfloat16, device=DEV)
    ids = torch.empty(cfg.T * cfg.k, dtype=torch.int32, device=DEV)
    M.ep_dispatch(x.view(torch.uint16), v["ids"], v["perm"], El, rows.view(torch.uint16), ids)
    perm = v["perm"].long()
    assert torch.equal(rows, x[perm // cfg.k])
    assert torch.equal(ids.long(), v["ids"].view(-1)[perm].long() % El)
    idx = torch.randperm(rows.shape[0], device=DEV).to(torch.int32)
    out = torch.empty_like(rows)
    M.gather_rows(rows, idx, out)
    assert torch.equal(out, rows[idx.long()])
