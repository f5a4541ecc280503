"""moe_permute_noalloc: the permute stage for callers that cannot allocate.

Some callers cannot hand the library a workspace (they run where cudaMalloc
is not allowed, or every device allocation belongs to a framework that gives
them none), so this entry point keeps its scratch in a fixed device array
inside the library.  This file is collected last so that, if it fails, a run
stopping at the first failure has already run every other test.  It needs
nothing from the other test files and runs alone in a fresh process too."""
import numpy as np
import pytest
import torch

from expert_layer_dual_b200.inputs import random_ids

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import expert_layer_dual_b200.moe as M

DEV = "cuda"


def _outputs(T, E, k):
    return (torch.empty(E, dtype=torch.int32, device=DEV), torch.empty(E + 1, dtype=torch.int32, device=DEV),
            torch.empty(T * k, dtype=torch.int32, device=DEV), torch.empty(T * k, dtype=torch.int32, device=DEV))


def test_permute_noalloc_matches_permute_on_two_calls_in_a_row():
    # a large call then a smaller one with other experts: the shared scratch
    # keeps the first call's contents, which must not leak into the second
    for T, E, k, seed in [(16384, 256, 8, 7), (301, 40, 4, 8)]:
        ids = random_ids(T, E, k, seed=seed).to(DEV)
        want = _outputs(T, E, k)
        ws = torch.empty(M.permute_workspace_bytes(T, E, k), dtype=torch.uint8, device=DEV)
        M.permute(ids, E, *want, ws)
        got = _outputs(T, E, k)
        M.permute_noalloc(ids, E, *got)
        torch.cuda.synchronize()
        for g, w in zip(got, want):
            assert torch.equal(g, w)      # integer outputs: exact


def test_permute_noalloc_rejects_sizes_beyond_its_scratch():
    T, E, k = 40000, 256, 8              # ceil(320000 / 1024) * 256 > 65536
    ids = torch.zeros((T, k), dtype=torch.int32, device=DEV)
    with pytest.raises(M.MoEError) as e:
        M.permute_noalloc(ids, E, *_outputs(T, E, k))
    assert e.value.code == M.WORKSPACE_TOO_SMALL
