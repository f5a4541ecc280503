"""CPU checks of the C ABI: the shared library builds, loads and exports every
entry point include/moe.h declares; host-only calls (sizes, status strings,
argument validation) behave as documented.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared():
    src = open(HEADER, encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from expert_layer_dual_b200 import build
    build.build()
    return ctypes.CDLL(build.LIB)


def test_every_declared_entry_point_is_exported(lib):
    names = _declared()
    assert len(names) >= 16
    for n in names:
        assert hasattr(lib, n), f"{n} declared in moe.h but not exported"
    from expert_layer_dual_b200 import moe
    assert sorted(moe.EXPORTS) == names


def test_status_strings_and_sizes(lib):
    from expert_layer_dual_b200 import moe as M
    assert M.status_string(M.OK) == "ok"
    assert "workspace" in M.status_string(M.WORKSPACE_TOO_SMALL)
    s = M.moe_shape(64, 4096, 256, 8, 1536, 1536, 0, 1)
    n = M.workspace_bytes(s)
    R = 64 * 8 + 64
    assert n >= R * 4096 * 2 + R * 1536 * 2 and n % 256 == 0
    s8 = M.moe_shape(4096, 6144, 256, 8, 2048, 2048, 1, 1)
    assert M.workspace_bytes(s8) > 0
    assert M.workspace_bytes(M.moe_shape(64, 4000, 256, 8, 1536, 1536, 0, 1)) == 0   # d % 128
    assert M.workspace_bytes(M.moe_shape(64, 4096, 300, 8, 1536, 1536, 0, 1)) == 0   # E > 256
    assert M.workspace_bytes(M.moe_shape(64, 4096, 256, 9, 1536, 1536, 0, 1)) == 0   # k > 8
    assert M.workspace_bytes(M.moe_shape(64, 4096, 256, 8, 1536, 512, 0, 1)) == 0    # Is not in {0, I}
    assert M.permute_workspace_bytes(16384, 256, 8) >= 256 + 128 * 256 * 4


def test_validation_happens_before_any_launch(lib):
    from expert_layer_dual_b200 import moe as M
    s = M.moe_shape(16, 256, 8, 2, 128, 0, 0, 1)
    w = M.moe_weights()
    # null weights -> invalid argument, decided on the host
    assert lib.moe_forward(ctypes.byref(s), ctypes.byref(w), None, None, None, 0, None) == M.INVALID_ARG
    bad = M.moe_shape(16, 250, 8, 2, 128, 0, 0, 1)
    assert lib.moe_forward(ctypes.byref(bad), ctypes.byref(w), None, None, None, 0, None) == M.UNSUPPORTED
    zero = M.moe_shape(0, 256, 8, 2, 128, 0, 0, 1)
    w2 = M.moe_weights(*([ctypes.c_void_p(256)] * 10 + [None]))
    assert lib.moe_forward(ctypes.byref(zero), ctypes.byref(w2), None, None, None, 0, None) == M.OK
    assert lib.moe_route_topk(None, 4, 300, 2, 1, None, None, None) == M.UNSUPPORTED
    assert lib.moe_router_split(None, None, None, ctypes.c_int64(-1), None) == M.INVALID_ARG


def test_workspace_map_regions(lib):
    # moe_workspace_offsets is host-only: the regions are 256-byte aligned, inside the
    # workspace, and the quantised-activation regions exist exactly for the formats
    # that have them (xq for the FP8 formats; xs for block-scaled FP8 and MXFP8)
    from expert_layer_dual_b200 import moe as M
    for wd in (0, 1, 2, 3):
        s = M.moe_shape(200, 512, 16, 4, 256, 256, wd, 1)
        m = M.workspace_offsets(s)
        assert m.total == M.workspace_bytes(s)
        regs = {n: getattr(m, n) for n in ("logits", "ids", "w", "counts", "offsets", "perm", "inv",
                                           "xq", "xs", "h")}
        for n, off in regs.items():
            assert off % 256 == 0 and off < m.total, (wd, n)
        R = 200 * 4 + 200
        assert (regs["xq"] > 0) == (wd != 0)   # 200 x 4 rows over 16 experts: no pair gate-up
        assert (regs["xs"] > 0) == (wd in (1, 2))
        if wd:
            assert regs["xq"] + R * 512 <= m.total
    # BF16 with >= 256 rows per expert on average (the CTA-pair gate-up): xq holds x's
    # T*k routed rows in permuted order (the shared expert's rows are read from x), no xs
    T, d, E, k = 1100, 512, 8, 4
    s = M.moe_shape(T, d, E, k, 256, 256, 0, 1)
    m = M.workspace_offsets(s)
    regs = {n: getattr(m, n) for n in ("logits", "ids", "w", "counts", "offsets", "perm", "inv",
                                       "xq", "xs", "h")}
    assert regs["xq"] > 0 and regs["xs"] == 0
    nxt = min([off for off in regs.values() if off > regs["xq"]] + [m.total])
    assert nxt - regs["xq"] == T * k * d * 2


def test_misaligned_pointers_are_rejected_on_the_host(lib):
    # every case below is refused before any device work, so nothing is launched
    # (row buffers and weight matrices must start on a 16-byte boundary)
    from expert_layer_dual_b200 import moe as M
    V = ctypes.c_void_p
    s = M.moe_shape(16, 256, 8, 2, 128, 0, 0, 1)
    good = [V(256)] * 10 + [None]
    w = M.moe_weights(*good)
    nb = M.workspace_bytes(s)
    ws = V(1 << 20)
    for bad_x, bad_y in ((V(1024 + 2), V(2048)), (V(1024), V(2048 + 8))):
        assert lib.moe_forward(ctypes.byref(s), ctypes.byref(w), bad_x, bad_y, ws, nb, None) == M.INVALID_ARG
    for i in range(10):
        if i in (2, 3, 6, 7):   # scale arrays: no alignment rule
            continue
        fields = list(good)
        fields[i] = V(256 + 4)
        wb = M.moe_weights(*fields)
        assert lib.moe_forward(ctypes.byref(s), ctypes.byref(wb), V(1024), V(2048), ws, nb, None) == \
            M.INVALID_ARG, i
    assert lib.moe_combine(ctypes.byref(s), V(1024 + 2), V(4096), V(8192), V(2048), None) == M.INVALID_ARG
    assert lib.moe_combine(ctypes.byref(s), V(1024), V(4096), V(8192), V(2048 + 2), None) == M.INVALID_ARG
    assert lib.moe_router_logits(V(1024 + 2), V(256), V(512), None, V(2048), 16, 256, 8, None) == M.INVALID_ARG
    assert lib.moe_quantize_act_fp8(V(1024 + 2), ctypes.c_int64(16), 256, V(2048), V(4096), None) == \
        M.INVALID_ARG
    assert lib.moe_quantize_act_fp8(V(1024), ctypes.c_int64(16), 256, V(2048 + 1), V(4096), None) == \
        M.INVALID_ARG
    # the same calls with aligned pointers pass the host checks; without a GPU they
    # stop at the device check (only run where no GPU could launch anything)
    import torch
    if not torch.cuda.is_available():
        assert lib.moe_forward(ctypes.byref(s), ctypes.byref(w), V(1024), V(2048), ws, nb, None) == \
            M.UNSUPPORTED
        assert lib.moe_combine(ctypes.byref(s), V(1024), V(4096), V(8192), V(2048), None) == M.UNSUPPORTED
        assert lib.moe_quantize_act_fp8(V(1024), ctypes.c_int64(16), 256, V(2048), V(4096), None) == \
            M.UNSUPPORTED
