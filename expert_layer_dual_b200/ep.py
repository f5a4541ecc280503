"""Expert parallelism of the MoE layer over G ranks, one process per GPU.

"HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫", section HPC-Ops的主要功能,
"GroupGEMM FP8": the grouped expert GEMM is meant for expert-parallel
deployment; "PR #54160 完整报告", section 实现拆解: the 256-expert layer runs on
8 GPUs.  Rank r holds the router (replicated), the shared expert (replicated)
and the routed experts r*E/G .. (r+1)*E/G - 1.  One forward over a rank's own
tokens x:

  1. route (moe_route): logits, fused top-k and the permutation, over all E
     experts.  The permuted rows are grouped by expert, hence by owning rank;
  2. dispatch: the per-rank row counts are exchanged, then the rows
     themselves (moe_ep_dispatch packs them, each with its expert's id local
     to its owner) by an all-to-all-v;
  3. experts: the received rows are grouped by local expert (moe_permute with
     k = 1) and run through the grouped gate-up and down GEMMs; the outputs
     are put back in arrival order (moe_gather_rows);
  4. return: an all-to-all-v with the split sizes of step 2 reversed brings
     every row's expert output back to the rank that sent it, where it lands
     in the rows of the permuted order moe_combine reads;
  5. the shared expert on the rank's own tokens, then moe_combine.

Every step on the data runs in the library's kernels; the host only moves
the per-rank counts (the split sizes an all-to-all-v needs) and issues the
collectives.  Transport is `torch.distributed.all_to_all_single` (NCCL over
NVLink between GPUs): the rows land in this GPU's own memory before any
kernel reads them, and no kernel reads another GPU's memory.

The per-rank steps are exposed as three phases (`dispatch`, `experts`,
`finish`) around the two exchanges, so that `emulate` can run G ranks in one
process on one GPU (the exchanges become tensor copies) and `forward` runs one
rank of a real process group.  The arithmetic of every row is the one
`moe_forward` applies to it, so the result equals moe_forward's bit for bit.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch

from .configs import MoEConfig


class TorchExchange:
    """All-to-all-v over a torch.distributed process group (NCCL for CUDA
    tensors, gloo for CPU tensors)."""

    def __init__(self, group=None):
        self.group = group

    def counts(self, send: Sequence[int], device) -> List[int]:
        inp = torch.tensor(list(send), dtype=torch.int64, device=device)
        out = torch.empty_like(inp)
        torch.distributed.all_to_all_single(out, inp, group=self.group)
        return [int(v) for v in out.cpu().tolist()]

    def rows(self, out: torch.Tensor, inp: torch.Tensor, out_splits: Sequence[int],
             in_splits: Sequence[int]) -> None:
        torch.distributed.all_to_all_single(out, inp, output_split_sizes=list(out_splits),
                                            input_split_sizes=list(in_splits), group=self.group)


@dataclass
class Dispatch:
    """One rank's state between its phases."""
    T: int
    routing: dict            # ids, w, offsets, perm, inv of its own tokens
    send_rows: torch.Tensor  # [T*k, d] in permuted order
    send_ids: torch.Tensor   # [T*k] expert ids local to their owners
    send_counts: List[int]   # rows per destination rank
    o: torch.Tensor          # [T*k + T, d] expert outputs: routed rows, then shared rows
    x: torch.Tensor


def split_counts(offsets: Sequence[int], world: int, E: int) -> List[int]:
    """Rows bound for each rank: the permuted rows of its expert range."""
    El = E // world
    return [int(offsets[(r + 1) * El]) - int(offsets[r * El]) for r in range(world)]


class LibraryOps:
    """The EP steps on the GPU, through the library's C ABI."""

    def __init__(self, cfg: MoEConfig, inputs: dict, rank: int, world: int, device,
                 act_scales=None):
        from . import moe as M
        self.M = M
        self.cfg = cfg
        self.dev = torch.device(device)
        self.E_local = cfg.E // world
        lo, hi = rank * self.E_local, (rank + 1) * self.E_local
        # the layer object prepares the router split and, for FP8 layers, the weight
        # quantisation; it holds this rank's experts only (the static activation scales
        # of a per-tensor FP8 layer are a property of the whole layer: calibrated on it
        # when not given)
        if cfg.wdtype == M.WDTYPE_FP8_TENSOR and act_scales is None:
            act_scales = M.MoELayer(cfg, inputs, device=self.dev).act_scales
        local = {**inputs, "w_gu": inputs["w_gu"][lo:hi], "w_d": inputs["w_d"][lo:hi]}
        self.full = M.MoELayer(cfg, local, device=self.dev, act_scales=act_scales)
        f = self.full
        P = M._p

        def part(name, sl):
            t = f.mats[name]
            return None if t is None else t[sl]

        def part_scale(name, sl):
            t = f.scales[name]
            return None if t is None else t[sl]

        sl = slice(0, self.E_local)
        self.local_mats = (part("w_gu", sl), part("w_d", sl), part_scale("w_gu", sl),
                           part_scale("w_d", sl))
        self.w_local = M.moe_weights(*[P(t) for t in self.local_mats], None, None, None, None,
                                     P(f.router_hi), P(f.router_lo), P(f.router_bias),
                                     *f.act_scales)
        if cfg.Is:
            self.w_shared = M.moe_weights(P(f.mats["ws_gu"]), P(f.mats["ws_d"]),
                                          P(f.scales["ws_gu"]), P(f.scales["ws_d"]),
                                          None, None, None, None, P(f.router_hi), P(f.router_lo),
                                          P(f.router_bias), *f.act_scales)
        self.ws_route: Optional[torch.Tensor] = None

    # -- phase 1
    def route(self, x: torch.Tensor) -> dict:
        M, cfg = self.M, self.cfg
        shape = M.shape_of(cfg, x.shape[0])
        need = M.workspace_bytes(shape)
        if self.ws_route is None or self.ws_route.numel() < need:
            self.ws_route = torch.empty(need, dtype=torch.uint8, device=self.dev)
        M.route(shape, self.full.weights, x.view(torch.uint16), self.ws_route)
        v = M.workspace_view(self.ws_route, shape)
        return {n: v[n] for n in ("ids", "w", "offsets", "perm", "inv")}

    def host_offsets(self, routing: dict) -> List[int]:
        return routing["offsets"].cpu().tolist()

    def dispatch(self, x: torch.Tensor, routing: dict):
        T, d, k = x.shape[0], self.cfg.d, self.cfg.k
        rows = torch.empty((T * k, d), dtype=torch.bfloat16, device=self.dev)
        ids = torch.empty(T * k, dtype=torch.int32, device=self.dev)
        self.M.ep_dispatch(x.view(torch.uint16), routing["ids"], routing["perm"], self.E_local,
                           rows.view(torch.uint16), ids)
        return rows, ids

    def empty_rows(self, n: int) -> torch.Tensor:
        return torch.empty((n, self.cfg.d), dtype=torch.bfloat16, device=self.dev)

    def empty_ids(self, n: int) -> torch.Tensor:
        return torch.empty(n, dtype=torch.int32, device=self.dev)

    def empty_out(self, n: int) -> torch.Tensor:
        return torch.empty((n, self.cfg.d), dtype=torch.float16, device=self.dev)

    # -- the grouped GEMMs of one group set: rows x (bf16 [T, d]) through perm / offsets
    def _ffn(self, shape, weights, x, perm, offsets, o):
        M, cfg = self.M, self.cfg
        R = shape.T * shape.k
        ws = torch.empty(4096, dtype=torch.uint8, device=self.dev)
        wd = cfg.wdtype
        a_in, a_scale = x.view(torch.uint16), None
        if wd == M.WDTYPE_FP8_BLOCK128:
            a_in = torch.empty((R, cfg.d), dtype=torch.uint8, device=self.dev)
            a_scale = torch.empty((R, cfg.d // 128), dtype=torch.float32, device=self.dev)
            M.quantize_act_fp8_permuted(x.view(torch.uint16), perm, shape.k, False, a_in, a_scale)
        elif wd == M.WDTYPE_MXFP8:
            a_in = torch.empty((R, cfg.d), dtype=torch.uint8, device=self.dev)
            a_scale = torch.empty(R * cfg.d // 32, dtype=torch.uint8, device=self.dev)
            M.quantize_act_mxfp8_permuted(x.view(torch.uint16), perm, shape.k, False, a_in, a_scale)
        elif wd == M.WDTYPE_FP8_TENSOR:
            a_in = torch.empty((R, cfg.d), dtype=torch.uint8, device=self.dev)
            M.quantize_act_fp8_static_permuted(x.view(torch.uint16), perm, shape.k, False,
                                               weights.act_scale_x, a_in)
        if wd == M.WDTYPE_BF16:
            h = torch.empty((R, shape.I), dtype=torch.uint16, device=self.dev)
            hs = None
        else:
            h = torch.empty((R, shape.I), dtype=torch.uint8, device=self.dev)
            hs = (None if wd == M.WDTYPE_FP8_TENSOR else
                  torch.empty((R, shape.I // 128), dtype=torch.float32, device=self.dev)
                  if wd == M.WDTYPE_FP8_BLOCK128 else
                  torch.empty(R * shape.I // 32, dtype=torch.uint8, device=self.dev))
        M.gemm_gateup(shape, weights, a_in, a_scale, perm, offsets, h, hs, ws)
        M.gemm_down(shape, weights, h, hs, offsets, o, ws)
        if M.read_device_status(ws) != M.OK:
            raise M.MoEError(M.read_device_status(ws), "expert-parallel grouped GEMMs")

    # -- phase 2: this rank's experts on the rows it received
    def experts(self, rows: torch.Tensor, ids: torch.Tensor) -> torch.Tensor:
        M, cfg = self.M, self.cfg
        R = rows.shape[0]
        out = self.empty_out(R)
        if R == 0:
            return out
        El = self.E_local
        counts = torch.empty(El, dtype=torch.int32, device=self.dev)
        offsets = torch.empty(El + 1, dtype=torch.int32, device=self.dev)
        perm = torch.empty(R, dtype=torch.int32, device=self.dev)
        inv = torch.empty(R, dtype=torch.int32, device=self.dev)
        pws = torch.empty(M.permute_workspace_bytes(R, El, 1), dtype=torch.uint8, device=self.dev)
        M.permute(ids.view(R, 1), El, counts, offsets, perm, inv, pws)
        shape = M.moe_shape(R, cfg.d, El, 1, cfg.I, 0, cfg.wdtype, int(cfg.renorm))
        o = self.empty_out(R)
        self._ffn(shape, self.w_local, rows, perm, offsets, o)
        M.gather_rows(o, inv, out)           # grouped order -> arrival order
        return out

    # -- phase 3: the shared expert on the rank's own tokens, then the combine
    def shared(self, x: torch.Tensor, o_shared: torch.Tensor) -> None:
        M, cfg = self.M, self.cfg
        T = x.shape[0]
        perm = torch.arange(T, dtype=torch.int32, device=self.dev)
        offsets = torch.tensor([0, T], dtype=torch.int32, device=self.dev)
        shape = M.moe_shape(T, cfg.d, 1, 1, cfg.Is, 0, cfg.wdtype, int(cfg.renorm))
        self._ffn(shape, self.w_shared, x, perm, offsets, o_shared)

    def combine(self, T: int, o: torch.Tensor, routing: dict) -> torch.Tensor:
        M = self.M
        y = torch.empty((T, self.cfg.d), dtype=torch.bfloat16, device=self.dev)
        M.combine(M.shape_of(self.cfg, T), o, routing["inv"], routing["w"], y.view(torch.uint16))
        return y


class EPLayer:
    """One rank of an expert-parallel MoE layer.  `ops` performs the steps on
    the data (default: the library's kernels on `device`)."""

    def __init__(self, cfg: MoEConfig, inputs: dict, rank: int, world: int, device="cuda",
                 ops=None):
        if cfg.E % world != 0:
            raise ValueError(f"E={cfg.E} experts do not split evenly over {world} ranks")
        self.cfg, self.rank, self.world = cfg, rank, world
        self.ops = ops if ops is not None else LibraryOps(cfg, inputs, rank, world, device)

    def dispatch(self, x: torch.Tensor) -> Dispatch:
        T, k = x.shape[0], self.cfg.k
        routing = self.ops.route(x)
        counts = split_counts(self.ops.host_offsets(routing), self.world, self.cfg.E)
        rows, ids = self.ops.dispatch(x, routing)
        o = self.ops.empty_out(T * k + (T if self.cfg.Is else 0))
        return Dispatch(T=T, routing=routing, send_rows=rows, send_ids=ids, send_counts=counts,
                        o=o, x=x)

    def experts(self, rows: torch.Tensor, ids: torch.Tensor) -> torch.Tensor:
        return self.ops.experts(rows, ids)

    def finish(self, st: Dispatch) -> torch.Tensor:
        """After the returned rows are in st.o[:T*k]: shared expert and combine."""
        T, k = st.T, self.cfg.k
        if self.cfg.Is:
            self.ops.shared(st.x, st.o[T * k:])
        return self.ops.combine(T, st.o, st.routing)

    def forward(self, x: torch.Tensor, exchange: Optional[TorchExchange] = None) -> torch.Tensor:
        """This rank's tokens through the layer; every rank of the group calls
        it with its own x (the collectives pair up in the same order)."""
        ex = exchange if exchange is not None else TorchExchange()
        st = self.dispatch(x)
        recv_counts = ex.counts(st.send_counts, st.send_rows.device)
        R = sum(recv_counts)
        rows = self.ops.empty_rows(R)
        ids = self.ops.empty_ids(R)
        ex.rows(rows, st.send_rows, recv_counts, st.send_counts)
        ex.rows(ids, st.send_ids, recv_counts, st.send_counts)
        out = self.experts(rows, ids)
        ex.rows(st.o[: st.T * self.cfg.k], out, st.send_counts, recv_counts)
        return self.finish(st)


def emulate(layers: Sequence[EPLayer], xs: Sequence[torch.Tensor]) -> List[torch.Tensor]:
    """G ranks in one process: the same phases as EPLayer.forward, the two
    all-to-all-v exchanges done as tensor copies between the ranks' buffers.
    Ranks run one after another, so nothing waits on another rank."""
    G = len(layers)
    sts = [layer.dispatch(x) for layer, x in zip(layers, xs)]
    starts = []
    for st in sts:
        acc, s = 0, []
        for c in st.send_counts:
            s.append(acc)
            acc += c
        starts.append(s)
    outs = []
    for r, layer in enumerate(layers):
        rows = torch.cat([sts[s].send_rows[starts[s][r]: starts[s][r] + sts[s].send_counts[r]]
                          for s in range(G)])
        ids = torch.cat([sts[s].send_ids[starts[s][r]: starts[s][r] + sts[s].send_counts[r]]
                         for s in range(G)])
        outs.append((layer.experts(rows, ids), [sts[s].send_counts[r] for s in range(G)]))
    for r in range(G):
        # rank r's rows come back from every owner, in owner order
        back = []
        for s in range(G):
            out_s, recv_s = outs[s]
            off = sum(recv_s[:r])
            back.append(out_s[off: off + sts[r].send_counts[s]])
        T, k = sts[r].T, layers[r].cfg.k
        sts[r].o[: T * k].copy_(torch.cat(back))
    return [layer.finish(st) for layer, st in zip(layers, sts)]
