"""The steps of expert_layer_dual_b200.ep.EPLayer computed by the oracle on
host tensors, so that the expert-parallel host logic (split sizes, the two
all-to-all-v exchanges, where returned rows land) runs over real gloo ranks
on the CPU.  TEST INFRASTRUCTURE: the product path runs the same steps in the
library's kernels (ep.LibraryOps).

Rows travel as bf16 tensors, expert outputs as float64 (the oracle's
precision), ids as int32."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from gpu_util import bits


class OracleOps:
    def __init__(self, cfg, inputs: dict, rank: int, world: int):
        self.cfg = cfg
        self.El = cfg.E // world
        lo, hi = rank * self.El, (rank + 1) * self.El
        self.w_gu = bits(inputs["w_gu"])
        self.w_d = bits(inputs["w_d"])
        self.local_gu = self.w_gu[lo:hi]
        self.local_d = self.w_d[lo:hi]
        self.ws_gu = None if inputs.get("ws_gu") is None else bits(inputs["ws_gu"])
        self.ws_d = None if inputs.get("ws_d") is None else bits(inputs["ws_d"])
        self.router_w = inputs["router_w"].numpy()
        self.bias = None if inputs.get("router_bias") is None else inputs["router_bias"].numpy()
        self.hi, self.lo = oracle.router_split(self.router_w)

    def _layer(self, T, E, k, I, Is, w_gu, w_d, ws_gu=None, ws_d=None):
        return oracle.Layer(T=T, d=self.cfg.d, E=E, k=k, I=I, Is=Is, w_gu=w_gu, w_d=w_d,
                            ws_gu=ws_gu, ws_d=ws_d, router_w=np.zeros((E, self.cfg.d), np.float32),
                            wdtype=self.cfg.wdtype, renorm=self.cfg.renorm)

    def route(self, x: torch.Tensor) -> dict:
        xb = bits(x)
        lg = oracle.router_logits(xb, self.hi, self.lo, self.bias)
        ids, w = oracle.route_topk(lg.astype(np.float32), self.cfg.k, self.cfg.renorm)
        _, offsets, perm, inv = oracle.permute(ids, self.cfg.E)
        return {"ids": ids, "w": w, "offsets": offsets, "perm": perm, "inv": inv}

    def host_offsets(self, routing):
        return routing["offsets"].tolist()

    def dispatch(self, x: torch.Tensor, routing):
        perm = routing["perm"]
        rows = x[torch.from_numpy(perm // self.cfg.k).long()].contiguous()
        ids = torch.from_numpy((routing["ids"].reshape(-1)[perm] % self.El).astype(np.int32))
        return rows, ids

    def empty_rows(self, n):
        return torch.empty((n, self.cfg.d), dtype=torch.bfloat16)

    def empty_ids(self, n):
        return torch.empty(n, dtype=torch.int32)

    def empty_out(self, n):
        return torch.empty((n, self.cfg.d), dtype=torch.float64)

    def experts(self, rows: torch.Tensor, ids: torch.Tensor) -> torch.Tensor:
        R = rows.shape[0]
        if R == 0:
            return self.empty_out(0)
        _, offsets, perm, inv = oracle.permute(ids.numpy().reshape(R, 1), self.El)
        L = self._layer(R, self.El, 1, self.cfg.I, 0, self.local_gu, self.local_d)
        h = oracle.gateup(L, bits(rows), perm, offsets)
        o = oracle.down(L, h, offsets, R)
        return torch.from_numpy(np.ascontiguousarray(o[inv]))   # grouped -> arrival order

    def shared(self, x: torch.Tensor, o_shared: torch.Tensor) -> None:
        T = x.shape[0]
        L = self._layer(T, 1, 1, self.cfg.Is, 0, self.ws_gu[None], self.ws_d[None])
        h = oracle.gateup(L, bits(x), np.arange(T, dtype=np.int32), np.array([0, T], np.int32))
        o_shared.copy_(torch.from_numpy(oracle.down(L, h, np.array([0, T], np.int32), T)))

    def combine(self, T, o: torch.Tensor, routing) -> torch.Tensor:
        c = self.cfg
        L = oracle.Layer(T=T, d=c.d, E=c.E, k=c.k, I=c.I, Is=c.Is, w_gu=self.w_gu, w_d=self.w_d,
                         ws_gu=self.ws_gu, ws_d=self.ws_d, router_w=self.router_w,
                         wdtype=c.wdtype, renorm=c.renorm)
        return torch.from_numpy(oracle.combine(L, o.numpy(), routing["inv"], routing["w"], T))
