"""DiT-MoE sparse expert layer on one GPU: buffers plus the four C-ABI calls.

``MoELayer`` owns the device buffers of one configuration (allocated once with
torch, which is only the allocator and the stream provider here) and runs

    moe_route -> moe_dispatch -> moe_expert_gemm1 -> moe_expert_gemm2 -> moe_combine

on the current CUDA stream.  Nothing in this file computes any part of the
layer: it moves arguments to the library.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

from . import binding as B


def _dev(a, dtype, device):
    if a is None:
        return None
    t = torch.as_tensor(np.ascontiguousarray(a)) if isinstance(a, np.ndarray) else a
    return t.to(device=device, dtype=dtype).contiguous()


def global_balance_loss(layer, group=None):
    """The cross-rank exchange of a data-parallel layer: each rank's [counts, score sums]
    are summed by one all-reduce of 2E values, and every rank then computes the loss of
    the whole batch.  Every rank must route the same number of tokens (T_total = T x world
    size) and call this in the same order as the other collectives."""
    import torch.distributed as dist
    if layer.s.seq_len:
        raise ValueError("the cross-rank loss is the whole-batch loss; seq_len must be 0")
    stats = layer.balance_stats(getattr(layer, "_stats", None))
    layer._stats = stats
    world = 1
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(stats, op=dist.ReduceOp.SUM, group=group)
        world = dist.get_world_size(group)
    return layer.balance_loss_from_stats(stats, layer.cfg.T * world)


@dataclass
class LayerShape:
    T: int
    D: int
    H: int
    E: int
    K: int
    n_shared: int
    dtype: str = "bf16"
    routing: str = "topk"
    alpha: float = 0.01
    act: str = "tanh"
    gemm_impl: str = "auto"
    seq_len: int = 0          # tokens per image for the balance loss (0 = the whole call)
    fuse_combine: bool = True  # fold the combine into the shared experts' GEMM2 where supported
    gather_rows: bool = False  # GEMM1 gathers its routed rows from x itself (no x_perm)
    gemm_pairs: int = 0        # CTA pairs the tensor-core GEMMs may occupy at once (0 = as many as fit)


class MoELayer:
    """Weights and buffers of one layer configuration on one CUDA device."""

    def __init__(self, shape: LayerShape, params: dict, device="cuda:0"):
        self.s = shape
        self.device = torch.device(device)
        self.cfg = B.make_config(shape.T, shape.D, shape.H, shape.E, shape.K, shape.n_shared, shape.dtype,
                                 shape.routing, shape.alpha, shape.act, shape.gemm_impl, shape.seq_len,
                                 shape.gemm_pairs)
        self.act_dtype = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[shape.dtype]
        dt, dev = self.act_dtype, self.device
        self.wg = _dev(params["wg"], dt, dev)
        self.router_bias = _dev(params.get("router_bias"), torch.float32, dev)
        self.w1 = _dev(params["w1"], dt, dev)
        self.b1 = _dev(params.get("b1"), dt, dev)
        self.w2 = _dev(params["w2"], dt, dev)
        self.b2 = _dev(params.get("b2"), dt, dev)
        ns = shape.n_shared
        self.ws1 = _dev(params["ws1"], dt, dev) if ns else None
        self.bs1 = _dev(params.get("bs1"), dt, dev) if ns else None
        self.ws2 = _dev(params["ws2"], dt, dev) if ns else None
        self.bs2 = _dev(params.get("bs2"), dt, dev) if ns else None
        self._alloc(shape.T)

    def _alloc(self, T: int):
        s, dev, dt = self.s, self.device, self.act_dtype
        self.cfg.T = T
        kmax = s.E if s.routing == "race" else s.K
        self.kmax = kmax
        self.R = B.moe_max_rows(self.cfg)
        self.ws_bytes = B.moe_workspace_size(self.cfg)
        i32, f32 = torch.int32, torch.float32
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.topk_idx = torch.empty((T, kmax), dtype=i32, device=dev)
        self.topk_w = torch.empty((T, kmax), dtype=f32, device=dev)
        self.n_sel = torch.empty((T,), dtype=i32, device=dev)
        self.counts = torch.empty((s.E,), dtype=i32, device=dev)
        self.aux = torch.empty((1,), dtype=f32, device=dev)
        self.offsets = torch.empty((s.E + 1,), dtype=i32, device=dev)
        self.pos = torch.empty((T, kmax), dtype=i32, device=dev)
        self.row_token = torch.empty((self.R,), dtype=i32, device=dev)
        self.row_gate = torch.empty((self.R,), dtype=f32, device=dev)
        # GEMM1 reads the routed rows of x itself (cp.async gather warps) on the 16-bit CTA-pair path:
        # no x_perm
        self.gathered = bool(s.gather_rows and s.dtype in ("bf16", "f16") and s.gemm_impl == "auto")
        self.x_perm = None if self.gathered else torch.empty((self.R, s.D), dtype=dt, device=dev)
        self.h_perm = torch.empty((self.R, s.H), dtype=dt, device=dev)
        self.y_perm = torch.empty((self.R, s.D), dtype=dt, device=dev)
        ns = s.n_shared
        # the combine folds into the shared experts' GEMM2 for 16-bit types on the CTA-pair GEMM with n_s >= 1
        self.fused = bool(s.fuse_combine and ns > 0 and s.dtype in ("bf16", "f16") and s.gemm_impl == "auto")
        self.h_sh = torch.empty((T, ns * s.H), dtype=dt, device=dev) if ns else None
        self.y_sh = torch.empty((T, s.D), dtype=dt, device=dev) if ns and not self.fused else None
        self.out = torch.empty((T, s.D), dtype=dt, device=dev)
        B.moe_workspace_init(self.ws, self.ws_bytes, self.stream())

    def stream(self) -> int:
        return torch.cuda.current_stream(self.device).cuda_stream

    # ------------------------------------------------------------ the four calls
    def route(self, x: torch.Tensor, mod=None):
        B.moe_route(self.cfg, x, self.wg, self.router_bias, self.topk_idx, self.topk_w, self.n_sel, self.counts,
                    self.aux, self.ws, self.ws_bytes, self.stream(), mod=mod)

    def dispatch(self, x: torch.Tensor):
        B.moe_dispatch(self.cfg, x, self.topk_idx, self.topk_w, self.n_sel, self.offsets, self.pos,
                       self.row_token, self.row_gate, self.x_perm, self.ws, self.ws_bytes, self.stream())

    def gemm1(self, x: torch.Tensor):
        if self.gathered:
            B.moe_expert_gemm1_gather(self.cfg, self.offsets, self.row_token, x, self.w1, self.b1, self.ws1,
                                      self.bs1, self.h_perm, self.h_sh, self.ws, self.ws_bytes, self.stream())
            return
        B.moe_expert_gemm1(self.cfg, self.offsets, self.x_perm, x, self.w1, self.b1, self.ws1, self.bs1,
                           self.h_perm, self.h_sh, self.ws, self.ws_bytes, self.stream())

    def gemm2(self):
        B.moe_expert_gemm2(self.cfg, self.offsets, self.h_perm, self.h_sh, self.w2, self.b2, self.ws2, self.bs2,
                           self.row_gate, self.y_perm, self.y_sh, self.ws, self.ws_bytes, self.stream())

    def combine(self, res=None):
        B.moe_combine(self.cfg, self.y_perm, self.y_sh, self.pos, self.n_sel, self.out, self.stream(), res=res)

    def gemm2_combine(self, res=None):
        B.moe_expert_gemm2_combine(self.cfg, self.offsets, self.h_perm, self.h_sh, self.w2, self.b2, self.ws2,
                                   self.bs2, self.row_gate, self.pos, self.n_sel, self.y_perm, self.out, self.ws,
                                   self.ws_bytes, self.stream(), res=res)

    def forward(self, x: torch.Tensor, x_res: Optional[torch.Tensor] = None, alpha: Optional[torch.Tensor] = None,
                img_len: Optional[int] = None, gamma: Optional[torch.Tensor] = None,
                beta: Optional[torch.Tensor] = None, eps: float = 1e-5) -> torch.Tensor:
        """Whole layer on device-resident x [T,D]; returns the output buffer.

        adaLN-Zero around the layer (all per-image tensors [T/img_len, D], act dtype):
        ``gamma``/``beta`` make the router route on m = gamma * LayerNorm(x) + beta (written to
        ``self.x_mod``, which dispatch and the shared GEMM1 then read); ``alpha`` makes the output
        x_res + alpha * MoE(m), with x_res = x unless given.
        """
        assert x.shape == (self.cfg.T, self.s.D) and x.dtype == self.act_dtype and x.is_contiguous()
        per_image = (self.cfg.T // img_len, self.s.D) if img_len else None
        mod = None
        x_in = x
        if gamma is not None:
            for t in (gamma, beta):
                assert t.dtype == x.dtype and t.is_contiguous() and t.shape == per_image
            if getattr(self, "x_mod", None) is None or self.x_mod.shape != x.shape:
                self.x_mod = torch.empty_like(x)
            mod = B.make_adaln(gamma, beta, img_len, eps, self.x_mod)
            x_in = self.x_mod
        res = None
        if alpha is not None:
            x_res = x if x_res is None else x_res
            assert x_res.shape == x.shape and x_res.dtype == x.dtype and x_res.is_contiguous()
            assert alpha.dtype == x.dtype and alpha.is_contiguous() and alpha.shape == per_image
            res = B.make_residual(x_res, alpha, img_len)
        self.route(x, mod)
        self.dispatch(x_in)
        self.gemm1(x_in)
        if self.fused:
            self.gemm2_combine(res)
        else:
            self.gemm2()
            self.combine(res)
        return self.out

    def capture(self, x: torch.Tensor, **kwargs) -> "torch.cuda.CUDAGraph":
        """Record one forward on the fixed input buffer ``x`` into a CUDA graph.

        ``graph.replay()`` then reruns the whole layer with one launch from the host
        (whatever is in ``x`` at replay time).  Every counter the kernels keep in the
        workspace between launches is reset by the kernels themselves, so replays need
        no host work in between.
        """
        self.forward(x, **kwargs)                 # warm: lazy buffers, kernel attributes
        torch.cuda.synchronize(self.device)
        side = torch.cuda.Stream(self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                self.forward(x, **kwargs)
        torch.cuda.current_stream(self.device).wait_stream(side)
        return graph

    def expert_frequency(self, seq_len: int, seq_labels: Optional[torch.Tensor] = None,
                         n_labels: Optional[int] = None) -> torch.Tensor:
        """Counts [n_labels, E] of the last routing's selections per label: per patch position
        (t mod seq_len) without labels, else per image label (class or timestep)."""
        n = seq_len if seq_labels is None else int(n_labels)
        hist = torch.empty((n, self.s.E), dtype=torch.int32, device=self.device)
        B.moe_expert_frequency(self.cfg, self.topk_idx, self.n_sel, seq_len, seq_labels, n, hist, self.ws,
                               self.stream())
        return hist

    def balance_stats(self, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """[2E] fp64 statistics of the last routing: per-expert counts, then score sums."""
        if out is None:
            out = torch.empty((2 * self.s.E,), dtype=torch.float64, device=self.device)
        B.moe_balance_stats(self.cfg, self.counts, self.ws, self.ws_bytes, out, self.stream())
        return out

    def balance_loss_from_stats(self, stats: torch.Tensor, T_total: int) -> torch.Tensor:
        """Overwrite ``self.aux`` with the balance loss of a batch of T_total tokens whose
        statistics (summed over its parts) are ``stats``."""
        B.moe_balance_loss_from_stats(self.cfg, stats, T_total, self.aux, self.stream())
        return self.aux

    def global_balance_loss(self, group=None) -> torch.Tensor:
        """Balance loss over the batch of every rank of ``group``: one all-reduce of the 2E
        statistics (NCCL on GPUs), then the loss with T = the tokens of all ranks.
        Overwrites ``self.aux`` on every rank with the same value."""
        return global_balance_loss(self, group)

    def check(self):
        B.moe_check_status(self.ws, self.stream())

    # ------------------------------------------------------------ backward
    def backward(self, x: torch.Tensor, dout: torch.Tensor, aux_scale: float = 1.0) -> dict:
        """Gradients of J = <dout, MoE(x)> + aux_scale * L_balance after ``forward(x)``.

        Returns fp32 gradients of every weight and bias (dw1, db1, dw2, db2, dws1, dbs1, dws2,
        dbs2, dwg, dbias), the gates' gradient ``dgate`` [T, Kmax] and ``dx`` (act dtype).  The
        selection is the forward's (discrete, no gradient).  Needs the forward's x_perm (the
        default dispatch, not the gathered GEMM1)."""
        if self.x_perm is None:
            raise ValueError("the backward reads x_perm: run the forward without gather_rows")
        s, dev, T = self.s, self.device, self.cfg.T
        f32 = torch.float32
        E, D, H, ns = s.E, s.D, s.H, s.n_shared
        if getattr(self, "_ebws", None) is None:
            self._ebws_bytes = B.moe_expert_backward_workspace_size(self.cfg)
            self._ebws = torch.empty(self._ebws_bytes, dtype=torch.uint8, device=dev)
            self._rbws_bytes = B.moe_backward_workspace_size(self.cfg)
            self._rbws = torch.empty(self._rbws_bytes, dtype=torch.uint8, device=dev)
        e = lambda *shape: torch.empty(shape, dtype=f32, device=dev)
        g = {"dw1": e(E, H, D), "db1": e(E, H), "dw2": e(E, D, H), "db2": e(E, D),
             "dws1": e(ns, H, D) if ns else None, "dbs1": e(ns, H) if ns else None,
             "dws2": e(ns, D, H) if ns else None, "dbs2": e(ns, D) if ns else None,
             "dwg": e(E, D), "dbias": e(E), "dgate": e(T, self.kmax),
             "dx": torch.empty((T, D), dtype=self.act_dtype, device=dev)}
        wts = B.make_expert_weights(self.w1, self.b1, self.w2, self.b2, self.ws1, self.bs1, self.ws2, self.bs2)
        grads = B.make_expert_grads(g["dw1"], g["db1"], g["dw2"], g["db2"], g["dws1"], g["dbs1"], g["dws2"],
                                    g["dbs2"])
        B.moe_expert_backward(self.cfg, x, self.x_perm, self.offsets, self.pos, self.topk_idx, self.n_sel,
                              self.row_token, self.row_gate, wts, self.h_perm, self.h_sh, dout, grads, g["dgate"],
                              g["dx"], self.ws, self.ws_bytes, self._ebws, self._ebws_bytes, self.stream())
        B.moe_router_backward(self.cfg, x, self.wg, self.router_bias, self.counts, self.topk_idx, self.n_sel,
                              g["dgate"], aux_scale, g["dwg"], g["dbias"], g["dx"], 1, self._rbws, self._rbws_bytes,
                              self.stream())
        return g

    # ------------------------------------------------------------ serving from host memory
    def forward_host_pipelined(self, x_host, out_host, aux_host=None):
        """Run the layer over a sequence of host batches, overlapping transfers with compute.

        ``x_host`` / ``out_host`` are lists of pinned host tensors [T, D] (act dtype);
        ``aux_host`` an optional list of pinned fp32 [1] tensors for each batch's balance
        loss.  Batch i+1's host-to-device copy and batch i-1's device-to-host copy run on
        their own streams while batch i computes (two device input and output buffers).
        Returns when every copy back has finished.
        """
        n = len(x_host)
        dev = self.device
        own_out, own_aux = self.out, self.aux
        if not hasattr(self, "_pipe"):
            self._pipe = {
                "x": [torch.empty((self.cfg.T, self.s.D), dtype=self.act_dtype, device=dev) for _ in range(2)],
                "out": [torch.empty((self.cfg.T, self.s.D), dtype=self.act_dtype, device=dev) for _ in range(2)],
                "aux": [torch.empty((1,), dtype=torch.float32, device=dev) for _ in range(2)],
                "h2d": torch.cuda.Stream(dev), "d2h": torch.cuda.Stream(dev),
            }
        P = self._pipe
        comp = torch.cuda.current_stream(dev)
        loaded = [torch.cuda.Event() for _ in range(n)]
        computed = [torch.cuda.Event() for _ in range(n)]
        drained = [torch.cuda.Event() for _ in range(n)]
        consumed = [torch.cuda.Event() for _ in range(n)]

        def load(i):
            with torch.cuda.stream(P["h2d"]):
                if i >= 2:
                    P["h2d"].wait_event(consumed[i - 2])      # buffer i%2 free again
                P["x"][i % 2].copy_(x_host[i], non_blocking=True)
                loaded[i].record(P["h2d"])

        load(0)
        try:
            self._pipeline(n, P, comp, load, loaded, computed, drained, consumed, out_host, aux_host)
        finally:
            self.out, self.aux = own_out, own_aux
        drained[n - 1].synchronize()

    def _pipeline(self, n, P, comp, load, loaded, computed, drained, consumed, out_host, aux_host):
        for i in range(n):
            if i + 1 < n:
                load(i + 1)
            comp.wait_event(loaded[i])
            if i >= 2:
                comp.wait_event(drained[i - 2])               # output buffer i%2 copied out
            # the layer writes straight into this batch's output buffers
            self.out, self.aux = P["out"][i % 2], P["aux"][i % 2]
            self.forward(P["x"][i % 2])
            consumed[i].record(comp)
            computed[i].record(comp)
            with torch.cuda.stream(P["d2h"]):
                P["d2h"].wait_event(computed[i])
                out_host[i].copy_(P["out"][i % 2], non_blocking=True)
                if aux_host is not None:
                    aux_host[i].copy_(P["aux"][i % 2], non_blocking=True)
                drained[i].record(P["d2h"])
