"""Run the layer a few times on one workload, for profilers (ncu) to capture.

    python -m sparse_moe_layer_03_b200.profile_layer --workload xl2_8e2a_512 [--tokens T] [--iters N]

No timing and no checking: the seeded inputs of the workload (optionally cut
to T tokens) go through N forward passes on cuda:0 (with ``--backward``, each
followed by the layer's backward for a seeded dY: moe_expert_backward then
moe_router_backward).  Each pass launches the
layer's kernels in order: route (its last CTA finalizes counts and loss;
Expert-Race adds one select kernel), dispatch count, dispatch gather, GEMM1,
and GEMM2 with the combine folded in (16-bit types with shared experts; else
GEMM2 and a combine kernel).
"""
from __future__ import annotations

import argparse

import torch

from . import inputs as I
from .layer import LayerShape, MoELayer


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="xl2_8e2a_512", choices=sorted(I.WORKLOADS))
    ap.add_argument("--tokens", type=int, default=0, help="cut the workload to this many tokens")
    ap.add_argument("--iters", type=int, default=2)
    ap.add_argument("--backward", action="store_true", help="run the layer's backward after each forward")
    a = ap.parse_args(argv)
    w = I.WORKLOADS[a.workload]
    if a.tokens:
        w = w.with_tokens(a.tokens)
    inp = I.make_inputs(w)
    shape = LayerShape(w.T, w.D, w.H, w.E, w.K, w.n_shared, w.dtype, w.routing, w.alpha)
    L = MoELayer(shape, inp, "cuda:0")
    x = torch.as_tensor(inp["x"]).to("cuda:0", L.act_dtype)
    dout = None
    if a.backward:
        dout = torch.randn((w.T, w.D), generator=torch.Generator().manual_seed(5)).to("cuda:0", L.act_dtype)
    for _ in range(a.iters):
        L.forward(x)
        if dout is not None:
            L.backward(x, dout)
    torch.cuda.synchronize()
    L.check()
    print(f"{w.name}: T={w.T} ran {a.iters} forward passes")


if __name__ == "__main__":
    main()
