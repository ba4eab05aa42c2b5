"""moe_route_static: the router for callers that cannot allocate device memory.

Some callers cannot allocate: their host framework owns every device
allocation, or their runtime forbids cudaMalloc after start-up.  For them the
library offers moe_route_static, whose scratch is a fixed array built into the
library instead of a caller workspace.  These tests call it through the C ABI
and hold its results to those of moe_route (the workspace entry point) on the
same inputs, twice in a row (the array keeps the previous call's contents, so
the second call checks that each call starts clean).  This file is collected
last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_moe_layer_03_b200 import binding as B
from sparse_moe_layer_03_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _route_both(w, inp, dev="cuda:0", seq_len=0):
    cfg = B.make_config(w.T, w.D, w.H, w.E, w.K, w.n_shared, w.dtype, w.routing, w.alpha, seq_len=seq_len)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    x = torch.as_tensor(inp["x"]).to(dev, dt)
    wg = torch.as_tensor(inp["wg"]).to(dev, dt)
    bias = None if inp["router_bias"] is None else torch.as_tensor(inp["router_bias"]).to(dev)
    kmax = w.E if w.routing == "race" else w.K

    def outs():
        return (torch.full((w.T, kmax), -7, dtype=torch.int32, device=dev),
                torch.full((w.T, kmax), -7.0, dtype=torch.float32, device=dev),
                torch.full((w.T,), -7, dtype=torch.int32, device=dev),
                torch.full((w.E,), -7, dtype=torch.int32, device=dev),
                torch.full((1,), -7.0, dtype=torch.float32, device=dev))

    stream = torch.cuda.current_stream().cuda_stream
    ref = outs()
    ws_bytes = B.moe_workspace_size(cfg)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    B.moe_route(cfg, x, wg, bias, *ref, ws, ws_bytes, stream)
    runs = []
    for _ in range(2):                       # two calls in a row on the shared array
        o = outs()
        B.moe_route_static(cfg, x, wg, bias, *o, stream)
        runs.append(o)
    torch.cuda.synchronize()
    B.moe_route_static_check_status(stream)   # no device-detected error in either call
    B.moe_check_status(ws, stream)
    return ref, runs


@pytest.mark.parametrize("key,T,seq_len", [("xl2_8e2a_512", 4096, 0), ("s2_8e2a_f32", 512, 0),
                                           ("xl_race_16e", 3000, 0), ("xl2_8e2a_512", 32768, 0),
                                           ("xl2_8e2a_512", 8192, 1024)])
def test_static_scratch_router_matches_workspace_router(key, T, seq_len):
    # seq_len > 0: per-image losses, whose T x E score matrix also lives in the scratch
    w = I.WORKLOADS[key].with_tokens(T)
    inp = I.make_inputs(w)
    ref, runs = _route_both(w, inp, seq_len=seq_len)
    for o in runs:
        assert torch.equal(o[0], ref[0])                               # topk_idx: exact
        assert torch.allclose(o[1], ref[1], rtol=0, atol=1e-6)         # gates
        assert torch.equal(o[2], ref[2])                               # n_sel
        assert torch.equal(o[3], ref[3])                               # counts: exact
        tol = 1e-5 if w.dtype == "f32" else 1e-4
        assert abs(float(o[4]) - float(ref[4])) <= tol * abs(float(ref[4]))   # balance loss


def test_static_scratch_rejects_oversized_config_without_launching():
    # Expert-Race keeps a T x E fp32 score matrix in scratch: 262144 x 32 x 4 bytes > 4 MiB
    cfg = B.make_config(262144, 64, 128, 32, 2, 0, routing="race")
    rc = B.lib.moe_route_static(ctypes.byref(cfg), None, None, None, None, None, None, None, None, None)
    assert rc == B.MOE_ERR_WORKSPACE
    assert b"4194304" in B.lib.moe_last_error()
    # per-image losses keep the T x E score matrix in the scratch too: top-K at E = 8 then fits
    # about 113k tokens, not the 262144 of the whole-call loss
    ok = B.make_config(65536, 1152, 4608, 8, 2, 2, seq_len=1024)
    big = B.make_config(131072, 1152, 4608, 8, 2, 2, seq_len=1024)
    assert B.moe_workspace_size(ok) <= 4194304 < B.moe_workspace_size(big)
    rc = B.lib.moe_route_static(ctypes.byref(big), None, None, None, None, None, None, None, None, None)
    assert rc == B.MOE_ERR_WORKSPACE
