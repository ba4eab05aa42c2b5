"""GPU parity of the layer's backward: moe_expert_backward + moe_router_backward, called
through the C ABI (MoELayer.backward), against the oracle's layer_backward (fp64, pinned to
torch autograd on the CPU).

Every gradient (weights, biases, router, gates, input) is compared normwise, max|g - g_ref| /
max|g_ref|, with the output bound of the storage type: 2e-2 for bf16, 5e-3 for fp16.  The few
16-bit roundings on each path (dY times the gate, the recomputed pre-activation, dU, dx per
routed row, and the forward's h that the weight gradients read) are each about 2^-9 of the
values (2^-12 for fp16), the same budget as the forward's output.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_moe_layer_03_b200 import inputs as I
from tests import parity as PA

pytestmark = pytest.mark.gpu

BWD_CASES = [  # T, D, H, E, K, n_s, dtype, routing
    (600, 256, 512, 8, 2, 2, "bf16", "topk"),
    (900, 320, 640, 16, 3, 1, "bf16", "race"),
    (500, 192, 384, 4, 1, 0, "bf16", "topk"),      # no shared experts: separate combine of dx
    (777, 384, 1536, 16, 2, 2, "f16", "topk"),
    (1000, 256, 768, 8, 2, 1, "bf16", "topk"),     # H not a multiple of 256: narrower column tiles
]


def _grads_ref(inp, idx, dout, w, aux_scale):
    return O.layer_backward(inp, idx, dout, w.K, w.alpha, aux_scale=aux_scale)


def _compare(g, ref, w, names):
    tol = PA.out_tol(w)
    errs = {}
    for n in names:
        got = g[n].float().cpu().numpy() if g[n] is not None else None
        want = ref[n]
        if want.size == 0:
            continue
        errs[n] = PA.rel_err(got.reshape(want.shape), want)
    bad = {n: e for n, e in errs.items() if not e <= tol}
    assert not bad, f"gradients off (tol {tol:.0e}): {bad}; all: {errs}"
    return errs


def _dgate_ref(inp, idx, dout):
    # dJ/dg for each selected slot: <dout_t, e_i(x_t)>
    x = O.as_f64(inp["x"])
    out = np.zeros(idx.shape)
    for e in range(inp["w1"].shape[0]):
        rows, slots = np.nonzero(idx == e)
        if rows.size == 0:
            continue
        y = O.expert_mlp(x[rows], inp["w1"][e], O._bias_row(inp.get("b1"), e), inp["w2"][e],
                         O._bias_row(inp.get("b2"), e))
        out[rows, slots] = np.sum(O.as_f64(dout)[rows] * y, axis=1)
    return out


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "T%d_D%d_H%d_E%d_K%d_ns%d_%s_%s" % c)
def test_layer_backward_against_oracle(case):
    T, D, H, E, K, ns, dt, routing = case
    w = I.small_workload(T, D, H, E, K, ns, dt, routing, seed=91 + T)
    inp = I.make_inputs(w, bias_std=0.2)
    L, x = PA.run_layer(w, inp)
    rng = np.random.default_rng(T)
    dout = I._store(rng.standard_normal((T, D)), dt)
    dout_d = torch.as_tensor(dout).to(device=x.device, dtype=L.act_dtype)
    g = L.backward(x, dout_d, aux_scale=3.0)
    torch.cuda.synchronize()
    L.check()
    r = PA.fetch(L)
    idx = PA.gpu_selection(r)
    ref = _grads_ref(inp, idx, dout, w, 3.0)
    names = ["dx", "dwg", "dbias", "dw1", "db1", "dw2", "db2"] + (["dws1", "dbs1", "dws2", "dbs2"] if ns else [])
    _compare(g, ref, w, names)
    # the gates' gradient per slot
    got = g["dgate"].cpu().numpy()
    want = _dgate_ref(inp, idx, dout)
    used = idx >= 0
    assert PA.rel_err(got[used], want[used]) <= PA.out_tol(w)
    assert np.all(got[~used] == 0)


def test_backward_is_deterministic():
    w = I.small_workload(1200, 256, 512, 8, 2, 2, "bf16", "race", seed=95)
    inp = I.make_inputs(w, bias_std=0.2)
    L, x = PA.run_layer(w, inp)
    dout = torch.randn((w.T, w.D), generator=torch.Generator().manual_seed(3)).to(device=x.device,
                                                                                     dtype=L.act_dtype)
    first = {k: v.clone() for k, v in L.backward(x, dout).items() if v is not None}
    for _ in range(2):
        again = L.backward(x, dout)
        torch.cuda.synchronize()
        for k, v in first.items():
            assert torch.equal(v, again[k]), k
    L.check()


def test_backward_with_an_empty_expert():
    # an expert nobody takes gets zero weight gradients (its tiles reduce over no rows)
    w = I.small_workload(700, 128, 256, 8, 2, 1, "bf16", "topk", seed=97)
    inp = dict(I.make_inputs(w, bias_std=0.2))
    b = np.zeros(8, np.float32)
    b[5] = -40.0
    inp["router_bias"] = b
    L, x = PA.run_layer(w, inp)
    r = PA.fetch(L)
    assert r["counts"][5] == 0
    dout = I._store(np.random.default_rng(1).standard_normal((w.T, w.D)), "bf16")
    g = L.backward(x, torch.as_tensor(dout).to(device=x.device, dtype=L.act_dtype))
    torch.cuda.synchronize()
    assert torch.count_nonzero(g["dw1"][5]) == 0 and torch.count_nonzero(g["dw2"][5]) == 0
    idx = PA.gpu_selection(r)
    ref = _grads_ref(inp, idx, dout, w, 1.0)
    _compare(g, ref, w, ["dx", "dwg", "dw1", "db1", "dw2", "db2", "dws1", "dws2"])


def test_backward_full_size_xl_on_sampled_tokens():
    # XL/2-8E2A at full size: dout is zero outside 2048 sampled tokens and the balance term is off,
    # so every gradient is the oracle's backward of those tokens alone
    w = I.WORKLOADS["xl2_8e2a_512"]
    inp = I.make_inputs(w)
    L, x = PA.run_layer(w, inp)
    tok = PA.sample_tokens(w.T, 2048)
    rng = np.random.default_rng(11)
    dout = np.zeros((w.T, w.D), np.float32)
    dout[tok] = I._store(rng.standard_normal((tok.size, w.D)), "bf16")
    g = L.backward(x, torch.as_tensor(dout).to(device=x.device, dtype=L.act_dtype), aux_scale=0.0)
    torch.cuda.synchronize()
    L.check()
    r = PA.fetch(L)
    idx = PA.gpu_selection(r)[tok]
    sub = dict(inp, x=inp["x"][tok])
    ref = _grads_ref(sub, idx, dout[tok], w, 0.0)
    g_sub = dict(g)
    g_sub["dx"] = g["dx"][torch.as_tensor(tok, device=x.device)]
    _compare(g_sub, ref, w, ["dx", "dwg", "dbias", "dw1", "db1", "dw2", "db2", "dws1", "dbs1", "dws2", "dbs2"])
    # tokens outside the sample get no gradient
    rest = np.setdiff1d(np.arange(w.T), tok)
    assert int(torch.count_nonzero(g["dx"][torch.as_tensor(rest, device=x.device)])) == 0
