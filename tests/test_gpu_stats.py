"""GPU parity of the per-image balance loss and of the expert-selection frequencies.

Both are checked against the oracle evaluated on the GPU's own selection: the
loss to the same relative tolerance as the whole-call loss, the frequencies
bit for bit (integer counts).
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_moe_layer_03_b200 import binding as B
from sparse_moe_layer_03_b200 import inputs as I
from tests import parity as PA

pytestmark = pytest.mark.gpu


def _run(w, inp, seq_len):
    from sparse_moe_layer_03_b200.layer import LayerShape, MoELayer
    shape = LayerShape(w.T, w.D, w.H, w.E, w.K, w.n_shared, w.dtype, w.routing, w.alpha, seq_len=seq_len)
    L = MoELayer(shape, inp, "cuda:0")
    x = torch.as_tensor(inp["x"]).to(device="cuda:0", dtype=L.act_dtype).contiguous()
    L.forward(x)
    torch.cuda.synchronize()
    L.check()
    return L, PA.fetch(L)


def _check_loss(w, inp, L, r, seq_len):
    P = O.softmax_scores(O.gate_logits(inp["x"], inp["wg"], inp.get("router_bias")))
    PA.check_routing(w, P, r, inp)
    idx = PA.gpu_selection(r)
    assert np.array_equal(r["counts"].astype(np.int64), O.expert_counts(idx, w.E))
    ref = O.balance_loss_per_sequence(idx, P, w.K, w.alpha, seq_len)
    got = float(r["aux"][0])
    assert abs(got - ref) <= PA.aux_tol(w) * abs(ref), (got, ref)
    return idx


CASES = [  # T, D, H, E, K, n_s, dtype, routing, seq_len
    (1024, 128, 256, 8, 2, 1, "bf16", "topk", 256),
    (1024, 128, 256, 16, 2, 1, "bf16", "race", 256),
    (960, 64, 128, 8, 1, 0, "f32", "topk", 64),
    (960, 64, 128, 8, 3, 0, "f32", "race", 320),
    (600, 192, 384, 32, 4, 2, "bf16", "topk", 1),      # one token per image
    (600, 192, 384, 4, 2, 0, "bf16", "race", 600),     # one image: the whole-call loss
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T%d_D%d_E%d_K%d_%s_%s_L%d" % (c[0], c[1], c[3], c[4], c[6], c[7], c[8]))
def test_per_image_loss_and_frequencies(case):
    T, D, H, E, K, ns, dt, routing, L_img = case
    w = I.small_workload(T, D, H, E, K, ns, dt, routing, seed=31 + T + E)
    inp = I.make_inputs(w)
    L, r = _run(w, inp, L_img)
    idx = _check_loss(w, inp, L, r, L_img)
    if L_img == T:
        assert abs(float(r["aux"][0]) - O.balance_loss(O.expert_counts(idx, E), O.softmax_scores(
            O.gate_logits(inp["x"], inp["wg"], inp.get("router_bias"))), K, w.alpha)) <= 1e-4 * float(r["aux"][0])
    # per patch position
    hp = L.expert_frequency(L_img).cpu().numpy()
    assert np.array_equal(hp, O.expert_frequency(idx, E, O.position_labels(T, L_img), L_img))
    # per image label (a class out of 1000, or a timestep out of 250 DDPM steps)
    nimg = T // L_img
    rng = np.random.default_rng(5)
    for n_labels in (1000, 250):
        lab = rng.integers(0, n_labels, nimg).astype(np.int32)
        hl = L.expert_frequency(L_img, torch.as_tensor(lab, device="cuda:0"), n_labels).cpu().numpy()
        assert np.array_equal(hl, O.expert_frequency(idx, E, O.image_labels(T, L_img, lab), n_labels))
    L.check()


@pytest.mark.parametrize("key", ["xl2_8e2a_512", "xl_race_16e"])
def test_per_image_loss_full_size(key):
    # 512x512 images: 1024 patch tokens each, 32 images per call
    w = I.WORKLOADS[key]
    inp = I.make_inputs(w)
    L, r = _run(w, inp, 1024)
    idx = _check_loss(w, inp, L, r, 1024)
    hp = L.expert_frequency(1024).cpu().numpy()
    assert np.array_equal(hp, O.expert_frequency(idx, w.E, O.position_labels(w.T, 1024), 1024))
    lab = (np.arange(32) * 7 % 250).astype(np.int32)
    hl = L.expert_frequency(1024, torch.as_tensor(lab, device="cuda:0"), 250).cpu().numpy()
    assert np.array_equal(hl, O.expert_frequency(idx, w.E, O.image_labels(w.T, 1024, lab), 250))


def test_label_out_of_range_is_reported_not_faulted():
    w = I.small_workload(512, 64, 128, 8, 2, 0, "bf16", "topk", seed=3)
    inp = I.make_inputs(w)
    L, r = _run(w, inp, 128)
    lab = torch.tensor([0, 5, 12, 1], dtype=torch.int32, device="cuda:0")   # 12 is outside 0..9
    hist = L.expert_frequency(128, lab, 10)
    torch.cuda.synchronize()
    with pytest.raises(B.MoeError) as ei:
        L.check()
    assert ei.value.code == B.MOE_ERR_DEVICE_CHECK
    idx = PA.gpu_selection(r)
    tok_lab = O.image_labels(512, 128, [0, 5, 12, 1])
    keep = tok_lab < 10
    want = O.expert_frequency(idx[keep], 8, tok_lab[keep], 10)
    assert np.array_equal(hist.cpu().numpy(), want)      # the image with the bad label is skipped
    L.check()                                            # the status word was cleared


BWD_CASES = [  # T, D, E, K, dtype, routing
    (1000, 256, 8, 2, "bf16", "topk"),
    (1024, 384, 16, 2, "bf16", "race"),
    (777, 128, 4, 1, "f32", "topk"),
    (600, 192, 32, 4, "f16", "topk"),
    (32768, 1152, 8, 2, "bf16", "topk"),       # XL/2-8E2A router
]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "T%d_D%d_E%d_K%d_%s_%s" % c)
def test_balance_loss_backward(case):
    T, D, E, K, dt, routing = case
    w = I.small_workload(T, D, 2 * D, E, K, 0, dt, routing, seed=3 + T + E, router_bias="normal")
    inp = I.make_inputs(w)
    L, r = _run(w, inp, 0)
    dev = L.device
    bws = torch.empty(B.moe_backward_workspace_size(L.cfg), dtype=torch.uint8, device=dev)
    outs = []
    for _ in range(2):
        dwg = torch.empty((E, D), dtype=torch.float32, device=dev)
        db = torch.empty((E,), dtype=torch.float32, device=dev)
        dx = torch.empty((T, D), dtype=L.act_dtype, device=dev)
        x = torch.as_tensor(inp["x"]).to(device=dev, dtype=L.act_dtype).contiguous()
        B.moe_balance_loss_backward(L.cfg, x, L.wg, L.router_bias, L.counts, 1.0, dwg, db, dx, bws, bws.numel(),
                                    L.stream())
        torch.cuda.synchronize()
        outs.append((dwg.cpu().numpy(), db.cpu().numpy(), dx.float().cpu().numpy()))
    for a, b in zip(outs[0], outs[1]):
        assert np.array_equal(a, b)                     # fixed summation order
    P = O.softmax_scores(O.gate_logits(inp["x"], inp["wg"], inp.get("router_bias")))
    dl = O.balance_loss_grad_logits(P, r["counts"], K, w.alpha)
    ref_dwg, ref_db, ref_dx = O.router_backward(inp["x"], inp["wg"], dl)
    dwg, db, dx = outs[0]
    # fp32 logits against fp64 and fp32 sums: the gradient is a difference of nearby terms
    # (P (c - P.c)), so it is held to 1e-3 of its largest entry; dx is also rounded to the act type
    assert PA.rel_err(dwg, ref_dwg) < 1e-3
    assert PA.rel_err(db, ref_db) < 1e-3
    assert PA.rel_err(dx, ref_dx) < (1e-3 if dt == "f32" else 1e-2)


STATS_CASES = [  # T (two halves of T/2), D, E, K, dtype, routing
    (2048, 128, 8, 2, "bf16", "topk"),
    (2048, 128, 16, 2, "bf16", "race"),
    (1000, 64, 8, 1, "f32", "topk"),
    (1200, 192, 4, 2, "f16", "topk"),
]


@pytest.mark.parametrize("case", STATS_CASES, ids=lambda c: "T%d_D%d_E%d_K%d_%s_%s" % c)
def test_balance_stats_and_loss_of_two_calls(case):
    # one layer routes the two halves of a batch in two calls (as two ranks would); the sum of
    # their statistics gives the loss of the whole batch under the union of the two selections
    from sparse_moe_layer_03_b200.layer import LayerShape, MoELayer
    T, D, E, K, dt, routing = case
    Th = T // 2
    w = I.small_workload(T, D, 2 * D, E, K, 0, dt, routing, seed=11 + T + E, router_bias="normal")
    inp = I.make_inputs(w)
    L = MoELayer(LayerShape(Th, D, 2 * D, E, K, 0, dt, routing, w.alpha), inp, "cuda:0")
    xs = torch.as_tensor(inp["x"]).to(device="cuda:0", dtype=L.act_dtype).contiguous()
    stats, sels, own = [], [], []
    for h in range(2):
        L.route(xs[h * Th:(h + 1) * Th].contiguous())
        st = L.balance_stats().clone()
        own.append(L.aux.clone())
        L.balance_loss_from_stats(st, Th)                # one call's statistics: that call's own loss
        torch.cuda.synchronize()
        L.check()
        assert torch.equal(L.aux, own[-1])              # same terms, same order
        r = PA.fetch(L)
        idx = PA.gpu_selection(r)
        half = slice(h * Th, (h + 1) * Th)
        P = O.softmax_scores(O.gate_logits(inp["x"][half], inp["wg"], inp.get("router_bias")))
        PA.check_routing(w, P, r, dict(inp, x=inp["x"][half]))
        got = st.cpu().numpy()
        assert np.array_equal(got[:E], r["counts"].astype(np.float64))
        assert np.max(np.abs(got[E:] - P.sum(axis=0))) <= 1e-5 * Th
        stats.append(st)
        sels.append((idx, P))
    total = stats[0] + stats[1]
    L.balance_loss_from_stats(total, T)
    torch.cuda.synchronize()
    idx = np.concatenate([s[0] for s in sels])
    P = np.concatenate([s[1] for s in sels])
    ref = O.balance_loss_from_stats(O.balance_stats(idx, P, E), K, T, w.alpha)
    got = float(L.aux[0])
    assert abs(got - ref) <= PA.aux_tol(w) * abs(ref), (got, ref)
    if routing == "topk":                               # per-token selection: the whole batch's own loss
        assert abs(ref - O.balance_loss(O.expert_counts(idx, E), P, K, w.alpha)) <= 1e-12 * ref
    L.check()


def test_balance_stats_of_an_empty_call():
    from sparse_moe_layer_03_b200.layer import LayerShape, MoELayer
    w = I.small_workload(0, 128, 256, 8, 2, 0, "bf16", "topk", seed=5)
    inp = I.make_inputs(w)
    L = MoELayer(LayerShape(0, 128, 256, 8, 2, 0, "bf16", "topk", w.alpha), inp, "cuda:0")
    L.route(torch.empty((0, 128), dtype=torch.bfloat16, device="cuda:0"))
    st = L.balance_stats()
    L.balance_loss_from_stats(st, 0)
    torch.cuda.synchronize()
    assert torch.all(st == 0) and float(L.aux[0]) == 0.0
    L.check()
