"""GPU parity: the CUDA layer, called through the C ABI, against the fp64 oracle.

Small shapes (oracle in seconds) span several 256-row tiles and a ragged tail;
the five named workloads run at full size in the launch configuration the
benchmark times, with routing, permutation and output checked on every token.
Other GEMM paths at full size are checked on 2048 sampled tokens, which put
about 16 rows into every 256-row tile of each GEMM.
"""
import numpy as np
import pytest
import torch

from sparse_moe_layer_03_b200 import inputs as I
from oracle import moe_oracle as O
from tests import parity as PA

pytestmark = pytest.mark.gpu


def _small(T, D, H, E, K, ns, dtype="bf16", routing="topk", seed=100, bias="none", bias_std=0.2):
    w = I.small_workload(T, D, H, E, K, ns, dtype, routing, seed, bias)
    return w, I.make_inputs(w, bias_std=bias_std)


SMALL = [
    # T, D, H, E, K, ns, dtype, routing
    (1000, 256, 512, 8, 2, 2, "bf16", "topk"),
    (1000, 256, 512, 8, 2, 2, "f32", "topk"),
    (777, 384, 1536, 16, 2, 2, "bf16", "topk"),
    (999, 128, 256, 4, 1, 0, "bf16", "topk"),
    (1300, 192, 384, 8, 3, 1, "f32", "topk"),
    (1000, 256, 512, 8, 2, 2, "bf16", "race"),
    (513, 128, 256, 16, 2, 1, "f32", "race"),
    (640, 64, 128, 32, 4, 2, "bf16", "topk"),
    (1111, 192, 384, 8, 2, 1, "bf16", "topk"),     # odd number of 64-column blocks in the router
    (900, 320, 640, 16, 3, 2, "bf16", "race"),
    (1000, 256, 512, 8, 2, 2, "f16", "topk"),     # fp16 storage (DiT inference default)
    (900, 320, 640, 16, 3, 2, "f16", "race"),
    (999, 128, 256, 4, 1, 0, "f16", "topk"),       # no shared experts: separate combine
    (1200, 640, 1280, 8, 2, 2, "bf16", "topk"),     # 512 + 128-wide column tiles in GEMM2 + combine
    (900, 1152, 768, 8, 2, 1, "f16", "topk"),      # 2 x 512 + 128
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "T%d_D%d_H%d_E%d_K%d_ns%d_%s_%s" % c)
def test_small_layer_parity(case):
    w, inp = _small(*case)
    rep = PA.full_check(w, inp)
    assert rep["err"] <= PA.out_tol(w)


@pytest.mark.parametrize("impl", ["auto", "tc1"])
def test_tensor_core_paths_match_ffma_path(impl):
    # auto = tcgen05 on CTA pairs (256-row tiles), tc1 = tcgen05 on single CTAs
    w, inp = _small(1000, 256, 512, 8, 2, 2, "bf16")
    a = PA.full_check(w, inp, gemm_impl=impl)
    b = PA.full_check(w, inp, gemm_impl="simt")
    # both against the oracle already; against each other: same rounding points
    assert PA.rel_err(a["res"]["out"], b["res"]["out"]) < 1e-2


@pytest.mark.parametrize("impl", ["tc1", "simt"])
def test_other_gemm_paths_full_size_xl(impl):
    w = I.WORKLOADS["xl2_8e2a_512"]
    inp = I.make_inputs(w)
    PA.full_check(w, inp, gemm_impl=impl, tokens=PA.sample_tokens(w.T, 2048))


def test_erf_gelu_option():
    w, inp = _small(300, 128, 256, 4, 2, 1, "f32")
    rep = PA.full_check(w, inp, act="erf")
    assert rep["err"] <= 1e-5


def test_deterministic_repeat():
    w, inp = _small(2000, 256, 512, 8, 2, 2, "bf16", routing="race")
    L, x = PA.run_layer(w, inp)
    valid = L.row_token >= 0          # padding rows of x_perm are never written
    pick = lambda: (L.out, L.topk_idx, L.topk_w, L.pos, L.aux, L.counts, L.h_perm[valid], L.y_perm[valid])
    first = [t.clone() for t in pick()]
    for _ in range(2):
        L.forward(x)
        torch.cuda.synchronize()
        for a, b in zip(first, pick()):
            assert torch.equal(a, b)


# ------------------------------------------------------------------ edge cases

def test_empty_batch():
    w, inp = _small(0, 128, 256, 8, 2, 1)
    L, x = PA.run_layer(w, inp)
    assert torch.all(L.counts == 0) and float(L.aux[0]) == 0.0
    assert torch.all(L.offsets == 0) and torch.all(L.row_token == -1)


def test_single_token_and_race_single_token():
    for routing in ("topk", "race"):
        w, inp = _small(1, 128, 256, 8, 2, 1, routing=routing)
        PA.full_check(w, inp)


def test_dense_mlp_special_case():
    # E = 1, K = 1, n_s = 0: every token takes the one expert with g = 1
    w, inp = _small(333, 128, 256, 1, 1, 0, "f32")
    rep = PA.full_check(w, inp)
    assert np.all(rep["res"]["topk_w"] == 1.0)


def test_all_experts_selected():
    w, inp = _small(500, 128, 256, 4, 4, 1, "bf16")
    PA.full_check(w, inp)
    w, inp = _small(300, 128, 256, 4, 4, 1, "bf16", routing="race")
    rep = PA.full_check(w, inp)
    assert np.all(rep["res"]["n_sel"] == 4)


def test_skewed_experts_one_full_one_empty():
    w, inp = _small(700, 128, 256, 8, 2, 1, "bf16")
    inp = dict(inp)
    b = np.zeros(8, np.float32)
    b[3] = 40.0        # every token takes expert 3 first
    b[5] = -40.0       # nobody ever takes expert 5
    inp["router_bias"] = b
    rep = PA.full_check(w, inp)
    c = rep["res"]["counts"]
    assert c[3] == 700 and c[5] == 0


def test_uniform_router_gives_alpha():
    # Wg = 0, no bias: all scores 1/E, ties broken by expert id, L = alpha exactly
    w, inp = _small(512, 128, 256, 8, 2, 1, "bf16")
    inp = dict(inp)
    inp["wg"] = np.zeros_like(inp["wg"])
    rep = PA.full_check(w, inp)
    assert abs(float(rep["res"]["aux"][0]) - w.alpha) < 1e-7
    assert np.all(rep["res"]["topk_idx"] == np.array([0, 1]))


def test_planted_bad_index_reported_not_faulted():
    from sparse_moe_layer_03_b200 import binding as B
    w, inp = _small(256, 128, 256, 8, 2, 1, "bf16")
    L, x = PA.run_layer(w, inp)
    L.topk_idx[7, 1] = 8 + 3                    # out-of-range expert planted on the host side
    L.dispatch(x)
    with pytest.raises(B.MoeError) as ei:
        L.check()
    assert ei.value.code == B.MOE_ERR_DEVICE_CHECK
    L.check()                                  # status cleared
    assert int(L.pos[7, 1]) == -1


# ------------------------------------------------------------------ full-size workloads

@pytest.mark.parametrize("key", I.WORKLOAD_ORDER)
def test_named_workload_full_size(key):
    # every output token of the workload against the oracle (about 40 s of oracle at XL)
    w = I.WORKLOADS[key]
    inp = I.make_inputs(w)
    rep = PA.full_check(w, inp)
    assert rep["err"] <= PA.out_tol(w)


def test_pipelined_host_batches_match_device_forward():
    # three different batches through the copy/compute-overlapped host path
    w, inp = _small(700, 256, 512, 8, 2, 2, "bf16")
    L, x = PA.run_layer(w, inp)
    xs = [torch.randn((700, 256), generator=torch.Generator().manual_seed(i)).to(torch.bfloat16).pin_memory()
          for i in range(3)]
    outs = [torch.empty((700, 256), dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    auxs = [torch.empty((1,), dtype=torch.float32).pin_memory() for _ in range(3)]
    L.forward_host_pipelined(xs, outs, auxs)
    for i in range(3):
        ref = L.forward(xs[i].to("cuda:0")).cpu()
        torch.cuda.synchronize()
        assert torch.equal(outs[i], ref)
        assert float(auxs[i][0]) == float(L.aux[0].cpu())


FUSED_CASES = [  # T, D, H, E, K, n_s, routing
    (600, 192, 384, 8, 2, 1, "topk"),
    (1111, 128, 256, 16, 2, 2, "race"),
    (300, 64, 128, 4, 4, 3, "topk"),        # every token takes every expert
]


@pytest.mark.parametrize("case", FUSED_CASES, ids=lambda c: "T%d_D%d_E%d_K%d_ns%d_%s" % (c[0], c[1], c[3], c[4], c[5], c[6]))
def test_combine_folded_into_gemm2_matches_separate_combine(case):
    from sparse_moe_layer_03_b200.layer import LayerShape, MoELayer
    T, D, H, E, K, ns, routing = case
    w = I.small_workload(T, D, H, E, K, ns, "bf16", routing, seed=77 + T)
    inp = I.make_inputs(w, bias_std=0.3)
    outs = {}
    for fuse in (True, False):
        shape = LayerShape(T, D, H, E, K, ns, "bf16", routing, w.alpha, fuse_combine=fuse)
        L = MoELayer(shape, inp, "cuda:0")
        assert L.fused == fuse
        x = torch.as_tensor(inp["x"]).to(device="cuda:0", dtype=L.act_dtype).contiguous()
        for _ in range(2):                   # the second call checks the counters were left at zero
            L.forward(x)
        torch.cuda.synchronize()
        L.check()
        r = PA.fetch(L)
        P = O.softmax_scores(O.gate_logits(inp["x"], inp["wg"], inp.get("router_bias")))
        PA.check_routing(w, P, r, inp)
        PA.check_output(w, inp, P, r)
        outs[fuse] = r["out"]
    # the folded path skips one bf16 rounding of the shared output: at most a couple of bf16 ulps apart
    assert PA.rel_err(outs[True], outs[False]) < 2e-2


@pytest.mark.parametrize("impl", ["tc1", "simt"])
def test_f16_other_gemm_paths(impl):
    w = I.small_workload(777, 384, 1536, 16, 2, 2, "f16", "topk", seed=21)
    inp = I.make_inputs(w, bias_std=0.25)
    PA.full_check(w, inp, gemm_impl=impl)


def test_f16_full_size_xl():
    # the XL/2-8E2A layer with fp16 storage: every output token against the oracle
    import dataclasses
    w = dataclasses.replace(I.WORKLOADS["xl2_8e2a_512"], dtype="f16", name="DiT-MoE-XL/2-8E2A layer at 512x512, fp16")
    inp = I.make_inputs(w)
    PA.full_check(w, inp)


RESIDUAL_CASES = [  # T, D, H, E, K, n_s, dtype, routing, img_len, fuse
    (1024, 256, 512, 8, 2, 2, "bf16", "topk", 256, True),
    (1024, 256, 512, 8, 2, 2, "bf16", "topk", 256, False),
    (900, 320, 640, 16, 3, 1, "bf16", "race", 300, True),
    (999, 128, 256, 4, 1, 0, "bf16", "topk", 333, True),     # n_s = 0: the separate combine applies it
    (1000, 256, 512, 8, 2, 2, "f16", "topk", 250, True),
]


@pytest.mark.parametrize("case", RESIDUAL_CASES,
                         ids=lambda c: "T%d_E%d_K%d_ns%d_%s_%s_L%d_%s" % (c[0], c[3], c[4], c[5], c[6], c[7], c[8],
                                                                         "fused" if c[9] else "separate"))
def test_adaln_zero_residual_in_combine(case):
    from sparse_moe_layer_03_b200.layer import LayerShape, MoELayer
    T, D, H, E, K, ns, dt, routing, L_img, fuse = case
    w = I.small_workload(T, D, H, E, K, ns, dt, routing, seed=5 + T + E)
    inp = I.make_inputs(w, bias_std=0.2)
    rng = np.random.default_rng(T)
    x_res = I._store(rng.standard_normal((T, D)), dt)
    alpha = I._store(rng.standard_normal((T // L_img, D)) * 0.5, dt)
    L = MoELayer(LayerShape(T, D, H, E, K, ns, dt, routing, w.alpha, fuse_combine=fuse), inp, "cuda:0")
    dev = lambda a: torch.as_tensor(a).to(device="cuda:0", dtype=L.act_dtype).contiguous()
    L.forward(dev(inp["x"]), dev(x_res), dev(alpha), L_img)
    torch.cuda.synchronize()
    L.check()
    r = PA.fetch(L)
    P = O.softmax_scores(O.gate_logits(inp["x"], inp["wg"], inp.get("router_bias")))
    PA.check_routing(w, P, r, inp)
    idx = PA.gpu_selection(r)
    g = np.where(idx >= 0, np.take_along_axis(P, np.maximum(idx, 0), axis=1), 0.0)
    ref = O.gated_residual(x_res, O.layer_output(inp, idx, g), alpha, L_img)
    err = PA.rel_err(r["out"], ref)
    assert err <= PA.out_tol(w), err
    # a zero gate leaves the residual stream unchanged (adaLN-Zero at initialisation)
    L.forward(dev(inp["x"]), dev(x_res), torch.zeros_like(dev(alpha)), L_img)
    torch.cuda.synchronize()
    assert torch.equal(L.out, dev(x_res))


ADALN_CASES = [  # T, D, H, E, K, n_s, dtype, routing, img_len, gate
    (1024, 256, 512, 8, 2, 2, "bf16", "topk", 256, True),
    (1024, 384, 1536, 16, 2, 1, "bf16", "race", 512, True),
    (1000, 192, 384, 8, 2, 1, "bf16", "topk", 40, False),     # img_len not a multiple of 16; odd 64-column blocks
    (1024, 256, 512, 8, 2, 2, "f16", "topk", 128, True),
]


@pytest.mark.parametrize("case", ADALN_CASES,
                         ids=lambda c: "T%d_D%d_E%d_%s_%s_L%d_%s" % (c[0], c[1], c[3], c[6], c[7], c[8],
                                                                     "gate" if c[9] else "nogate"))
def test_adaln_modulation_in_router(case):
    from sparse_moe_layer_03_b200.layer import LayerShape, MoELayer
    T, D, H, E, K, ns, dt, routing, L_img, gate = case
    w = I.small_workload(T, D, H, E, K, ns, dt, routing, seed=9 + T + D)
    inp = I.make_inputs(w)
    rng = np.random.default_rng(D)
    nimg = T // L_img
    x = I._store(rng.standard_normal((T, D)) * 2.0 + 0.5, dt)          # a residual stream with an offset
    gamma = I._store(1.0 + 0.3 * rng.standard_normal((nimg, D)), dt)
    beta = I._store(0.3 * rng.standard_normal((nimg, D)), dt)
    alpha = I._store(0.5 * rng.standard_normal((nimg, D)), dt) if gate else None
    L = MoELayer(LayerShape(T, D, H, E, K, ns, dt, routing, w.alpha), inp, "cuda:0")
    dev = lambda a: torch.as_tensor(a).to(device="cuda:0", dtype=L.act_dtype).contiguous()
    L.forward(dev(x), alpha=dev(alpha) if gate else None, img_len=L_img, gamma=dev(gamma), beta=dev(beta))
    torch.cuda.synchronize()
    L.check()
    # m as the layer stores it: the oracle's adaLN rounded to the act type; the GPU's fp32 statistics may
    # land a value on the other side of a rounding boundary, so one unit in the last place is allowed
    m = I._store(O.adaln(x, gamma, beta, L_img).astype(np.float32), dt)
    got = L.x_mod.float().cpu().numpy()
    ulp = np.abs(m) * (2.0 ** (-7 if dt == "bf16" else -10)) + 1e-30
    # where gamma * LayerNorm(x) and beta nearly cancel, the fp32 row statistics (mean, variance over
    # D values, error about D * 2^-24 relative) matter against a small m: allow 2^-16 of the terms' size
    b = np.arange(T) // L_img
    terms = np.abs(gamma[b] * O.layer_norm(x)) + np.abs(beta[b])
    assert np.all(np.abs(got - m) <= ulp * 1.01 + terms * 2.0 ** -16)
    assert np.mean(got == m) > 0.99
    # routing and output on the layer's own m
    inp_m = dict(inp, x=got.astype(np.float64))
    r = PA.fetch(L)
    P = O.softmax_scores(O.gate_logits(inp_m["x"], inp["wg"], inp.get("router_bias")))
    PA.check_routing(w, P, r, inp_m)
    idx = PA.gpu_selection(r)
    g = np.where(idx >= 0, np.take_along_axis(P, np.maximum(idx, 0), axis=1), 0.0)
    y = O.layer_output(inp_m, idx, g)
    ref = O.gated_residual(x, y, alpha, L_img) if gate else y
    err = PA.rel_err(r["out"], ref)
    assert err <= PA.out_tol(w), err



@pytest.mark.parametrize("routing", ["topk", "race"])
def test_gathered_gemm1_rows_against_oracle(routing):
    # GEMM1 reading its routed rows straight from x (no x_perm): routing, positions and output
    # against the oracle
    w = I.small_workload(1500, 384, 768, 16 if routing == "race" else 8, 2, 2, "bf16", routing, seed=63)
    inp = I.make_inputs(w, bias_std=0.2)
    rep = PA.full_check(w, inp, gather_rows=True)
    assert rep["layer"].gathered and rep["layer"].x_perm is None
    assert rep["err"] <= PA.out_tol(w)


def test_gathered_gemm1_full_size_xl():
    w = I.WORKLOADS["xl2_8e2a_512"]
    inp = I.make_inputs(w)
    rep = PA.full_check(w, inp, gather_rows=True, tokens=PA.sample_tokens(w.T, 2048))
    assert rep["layer"].gathered


@pytest.mark.parametrize("routing", ["topk", "race"])
def test_gathered_gemm1_rows_equal_permuted_copy(routing):
    # GEMM1 reading its rows from x (cp.async gather warps) computes bit for bit what it computes on x_perm
    from sparse_moe_layer_03_b200.layer import LayerShape, MoELayer
    w = I.small_workload(1500, 384, 768, 16 if routing == "race" else 8, 2, 2, "bf16", routing, seed=61)
    inp = I.make_inputs(w, bias_std=0.2)
    res = {}
    for gather in (True, False):
        L = MoELayer(LayerShape(w.T, w.D, w.H, w.E, w.K, w.n_shared, "bf16", routing, w.alpha, gather_rows=gather),
                     inp, "cuda:0")
        assert L.gathered == gather and (L.x_perm is None) == gather
        x = torch.as_tensor(inp["x"]).to(device="cuda:0", dtype=L.act_dtype).contiguous()
        L.forward(x)
        torch.cuda.synchronize()
        L.check()
        valid = L.row_token >= 0
        res[gather] = (L.h_perm[valid].clone(), L.out.clone())
    assert torch.equal(res[True][0], res[False][0])
    assert torch.equal(res[True][1], res[False][1])


@pytest.mark.parametrize("routing", ["topk", "race"])
def test_forward_captured_in_a_cuda_graph(routing):
    # one graph launch reruns the whole layer; replays match the eager forward bit for bit
    from sparse_moe_layer_03_b200.layer import LayerShape, MoELayer
    w = I.small_workload(2048, 384, 768, 16 if routing == "race" else 8, 2, 2, "bf16", routing, seed=71)
    inp = I.make_inputs(w, bias_std=0.2)
    L = MoELayer(LayerShape(w.T, w.D, w.H, w.E, w.K, w.n_shared, "bf16", routing, w.alpha), inp, "cuda:0")
    x = torch.as_tensor(inp["x"]).to(device="cuda:0", dtype=L.act_dtype).contiguous()
    eager = L.forward(x).clone()
    eager_aux = L.aux.clone()
    g = L.capture(x)
    for _ in range(3):
        L.out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(L.out, eager) and torch.equal(L.aux, eager_aux)
    L.check()
    # a new input in the captured buffer is routed afresh
    x2 = torch.as_tensor(I.make_inputs(I.small_workload(2048, 384, 768, w.E, 2, 2, "bf16", routing, seed=72))["x"])
    x.copy_(x2.to(device="cuda:0", dtype=L.act_dtype))
    g.replay()
    torch.cuda.synchronize()
    fresh = L.forward(x).clone()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(L.out, fresh)


MLP_CASES = [  # T, D, H, E, K, n_s, dtype, routing
    (1000, 256, 512, 8, 2, 2, "bf16", "topk"),
    (900, 320, 640, 16, 3, 1, "bf16", "race"),
    (700, 256, 512, 8, 2, 1, "f32", "topk"),
    (999, 128, 256, 4, 1, 0, "f16", "topk"),
]


@pytest.mark.parametrize("case", MLP_CASES, ids=lambda c: "T%d_D%d_E%d_K%d_ns%d_%s_%s" % (c[0], c[1], c[3], c[4], c[5],
                                                                                         c[6], c[7]))
def test_expert_mlp_call_then_combine(case):
    # moe_expert_mlp (GEMM1 then GEMM2 in one call) and moe_combine, called through the C ABI into
    # buffers of their own after the layer's route and dispatch, against the oracle
    from sparse_moe_layer_03_b200 import binding as B
    T, D, H, E, K, ns, dt, routing = case
    w = I.small_workload(T, D, H, E, K, ns, dt, routing, seed=31 + T)
    inp = I.make_inputs(w, bias_std=0.2)
    L, x = PA.run_layer(w, inp)
    r = PA.fetch(L)
    h_perm = torch.zeros_like(L.h_perm)
    y_perm = torch.zeros_like(L.y_perm)
    h_sh = torch.zeros((T, ns * H), dtype=L.act_dtype, device=x.device) if ns else None
    y_sh = torch.zeros((T, D), dtype=L.act_dtype, device=x.device) if ns else None
    out = torch.zeros_like(L.out)
    B.moe_expert_mlp(L.cfg, L.offsets, L.x_perm, x, L.w1, L.b1, L.w2, L.b2, L.ws1, L.bs1, L.ws2, L.bs2, L.row_gate,
                     h_perm, h_sh, y_perm, y_sh, L.ws, L.ws_bytes, L.stream())
    B.moe_combine(L.cfg, y_perm, y_sh, L.pos, L.n_sel, out, L.stream())
    torch.cuda.synchronize()
    L.check()
    r["out"] = out.float().cpu().numpy()
    P = O.softmax_scores(O.gate_logits(inp["x"], inp["wg"], inp.get("router_bias")))
    err = PA.check_output(w, inp, P, r)
    assert err <= PA.out_tol(w)
