"""Parity harness: run the CUDA layer through the C ABI and hold it to the oracle.

Rules (from the method's workload description):
* routing indices, counts and permutations are bit-exact wherever the K-th and
  (K+1)-th oracle scores (race: the S-th and (S+1)-th of the whole matrix)
  differ by more than 1e-4; inside that band either choice is accepted;
* counts, offsets, positions, row order and x_perm rows are then compared bit
  for bit with the oracle's canonical permutation of the GPU's own selection;
* the output is compared with the oracle evaluated on the GPU's selection
  (so a tie flip costs no output tolerance): normwise max relative error
  max|y - y_ref| / max|y_ref| <= 1e-5 (fp32), <= 2e-2 (bf16), <= 5e-3 (fp16);
* the balance loss to 1e-5 (fp32) / 1e-4 (bf16, fp16) relative;
* the gates (the GPU's fp32 softmax scores of the chosen experts) within the
  rounding-error bound of ``score_error_bound``, derived below.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_oracle as O
from sparse_moe_layer_03_b200.inputs import Workload

TIE = 1e-4
SEG_ALIGN = 256      # expert segments of the permuted buffers start on multiples of this
U32 = 2.0 ** -23     # one unit in the last place of an fp32 value, relative (2x the round-to-nearest unit)


def score_error_bound(inp: dict) -> np.ndarray:
    """[T,E] bound on |P_gpu - P| for softmax scores computed in fp32 from the stored inputs.

    The GPU forms each logit l = sum_d x_d w_d + b in fp32 from the same stored values the
    oracle reads, in an order of its own (tensor-core chains for 16-bit inputs, FMA chains for
    fp32).  Whatever the order, a sum of n terms whose every addition (or FMA, or product) is
    off by at most one unit in the last place has |error| <= gamma_n * sum |terms| with
    gamma_n = n u / (1 - n u), u = 2^-23 (this covers round-to-nearest and accumulators that
    truncate).  With n = D + 2 (D - 1 additions, the product rounding of fp32 inputs, the bias):
        |dl_i| <= gamma_{D+2} (sum_d |x_d w_id| + |b_i|) <= Delta = max_i of that.
    The exact softmax of logits each moved by at most Delta moves each score by a factor in
    [e^{-2 Delta}, e^{2 Delta}].  Evaluating it in fp32 adds the rounding of l_i - m (relative
    u |l_i - m| after exp), expf (2 units), the sum of E positive terms (E - 1 units), the
    reciprocal and the product (one unit each):
        |P_gpu - P| <= P (e^{2 Delta} - 1) + P e^{2 Delta} u (|l_i - m| + 2 Delta + E + 4).
    A 1% margin covers the second-order terms.
    """
    x = np.asarray(inp["x"], dtype=np.float64)
    wg = np.asarray(inp["wg"], dtype=np.float64)
    T, D = x.shape
    E = wg.shape[0]
    b = inp.get("router_bias")
    b = np.zeros(E) if b is None else np.asarray(b, dtype=np.float64)
    logits = x @ wg.T + b
    n = D + 2
    gam = n * U32 / (1.0 - n * U32)
    dl = gam * (np.abs(x) @ np.abs(wg).T + np.abs(b))
    delta = dl.max(axis=1, keepdims=True) if T else np.zeros((0, 1))
    P = O.softmax_scores(logits)
    spread = np.abs(logits - (logits.max(axis=1, keepdims=True) if T else 0.0))
    rel = np.expm1(2 * delta) + np.exp(2 * delta) * U32 * (spread + 2 * delta + E + 4)
    return P * rel * 1.01


def out_tol(w: Workload) -> float:
    # fp16 carries 3 more mantissa bits than bf16 (unit roundoff 2^-11 against 2^-8), so the same
    # few roundings (h, y, out) sit 8x lower; 5e-3 keeps the bf16 bound's margin of about 4
    return {"f32": 1e-5, "bf16": 2e-2, "f16": 5e-3}[w.dtype]


def aux_tol(w: Workload) -> float:
    return 1e-5 if w.dtype == "f32" else 1e-4


def rel_err(y, ref) -> float:
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(y - ref)) / (den if den > 0 else 1.0))


def run_layer(w: Workload, inp: dict, gemm_impl: str = "auto", device: str = "cuda:0", act: str = "tanh",
              **layer_opts):
    """Run the whole layer once; returns the layer object (buffers on device).  ``layer_opts`` are
    further ``LayerShape`` fields (gather_rows, fuse_combine, max_clusters, ...)."""
    from sparse_moe_layer_03_b200.layer import LayerShape, MoELayer
    shape = LayerShape(w.T, w.D, w.H, w.E, w.K, w.n_shared, w.dtype, w.routing, w.alpha, act, gemm_impl,
                       **layer_opts)
    L = MoELayer(shape, inp, device)
    x = torch.as_tensor(inp["x"]).to(device=device, dtype=L.act_dtype).contiguous()
    L.forward(x)
    torch.cuda.synchronize()
    L.check()
    return L, x


def fetch(L) -> dict:
    g = lambda t: None if t is None else t.detach().cpu()
    r = {k: g(getattr(L, k)) for k in ("topk_idx", "topk_w", "n_sel", "counts", "aux", "offsets", "pos",
                                       "row_token", "row_gate", "out")}
    r = {k: (v.float().numpy() if v is not None and v.dtype == torch.bfloat16 else
             (v.numpy() if v is not None else None)) for k, v in r.items()}
    return r


def check_routing(w: Workload, P: np.ndarray, r: dict, inp: dict) -> dict:
    """Selection vs the oracle scores P (fp64), with the near-tie band; gates within the fp32
    rounding bound of the scores (``score_error_bound`` of the inputs ``inp`` the GPU routed on)."""
    T, E = P.shape
    idx, n_sel, gw = r["topk_idx"].astype(np.int64), r["n_sel"].astype(np.int64), r["topk_w"]
    kmax = idx.shape[1]
    sel = np.zeros((T, E), dtype=bool)
    for k in range(kmax):
        ok = (np.arange(kmax)[k] < n_sel) & (idx[:, k] >= 0)
        assert np.all(idx[ok, k] < E)
        rows = np.nonzero(ok)[0]
        assert not np.any(sel[rows, idx[rows, k]]), "an expert chosen twice by one token"
        sel[rows, idx[rows, k]] = True
        if w.routing == "race":                       # unused slots are padded with -1
            assert np.all(idx[k >= n_sel, k] == -1)
    if w.routing == "topk":
        assert np.all(n_sel == w.K)
        assert np.all(sel.sum(1) == w.K)
        s = -np.sort(-P, axis=1)
        thr = (s[:, w.K - 1] + s[:, w.K]) / 2 if w.K < E else np.full(T, -1.0)
        thr = thr[:, None]
    else:
        S = w.K * T
        assert sel.sum() == S, (sel.sum(), S)
        f = -np.sort(-P.reshape(-1))
        thr = (f[S - 1] + f[S]) / 2 if S < T * E else -1.0
    free = np.abs(P - thr) <= TIE
    want = P > thr
    bad = (~free) & (sel != want)
    assert not np.any(bad), f"{int(bad.sum())} routing decisions differ outside the 1e-4 band"
    # gates: the GPU's fp32 scores of its chosen experts, within the derived rounding bound
    bound = score_error_bound(inp)
    for k in range(kmax):
        ok = (k < n_sel) & (idx[:, k] >= 0)
        d = np.abs(gw[ok, k] - P[ok, idx[ok, k]])
        lim = bound[ok, idx[ok, k]]
        assert np.all(d <= lim), f"gate error {d.max():.3e} above its rounding bound ({int((d > lim).sum())} gates)"
        if k + 1 < kmax:
            nxt = (k + 1 < n_sel) & ok
            assert np.all(gw[nxt, k] >= gw[nxt, k + 1]), "slots not in descending score"
            eq = nxt & (gw[:, k] == gw[:, k + 1])
            assert np.all(idx[eq, k] < idx[eq, k + 1]), "equal scores not in ascending expert id"
    return {"sel": sel, "free": int(free.sum()), "flips": int(((sel != want) & free).sum())}


def check_counts_loss(w: Workload, P: np.ndarray, r: dict):
    idx = r["topk_idx"].astype(np.int64)
    counts = O.expert_counts(np.where(np.arange(idx.shape[1])[None, :] < r["n_sel"][:, None], idx, -1), w.E)
    assert np.array_equal(r["counts"].astype(np.int64), counts)
    assert counts.sum() == w.K * w.T
    ref = O.balance_loss(counts, P, w.K, w.alpha)
    got = float(r["aux"][0])
    assert abs(got - ref) <= aux_tol(w) * abs(ref), (got, ref)
    return ref


def gpu_selection(r: dict) -> np.ndarray:
    idx = r["topk_idx"].astype(np.int64).copy()
    kmax = idx.shape[1]
    idx[np.arange(kmax)[None, :] >= r["n_sel"][:, None]] = -1
    return idx


def check_permutation(w: Workload, L, r: dict, x_dev: torch.Tensor, rows_to_check: int = 4096):
    idx = gpu_selection(r)
    cp = O.canonical_permutation(idx, w.E, tile=SEG_ALIGN)
    assert np.array_equal(r["offsets"].astype(np.int64), cp["offsets"])
    assert np.array_equal(r["pos"].astype(np.int64), cp["pos"])
    Rv = int(cp["padded_offsets"][-1])
    assert np.array_equal(r["row_token"][:Rv].astype(np.int64), cp["row_token"])
    assert np.all(r["row_token"][Rv:] == -1) and np.all(r["row_gate"][Rv:] == 0)
    valid = cp["row_token"] >= 0
    rt, rs = cp["row_token"][valid], cp["row_slot"][valid]
    assert np.array_equal(r["row_gate"][:Rv][valid], r["topk_w"][rt, rs])
    assert np.all(r["row_gate"][:Rv][~valid] == 0)
    if L.x_perm is None:             # GEMM1 gathered the rows from x itself: nothing permuted to compare
        return cp
    # the padding rows inside the expert segments are zero
    pad = torch.as_tensor(np.nonzero(~valid)[0], device=x_dev.device)
    if pad.numel():
        assert int(torch.count_nonzero(L.x_perm.index_select(0, pad))) == 0
    # x_perm rows are exact copies of x rows (sampled rows when large)
    rows = np.nonzero(valid)[0]
    if rows.size > rows_to_check:
        rows = np.random.default_rng(0).choice(rows, rows_to_check, replace=False)
    rows_t = torch.as_tensor(rows, device=x_dev.device)
    xp = L.x_perm.index_select(0, rows_t)
    xs = x_dev.index_select(0, torch.as_tensor(cp["row_token"][rows], device=x_dev.device))
    assert torch.equal(xp, xs)
    return cp


def sample_tokens(T: int, n: int, seed: int = 0) -> np.ndarray:
    if T <= n:
        return np.arange(T)
    rng = np.random.default_rng(seed)
    s = set(rng.choice(T, n - 4, replace=False).tolist()) | {0, 1, T - 2, T - 1}
    return np.array(sorted(s))


def check_output(w: Workload, inp: dict, P: np.ndarray, r: dict, tokens=None, act="tanh") -> float:
    idx = gpu_selection(r)
    g = np.where(idx >= 0, np.take_along_axis(P, np.maximum(idx, 0), axis=1), 0.0)
    tok = np.arange(w.T) if tokens is None else np.asarray(tokens)
    ref = O.layer_output(inp, idx, g, tokens=tok, act=act)
    err = rel_err(r["out"][tok], ref)
    assert err <= out_tol(w), f"output normwise max rel err {err:.3e} > {out_tol(w):.0e}"
    return err


def full_check(w: Workload, inp: dict, gemm_impl="auto", tokens=None, act="tanh", **layer_opts) -> dict:
    L, x = run_layer(w, inp, gemm_impl, act=act, **layer_opts)
    r = fetch(L)
    P = O.softmax_scores(O.gate_logits(inp["x"], inp["wg"], inp.get("router_bias")))
    rep = check_routing(w, P, r, inp)
    loss = check_counts_loss(w, P, r)
    check_permutation(w, L, r, x)
    err = check_output(w, inp, P, r, tokens, act)
    return {"err": err, "aux_ref": loss, "flips": rep["flips"], "free": rep["free"], "layer": L, "res": r}
