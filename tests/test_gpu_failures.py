"""Failure detection on the GPU without faulting it.

The two waits on global memory (the fused GEMM2's wait for the routed tiles, the
Expert-Race selection's grid barriers) are bounded.  Two test words in the
workspace header, written only by the host, make each wait impossible to satisfy
and shorten its limit to a millisecond: the kernel must then return, the status
word must report MOE_ERR_TIMEOUT, and the next call on the same workspace (words
cleared) must be correct again.  Also here: the expert GEMMs restricted to a few
CTA pairs (``gemm_pairs``) give the oracle's result, with the combine folded in.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_moe_layer_03_b200 import binding as B
from sparse_moe_layer_03_b200 import inputs as I
from tests import parity as PA

pytestmark = pytest.mark.gpu

SKIP_ROUTED_COUNT = 1      # bit 0 of the flags word
RACE_EXTRA_ARRIVAL = 2     # bit 1


def _set_test_words(L, flags: int, limit_us: int):
    L.ws[240:248].view(torch.int32).copy_(torch.tensor([flags, limit_us], dtype=torch.int32))


def _expect_timeout(L):
    torch.cuda.synchronize()
    with pytest.raises(B.MoeError) as ei:
        L.check()
    assert ei.value.code == B.MOE_ERR_TIMEOUT
    # moe_check_status clears the header (status, counters and test words) after an error
    assert int(L.ws[:256].count_nonzero()) == 0


def test_fused_combine_wait_runs_out_and_the_next_call_is_clean():
    w = I.small_workload(1000, 256, 512, 8, 2, 2, "bf16", "topk", seed=41)
    inp = I.make_inputs(w, bias_std=0.2)
    L, x = PA.run_layer(w, inp)
    assert L.fused
    _set_test_words(L, SKIP_ROUTED_COUNT, 1000)
    L.forward(x)
    _expect_timeout(L)
    # same workspace, words cleared: correct again
    L.out.zero_()
    L.forward(x)
    torch.cuda.synchronize()
    L.check()
    r = PA.fetch(L)
    P = O.softmax_scores(O.gate_logits(inp["x"], inp["wg"], inp.get("router_bias")))
    PA.check_output(w, inp, P, r)


def test_race_grid_barrier_runs_out_and_the_next_call_is_clean():
    w = I.small_workload(2000, 256, 512, 16, 2, 1, "bf16", "race", seed=43)
    inp = I.make_inputs(w, bias_std=0.2)
    L, x = PA.run_layer(w, inp)
    _set_test_words(L, RACE_EXTRA_ARRIVAL, 1000)
    L.route(x)
    _expect_timeout(L)
    rep = PA.full_check(w, inp)          # a fresh layer: the normal path
    L.forward(x)                          # and the old workspace, words cleared
    torch.cuda.synchronize()
    L.check()
    assert torch.equal(L.topk_idx.cpu(), torch.as_tensor(rep["res"]["topk_idx"]))
    r = PA.fetch(L)
    P = O.softmax_scores(O.gate_logits(inp["x"], inp["wg"], inp.get("router_bias")))
    PA.check_routing(w, P, r, inp)
    PA.check_output(w, inp, P, r)


@pytest.mark.parametrize("pairs", [1, 3, 17])
def test_expert_gemms_on_few_cta_pairs(pairs):
    # the folded combine's shared tiles wait for routed tiles: with one pair the same pair
    # runs every routed tile before any shared one
    for routing in ("topk", "race"):
        w = I.small_workload(1200, 256, 512, 8, 2, 2, "bf16", routing, seed=47 + pairs)
        inp = I.make_inputs(w, bias_std=0.2)
        rep = PA.full_check(w, inp, gemm_pairs=pairs)
        assert rep["layer"].fused and rep["layer"].cfg.gemm_pairs == pairs
        assert rep["err"] <= PA.out_tol(w)


def test_few_pairs_full_size_xl_matches_all_pairs():
    # the result does not depend on how many pairs run: bit-identical at XL
    w = I.WORKLOADS["xl2_8e2a_512"]
    inp = I.make_inputs(w)
    a, _ = PA.run_layer(w, inp)
    out_all = a.out.clone()
    del a
    b, _ = PA.run_layer(w, inp, gemm_pairs=5)
    assert torch.equal(b.out, out_all)
