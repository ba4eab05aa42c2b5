"""The C-ABI library loads and exports every function include/moe.h declares.

Runs without a GPU: only host-side entry points that touch no device memory
are called (version, workspace sizing, row capacity, argument validation).
"""
import ctypes

import pytest

from sparse_moe_layer_03_b200 import binding as B


def test_library_exports_every_declared_symbol():
    names = B.header_symbols()
    assert len(names) >= 11
    for n in names:
        assert hasattr(B.lib, n), n
    # and the binding wraps each of them under the same name
    for n in names:
        assert hasattr(B, n), n


def test_version_and_sizes():
    assert B.moe_version() == 100
    cfg = B.make_config(32768, 1152, 4608, 8, 2, 2)
    assert B.moe_max_rows(cfg) == 67584     # round_up(65536 + 255*8, 256)
    assert B.moe_workspace_size(cfg) > 0
    race = B.make_config(32768, 1152, 4608, 16, 2, 1, routing="race")
    assert B.moe_workspace_size(race) > 32768 * 16 * 4
    f16 = B.make_config(32768, 1152, 4608, 8, 2, 2, dtype="f16")
    assert B.moe_workspace_size(f16) == B.moe_workspace_size(cfg)


@pytest.mark.parametrize("field,value,code", [
    ("K", 9, B.MOE_ERR_INVALID_ARG), ("E", 33, B.MOE_ERR_UNSUPPORTED), ("D", 100, B.MOE_ERR_UNSUPPORTED),
    ("T", -1, B.MOE_ERR_INVALID_ARG), ("n_shared", 9, B.MOE_ERR_UNSUPPORTED), ("dtype", 7, B.MOE_ERR_INVALID_ARG),
    ("routing", 3, B.MOE_ERR_INVALID_ARG), ("seq_len", -1, B.MOE_ERR_INVALID_ARG), ("seq_len", 7, B.MOE_ERR_INVALID_ARG),
])
def test_invalid_config_is_rejected_on_host(field, value, code):
    cfg = B.make_config(1024, 384, 1536, 8, 2, 2)
    setattr(cfg, field, value)
    assert B.lib.moe_workspace_size(ctypes.byref(cfg)) == 0
    rc = B.lib.moe_route(ctypes.byref(cfg), None, None, None, None, None, None, None, None, None, None, 0, None)
    assert rc == code
    assert B.lib.moe_last_error()


def test_null_and_misaligned_pointers_rejected_before_launch():
    cfg = B.make_config(1024, 384, 1536, 8, 2, 2)
    n = B.moe_workspace_size(cfg)
    fake = 1 << 40                          # never dereferenced: validation fails first
    rc = B.lib.moe_route(ctypes.byref(cfg), fake, fake, None, fake, fake, None, fake, None, None, fake, n, None)
    assert rc == B.MOE_ERR_INVALID_ARG and b"aux_loss" in B.lib.moe_last_error()
    rc = B.lib.moe_route(ctypes.byref(cfg), fake + 8, fake, None, fake, fake, None, fake, fake, None, fake, n, None)
    assert rc == B.MOE_ERR_INVALID_ARG and b"aligned" in B.lib.moe_last_error()
    rc = B.lib.moe_route(ctypes.byref(cfg), fake, fake, None, fake, fake, None, fake, fake, None, fake, n - 256, None)
    assert rc == B.MOE_ERR_WORKSPACE
    rc = B.lib.moe_route(ctypes.byref(cfg), fake, fake, None, fake, fake, None, fake, fake, None, fake + 16, n, None)
    assert rc == B.MOE_ERR_INVALID_ARG      # ws not 256-byte aligned
    race = B.make_config(1024, 384, 1536, 8, 2, 2, routing="race")
    n = B.moe_workspace_size(race)
    rc = B.lib.moe_route(ctypes.byref(race), fake, fake, None, fake, fake, None, fake, fake, None, fake, n, None)
    assert rc == B.MOE_ERR_INVALID_ARG and b"n_sel" in B.lib.moe_last_error()
    rc = B.lib.moe_combine(ctypes.byref(race), fake, fake, fake, None, None, fake, None)
    assert rc == B.MOE_ERR_INVALID_ARG
    # adaLN-Zero residual: img_len must divide T, pointers set and aligned
    cfg = B.make_config(1024, 384, 1536, 8, 2, 2)
    for res, word in [(B.MoeResidual(fake, fake, 300), b"img_len"), (B.MoeResidual(fake, None, 256), b"alpha"),
                      (B.MoeResidual(fake + 2, fake, 256), b"aligned")]:
        rc = B.lib.moe_combine(ctypes.byref(cfg), fake, fake, fake, None, ctypes.byref(res), fake, None)
        assert rc == B.MOE_ERR_INVALID_ARG and word in B.lib.moe_last_error()


def test_frequency_arguments_rejected_before_launch():
    cfg = B.make_config(1024, 384, 1536, 8, 2, 2)
    fake = 1 << 40                          # never dereferenced: validation fails first
    f = B.lib.moe_expert_frequency
    cases = [
        (0, None, 0, fake, b"seq_len"),          # seq_len < 1
        (100, None, 100, fake, b"divide"),        # 100 does not divide 1024
        (256, None, 255, fake, b"n_labels"),      # position labels need n_labels == seq_len
        (256, fake, 0, fake, b"n_labels"),        # no rows
        (256, None, 256, None, b"hist"),          # no output
    ]
    for seq_len, labels, n_labels, hist, word in cases:
        rc = f(ctypes.byref(cfg), fake, None, seq_len, labels, n_labels, hist, fake, None)
        assert rc == B.MOE_ERR_INVALID_ARG, (seq_len, n_labels)
        assert word in B.lib.moe_last_error()
    race = B.make_config(1024, 384, 1536, 8, 2, 2, routing="race")
    rc = f(ctypes.byref(race), fake, None, 256, None, 256, fake, fake, None)
    assert rc == B.MOE_ERR_INVALID_ARG and b"n_sel" in B.lib.moe_last_error()


def test_fused_combine_refuses_unsupported_configs_before_launch():
    fake = 1 << 40
    f = B.lib.moe_expert_gemm2_combine
    for cfg, why in [(B.make_config(1024, 384, 1536, 8, 2, 2, dtype="f32"), b"bf16"),
                     (B.make_config(1024, 384, 1536, 8, 2, 0), b"n_shared"),
                     (B.make_config(1024, 384, 1536, 8, 2, 2, gemm_impl="tc1"), b"AUTO")]:
        n = B.moe_workspace_size(cfg)
        rc = f(ctypes.byref(cfg), fake, fake, fake, fake, None, fake, None, fake, fake, None, fake, None, fake, fake, n,
               None)
        assert rc == B.MOE_ERR_UNSUPPORTED and why in B.lib.moe_last_error()
    cfg = B.make_config(1024, 384, 1536, 8, 2, 2)
    n = B.moe_workspace_size(cfg)
    rc = f(ctypes.byref(cfg), fake, fake, fake, fake, None, fake, None, fake, None, None, fake, None, fake, fake, n, None)
    assert rc == B.MOE_ERR_INVALID_ARG and b"pos" in B.lib.moe_last_error()


def test_python_wrappers_reach_the_library():
    # every wrapper marshals its arguments and reaches the C ABI (which then fails without a GPU,
    # or on the fake pointers, with its own error code rather than a Python TypeError)
    cfg = B.make_config(1024, 384, 1536, 8, 2, 2)
    n = B.moe_workspace_size(cfg)
    f = 1 << 40
    res = B.make_residual(f, f, 256)
    calls = [
        lambda: B.moe_route(cfg, f, f, None, f, f, f, f, f, f, n),
        lambda: B.moe_dispatch(cfg, f, f, f, f, f, f, f, f, f, f, n),
        lambda: B.moe_expert_gemm1(cfg, f, f, f, f, None, f, None, f, f, f, n),
        lambda: B.moe_expert_gemm2(cfg, f, f, f, f, None, f, None, f, f, f, f, n),
        lambda: B.moe_expert_gemm2_combine(cfg, f, f, f, f, None, f, None, f, f, None, f, f, f, n, res=res),
        lambda: B.moe_combine(cfg, f, f, f, None, f, res=res),
        lambda: B.moe_expert_frequency(cfg, f, None, 256, None, 256, f, f),
        lambda: B.moe_balance_stats(cfg, f, f, n, f),
        lambda: B.moe_balance_loss_from_stats(cfg, f, 2048, f),
    ]
    for c in calls:
        with pytest.raises(B.MoeError):
            c()



def test_modulation_arguments_rejected_before_launch():
    fake = 1 << 40
    cfg = B.make_config(1024, 384, 1536, 8, 2, 2)
    n = B.moe_workspace_size(cfg)
    f32 = B.make_config(1024, 384, 1536, 8, 2, 2, dtype="f32")
    nf = B.moe_workspace_size(f32)
    cases = [(cfg, n, B.MoeAdaln(fake, fake, 300, 1e-5, fake), B.MOE_ERR_INVALID_ARG, b"img_len"),
             (cfg, n, B.MoeAdaln(fake, fake, 256, 0.0, fake), B.MOE_ERR_INVALID_ARG, b"eps"),
             (cfg, n, B.MoeAdaln(fake, fake, 256, 1e-5, None), B.MOE_ERR_INVALID_ARG, b"x_mod"),
             (f32, nf, B.MoeAdaln(fake, fake, 256, 1e-5, fake), B.MOE_ERR_UNSUPPORTED, b"16-bit")]
    for c, nb, mod, code, word in cases:
        rc = B.lib.moe_route(ctypes.byref(c), fake, fake, None, fake, fake, None, fake, fake, ctypes.byref(mod),
                             fake, nb, None)
        assert rc == code and word in B.lib.moe_last_error(), B.lib.moe_last_error()


def test_balance_backward_arguments_rejected_before_launch():
    fake = 1 << 40
    cfg = B.make_config(1024, 384, 1536, 8, 2, 2)
    n = B.moe_backward_workspace_size(cfg)
    assert n >= 8 * 385 * 4
    f = B.lib.moe_balance_loss_backward
    assert f(ctypes.byref(cfg), fake, fake, None, fake, ctypes.c_float(1.0), None, None, None, fake, n, None) == \
        B.MOE_ERR_INVALID_ARG
    assert f(ctypes.byref(cfg), fake, fake, None, fake, ctypes.c_float(1.0), fake, None, None, fake, n - 4, None) == \
        B.MOE_ERR_WORKSPACE
    per_image = B.make_config(1024, 384, 1536, 8, 2, 2, seq_len=256)
    assert f(ctypes.byref(per_image), fake, fake, None, fake, ctypes.c_float(1.0), fake, None, None, fake, n, None) == \
        B.MOE_ERR_UNSUPPORTED


def test_balance_statistics_arguments_rejected_before_launch():
    fake = 1 << 40
    cfg = B.make_config(1024, 384, 1536, 8, 2, 2)
    n = B.moe_workspace_size(cfg)
    st = B.lib.moe_balance_stats
    assert st(ctypes.byref(cfg), fake, fake, n, None, None) == B.MOE_ERR_INVALID_ARG
    assert b"stats" in B.lib.moe_last_error()
    assert st(ctypes.byref(cfg), None, fake, n, fake, None) == B.MOE_ERR_INVALID_ARG
    assert st(ctypes.byref(cfg), fake, fake, n - 8, fake, None) == B.MOE_ERR_WORKSPACE
    lf = B.lib.moe_balance_loss_from_stats
    assert lf(ctypes.byref(cfg), fake, -1, fake, None) == B.MOE_ERR_INVALID_ARG
    assert b"T_total" in B.lib.moe_last_error()
    assert lf(ctypes.byref(cfg), fake, 1024, None, None) == B.MOE_ERR_INVALID_ARG
    assert lf(ctypes.byref(cfg), None, 1024, fake, None) == B.MOE_ERR_INVALID_ARG
    bad = B.make_config(1024, 384, 1536, 8, 9, 2)          # K > E
    assert lf(ctypes.byref(bad), fake, 1024, fake, None) == B.MOE_ERR_INVALID_ARG



def test_negative_gemm_pairs_rejected():
    fake = 1 << 40
    cfg = B.make_config(1024, 384, 1536, 8, 2, 2, gemm_pairs=-1)
    assert B.lib.moe_workspace_size(ctypes.byref(cfg)) == 0
    assert b"gemm_pairs" in B.lib.moe_last_error()
    ok = B.make_config(1024, 384, 1536, 8, 2, 2, gemm_pairs=3)
    assert B.lib.moe_workspace_size(ctypes.byref(ok)) > 0
    f = B.lib.moe_expert_gemm1
    assert f(ctypes.byref(cfg), fake, fake, fake, fake, None, fake, None, fake, fake, fake, 1 << 20, None) == \
        B.MOE_ERR_INVALID_ARG


def test_expert_backward_arguments_rejected_before_launch():
    fake = 1 << 40
    cfg = B.make_config(1024, 384, 1536, 8, 2, 2)
    n = B.moe_expert_backward_workspace_size(cfg)
    assert n > 0 and n % 256 == 0
    wsz = B.moe_workspace_size(cfg)
    w = B.MoeExpertWeights(*([fake] * 8))
    g = B.MoeExpertGrads(*([fake] * 8))
    f = B.lib.moe_expert_backward

    def call(c=cfg, wts=w, grads=g, bws_bytes=n, dgate=fake):
        return f(ctypes.byref(c), fake, fake, fake, fake, fake, fake, fake, fake,
                 ctypes.byref(wts) if wts is not None else None, fake, fake, fake,
                 ctypes.byref(grads) if grads is not None else None, dgate, fake, fake, wsz, fake, bws_bytes, None)
    f32 = B.make_config(1024, 384, 1536, 8, 2, 2, dtype="f32")
    assert call(c=f32) == B.MOE_ERR_UNSUPPORTED and b"bf16" in B.lib.moe_last_error()
    erf = B.make_config(1024, 384, 1536, 8, 2, 2, act="erf")
    assert call(c=erf) == B.MOE_ERR_UNSUPPORTED
    assert call(wts=None) == B.MOE_ERR_INVALID_ARG
    assert call(bws_bytes=n - 256) == B.MOE_ERR_WORKSPACE
    assert call(dgate=None) == B.MOE_ERR_INVALID_ARG and b"dgate" in B.lib.moe_last_error()
    bad = B.MoeExpertGrads(None, fake, fake, fake, fake, fake, fake, fake)
    assert call(grads=bad) == B.MOE_ERR_INVALID_ARG and b"dw1" in B.lib.moe_last_error()
    rb = B.lib.moe_router_backward
    nb = B.moe_backward_workspace_size(cfg)
    # accumulating into dx needs dx; the gates' gradient needs the selection
    assert rb(ctypes.byref(cfg), fake, fake, None, fake, fake, None, None, ctypes.c_float(1.0), fake, None, None, 1,
              fake, nb, None) == B.MOE_ERR_INVALID_ARG
    assert rb(ctypes.byref(cfg), fake, fake, None, fake, None, None, fake, ctypes.c_float(1.0), fake, None, None, 0,
              fake, nb, None) == B.MOE_ERR_INVALID_ARG
