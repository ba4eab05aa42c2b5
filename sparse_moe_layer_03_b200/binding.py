"""ctypes binding of ``libmoe.so``: the C-ABI entry points under the same names.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Tensors are passed as device pointers (``torch.Tensor.data_ptr()``)
and the stream as a raw ``cudaStream_t``.  Importing this module loads the
library and raises if it is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "moe.h")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE = 0, -1, -2, -3
MOE_ERR_CUDA, MOE_ERR_DEVICE_CHECK, MOE_ERR_TIMEOUT = -4, -5, -6
MOE_F32, MOE_BF16, MOE_F16 = 0, 1, 2
MOE_ROUTE_TOPK, MOE_ROUTE_RACE = 0, 1
MOE_GEMM_AUTO, MOE_GEMM_SIMT, MOE_GEMM_TC1 = 0, 1, 2


class MoeConfig(C.Structure):
    _fields_ = [("T", C.c_int32), ("D", C.c_int32), ("H", C.c_int32), ("E", C.c_int32),
                ("K", C.c_int32), ("n_shared", C.c_int32), ("dtype", C.c_int32),
                ("routing", C.c_int32), ("alpha", C.c_float), ("act", C.c_int32),
                ("gemm_impl", C.c_int32), ("seq_len", C.c_int32), ("gemm_pairs", C.c_int32)]


class MoeAdaln(C.Structure):
    _fields_ = [("gamma", C.c_void_p), ("beta", C.c_void_p), ("img_len", C.c_int32), ("eps", C.c_float),
                ("x_mod", C.c_void_p)]


def make_adaln(gamma, beta, img_len, eps, x_mod):
    """adaLN modulation done by the router: x_mod = gamma[image] * LayerNorm(x) + beta[image]; None for none."""
    if gamma is None:
        return None
    return MoeAdaln(_ptr(gamma), _ptr(beta), img_len, eps, _ptr(x_mod))


class MoeResidual(C.Structure):
    _fields_ = [("x_res", C.c_void_p), ("alpha", C.c_void_p), ("img_len", C.c_int32)]


def make_residual(x_res, alpha, img_len):
    """adaLN-Zero residual for the combine: out = x_res + alpha[image] * MoE(x); None for MoE(x) alone."""
    if x_res is None:
        return None
    return MoeResidual(_ptr(x_res), _ptr(alpha), img_len)


def _res_ref(r):
    return None if r is None else C.byref(r)


class MoeExpertWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("w1", "b1", "w2", "b2", "w1s", "b1s", "w2s", "b2s")]


class MoeExpertGrads(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("dw1", "db1", "dw2", "db2", "dws1", "dbs1", "dws2", "dbs2")]


def make_expert_weights(w1, b1, w2, b2, w1s, b1s, w2s, b2s):
    return MoeExpertWeights(*[_ptr(t) for t in (w1, b1, w2, b2, w1s, b1s, w2s, b2s)])


def make_expert_grads(dw1, db1, dw2, db2, dws1, dbs1, dws2, dbs2):
    return MoeExpertGrads(*[_ptr(t) for t in (dw1, db1, dw2, db2, dws1, dbs1, dws2, dbs2)])


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"moe error {code}: {msg}")
        self.code = code


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m sparse_moe_layer_03_b200.build` "
                      "(the CUDA library is required; there is no CPU path)")
lib = C.CDLL(LIB_PATH)

_P = C.c_void_p
_CFG = C.POINTER(MoeConfig)
_SIGS = {
    "moe_version": (C.c_int32, []),
    "moe_last_error": (C.c_char_p, []),
    "moe_workspace_size": (C.c_size_t, [_CFG]),
    "moe_max_rows": (C.c_int64, [_CFG]),
    "moe_workspace_init": (C.c_int, [_P, C.c_size_t, _P]),
    "moe_check_status": (C.c_int, [_P, _P]),
    "moe_route": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, C.c_size_t, _P]),
    "moe_dispatch": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, C.c_size_t, _P]),
    "moe_expert_gemm1": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, C.c_size_t, _P]),
    "moe_expert_gemm1_gather": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, C.c_size_t, _P]),
    "moe_expert_gemm2": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, C.c_size_t, _P]),
    "moe_expert_mlp": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                 _P, C.c_size_t, _P]),
    "moe_combine": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P]),
    "moe_route_static": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_route_static_check_status": (C.c_int, [_P]),
    "moe_expert_frequency": (C.c_int, [_CFG, _P, _P, C.c_int32, _P, C.c_int32, _P, _P, _P]),
    "moe_backward_workspace_size": (C.c_size_t, [_CFG]),
    "moe_balance_loss_backward": (C.c_int, [_CFG, _P, _P, _P, _P, C.c_float, _P, _P, _P, _P, C.c_size_t, _P]),
    "moe_balance_stats": (C.c_int, [_CFG, _P, _P, C.c_size_t, _P, _P]),
    "moe_balance_loss_from_stats": (C.c_int, [_CFG, _P, C.c_longlong, _P, _P]),
    "moe_expert_gemm2_combine": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                           C.c_size_t, _P]),
    "moe_expert_backward_workspace_size": (C.c_size_t, [_CFG]),
    "moe_expert_backward": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, C.POINTER(MoeExpertWeights), _P, _P,
                                      _P, C.POINTER(MoeExpertGrads), _P, _P, _P, C.c_size_t, _P, C.c_size_t, _P]),
    "moe_router_backward": (C.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, C.c_float, _P, _P, _P, C.c_int32, _P,
                                      C.c_size_t, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def header_symbols(path: str = HEADER) -> list:
    """Names of the functions that include/moe.h declares."""
    text = open(path).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\*\s]+?\b(moe_\w+)\s*\(", text, re.M)))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _check(rc: int):
    if rc != MOE_OK:
        raise MoeError(rc, lib.moe_last_error().decode())


def make_config(T, D, H, E, K, n_shared, dtype="bf16", routing="topk", alpha=0.01, act="tanh",
                gemm_impl="auto", seq_len=0, gemm_pairs=0) -> MoeConfig:
    return MoeConfig(T, D, H, E, K, n_shared, {"f32": MOE_F32, "bf16": MOE_BF16, "f16": MOE_F16}[dtype],
                     MOE_ROUTE_RACE if routing == "race" else MOE_ROUTE_TOPK, alpha,
                     1 if act == "erf" else 0,
                     {"auto": MOE_GEMM_AUTO, "simt": MOE_GEMM_SIMT, "tc1": MOE_GEMM_TC1}[gemm_impl], seq_len,
                     gemm_pairs)


def moe_version() -> int:
    return lib.moe_version()


def moe_workspace_size(cfg: MoeConfig) -> int:
    n = lib.moe_workspace_size(C.byref(cfg))
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, lib.moe_last_error().decode())
    return n


def moe_max_rows(cfg: MoeConfig) -> int:
    n = lib.moe_max_rows(C.byref(cfg))
    if n < 0:
        raise MoeError(MOE_ERR_INVALID_ARG, lib.moe_last_error().decode())
    return n


def moe_workspace_init(ws, ws_bytes, stream=0):
    _check(lib.moe_workspace_init(_ptr(ws), ws_bytes, stream))


def moe_check_status(ws, stream=0):
    _check(lib.moe_check_status(_ptr(ws), stream))


def moe_route(cfg, x, wg, router_bias, topk_idx, topk_w, n_sel, counts, aux_loss, ws, ws_bytes, stream=0, mod=None):
    _check(lib.moe_route(C.byref(cfg), _ptr(x), _ptr(wg), _ptr(router_bias), _ptr(topk_idx), _ptr(topk_w),
                         _ptr(n_sel), _ptr(counts), _ptr(aux_loss), _res_ref(mod), _ptr(ws), ws_bytes, stream))


def moe_dispatch(cfg, x, topk_idx, topk_w, n_sel, offsets, pos, row_token, row_gate, x_perm, ws, ws_bytes,
                 stream=0):
    _check(lib.moe_dispatch(C.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(topk_w), _ptr(n_sel), _ptr(offsets),
                            _ptr(pos), _ptr(row_token), _ptr(row_gate), _ptr(x_perm), _ptr(ws), ws_bytes, stream))


def moe_expert_gemm1(cfg, offsets, x_perm, x, w1, b1, w1s, b1s, h_perm, h_sh, ws, ws_bytes, stream=0):
    _check(lib.moe_expert_gemm1(C.byref(cfg), _ptr(offsets), _ptr(x_perm), _ptr(x), _ptr(w1), _ptr(b1),
                                _ptr(w1s), _ptr(b1s), _ptr(h_perm), _ptr(h_sh), _ptr(ws), ws_bytes, stream))


def moe_expert_gemm1_gather(cfg, offsets, row_token, x, w1, b1, w1s, b1s, h_perm, h_sh, ws, ws_bytes, stream=0):
    """GEMM1 reading its routed rows straight from x (cp.async by row_token): no x_perm."""
    _check(lib.moe_expert_gemm1_gather(C.byref(cfg), _ptr(offsets), _ptr(row_token), _ptr(x), _ptr(w1), _ptr(b1),
                                       _ptr(w1s), _ptr(b1s), _ptr(h_perm), _ptr(h_sh), _ptr(ws), ws_bytes, stream))


def moe_expert_gemm2(cfg, offsets, h_perm, h_sh, w2, b2, w2s, b2s, row_gate, y_perm, y_sh, ws, ws_bytes,
                     stream=0):
    _check(lib.moe_expert_gemm2(C.byref(cfg), _ptr(offsets), _ptr(h_perm), _ptr(h_sh), _ptr(w2), _ptr(b2),
                                _ptr(w2s), _ptr(b2s), _ptr(row_gate), _ptr(y_perm), _ptr(y_sh), _ptr(ws),
                                ws_bytes, stream))


def moe_expert_mlp(cfg, offsets, x_perm, x, w1, b1, w2, b2, w1s, b1s, w2s, b2s, row_gate, h_perm, h_sh, y_perm,
                   y_sh, ws, ws_bytes, stream=0):
    _check(lib.moe_expert_mlp(C.byref(cfg), _ptr(offsets), _ptr(x_perm), _ptr(x), _ptr(w1), _ptr(b1), _ptr(w2),
                              _ptr(b2), _ptr(w1s), _ptr(b1s), _ptr(w2s), _ptr(b2s), _ptr(row_gate), _ptr(h_perm),
                              _ptr(h_sh), _ptr(y_perm), _ptr(y_sh), _ptr(ws), ws_bytes, stream))


def moe_combine(cfg, y_perm, y_sh, pos, n_sel, out, stream=0, res=None):
    _check(lib.moe_combine(C.byref(cfg), _ptr(y_perm), _ptr(y_sh), _ptr(pos), _ptr(n_sel), _res_ref(res), _ptr(out),
                           stream))


def moe_last_error() -> str:
    return lib.moe_last_error().decode()


def moe_route_static(cfg, x, wg, router_bias, topk_idx, topk_w, n_sel, counts, aux_loss, stream=0):
    """moe_route without a workspace: scratch comes from the library's built-in 4 MiB array."""
    _check(lib.moe_route_static(C.byref(cfg), _ptr(x), _ptr(wg), _ptr(router_bias), _ptr(topk_idx), _ptr(topk_w),
                                _ptr(n_sel), _ptr(counts), _ptr(aux_loss), stream))


def moe_route_static_check_status(stream=0):
    """Read and clear the first device-detected error of moe_route_static's calls (blocks)."""
    _check(lib.moe_route_static_check_status(stream))


def moe_expert_frequency(cfg, topk_idx, n_sel, seq_len, seq_labels, n_labels, hist, ws, stream=0):
    """Expert-selection counts per label: patch position (seq_labels None) or each image's label."""
    _check(lib.moe_expert_frequency(C.byref(cfg), _ptr(topk_idx), _ptr(n_sel), seq_len, _ptr(seq_labels),
                                    n_labels, _ptr(hist), _ptr(ws), stream))


def moe_expert_gemm2_combine(cfg, offsets, h_perm, h_sh, w2, b2, w2s, b2s, row_gate, pos, n_sel, y_perm, out, ws,
                             ws_bytes, stream=0, res=None):
    """GEMM2 with the combine folded into the shared experts' tiles: writes out [T,D] directly."""
    _check(lib.moe_expert_gemm2_combine(C.byref(cfg), _ptr(offsets), _ptr(h_perm), _ptr(h_sh), _ptr(w2), _ptr(b2),
                                        _ptr(w2s), _ptr(b2s), _ptr(row_gate), _ptr(pos), _ptr(n_sel), _ptr(y_perm),
                                        _res_ref(res), _ptr(out), _ptr(ws), ws_bytes, stream))


def moe_backward_workspace_size(cfg) -> int:
    n = lib.moe_backward_workspace_size(C.byref(cfg))
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, lib.moe_last_error().decode())
    return n


def moe_balance_stats(cfg, counts, ws, ws_bytes, stats, stream=0):
    """[counts, score sums] of the last moe_route on ws, as [2E] fp64 (summable over ranks)."""
    _check(lib.moe_balance_stats(C.byref(cfg), _ptr(counts), _ptr(ws), ws_bytes, _ptr(stats), stream))


def moe_balance_loss_from_stats(cfg, stats, T_total, aux_loss, stream=0):
    """Balance loss of a whole batch from its summed [2E] statistics and its token count."""
    _check(lib.moe_balance_loss_from_stats(C.byref(cfg), _ptr(stats), int(T_total), _ptr(aux_loss), stream))


def moe_balance_loss_backward(cfg, x, wg, router_bias, counts, grad_scale, dwg, dbias, dx, bws, bws_bytes, stream=0):
    """Gradient of the balance loss through the router: dWg [E,D], db [E] (fp32) and dx [T,D] (act)."""
    _check(lib.moe_balance_loss_backward(C.byref(cfg), _ptr(x), _ptr(wg), _ptr(router_bias), _ptr(counts),
                                         grad_scale, _ptr(dwg), _ptr(dbias), _ptr(dx), _ptr(bws), bws_bytes, stream))


def moe_expert_backward_workspace_size(cfg) -> int:
    n = lib.moe_expert_backward_workspace_size(C.byref(cfg))
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, lib.moe_last_error().decode())
    return n


def moe_expert_backward(cfg, x, x_perm, offsets, pos, topk_idx, n_sel, row_token, row_gate, weights, h_perm, h_sh,
                        dout, grads, dgate, dx, ws, ws_bytes, bws, bws_bytes, stream=0):
    """Gradients of the expert MLPs (weights, biases), of the gates and the experts' part of dx."""
    _check(lib.moe_expert_backward(C.byref(cfg), _ptr(x), _ptr(x_perm), _ptr(offsets), _ptr(pos), _ptr(topk_idx),
                                   _ptr(n_sel), _ptr(row_token), _ptr(row_gate), C.byref(weights), _ptr(h_perm),
                                   _ptr(h_sh), _ptr(dout), C.byref(grads), _ptr(dgate), _ptr(dx), _ptr(ws), ws_bytes,
                                   _ptr(bws), bws_bytes, stream))


def moe_router_backward(cfg, x, wg, router_bias, counts, topk_idx, n_sel, dgate, aux_scale, dwg, dbias, dx,
                        dx_accumulate, bws, bws_bytes, stream=0):
    """The router's gradients (dWg, db, dx) from the gates' gradient and the balance loss."""
    _check(lib.moe_router_backward(C.byref(cfg), _ptr(x), _ptr(wg), _ptr(router_bias), _ptr(counts), _ptr(topk_idx),
                                   _ptr(n_sel), _ptr(dgate), aux_scale, _ptr(dwg), _ptr(dbias), _ptr(dx),
                                   int(dx_accumulate), _ptr(bws), bws_bytes, stream))
