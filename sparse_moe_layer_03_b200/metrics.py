"""Work accounting for the layer: algorithmic FLOPs and bytes per call.

FLOP convention: 2 FLOP per multiply-accumulate.  The DiT pages count model
cost with thop, whose "Gflops" are multiply-accumulates (the DiT-XL/2 figures
118.6 and 524.6 are reproduced by counting MACs; a test pins this).

Only the work the method asks for is counted: unselected experts and the
padding rows of the expert-contiguous layout are not.
"""
from __future__ import annotations


def mlp_macs_per_token(D: int, H: int) -> int:
    """Multiply-accumulates of one expert MLP W2 gelu(W1 x) on one token."""
    return 2 * D * H


def gemm_flops(T: int, D: int, H: int, K: int, n_shared: int) -> int:
    """Expert GEMM FLOPs of one layer call: S = K*T routed pairs plus n_s*T shared."""
    return 2 * mlp_macs_per_token(D, H) * (K * T + n_shared * T)


def gemm1_flops(T, D, H, K, n_shared):
    return 2 * D * H * (K * T + n_shared * T)


def gemm2_flops(T, D, H, K, n_shared):
    return 2 * D * H * (K * T + n_shared * T)


def route_bytes(T, D, E, K, elem, race=False):
    """x read once, plus the per-token selection written (index + weight)."""
    kmax = E if race else K
    b = T * D * elem + T * kmax * 8
    if race:
        b += T * E * 4 * 2 + T * 4      # score matrix written and re-read, n_sel
    return b


def dispatch_bytes(T, D, E, K, elem, race=False):
    """x read once, one row written per selected pair, plus index traffic."""
    S = K * T
    kmax = E if race else K
    return T * D * elem + S * D * elem + T * kmax * 4 * 2 + S * 8


def combine_bytes(T, D, K, n_shared, elem, y_elem=None):
    """Routed rows and the shared row read, output written, positions read."""
    S = K * T
    y_elem = elem if y_elem is None else y_elem      # expert outputs are stored in the act dtype
    b = S * D * y_elem + T * D * elem + T * K * 4
    if n_shared > 0:
        b += T * D * y_elem
    return b
