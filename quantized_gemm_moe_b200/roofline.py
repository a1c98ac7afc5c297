"""Algorithmic work of one QE linear layer: the operation and byte counts behind
the reported TOPS and roofline fractions.

Counts are of what the method must do, not of what a kernel happens to move:
* int ops: the quantized product, 2*T*K*N (one multiply and one add per MAC).
* bf16 flops: the adapters and the router. The shared expert costs
  2*T*(K+N)*r_s, the routed expert 2*T*(K+N)*r_r (one expert per token), and
  the router 2*T*K*N_r.
* bytes: X once (2 B per element for bf16), the packed codes (b_w/8 B per weight),
  the group scales (fp32, or fp16), the shared adapters, the routed adapters that are touched
  (at most min(T, N_r) experts), the router, and Y once.
With d_in = d_out = d and r_s = r_r = r/2, (int ops + bf16 flops)/2 equals the
QE row of the complexity table on the thelatestinai listing (Table 7):
s*d^2 + s*d*(2r + N_r) MACs. Memory in parameters is d^2 + r*d*(1 + N_r).
"""
from __future__ import annotations


def int_ops(T: int, K: int, N: int) -> int:
    return 2 * T * K * N


def adapter_flops(T: int, K: int, N: int, r_s: int, n_r: int, r_r: int) -> int:
    return 2 * T * (K + N) * (r_s + r_r) + 2 * T * K * n_r


def layer_bytes(T: int, K: int, N: int, group: int, w_bits: int, r_s: int, n_r: int, r_r: int,
                x_bytes: int = 2, y_bytes: int = 2, scale_bytes: int = 4) -> int:
    """scale_bytes: 4 for fp32 group scales, 2 for fp16."""
    return (x_bytes * T * K + (K * N * w_bits) // 8 + scale_bytes * N * (K // group) + 2 * (K + N) * r_s
            + min(T, n_r) * 2 * (K + N) * r_r + 2 * K * n_r + y_bytes * T * N)


def table7_macs(s: int, d: int, r: int, n_r: int) -> int:
    """QE linear computation from the complexity table: s*d^2 + s*d*(2r + N_r)."""
    return s * d * d + s * d * (2 * r + n_r)


def table7_params(d: int, r: int, n_r: int) -> int:
    """QE linear memory from the complexity table: d^2 + r*d*(1 + N_r)."""
    return d * d + r * d * (1 + n_r)


def layer_params(K: int, N: int, r_s: int, n_r: int, r_r: int) -> int:
    """Weights plus adapters (router excluded): K*N + (K+N)*r_s + N_r*(K+N)*r_r."""
    return K * N + (K + N) * r_s + n_r * (K + N) * r_r


def topk_bytes(T: int, K: int, k: int, x_bytes: int = 2) -> int:
    """The importance statistic reads X and w once and writes the indices and the histogram."""
    return x_bytes * T * K + 4 * K + 4 * T * k + 4 * K
