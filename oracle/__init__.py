"""CPU oracle for the Quant Experts (QE) linear layer -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
leg may import this package. The product path (quantized_gemm_moe_b200) never
does, and it shares no code with it.

The arithmetic lives in qe_oracle.c (plain loops, IEEE fp32 for the steps
that decide integer codes, then int64 / fp64). This module only marshals
numpy arrays through ctypes. fixtures.py builds the low-rank adapters of the
pages' construction (whitened SVD of the quantization error) for the
invariant checks.

Parity status per function (pins live in tests/test_oracle_pins.py):
  quantize_weights, act_quant  pinned: grid round-trip, per-row RTN at g=K, hand cases; fp16 scales:
                               numpy's binary16 rounding, an on-grid round trip, a hand case
  smoothing_inverse            pinned: nearest fp32 to 1/s (neighbour check in fp64), powers of two exact
  route, bucket                pinned: brute-force argmin / stable sort, permutation
  group_acc                    pinned: bound |acc| <= g*qmax_a*qmax_w, numpy int64
  qe_forward                   pinned: zero adapters = literal dequant matmul,
                               token independence, identical experts, SVD fixture
  topk                         pinned: brute force, sum(hist) = T*k, order
  split_channels               pinned: a hand-ranked example with ties, d_in < k + C, count order
  cooccurrence, npmi           pinned: a hand-counted example, symmetry, diagonal = channel counts,
                               closed-form NPMI cases (independent 0, always together 1, never -1)
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i = ctypes.c_int
        L.oracle_quantize_weights.argtypes = [P, P, i, i, i, i, i, P, P, P, P]
        L.oracle_act_quant.argtypes = [P, P, i, i, i, P, P]
        L.oracle_route.argtypes = [P, P, i, i, i, P, P]
        L.oracle_bucket.argtypes = [P, i, i, P, P]
        L.oracle_group_acc.argtypes = [P, P, i, i, i, i, P]
        L.oracle_qe_forward.argtypes = [P, i, i, i, i, i, P, P, P, P, P, i, P, P, i, i, P, P, i, P, P, P]
        L.oracle_topk.argtypes = [P, P, i, i, i, P, P]
        L.oracle_round_bf16.argtypes = [ctypes.c_float]
        L.oracle_round_bf16.restype = ctypes.c_float
        L.oracle_round_fp16.argtypes = [ctypes.c_float]
        L.oracle_round_fp16.restype = ctypes.c_float
        for name in ("oracle_quantize_weights", "oracle_act_quant", "oracle_route", "oracle_bucket",
                     "oracle_group_acc", "oracle_qe_forward", "oracle_topk"):
            getattr(L, name).restype = ctypes.c_int
        _LIB = L
    return _LIB


def _f32(a) -> np.ndarray:
    if hasattr(a, "float") and not isinstance(a, np.ndarray):  # torch tensor (bf16 or fp32)
        a = a.float().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def quantize_weights(W, s, group: int, bits: int, scale_fp16: bool = False):
    """codes [N,K] int8, scales [N,K/group] fp32, w_mean [K], w_colmax [K].

    scale_fp16: the group scales are stored as fp16 (the fp32 scale rounded to nearest even,
    saturating at 65504) and the codes are computed from the stored scale; `scales` then holds
    those fp16 values widened to fp32."""
    W = _f32(W)
    s = _f32(s)
    N, K = W.shape
    codes = np.zeros((N, K), np.int8)
    scales = np.zeros((N, K // group), np.float32)
    w_mean = np.zeros(K, np.float32)
    w_colmax = np.zeros(K, np.float32)
    _check(lib().oracle_quantize_weights(_p(W), _p(s), N, K, group, bits, 1 if scale_fp16 else 0, _p(codes),
                                         _p(scales), _p(w_mean), _p(w_colmax)), "quantize_weights")
    return codes, scales, w_mean, w_colmax


def smoothing_inverse(s) -> np.ndarray:
    """The stored smoothing factor of the activations ([DR] \u00a7Method, Shared Expert: activations are
    divided by s): s_inv[k] = fl32(1/s[k]), one IEEE fp32 division per channel (numpy float32
    division is correctly rounded)."""
    s = _f32(s)
    return (np.float32(1.0) / s).astype(np.float32)


def act_quant(X, s_inv, bits: int):
    """codes [T,K] int8, sa [T] fp32 (token order)."""
    X = _f32(X)
    s_inv = _f32(s_inv)
    T, K = X.shape
    q = np.zeros((T, K), np.int8)
    sa = np.zeros(T, np.float32)
    _check(lib().oracle_act_quant(_p(X), _p(s_inv), T, K, bits, _p(q), _p(sa)), "act_quant")
    return q, sa


def route(X, G):
    """L [T,Nr] fp64, e [T] int32."""
    X = _f32(X)
    G = _f32(G)
    T, K = X.shape
    Nr = G.shape[1]
    L = np.zeros((T, Nr), np.float64)
    e = np.zeros(T, np.int32)
    _check(lib().oracle_route(_p(X), _p(G), T, K, Nr, _p(L), _p(e)), "route")
    return L, e


def bucket(e, Nr: int):
    """perm [T] (sorted position -> token), offsets [Nr+1]."""
    e = np.ascontiguousarray(e, dtype=np.int32)
    T = e.shape[0]
    perm = np.zeros(T, np.int32)
    offsets = np.zeros(Nr + 1, np.int32)
    _check(lib().oracle_bucket(_p(e), T, Nr, _p(perm), _p(offsets)), "bucket")
    return perm, offsets


def group_acc(xq, wq, group: int):
    """int64 [T, N, K/group]."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    T, K = xq.shape
    N = wq.shape[0]
    acc = np.zeros((T, N, K // group), np.int64)
    _check(lib().oracle_group_acc(_p(xq), _p(wq), T, N, K, group, _p(acc)), "group_acc")
    return acc


def qe_forward(X, codes, scales, s_inv, A_s, B_s, A_r, B_r, G, group: int, a_bits: int,
               rows=None, expert_override=None):
    """Y [n_rows, N] fp64 and the expert of each evaluated row.

    codes [N,K] int8, scales [N,K/group] (natural layout), adapters in their
    natural layouts: A_s [K,rs], B_s [rs,N], A_r [Nr,K,rr], B_r [Nr,rr,N], G [K,Nr].
    """
    X = _f32(X)
    T, K = X.shape
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    N = codes.shape[0]
    scales = _f32(scales)
    s_inv = _f32(s_inv)
    A_s, B_s, A_r, B_r, G = (_f32(a) for a in (A_s, B_s, A_r, B_r, G))
    rs = A_s.shape[1]
    Nr, _, rr = A_r.shape
    if rows is None:
        rows_a = None
        n = T
    else:
        rows_a = np.ascontiguousarray(rows, dtype=np.int32)
        n = rows_a.shape[0]
    ov = None if expert_override is None else np.ascontiguousarray(expert_override, dtype=np.int32)
    Y = np.zeros((n, N), np.float64)
    ex = np.zeros(n, np.int32)
    rc = lib().oracle_qe_forward(
        _p(X), T, K, N, group, a_bits, _p(codes), _p(scales), _p(s_inv),
        _p(A_s), _p(B_s), rs, _p(A_r), _p(B_r), Nr, rr, _p(G),
        None if rows_a is None else _p(rows_a), n,
        None if ov is None else _p(ov), _p(Y), _p(ex))
    _check(rc, "qe_forward")
    return Y, ex


def topk(X, w_mean, k: int):
    """idx [T,k] int32 ordered by (score desc, channel asc), hist [K] int32."""
    X = _f32(X)
    w_mean = _f32(w_mean)
    T, K = X.shape
    idx = np.zeros((T, k), np.int32)
    hist = np.zeros(K, np.int32)
    _check(lib().oracle_topk(_p(X), _p(w_mean), T, K, k, _p(idx), _p(hist)), "topk")
    return idx, hist


def round_bf16(v: float) -> float:
    return float(lib().oracle_round_bf16(ctypes.c_float(v)))


def round_fp16(v: float) -> float:
    return float(lib().oracle_round_fp16(ctypes.c_float(v)))


def qmax(bits: int) -> int:
    return (1 << (bits - 1)) - 1


def router_near_tie_bound(X, G) -> np.ndarray:
    """Per-token bound on fp32 rounding of the router logits. Two experts whose
    fp64 logits differ by less than this may legitimately swap order under
    fp32 accumulation: delta_t = 2*K*2^-24*sum_k |x_k|*max_e |G_k,e|."""
    X = _f32(X).astype(np.float64)
    G = _f32(G).astype(np.float64)
    K = X.shape[1]
    return 2.0 * K * 2.0 ** -24 * (np.abs(X) @ np.abs(G).max(axis=1))


def split_channels(hist, k: int, C: int) -> np.ndarray:
    """Token-dependent channel positions from the calibration histogram ([DR] \u00a7Method).

    Channels are ranked by how often they were in a token's Top-k set (higher count first, equal
    counts by lower channel index). The first k of that ranking are the token-independent channels
    the shared expert covers; the next C (= N_r * k) are the token-dependent ones. Returns int32
    [d_in]: rank - k for those C channels, -1 for every other channel.
    """
    h = np.asarray(hist, dtype=np.int64)
    d = h.shape[0]
    order = np.lexsort((np.arange(d), -h))   # primary key: count desc; then index asc
    pos = np.full(d, -1, dtype=np.int32)
    for r in range(k, min(k + C, d)):
        pos[order[r]] = r - k
    return pos


def cooccurrence(idx, channel_pos, C: int) -> np.ndarray:
    """Co-occurrence counts of the token-dependent channels ([DR] \u00a7Method, routed experts).

    idx [T][k]: each token's Top-k channel indices (qe_topk_importance). channel_pos [d_in]: the
    position in [0, C) of each token-dependent channel, -1 for every other channel. O[i][j] is the
    number of tokens whose important set holds both channels i and j; O[i][i] is how many tokens
    hold channel i. Built as the 0/1 token x channel indicator M, then O = M^T M in int64.
    """
    idx = np.asarray(idx, dtype=np.int64)
    pos = np.asarray(channel_pos, dtype=np.int64)
    T = idx.shape[0]
    M = np.zeros((T, C), dtype=np.int64)
    rows = np.repeat(np.arange(T), idx.shape[1])
    cols = pos[idx.ravel()]
    keep = cols >= 0
    M[rows[keep], cols[keep]] = 1
    return M.T @ M


def npmi(O, T: int, threshold: float = -1.0) -> np.ndarray:
    """Normalized pointwise mutual information of channel pairs ([DR] \u00a7Method), in fp64.

    p(i) = O[i][i] / T, p(i,j) = O[i][j] / T and S[i][j] = ln(p(i,j) / (p(i) p(j))) / (-ln p(i,j)).
    Readings where the formula is undefined: S = -1 when p(i,j) = 0 (the pair never co-occurs) and
    S = 1 when p(i,j) = 1 (both channels are in every token's set). Entries below `threshold` are
    set to 0 (the pages suggest 0.2); threshold <= -1 keeps every entry.
    """
    O = np.asarray(O, dtype=np.float64)
    p = O / float(T)
    pi = np.diag(p).copy()
    S = np.full(p.shape, -1.0)
    C = p.shape[0]
    for i in range(C):
        for j in range(C):
            pij = p[i, j]
            if pij <= 0.0:
                continue
            if pij >= 1.0:
                S[i, j] = 1.0
                continue
            S[i, j] = np.log(pij / (pi[i] * pi[j])) / (-np.log(pij))
    if threshold > -1.0:
        S = np.where(S >= threshold, S, 0.0)
    return S
