"""GPU parity of the calibration statistics: channel split, co-occurrence counts and NPMI.

Channel positions and counts are integers and must match the oracle bit for bit. NPMI is
computed in fp64 on both sides and rounded once to fp32 on the GPU, so the two agree to
1e-6 absolute; thresholded entries are compared away from the threshold (|S - thr| > 1e-9).
"""
import numpy as np
import pytest
import torch

import oracle
import qe_inputs as qi
import quantized_gemm_moe_b200 as qe
from gpu_util import cuda

pytestmark = pytest.mark.gpu

S_TOL = 1e-6


def _i32(a):
    return cuda(np.ascontiguousarray(a, dtype=np.int32))


def _split(hist, k, C):
    pos = torch.full((len(hist),), 12345, dtype=torch.int32, device="cuda")
    qe.split_channels(_i32(hist), k, C, pos)
    torch.cuda.synchronize()
    return pos.cpu().numpy()


@pytest.mark.parametrize("d,k,C,hi,seed", [
    (7, 2, 3, 10, 0), (500, 16, 128, 6, 1), (1536, 32, 256, 4, 2), (29568, 32, 256, 8192, 3),
    (100, 0, 50, 3, 4), (40, 16, 128, 5, 5), (5000, 128, 4096, 2, 6), (3000, 8, 64, 1, 7),
    (1000, 8, 64, 0, 10), (40000, 32, 256, 3000, 11), (70000, 16, 1024, 1 << 20, 12),
])
def test_split_channels_bit_exact(d, k, C, hi, seed):
    hist = np.random.default_rng(seed).integers(0, hi + 1, size=d)
    if d > 10:
        hist[: d // 10] = hi                 # a block of equal top counts
    assert (_split(hist, k, C) == oracle.split_channels(hist, k, C)).all()


def test_split_channels_signed_and_large_counts():
    rng = np.random.default_rng(8)
    hist = rng.integers(-(1 << 31), (1 << 31) - 1, size=3000, dtype=np.int64)
    hist[100:140] = (1 << 31) - 1
    hist[200:260] = -(1 << 31)
    assert (_split(hist, 20, 100) == oracle.split_channels(hist, 20, 100)).all()
    assert (_split(hist, 0, 3000) == oracle.split_channels(hist, 0, 3000)).all()


def _cooc(idx, pos, C, threshold=-1.0, with_s=True):
    O = torch.full((C, C), -7, dtype=torch.int32, device="cuda")
    S = torch.full((C, C), 9.0, dtype=torch.float32, device="cuda") if with_s else None
    qe.cooccurrence_npmi(_i32(idx), _i32(pos), C, O, S, threshold)
    torch.cuda.synchronize()
    return O.cpu().numpy(), (S.cpu().numpy() if with_s else None)


def _check_npmi(S, O, T, threshold):
    threshold = float(np.float32(threshold))     # the C ABI takes the threshold as fp32
    S_ref = oracle.npmi(O.astype(np.int64), T, threshold)
    if threshold > -1.0:
        S_plain = oracle.npmi(O.astype(np.int64), T)
        keep = np.abs(S_plain - threshold) > 1e-9
    else:
        keep = np.ones_like(S_ref, dtype=bool)
    err = np.abs(S.astype(np.float64) - S_ref)[keep]
    assert err.max(initial=0.0) <= S_TOL, err.max()


@pytest.mark.parametrize("T,d,k,kind,C,seed", [
    (1, 64, 8, 0, 16, 10), (37, 64, 8, 2, 24, 11), (300, 256, 16, 4, 64, 12), (1000, 1536, 32, 32, 256, 13),
    (513, 4000, 128, 8, 1024, 14), (64, 200, 4, 1, 4, 15),
])
def test_cooccurrence_npmi_parity(T, d, k, kind, C, seed):
    idx = qi.topk_like_sets(T, d, k, seed)
    hist = np.bincount(idx.ravel(), minlength=d)
    pos = oracle.split_channels(hist, kind, C)
    O, S = _cooc(idx, pos, C)
    O_ref = oracle.cooccurrence(idx, pos, C)
    assert (O.astype(np.int64) == O_ref).all()
    _check_npmi(S, O_ref, T, -1.0)
    O2, S2 = _cooc(idx, pos, C, threshold=0.2)
    assert (O2 == O).all()
    _check_npmi(S2, O_ref, T, 0.2)


def test_cooccurrence_ignores_channels_without_position_and_out_of_range():
    idx = np.array([[5, 7, 3], [7, 9, 3], [5, 7, 9], [1, 2, 3]], dtype=np.int32)
    pos = np.full(10, -1, dtype=np.int32)
    pos[5], pos[7], pos[9] = 0, 1, 2
    pos[1] = 3                                   # position >= C: ignored
    O, S = _cooc(idx, pos, 3)
    assert O.tolist() == [[2, 2, 1], [2, 3, 2], [1, 2, 2]]
    # an index outside [0, d_in) is skipped too (d_in = len(pos))
    idx2 = idx.copy()
    idx2[0, 2] = 10
    idx2[1, 2] = -4
    O2, _ = _cooc(idx2, pos, 3)
    assert (O2 == O).all()


def test_cooccurrence_empty_batch_zeroes_counts():
    pos = np.arange(16, dtype=np.int32)
    O = torch.full((16, 16), 5, dtype=torch.int32, device="cuda")
    idx = torch.empty((0, 4), dtype=torch.int32, device="cuda")
    qe.cooccurrence_npmi(idx, _i32(pos), 16, O, None)
    torch.cuda.synchronize()
    assert (O.cpu().numpy() == 0).all()


def test_cooccurrence_rejects_bad_sizes():
    pos = _i32(np.arange(8))
    O = torch.zeros((8, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(qe.QEError):
        qe.cooccurrence_npmi(_i32(np.zeros((2, 129))), pos, 8, O)      # k > 128
    with pytest.raises(qe.QEError):
        qe.cooccurrence_npmi(_i32(np.zeros((2, 4))), pos, 4097, O)     # C > 4096


def test_calibration_chain_full_size_72b():
    # 72B-shaped statistic: T = 8192 tokens, d = 29568, k = 32, N_r = 8 -> C = 256. The split,
    # the counts and NPMI run on the GPU; the oracle checks each from the same seeded sets.
    T, d, k, C = 8192, 29568, 32, 256
    idx = qi.topk_like_sets(T, d, k, 21)
    hist = np.bincount(idx.ravel(), minlength=d)
    pos_ref = oracle.split_channels(hist, k, C)
    pos = torch.empty(d, dtype=torch.int32, device="cuda")
    qe.split_channels(_i32(hist), k, C, pos)
    O = torch.empty((C, C), dtype=torch.int32, device="cuda")
    S = torch.empty((C, C), dtype=torch.float32, device="cuda")
    qe.cooccurrence_npmi(_i32(idx), pos, C, O, S, 0.2)
    torch.cuda.synchronize()
    assert (pos.cpu().numpy() == pos_ref).all()
    O_ref = oracle.cooccurrence(idx, pos_ref, C)
    assert (O.cpu().numpy().astype(np.int64) == O_ref).all()
    _check_npmi(S.cpu().numpy(), O_ref, T, 0.2)


def test_calibration_chain_from_gpu_topk_properties():
    # Top-k on the GPU feeds the split and the counts; checked by properties that hold at any
    # size: O is symmetric, its diagonal is the histogram at the selected channels, every row
    # sum is at most k times the diagonal, and S is symmetric within [-1, 1].
    cfg = qi.CONFIGS["qwen2vl72b"]
    T, d, k, C = 2048, 8192, 32, 256
    X = qi.to_bf16(qi.outlier_activations(T, d, 31, cfg.outlier_spec(d)))
    w_mean = np.abs(qi.gaussian(d, 0.02, 32)).astype(np.float32)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    hist = torch.empty(d, dtype=torch.int32, device="cuda")
    qe.topk_importance(cuda(X), cuda(w_mean), k, idx, hist)
    pos = torch.empty(d, dtype=torch.int32, device="cuda")
    qe.split_channels(hist, k, C, pos)
    O = torch.empty((C, C), dtype=torch.int32, device="cuda")
    S = torch.empty((C, C), dtype=torch.float32, device="cuda")
    qe.cooccurrence_npmi(idx, pos, C, O, S)
    torch.cuda.synchronize()
    h, p, o, s = hist.cpu().numpy(), pos.cpu().numpy(), O.cpu().numpy(), S.cpu().numpy()
    sel = np.flatnonzero(p >= 0)
    assert sorted(p[sel].tolist()) == list(range(C))
    by_pos = sel[np.argsort(p[sel])]
    assert all(h[a] > h[b] or (h[a] == h[b] and a < b) for a, b in zip(by_pos[:-1], by_pos[1:]))
    above = (h > h[by_pos[0]]) | ((h == h[by_pos[0]]) & (np.arange(d) < by_pos[0]))
    assert above.sum() == k
    assert (o == o.T).all()
    assert (np.diag(o)[p[sel]] == h[sel]).all()
    assert (o.sum(axis=1) <= k * np.diag(o)).all()
    assert (np.abs(s - s.T) == 0).all() and s.min() >= -1.0 and s.max() <= 1.0
