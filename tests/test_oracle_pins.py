"""Pins of the CPU oracle against facts the pages and the mathematics fix.

Each test checks an oracle function against something other than itself: a
hand-worked value, a closed form, a textbook routine, brute force on tiny
inputs, or an invariant the method states. Each is chosen so that a
plausible slip in the oracle would fail at least one test: a dropped term, a
wrong sign or index, a transposed operand, the wrong rounding or tie rule.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import fixtures
import qe_inputs as qi


# ---------------------------------------------------------------- quantization

def test_rtn_hand_cases_fp32_division():
    # One row, s = 1, group 4, W4 (qmax 7).
    # absmax 1 -> scale = fl32(1/7) = 0.142857149...
    # 0.5/scale = 3.4999998 in fp32, which is not a tie, so the code is 3.
    # 0.25/scale = 1.7499999 -> 2; -1/scale = -6.9999995 -> -7.
    W = np.array([[0.5, -1.0, 0.25, 0.0]], np.float32)
    codes, scales, _, _ = oracle.quantize_weights(W, np.ones(4, np.float32), 4, 4)
    assert scales[0, 0] == np.float32(1.0) / np.float32(7.0)
    assert codes.tolist() == [[3, -7, 2, 0]]


def test_rtn_ties_go_to_even():
    # absmax 7/8 -> scale 1/8 exactly, so every quotient is exact:
    # 7, 3.5 -> 4 (even), 2.5 -> 2 (even), -0.5 -> 0 (even), -1.5 -> -2.
    W = np.array([[7 / 8, 3.5 / 8, 2.5 / 8, -0.5 / 8, -1.5 / 8, 0, 0, 0]], np.float32)
    codes, scales, _, _ = oracle.quantize_weights(W, np.ones(8, np.float32), 8, 4)
    assert scales[0, 0] == np.float32(0.125)
    assert codes.tolist() == [[7, 4, 2, 0, -2, 0, 0, 0]]


def test_zero_group_gives_zero_scale_and_codes():
    W = np.zeros((2, 8), np.float32)
    W[1, 4:] = [1, -2, 3, -4]
    codes, scales, _, _ = oracle.quantize_weights(W, np.ones(8, np.float32), 4, 4)
    assert scales[0].tolist() == [0.0, 0.0] and scales[1, 0] == 0.0
    assert (codes[0] == 0).all() and (codes[1, :4] == 0).all()
    # scale = fl32(4/7) = 0.571428597 (rounded up), so -2/scale = -3.4999998 in fp32: not a tie, -> -3
    assert codes[1, 4:].tolist() == [2, -3, 5, -7]


# ---------------------------------------------------------------- fp16 group scales

def test_fp16_rounding_matches_ieee_binary16():
    # round to nearest even on the binary16 grid, normal and subnormal, ties included; numpy's
    # float32 -> float16 cast is IEEE round-to-nearest-even
    g = np.random.default_rng(11)
    vals = np.concatenate([
        g.uniform(-2.0, 2.0, 3000), g.uniform(-60000, 60000, 500), g.uniform(-1e-4, 1e-4, 500),
        g.uniform(-1e-7, 1e-7, 200),
        # exact halfway points between neighbouring fp16 values (ties) in the normal and subnormal range
        (np.arange(1, 200, dtype=np.float32) + np.float32(0.5)) * np.float32(2.0 ** -24),
        (np.float32(1024) + np.arange(0, 64, dtype=np.float32) + np.float32(0.5)) * np.float32(2.0 ** -10),
    ]).astype(np.float32)
    ref = vals.astype(np.float16).astype(np.float32)
    got = np.array([oracle.round_fp16(float(v)) for v in vals], np.float32)
    assert (got == ref).all()
    # beyond the largest finite fp16 the stored scale saturates (it stays finite)
    assert oracle.round_fp16(70000.0) == 65504.0 and oracle.round_fp16(-1e9) == -65504.0


def test_fp16_scales_on_grid_weights_round_trip():
    # W' = 2^m * q with max |q| = qmax per group: the scale 2^m is exact in fp16 as in fp32,
    # so the codes come back exactly and the stored scales are the powers of two
    g = np.random.default_rng(12)
    for bits in (4, 3):
        qmax = 2 ** (bits - 1) - 1
        N, K, grp = 6, 256, 64
        q = g.integers(-qmax, qmax + 1, size=(N, K))
        q[:, ::grp] = qmax
        m = g.integers(-12, 4, size=(N, K // grp))
        W = (q * 2.0 ** np.repeat(m, grp, axis=1)).astype(np.float32)
        codes, scales, _, _ = oracle.quantize_weights(W, np.ones(K, np.float32), grp, bits, scale_fp16=True)
        assert (codes == q).all()
        assert (scales == (2.0 ** m).astype(np.float32)).all()


def test_fp16_scale_recomputes_the_codes():
    # absmax 1, W4: the fp32 scale fl32(1/7) = 0.142857149 becomes fp16 0.142822265625
    # (1/7 = 1.142857 * 2^-3; the 10-bit mantissa of 0.142857 * 1024 = 146.29 rounds to 146).
    # 0.5 / 0.142822265625 = 3.5009 -> 4, where the fp32 scale gives 3.4999998 -> 3; the other
    # codes are unchanged: 1 -> 7.0017 -> 7, 0.25 -> 1.7504 -> 2.
    W = np.array([[0.5, -1.0, 0.25, 0.0]], np.float32)
    c32, s32, _, _ = oracle.quantize_weights(W, np.ones(4, np.float32), 4, 4)
    c16, s16, _, _ = oracle.quantize_weights(W, np.ones(4, np.float32), 4, 4, scale_fp16=True)
    assert s16[0, 0] == np.float32(0.142822265625) and s32[0, 0] == np.float32(1.0) / np.float32(7.0)
    assert c32.tolist() == [[3, -7, 2, 0]] and c16.tolist() == [[4, -7, 2, 0]]
    # codes stay in range and every scale is an fp16 value
    g = np.random.default_rng(13)
    W = g.standard_normal((20, 384)).astype(np.float32) * 0.02
    codes, scales, _, _ = oracle.quantize_weights(W, np.ones(384, np.float32), 128, 4, scale_fp16=True)
    assert np.abs(codes).max() <= 7
    assert (scales.astype(np.float16).astype(np.float32) == scales).all()


def test_smoothing_inverse_is_the_nearest_fp32_reciprocal():
    # s_inv = fl32(1/s): no fp32 neighbour of the stored value is closer to the exact 1/s
    # (checked in fp64, where 1/s and the distances are exact enough), and powers of two invert exactly
    g = np.random.default_rng(5)
    s = np.concatenate([g.uniform(0.01, 100.0, 4000), 2.0 ** g.integers(-20, 20, 64)]).astype(np.float32)
    si = oracle.smoothing_inverse(s)
    assert si.dtype == np.float32
    exact = 1.0 / s.astype(np.float64)
    d0 = np.abs(si.astype(np.float64) - exact)
    for nb in (np.nextafter(si, np.float32(np.inf)), np.nextafter(si, np.float32(0))):
        assert (d0 <= np.abs(nb.astype(np.float64) - exact)).all()
    p2 = s[-64:]
    assert (si[-64:].astype(np.float64) * p2.astype(np.float64) == 1.0).all()


def test_channel_scale_multiplies_weights_and_divides_activations():
    # Scaling moves magnitude between X and W (Shared Expert paragraph): with s
    # a power of two the scaled weight W*s is exact, so the weight codes of
    # (W, s) must equal the codes of (W*s, 1). For activations, s_inv = 1/s
    # scales x down.
    g = np.random.default_rng(0)
    W = g.standard_normal((6, 16)).astype(np.float32)
    s = (2.0 ** g.integers(-3, 4, size=16)).astype(np.float32)
    c1, sc1, _, _ = oracle.quantize_weights(W, s, 8, 4)
    c2, sc2, _, _ = oracle.quantize_weights(W * s[None, :], np.ones(16, np.float32), 8, 4)
    assert (c1 == c2).all() and (sc1 == sc2).all()
    X = g.standard_normal((5, 16)).astype(np.float32)
    q1, sa1 = oracle.act_quant(X, (1 / s).astype(np.float32), 8)
    q2, sa2 = oracle.act_quant(X / s[None, :], np.ones(16, np.float32), 8)
    assert (q1 == q2).all() and (sa1 == sa2).all()


@pytest.mark.parametrize("bits", [3, 4])
def test_weights_on_grid_roundtrip_exactly(bits):
    # W = 2^m * q with |q| = qmax present in every group: the scale is 2^m exactly,
    # the codes come back unchanged, and dequant(W) - W = 0.
    qm = oracle.qmax(bits)
    g = np.random.default_rng(bits)
    N, K, grp = 5, 256, 64
    q = g.integers(-qm, qm + 1, size=(N, K))
    q[:, ::grp] = qm * np.where(g.random((N, K // grp)) < 0.5, -1, 1)
    m = g.integers(-8, 2, size=(N, K // grp)).astype(np.float64)
    W = (q * np.repeat(2.0 ** m, grp, axis=1)).astype(np.float32)
    codes, scales, _, _ = oracle.quantize_weights(W, np.ones(K, np.float32), grp, bits)
    assert (codes == q).all()
    assert (scales == (2.0 ** m).astype(np.float32)).all()
    deq = codes.astype(np.float64) * np.repeat(scales.astype(np.float64), grp, axis=1)
    assert (deq == W.astype(np.float64)).all()


@pytest.mark.parametrize("bits", [6, 8])
def test_activations_on_grid_roundtrip_exactly(bits):
    qm = oracle.qmax(bits)
    g = np.random.default_rng(bits)
    T, K = 7, 96
    q = g.integers(-qm, qm + 1, size=(T, K))
    q[:, 3] = qm
    m = g.integers(-6, 3, size=T).astype(np.float64)
    X = (q * (2.0 ** m)[:, None]).astype(np.float32)
    codes, sa = oracle.act_quant(X, np.ones(K, np.float32), bits)
    assert (codes == q).all() and (sa == (2.0 ** m).astype(np.float32)).all()


def test_group_equal_K_is_per_row_rtn():
    # Textbook per-row symmetric RTN in numpy fp32 (s = 1, one group per row).
    g = np.random.default_rng(4)
    W = (g.standard_normal((9, 128)) * 0.05).astype(np.float32)
    scale = (np.abs(W).max(axis=1) / np.float32(7)).astype(np.float32)
    ref = np.clip(np.rint((W / scale[:, None]).astype(np.float32)), -7, 7).astype(np.int8)
    codes, scales, _, _ = oracle.quantize_weights(W, np.ones(128, np.float32), 128, 4)
    assert (scales[:, 0] == scale).all()
    assert (codes == ref).all()


def test_activation_invariants():
    cfg = qi.CONFIGS["tiny"]
    inp = qi.layer_inputs(cfg, cfg.projections[0])
    X = inp["X"].copy()
    X[5] = 0.0  # an all-zero token
    for bits in (6, 8):
        qm = oracle.qmax(bits)
        q, sa = oracle.act_quant(X, oracle.smoothing_inverse(inp["s"]), bits)
        assert np.abs(q).max() <= qm
        nz = sa > 0
        assert (np.abs(q[nz]).max(axis=1) == qm).all()
        assert sa[5] == 0 and (q[5] == 0).all()


def test_w_mean_is_meanrow_of_abs_weight():
    # Meanrow(|W|) is the mean over the d_out rows for each input channel.
    g = np.random.default_rng(5)
    W = g.standard_normal((33, 40)).astype(np.float32)
    _, _, w_mean, w_colmax = oracle.quantize_weights(W, np.ones(40, np.float32), 8, 4)
    ref = np.abs(W.astype(np.float64)).sum(axis=0) / 33
    assert np.allclose(w_mean, ref.astype(np.float32), rtol=0, atol=0)
    assert (w_colmax == np.abs(W).max(axis=0)).all()


# ---------------------------------------------------------------- router + buckets

def test_router_is_argmin_with_lowest_index_ties():
    g = np.random.default_rng(6)
    X = g.standard_normal((50, 24)).astype(np.float32)
    G = g.standard_normal((24, 5)).astype(np.float32)
    G[:, 3] = G[:, 1]  # experts 1 and 3 always tie -> 1 must win whenever they are best
    L, e = oracle.route(X, G)
    Lref = X.astype(np.float64) @ G.astype(np.float64)
    assert np.allclose(L, Lref, rtol=1e-14, atol=1e-12)
    assert (e == np.argmin(Lref, axis=1)).all()  # numpy argmin keeps the first minimum
    assert not (e == 3).any()


def test_bucket_is_stable_permutation():
    g = np.random.default_rng(7)
    e = g.integers(0, 6, size=300).astype(np.int32)
    perm, offsets = oracle.bucket(e, 6)
    assert sorted(perm.tolist()) == list(range(300))
    assert (np.diff(offsets) == np.bincount(e, minlength=6)).all()
    assert (perm == np.argsort(e, kind="stable")).all()


# ---------------------------------------------------------------- forward

def _tiny_layer(seed_shift=0, a_bits=8, zero_adapters=False):
    cfg = qi.CONFIGS["tiny"]
    inp = qi.layer_inputs(cfg, cfg.projections[0], proj_index=seed_shift)
    codes, scales, w_mean, _ = oracle.quantize_weights(inp["W"], inp["s"], cfg.group, cfg.w_bits)
    ad = {k: inp[k] for k in ("A_s", "B_s", "A_r", "B_r")}
    if zero_adapters:
        ad = {k: torch.zeros_like(v) for k, v in ad.items()}
    return cfg, inp, codes, scales, ad


def test_zero_adapters_equal_literal_dequant_matmul():
    # With every adapter zero, QE reduces to RTN + smoothing (the RTN/SQ rows of
    # the accuracy tables). The oracle's per-group int64 form must match the
    # literal (sa*q_x) . (sw*q_w)^T computed as one fp64 matmul.
    cfg, inp, codes, scales, ad = _tiny_layer(zero_adapters=True)
    Y, _ = oracle.qe_forward(inp["X"], codes, scales, oracle.smoothing_inverse(inp["s"]), ad["A_s"], ad["B_s"], ad["A_r"],
                             ad["B_r"], inp["G"], cfg.group, 8)
    xq, sa = oracle.act_quant(inp["X"], oracle.smoothing_inverse(inp["s"]), 8)
    deq_x = xq.astype(np.float64) * sa.astype(np.float64)[:, None]
    deq_w = codes.astype(np.float64) * np.repeat(scales.astype(np.float64), cfg.group, axis=1)
    Ylit = deq_x @ deq_w.T
    assert np.abs(Y - Ylit).max() <= 1e-12 * np.abs(Ylit).max()


def test_adapter_terms_match_formula():
    # Y - Y(adapters=0) = (X A_s) B_s + (X A_r[e]) B_r[e] for the routed e.
    cfg, inp, codes, scales, ad = _tiny_layer()
    Y, e = oracle.qe_forward(inp["X"], codes, scales, oracle.smoothing_inverse(inp["s"]), ad["A_s"], ad["B_s"], ad["A_r"],
                             ad["B_r"], inp["G"], cfg.group, 8)
    z = {k: torch.zeros_like(v) for k, v in ad.items()}
    Y0, e0 = oracle.qe_forward(inp["X"], codes, scales, oracle.smoothing_inverse(inp["s"]), z["A_s"], z["B_s"], z["A_r"],
                               z["B_r"], inp["G"], cfg.group, 8)
    assert (e == e0).all()
    X = np.asarray(inp["X"], np.float64)
    f = {k: v.double().numpy() for k, v in ad.items()}
    ref = (X @ f["A_s"]) @ f["B_s"]
    for t in range(X.shape[0]):
        ref[t] += (X[t] @ f["A_r"][e[t]]) @ f["B_r"][e[t]]
    _, e_ref = oracle.route(inp["X"], inp["G"])
    assert (e == e_ref).all()
    assert np.abs((Y - Y0) - ref).max() <= 1e-12 * np.abs(ref).max()


def test_token_independence_rows_permute():
    cfg, inp, codes, scales, ad = _tiny_layer()
    X = np.asarray(inp["X"])
    p = np.random.default_rng(8).permutation(X.shape[0])
    args = (codes, scales, oracle.smoothing_inverse(inp["s"]), ad["A_s"], ad["B_s"], ad["A_r"], ad["B_r"], inp["G"], cfg.group, 8)
    Y, e = oracle.qe_forward(X, *args)
    Yp, ep = oracle.qe_forward(X[p], *args)
    assert (Yp == Y[p]).all() and (ep == e[p]).all()
    rows = np.array([3, 0, 17], np.int32)
    Yr, er = oracle.qe_forward(X, *args, rows=rows)
    assert (Yr == Y[rows]).all() and (er == e[rows]).all()


def test_identical_experts_make_routing_irrelevant():
    cfg, inp, codes, scales, ad = _tiny_layer()
    A_r = ad["A_r"].clone()
    B_r = ad["B_r"].clone()
    A_r[:] = A_r[0]
    B_r[:] = B_r[0]
    args = (codes, scales, oracle.smoothing_inverse(inp["s"]), ad["A_s"], ad["B_s"], A_r, B_r, inp["G"], cfg.group, 8)
    Y, _ = oracle.qe_forward(inp["X"], *args)
    T = Y.shape[0]
    for ov in (np.zeros(T), np.full(T, 3), np.arange(T) % 4):
        Yo, eo = oracle.qe_forward(inp["X"], *args, expert_override=ov)
        assert (eo == ov).all()
        assert (Yo == Y).all()


def test_svd_experts_strictly_reduce_reconstruction_error():
    # The objective min ||(E - A_sB_s - A_rB_r) x||: a whitened SVD shared expert
    # strictly lowers the error of the calibration tokens, and the per-cluster
    # routed experts lower it again (Eckart-Young with whitening).
    cfg = qi.CONFIGS["tiny"]
    inp = qi.layer_inputs(cfg, cfg.projections[0], T=512)
    codes, scales, _, _ = oracle.quantize_weights(inp["W"], inp["s"], cfg.group, cfg.w_bits)
    _, experts = oracle.route(inp["X"], inp["G"])
    A_s, B_s, A_r, B_r = fixtures.qe_adapters(inp["W"], codes, scales, inp["s"], cfg.group, inp["X"],
                                             experts, cfg.rank_shared, cfg.n_routed, cfg.rank_routed)
    e0, e1, e2 = fixtures.reconstruction_errors(inp["W"], codes, scales, inp["s"], cfg.group, inp["X"],
                                                experts, A_s, B_s, A_r, B_r)
    assert e0 > e1 > e2 > 0
    # Full rank reconstructs E to rounding.
    A, B = fixtures.whitened_lowrank(
        (np.asarray(inp["W"], np.float64)
         - fixtures.effective_quantized_weight(codes, scales, inp["s"], cfg.group)).T, inp["X"], 256)
    Et = (np.asarray(inp["W"], np.float64) - fixtures.effective_quantized_weight(codes, scales, inp["s"], cfg.group)).T
    assert np.abs(A @ B - Et).max() <= 1e-9 * np.abs(Et).max()


def test_svd_adapters_reduce_layer_output_error_through_oracle():
    # End to end through oracle.qe_forward: with the fixture adapters, the QE
    # output is closer to the full-precision x W^T than RTN alone.
    cfg = qi.CONFIGS["tiny"]
    inp = qi.layer_inputs(cfg, cfg.projections[0], T=512)
    codes, scales, _, _ = oracle.quantize_weights(inp["W"], inp["s"], cfg.group, cfg.w_bits)
    _, experts = oracle.route(inp["X"], inp["G"])
    A_s, B_s, A_r, B_r = fixtures.qe_adapters(inp["W"], codes, scales, inp["s"], cfg.group, inp["X"],
                                             experts, cfg.rank_shared, cfg.n_routed, cfg.rank_routed)
    X = np.asarray(inp["X"])
    Yfp = X.astype(np.float64) @ np.asarray(inp["W"], np.float64).T
    z = np.zeros_like
    Yq, _ = oracle.qe_forward(X, codes, scales, oracle.smoothing_inverse(inp["s"]), z(A_s), z(B_s), z(A_r), z(B_r), inp["G"],
                              cfg.group, 16)
    Yqe, _ = oracle.qe_forward(X, codes, scales, oracle.smoothing_inverse(inp["s"]), A_s, B_s, A_r, B_r, inp["G"], cfg.group, 16)
    err_q = ((Yq - Yfp) ** 2).sum()
    err_qe = ((Yqe - Yfp) ** 2).sum()
    # a_bits=16 leaves only the bf16 activation rounding besides the weight error
    assert err_qe < 0.5 * err_q


def test_group_accumulator_bound_and_numpy():
    cfg, inp, codes, scales, ad = _tiny_layer()
    xq, _ = oracle.act_quant(inp["X"], oracle.smoothing_inverse(inp["s"]), 8)
    acc = oracle.group_acc(xq, codes, cfg.group)
    ref = np.einsum("tjg,ojg->toj", xq.reshape(64, 4, 64).astype(np.int64),
                    codes.reshape(256, 4, 64).astype(np.int64))
    assert (acc == ref).all()
    assert np.abs(acc).max() <= cfg.group * 127 * 7


def test_weight_only_on_grid_is_bf16_matmul():
    # W3A16 with s = 1 and weights on the grid: the layer is x_bf16 . W^T, which
    # torch's fp64 matmul computes independently.
    g = np.random.default_rng(9)
    T, K, N, grp = 6, 256, 40, 128
    q = g.integers(-3, 4, size=(N, K))
    q[:, ::grp] = 3
    sw = 2.0 ** g.integers(-7, -2, size=(N, K // grp))
    W = (q * np.repeat(sw, grp, axis=1)).astype(np.float32)
    codes, scales, _, _ = oracle.quantize_weights(W, np.ones(K, np.float32), grp, 3)
    X = g.standard_normal((T, K)).astype(np.float32)
    Gr = np.zeros((K, 2), np.float32)
    z = np.zeros
    Y, _ = oracle.qe_forward(X, codes, scales, np.ones(K, np.float32), z((K, 1)), z((1, N)), z((2, K, 1)),
                             z((2, 1, N)), Gr, grp, 16)
    xb = torch.from_numpy(X).to(torch.bfloat16).double()
    ref = (xb @ torch.from_numpy(W.astype(np.float64)).T).numpy()
    assert np.abs(Y - ref).max() <= 1e-12 * np.abs(ref).max()


def test_round_bf16_matches_torch():
    g = np.random.default_rng(10)
    v = np.concatenate([g.standard_normal(2000).astype(np.float32) * 100,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0], np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).float().numpy()
    got = np.array([oracle.round_bf16(float(x)) for x in v], np.float32)
    assert (got == ref).all()


# ---------------------------------------------------------------- top-k

def test_topk_brute_force_and_hist():
    g = np.random.default_rng(11)
    T, K, k = 40, 50, 7
    X = g.standard_normal((T, K)).astype(np.float32)
    X[0, :] = 1.0  # all-equal scores on token 0: ties go to the lowest channels
    w = np.abs(g.standard_normal(K)).astype(np.float32)
    w[:] = np.where(np.arange(K) < 3, 1.0, w)
    idx, hist = oracle.topk(X, w, k)
    score = (np.abs(X) * w[None, :]).astype(np.float32)
    for t in range(T):
        order = np.lexsort((np.arange(K), -score[t].astype(np.float64)))
        assert idx[t].tolist() == order[:k].tolist()
        chosen = score[t, idx[t]]
        rest = np.delete(score[t], idx[t])
        assert chosen.min() >= rest.max()
    assert hist.sum() == T * k
    assert (hist == np.bincount(idx.ravel(), minlength=K)).all()
    # token 0: scores are w; the three channels with w = 1 tie and must come in index order
    assert idx[0, :3].tolist() == sorted(idx[0, :3].tolist())


def test_topk_all_zero_row_takes_first_k_channels():
    X = np.zeros((1, 20), np.float32)
    idx, hist = oracle.topk(X, np.ones(20, np.float32), 5)
    assert idx[0].tolist() == [0, 1, 2, 3, 4]


# ---------------------------------------------------------------- co-occurrence and NPMI

def test_cooccurrence_hand_counted_example():
    # three tokens, channels 5, 7, 9 token-dependent (positions 0, 1, 2), channel 3 not:
    # token sets {5,7,3}, {7,9}, {5,7,9} -> pairs counted by hand
    idx = np.array([[5, 7, 3], [7, 9, 3], [5, 7, 9]])
    pos = np.full(12, -1)
    pos[5], pos[7], pos[9] = 0, 1, 2
    O = oracle.cooccurrence(idx, pos, 3)
    expect = np.array([[2, 2, 1],
                       [2, 3, 2],
                       [1, 2, 2]])
    assert (O == expect).all()


def test_cooccurrence_properties_on_topk_output():
    rng = np.random.default_rng(3)
    T, K, k, C = 200, 96, 8, 24
    X = rng.standard_normal((T, K)).astype(np.float32)
    w = np.abs(rng.standard_normal(K)).astype(np.float32)
    idx, hist = oracle.topk(X, w, k)
    dep = rng.permutation(K)[:C]           # some channels are token-dependent
    pos = np.full(K, -1)
    pos[dep] = np.arange(C)
    O = oracle.cooccurrence(idx, pos, C)
    assert (O == O.T).all()
    assert (np.diag(O) == hist[dep]).all()  # diagonal = how often the channel was picked
    # each token contributes |S_t ∩ dep|^2 pairs in total
    n_dep = (pos[idx] >= 0).sum(axis=1)
    assert O.sum() == (n_dep ** 2).sum()
    assert (O <= np.minimum.outer(np.diag(O), np.diag(O))).all()


def test_npmi_closed_forms():
    T = 8
    # channel 0 and 1 independent (p = 1/2 each, together 1/4), 0 and 2 always together,
    # 0 and 3 never together, channel 4 in every token
    O = np.array([[4, 2, 4, 0, 4],
                  [2, 4, 2, 2, 4],
                  [4, 2, 4, 0, 4],
                  [0, 2, 0, 4, 4],
                  [4, 4, 4, 4, 8]])
    S = oracle.npmi(O, T)
    assert S[0, 1] == pytest.approx(0.0, abs=1e-15)
    assert S[0, 2] == pytest.approx(1.0)
    assert S[0, 3] == -1.0
    assert S[4, 4] == 1.0                    # p = 1
    assert np.allclose(np.diag(S)[:4], 1.0)  # a channel with itself
    assert (S >= -1 - 1e-12).all() and (S <= 1 + 1e-12).all()
    assert (S == S.T).all()
    St = oracle.npmi(O, T, threshold=0.2)
    assert St[0, 1] == 0.0 and St[0, 3] == 0.0 and St[0, 2] == pytest.approx(1.0)


def test_split_channels_hand_ranked_example():
    # counts:   ch0 3, ch1 9, ch2 3, ch3 0, ch4 9, ch5 5, ch6 3
    # ranking:  ch1, ch4 (9; lower index first), ch5 (5), ch0, ch2, ch6 (3), ch3 (0)
    hist = [3, 9, 3, 0, 9, 5, 3]
    # k = 2 token-independent (ch1, ch4); C = 3 dependent: ch5 -> 0, ch0 -> 1, ch2 -> 2
    assert oracle.split_channels(hist, 2, 3).tolist() == [1, -1, 2, -1, -1, 0, -1]
    # C larger than what is left: every remaining channel gets a position
    assert oracle.split_channels(hist, 2, 10).tolist() == [1, -1, 2, 4, -1, 0, 3]
    # k = 0: the dependent set starts at the top of the ranking
    assert oracle.split_channels(hist, 0, 2).tolist() == [-1, 0, -1, -1, 1, -1, -1]


def test_split_channels_order_property():
    rng = np.random.default_rng(3)
    hist = rng.integers(0, 6, size=500)     # many ties
    k, C = 16, 128
    pos = oracle.split_channels(hist, k, C)
    sel = np.flatnonzero(pos >= 0)
    assert sorted(pos[sel].tolist()) == list(range(C))
    by_pos = sel[np.argsort(pos[sel])]
    # along the positions, counts never increase and equal counts go by index
    for a, b in zip(by_pos[:-1], by_pos[1:]):
        assert hist[a] > hist[b] or (hist[a] == hist[b] and a < b)
    rest = np.flatnonzero(pos < 0)
    # exactly k channels outrank every selected one; every unselected one is outranked by them
    outrank = [c for c in rest if hist[c] > hist[by_pos[0]] or (hist[c] == hist[by_pos[0]] and c < by_pos[0])]
    assert len(outrank) == k
    below = [c for c in rest if c not in outrank]
    last = by_pos[-1]
    assert all(hist[c] < hist[last] or (hist[c] == hist[last] and c > last) for c in below)
