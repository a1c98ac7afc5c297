"""GPU parity: the CUDA path through the C ABI against the CPU oracle, on the same seeded inputs.

Integer stages (weight codes and scales, activation codes and scales, int32
group accumulators, router choices, bucket order, Top-k index sets and
histograms) must match bit for bit. Router choices may differ only on
fp32 near-ties. Final fp outputs must be within 2e-3 (gpu_util.rel_err).
"""
import numpy as np
import pytest
import torch

import oracle
import qe_inputs as qi
import quantized_gemm_moe_b200 as qe
from gpu_util import Case, Y_TOL, check_routing, cuda, f32, rel_err

pytestmark = pytest.mark.gpu


def _cfg(base="tiny", **kw):
    return qi.CONFIGS[base].with_(**kw)


# ---------------------------------------------------------------- weight quantization

@pytest.mark.parametrize("N,K,group,bits,wdt,s16", [
    (256, 256, 64, 4, "f32", 0), (200, 384, 64, 4, "bf16", 0), (1536, 1536, 128, 4, "bf16", 0),
    (300, 256, 128, 3, "bf16", 0), (256, 320, 64, 3, "f32", 0), (8960, 1536, 128, 4, "bf16", 0),
    # fp16 group scales: the codes come from the stored fp16 scale
    (8960, 1536, 128, 4, "bf16", 1), (200, 384, 64, 4, "f32", 1), (300, 256, 128, 3, "bf16", 1),
])
def test_weight_quantization_bit_exact(N, K, group, bits, wdt, s16):
    cfg = _cfg(group=group, w_bits=bits, a_bits=8 if bits == 4 else 16, x_dtype=wdt)
    inp = qi.layer_inputs(cfg, qi.Projection("w", K, N), T=4)
    codes, scales, w_mean, colmax = oracle.quantize_weights(inp["W"], inp["s"], group, bits, scale_fp16=bool(s16))
    desc = qe.make_desc(K, N, group, bits, cfg.a_bits, 8, 4, 4, w_scale_fp16=s16)
    Wd = cuda(inp["W"])
    wp = torch.empty(qe.packed_weight_bytes(desc), dtype=torch.uint8, device="cuda")
    ws = torch.empty((K // group, N), dtype=torch.float16 if s16 else torch.float32, device="cuda")
    wm = torch.empty(K, dtype=torch.float32, device="cuda")
    wc = torch.empty(K, dtype=torch.float32, device="cuda")
    si = torch.empty(K, dtype=torch.float32, device="cuda")
    qe.quantize_weights(desc, Wd, cuda(inp["s"]), wp, ws, wm, wc, si)
    got = torch.empty((N, K), dtype=torch.int8, device="cuda")
    qe.unpack_weights(desc, wp, got)
    torch.cuda.synchronize()
    assert (got.cpu().numpy() == codes).all()
    assert (ws.float().cpu().numpy().T == scales).all()
    assert (wc.cpu().numpy() == colmax).all()
    # the stored smoothing factor is the correctly rounded fp32 reciprocal of s
    assert (si.cpu().numpy() == (np.float32(1.0) / inp["s"]).astype(np.float32)).all()
    np.testing.assert_allclose(wm.cpu().numpy(), w_mean, rtol=2e-7, atol=0)
    # padding rows of the last block hold zero codes (checked through the raw bytes)
    if N % 128:
        nb = (K + 127) // 128
        blk = 8192 if bits == 4 else 6144
        raw = wp.cpu().numpy().reshape(-1, nb, blk)[-1]
        rowb = blk // 128
        pad = raw[:, (N % 128) * rowb:]
        expect = 0 if bits == 4 else None
        if bits == 4:
            assert (pad == expect).all()


# ---------------------------------------------------------------- activations, router, buckets

@pytest.mark.parametrize("T,K,bits,xdt", [(1, 256, 8, "f32"), (3, 384, 6, "bf16"), (64, 256, 8, "f32"),
                                          (129, 1536, 6, "bf16"), (64, 8960, 6, "bf16")])
def test_activation_quantization_bit_exact(T, K, bits, xdt):
    cfg = _cfg(x_dtype=xdt, spec="qwen2b" if K >= 1024 else "tiny")
    inp = qi.layer_inputs(cfg, qi.Projection("x", K, 128), T=T)
    X = inp["X"]
    if T > 2:
        X = X.clone() if isinstance(X, torch.Tensor) else X.copy()
        X[1] = 0  # all-zero token: zero scale and codes
    q_ref, sa_ref = oracle.act_quant(X, oracle.smoothing_inverse(inp["s"]), bits)
    codes = torch.empty((T, K), dtype=torch.int8, device="cuda")
    sa = torch.empty(T, dtype=torch.float32, device="cuda")
    qe.act_quant(cuda(X), cuda(oracle.smoothing_inverse(inp["s"])), bits, codes, sa)
    torch.cuda.synchronize()
    assert (sa.cpu().numpy() == sa_ref).all()
    assert (codes.cpu().numpy() == q_ref).all()


@pytest.mark.parametrize("bits", [8, 6])
def test_activation_quantization_at_half_integers(bits):
    """Quotients x/sa on and next to half-integers: the kernel's division-free rounding must defer
    to the exact quotient there and give the oracle's codes (round half to even)."""
    qmax = 2 ** (bits - 1) - 1
    T, K = 6, 256
    rng = np.random.default_rng(77)
    X = np.zeros((T, K), np.float32)
    for t in range(T):
        S = np.float32(rng.uniform(0.003, 0.07))
        X[t, 0] = np.float32(qmax) * S                      # the row's absmax
        sa = np.float32(X[t, 0] / np.float32(qmax))         # what the oracle's scale will be
        n = rng.integers(-qmax, qmax, size=K - 1).astype(np.float32)
        x = (n + np.float32(0.5)) * sa                        # about half-integer quotients
        steps = rng.integers(-3, 4, size=K - 1)               # nudge by up to 3 ulps either way
        for i, st in enumerate(steps):
            for _ in range(abs(int(st))):
                x[i] = np.nextafter(x[i], np.float32(np.inf) if st > 0 else np.float32(-np.inf))
        X[t, 1:] = np.clip(x, -X[t, 0], X[t, 0])
    s_inv = np.ones(K, np.float32)
    q_ref, sa_ref = oracle.act_quant(X, s_inv, bits)
    codes = torch.empty((T, K), dtype=torch.int8, device="cuda")
    sa = torch.empty(T, dtype=torch.float32, device="cuda")
    qe.act_quant(cuda(X), cuda(s_inv), bits, codes, sa)
    torch.cuda.synchronize()
    assert (sa.cpu().numpy() == sa_ref).all()
    assert (codes.cpu().numpy() == q_ref).all()
    # the set really contains ties broken to even and quotients that miss the half-integer
    quot = X.astype(np.float64) / sa_ref.astype(np.float64)[:, None]
    frac = np.abs(quot - np.floor(quot) - 0.5)
    assert (frac == 0).sum() >= 1 and ((frac > 0) & (frac < 1e-6)).sum() >= 100


@pytest.mark.parametrize("T,K,Nr,xdt", [(1, 256, 4, "f32"), (64, 256, 4, "f32"), (300, 1536, 8, "bf16"),
                                        (2048, 1536, 8, "bf16"), (77, 512, 16, "bf16"), (40, 256, 3, "f32"),
                                        (33, 256, 1, "bf16")])
def test_router_and_buckets(T, K, Nr, xdt):
    cfg = _cfg(x_dtype=xdt, n_routed=Nr, spec="qwen2b" if K >= 1024 else "tiny")
    inp = qi.layer_inputs(cfg, qi.Projection("x", K, 128), T=T)
    L_ref, e_ref = oracle.route(inp["X"], inp["G"])
    expert = torch.empty(T, dtype=torch.int32, device="cuda")
    perm = torch.empty(T, dtype=torch.int32, device="cuda")
    offsets = torch.empty(Nr + 1, dtype=torch.int32, device="cuda")
    logits = torch.empty((T, Nr), dtype=torch.float32, device="cuda")
    qe.route(cuda(inp["X"]), cuda(inp["G"]), expert, perm, offsets, logits)
    torch.cuda.synchronize()
    e = expert.cpu().numpy()
    check_routing(inp["X"], inp["G"], e, e_ref)
    np.testing.assert_allclose(logits.cpu().numpy(), L_ref, rtol=1e-4, atol=1e-4 * np.abs(L_ref).max())
    # buckets are exactly the stable counting sort of the GPU's own choices
    p_ref, o_ref = oracle.bucket(e, Nr)
    assert (perm.cpu().numpy() == p_ref).all()
    assert (offsets.cpu().numpy() == o_ref).all()


def test_router_exact_ties_take_lowest_expert():
    cfg = _cfg()
    inp = qi.layer_inputs(cfg, qi.Projection("x", 256, 128), T=50)
    G = inp["G"].clone()
    G[:, 2] = G[:, 0]  # experts 0 and 2 tie exactly on every token
    G[:, 3] = G[:, 0]
    expert = torch.empty(50, dtype=torch.int32, device="cuda")
    perm = torch.empty(50, dtype=torch.int32, device="cuda")
    offsets = torch.empty(5, dtype=torch.int32, device="cuda")
    qe.route(cuda(inp["X"]), cuda(G), expert, perm, offsets)
    torch.cuda.synchronize()
    e = expert.cpu().numpy()
    assert not np.isin(e, [2, 3]).any()


# ---------------------------------------------------------------- Top-k importance

@pytest.mark.parametrize("T,K,k,xdt", [(1, 256, 1, "f32"), (64, 256, 8, "f32"), (100, 1536, 32, "bf16"),
                                       (37, 8960, 64, "bf16"), (5, 512, 128, "bf16"), (9, 29568, 32, "bf16")])
def test_topk_bit_exact(T, K, k, xdt):
    cfg = _cfg(x_dtype=xdt, spec="qwen2b" if K >= 1024 else "tiny")
    inp = qi.layer_inputs(cfg, qi.Projection("x", K, 128), T=T)
    X = f32(inp["X"]).copy()
    if T > 3:
        X[2] = 0.0              # all-zero token: ties everywhere, lowest channels win
        X[3, : K // 2] = 1.0    # many exact ties
    _, _, w_mean, _ = oracle.quantize_weights(inp["W"], inp["s"], 64, 4)
    w_mean = w_mean.copy()
    w_mean[:8] = w_mean[8]      # equal weights -> equal scores on equal |x|
    Xs = X if xdt == "f32" else qi.to_bf16(X)
    idx_ref, hist_ref = oracle.topk(Xs, w_mean, k)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    hist = torch.full((K,), 7, dtype=torch.int32, device="cuda")
    qe.topk_importance(cuda(Xs), cuda(w_mean), k, idx, hist)
    torch.cuda.synchronize()
    assert (idx.cpu().numpy() == idx_ref).all()
    assert (hist.cpu().numpy() == hist_ref).all()
    # accumulate mode adds a second pass on top
    qe.topk_importance(cuda(Xs), cuda(w_mean), k, idx, hist, accumulate=True)
    torch.cuda.synchronize()
    assert (hist.cpu().numpy() == 2 * hist_ref).all()


def test_topk_streaming_rows_with_degenerate_rows_mixed_in():
    # More tokens than SMs (the streaming kernel strides), with all-zero and constant rows that
    # it leaves to the radix-select kernel, spread over several CTAs and both row buffers.
    T, K, k = 400, 8192, 32
    cfg = _cfg(x_dtype="bf16", spec="qwen2b")
    X = qi.outlier_activations(T, K, 91, cfg.outlier_spec(K))
    for r in (0, 150, 151, 299, 399):
        X[r] = 0.0
    X[5] = 3.0
    X[6, ::2] = 0.0
    Xs = qi.to_bf16(X)
    w_mean = np.abs(qi.gaussian(K, 0.02, 92)).astype(np.float32)
    w_mean[100:140] = w_mean[99]
    idx_ref, hist_ref = oracle.topk(Xs, w_mean, k)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    hist = torch.empty(K, dtype=torch.int32, device="cuda")
    qe.topk_importance(cuda(Xs), cuda(w_mean), k, idx, hist)
    torch.cuda.synchronize()
    assert (idx.cpu().numpy() == idx_ref).all()
    assert (hist.cpu().numpy() == hist_ref).all()
    assert qe.device_error() == 0


def test_topk_full_size_sampled_rows():
    # 72B-shaped statistic: all 8192 tokens at d = 29568 on the GPU; the oracle checks a
    # seeded sample of rows, and sum(hist) = T*k, hist == bincount(idx) hold for the whole run.
    cfg = qi.CONFIGS["qwen2vl72b"]
    K, T, k = 29568, 8192, 32
    X = qi.to_bf16(qi.outlier_activations(T, K, 777, cfg.outlier_spec(K)))
    w_mean = np.abs(qi.gaussian(K, 0.02, 778)).astype(np.float32)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    hist = torch.empty(K, dtype=torch.int32, device="cuda")
    qe.topk_importance(cuda(X), cuda(w_mean), k, idx, hist)
    torch.cuda.synchronize()
    idx_c = idx.cpu().numpy()
    h = hist.cpu().numpy()
    assert h.sum() == T * k
    assert (h == np.bincount(idx_c.ravel(), minlength=K)).all()
    rows = np.random.default_rng(5).choice(T, 48, replace=False)
    idx_ref, _ = oracle.topk(X[rows], w_mean, k)
    assert (idx_c[rows] == idx_ref).all()


# ---------------------------------------------------------------- the forward

def _forward_check(case: Case, with_acc=True):
    Y, acc, expert, perm, sa = case.gpu_debug(with_acc)
    inp = case.inp
    _, e_ref = oracle.route(inp["X"], inp["G"])
    e = expert.cpu().numpy()
    check_routing(inp["X"], inp["G"], e, e_ref)
    xq_ref, sa_ref = oracle.act_quant(inp["X"], oracle.smoothing_inverse(inp["s"]), case.cfg.a_bits) if case.cfg.a_bits != 16 else (None, None)
    if sa_ref is not None:
        assert (sa.cpu().numpy() == sa_ref).all()
    p_ref, _ = oracle.bucket(e, case.cfg.n_routed)
    assert (perm.cpu().numpy() == p_ref).all()
    if with_acc:
        codes, _, _, _ = case.oracle_weights()
        acc_ref = oracle.group_acc(xq_ref, codes, case.cfg.group)
        assert (acc.cpu().numpy().astype(np.int64) == acc_ref).all()
    Y_ref, _ = case.oracle_forward(expert_override=e)
    err = rel_err(Y.cpu().numpy(), Y_ref)
    assert err <= Y_TOL, err
    return Y, Y_ref


def test_forward_tiny_layer():
    cfg = qi.CONFIGS["tiny"]
    _forward_check(Case(cfg, cfg.projections[0], cfg.T))


def test_forward_tiny_layer_with_svd_experts():
    # adapters built the pages' way (whitened SVD of E = W - W_q) on a calibration draw
    from oracle import fixtures
    cfg = qi.CONFIGS["tiny"]
    proj = cfg.projections[0]
    inp = qi.layer_inputs(cfg, proj, T=cfg.T)
    calib = qi.layer_inputs(cfg, proj, T=512, proj_index=9)
    codes, scales, _, _ = oracle.quantize_weights(inp["W"], inp["s"], cfg.group, cfg.w_bits)
    _, ec = oracle.route(calib["X"], inp["G"])
    A_s, B_s, A_r, B_r = fixtures.qe_adapters(inp["W"], codes, scales, inp["s"], cfg.group, calib["X"], ec,
                                             cfg.rank_shared, cfg.n_routed, cfg.rank_routed)
    for name, v in (("A_s", A_s), ("B_s", B_s), ("A_r", A_r), ("B_r", B_r)):
        inp[name] = qi.to_bf16(v)
    Y, Y_ref = _forward_check(Case(cfg, proj, cfg.T, inp=inp))
    # and the compensated layer is closer to the full-precision product than RTN alone
    X = np.asarray(inp["X"], np.float64)
    Yfp = X @ np.asarray(inp["W"], np.float64).T
    z = np.zeros_like
    Yq, _ = oracle.qe_forward(inp["X"], codes, scales, oracle.smoothing_inverse(inp["s"]), z(A_s), z(B_s), z(A_r), z(B_r), inp["G"],
                              cfg.group, cfg.a_bits)
    assert ((Y.cpu().numpy() - Yfp) ** 2).sum() < ((Yq - Yfp) ** 2).sum()


SHAPES = [
    # T, K, N, group, a_bits, r_s, N_r, r_r, x dtype
    (1, 256, 256, 64, 8, 8, 4, 4, "f32"),
    (3, 384, 200, 64, 8, 8, 4, 4, "bf16"),
    (16, 1024, 512, 128, 8, 32, 8, 4, "bf16"),
    (17, 256, 136, 128, 6, 32, 8, 4, "bf16"),
    (40, 512, 256, 128, 6, 32, 8, 4, "bf16"),
    (129, 512, 384, 128, 6, 32, 8, 4, "bf16"),
    (300, 256, 256, 64, 8, 0, 2, 16, "f32"),
    (257, 1024, 640, 128, 8, 32, 8, 32, "bf16"),
    (64, 256, 128, 128, 8, 0, 1, 0, "bf16"),
    (520, 640, 1152, 128, 6, 32, 8, 4, "bf16"),
]


@pytest.mark.parametrize("T,K,N,group,a_bits,rs,nr,rr,xdt", SHAPES)
def test_forward_shapes(T, K, N, group, a_bits, rs, nr, rr, xdt):
    cfg = _cfg(group=group, a_bits=a_bits, rank_shared=rs, n_routed=nr, rank_routed=rr, x_dtype=xdt,
               spec="qwen2b" if K >= 1024 else "tiny")
    _forward_check(Case(cfg, qi.Projection("p", K, N), T))


# Decode-sized batches (T <= 16) take the stream-K decode product: blocks split evenly over the
# SMs, the weights unpacked into TMEM, a per-tile fix-up of the segment partials. These shapes
# reach its corners: a K tail of one group (K % 128 = 64 at g = 64), ragged N, one output tile
# split over 64 CTAs (64 segments), many segments per tile at K = 29568, fewer blocks than SMs,
# no adapters, five adapter atoms, a single routed expert, A6 and A8 codes, W3 and W4 weight-only.
DECODE_SHAPES = [
    # T, K, N, group, a_bits, w_bits, r_s, N_r, r_r, x dtype
    (1, 320, 200, 64, 8, 4, 8, 4, 4, "f32"),
    (2, 320, 200, 64, 16, 3, 8, 4, 4, "bf16"),
    (7, 8192, 128, 128, 8, 4, 32, 8, 4, "bf16"),
    (16, 8192, 128, 128, 16, 4, 32, 8, 4, "bf16"),
    (16, 29568, 256, 128, 6, 4, 32, 8, 4, "bf16"),
    (5, 29568, 256, 128, 16, 3, 32, 8, 4, "bf16"),
    (16, 1024, 1000, 128, 8, 4, 0, 1, 0, "bf16"),
    (13, 1024, 640, 128, 6, 4, 32, 8, 32, "bf16"),
    (16, 1536, 8960, 128, 16, 3, 32, 8, 32, "bf16"),
    (3, 2048, 4096, 64, 8, 4, 32, 2, 8, "bf16"),
]


@pytest.mark.parametrize("T,K,N,group,a_bits,w_bits,rs,nr,rr,xdt", DECODE_SHAPES)
def test_forward_decode_batches(T, K, N, group, a_bits, w_bits, rs, nr, rr, xdt):
    cfg = _cfg(group=group, a_bits=a_bits, w_bits=w_bits, rank_shared=rs, n_routed=nr, rank_routed=rr,
               x_dtype=xdt, spec="qwen2b" if K >= 1024 else "tiny")
    c = Case(cfg, qi.Projection("p", K, N), T)
    assert qe.linear_plan(c.desc, T)["product_k_splits"] == 1
    Y, _ = _forward_check(c, with_acc=(a_bits != 16))
    # the fix-up adds the segment partials in a fixed order: repeats are bit-identical
    for _ in range(2):
        assert torch.equal(c.gpu_forward(), Y)
    assert torch.equal(c.gpu_forward(torch.bfloat16), c.gpu_forward().to(torch.bfloat16))


@pytest.mark.parametrize("T,K,N,group,bits,rs,nr,rr", [
    (1, 256, 200, 64, 3, 8, 4, 4), (5, 384, 256, 128, 3, 32, 8, 4), (16, 256, 384, 128, 4, 32, 8, 4),
    (33, 512, 136, 64, 3, 0, 2, 8), (4, 1024, 640, 128, 3, 32, 8, 32),
    # enough output tiles for 128-token tiles (two epilogue teams), with ragged token tails
    (300, 256, 8960, 128, 3, 32, 8, 4), (129, 384, 17920, 64, 4, 32, 8, 4),
])
def test_forward_weight_only(T, K, N, group, bits, rs, nr, rr):
    cfg = _cfg(group=group, w_bits=bits, a_bits=16, rank_shared=rs, n_routed=nr, rank_routed=rr, x_dtype="bf16")
    _forward_check(Case(cfg, qi.Projection("p", K, N), T), with_acc=False)


@pytest.mark.parametrize("T,K,N,group,a_bits,w_bits,rs,nr,rr,kc,xdt", [
    (64, 256, 256, 64, 8, 4, 8, 4, 4, 16, "f32"),         # adapter/router GEMM 32 wide
    (300, 1536, 1536, 128, 6, 4, 32, 8, 4, 32, "bf16"),   # 48 wide
    (129, 512, 384, 128, 8, 4, 32, 8, 32, 16, "bf16"),    # r_r = 32: U_cat 320 wide, GEMM 48 wide
    (16, 1024, 640, 128, 16, 3, 32, 8, 4, 32, "bf16"),    # weight-only
    (40, 512, 256, 128, 6, 4, 0, 4, 8, 24, "bf16"),       # no shared expert: GEMM 16 wide
])
def test_forward_cluster_sparse_routed(T, K, N, group, a_bits, w_bits, rs, nr, rr, kc, xdt):
    # Routed experts that touch only their cluster's channels: the forward gathers them per token;
    # the oracle runs the dense formula with A_r zero outside the clusters.
    cfg = _cfg(group=group, a_bits=a_bits, w_bits=w_bits, rank_shared=rs, n_routed=nr, rank_routed=rr,
               x_dtype=xdt, spec="qwen2b" if K >= 1024 else "tiny")
    _forward_check(Case(cfg, qi.Projection("p", K, N), T, routed_channels=kc), with_acc=(a_bits != 16))


def test_forward_bf16_output_is_rounded_fp32_output():
    cfg = _cfg(a_bits=6, x_dtype="bf16", group=128, rank_shared=32, n_routed=8)
    c = Case(cfg, qi.Projection("p", 512, 384), 70)
    y32 = c.gpu_forward(torch.float32)
    y16 = c.gpu_forward(torch.bfloat16)
    assert torch.equal(y16, y32.to(torch.bfloat16))


@pytest.mark.parametrize("cfg_name,proj_index,T,N", [
    ("qwen2vl2b", 0, 2048, None), ("qwen2vl2b", 2, 2048, None), ("qwen2vl2b", 4, 2048, None),
    ("qwen2vl2b", 0, 300, 1001), ("qwen2vl2b", 4, 1000, 1000), ("tiny", 0, 64, None),
])
def test_forward_bf16_output_full_size(cfg_name, proj_index, T, N):
    # bf16 output (the staged-tile store for tiles up to 192 tokens, the pass-wise store above)
    # equals the fp32 output (checked against the oracle elsewhere) rounded to bf16, element by element
    cfg = qi.CONFIGS[cfg_name]
    proj = cfg.projections[proj_index]
    if N is not None:
        proj = qi.Projection(proj.name, proj.d_in, N)
    c = Case(cfg, proj, T, proj_index=proj_index)
    y32 = c.gpu_forward(torch.float32)
    y16 = c.gpu_forward(torch.bfloat16)
    assert torch.equal(y16, y32.to(torch.bfloat16))


def test_forward_deterministic_and_token_independent():
    cfg = _cfg(a_bits=8, x_dtype="bf16", group=128, rank_shared=32, n_routed=8)
    c = Case(cfg, qi.Projection("p", 512, 384), 200)
    y1 = c.gpu_forward()
    y2 = c.gpu_forward()
    assert torch.equal(y1, y2)
    p = torch.randperm(200, generator=torch.Generator().manual_seed(3))
    Yp = c.layer.forward(c.Xd[p.cuda()].contiguous(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(Yp, y1[p.cuda()])


def test_forward_empty_batch_is_noop():
    cfg = _cfg()
    c = Case(cfg, cfg.projections[0], 4)
    X0 = torch.empty((0, 256), dtype=torch.float32, device="cuda")
    Y0 = c.layer.forward(X0, out_dtype=torch.float32)
    assert Y0.shape == (0, 256)


# ---------------------------------------------------------------- full-size layers, sampled rows

def _full_size(cfg_name, proj_index, n_rows=48, routed_channels=0):
    cfg = qi.CONFIGS[cfg_name]
    proj = cfg.projections[proj_index]
    c = Case(cfg, proj, cfg.T, proj_index=proj_index, routed_channels=routed_channels)
    _sampled_check(c, n_rows, proj_index)
    del c


def _sampled_check(c, n_rows, seed):
    # sampled output rows against the oracle (routing checked on the same rows), the whole
    # output finite, and the weight codes bit-exact
    cfg, proj = c.cfg, c.proj
    Y, _, expert, _, _ = c.gpu_debug(with_acc=False)
    e = expert.cpu().numpy()
    rows = np.random.default_rng(seed).choice(c.T, min(n_rows, c.T), replace=False).astype(np.int32)
    _, e_ref = oracle.route(f32(c.inp["X"])[rows], c.inp["G"])
    check_routing(f32(c.inp["X"])[rows], c.inp["G"], e[rows], e_ref)
    Y_ref, _ = c.oracle_forward(rows=rows, expert_override=e[rows])
    err = rel_err(Y.cpu().numpy()[rows], Y_ref)
    assert err <= Y_TOL, err
    # the whole output is finite and the integer stages are consistent
    assert torch.isfinite(Y).all()
    codes, scales, _, _ = c.oracle_weights()
    got = torch.empty((proj.d_out, proj.d_in), dtype=torch.int8, device="cuda")
    qe.unpack_weights(c.desc, c.layer.w_packed, got)
    torch.cuda.synchronize()
    assert (got.cpu().numpy() == codes).all()
    return Y


@pytest.mark.parametrize("T,K,N,group,a_bits,w_bits,rr", [
    (2048, 512, 2048, 128, 8, 4, 32),    # 256-token tiles (3 stages, 2 TMEM buffers), 5 adapter atoms
    (2048, 512, 2048, 64, 6, 4, 4),      # 256-token tiles, g = 64: two groups per stage on 2 buffers
    (2048, 512, 2048, 64, 8, 4, 32),     # both
    (2048, 1536, 1536, 64, 6, 4, 32),    # 192-token tiles
    (1000, 512, 1024, 128, 8, 4, 16),    # 128-token tiles (4 stages), 3 adapter atoms
    (1200, 512, 2048, 128, 16, 3, 32),   # weight-only 128-token tiles (2 operand slots), 5 atoms
    (1200, 512, 2048, 64, 16, 4, 32),
    (48, 512, 1024, 64, 16, 4, 32),      # weight-only 64-token tile (3 slots)
    (200, 512, 1024, 128, 16, 3, 16),
])
def test_forward_long_adapter_blocks_and_two_group_stages(T, K, N, group, a_bits, w_bits, rr):
    # Shapes where one MMA issuer skips more of the other's stages than the ring holds (an
    # adapter block of R_pad/64 atoms), or where a stage carries two groups on two TMEM
    # buffers: each issuer must still wait on the right barrier phase. Sampled rows against
    # the oracle, and a repeat must be bit-identical (a missed wait shows up as a race).
    cfg = _cfg(group=group, a_bits=a_bits, w_bits=w_bits, rank_shared=32, n_routed=8, rank_routed=rr,
               x_dtype="bf16", spec="qwen2b" if K >= 1024 else "tiny")
    c = Case(cfg, qi.Projection("p", K, N), T)
    Y = _sampled_check(c, 48, T + rr)
    for _ in range(3):
        assert torch.equal(c.gpu_forward(), Y)
    assert qe.device_error() == 0


@pytest.mark.parametrize("proj_index", range(5))
def test_full_size_qwen2vl2b_layer_set(proj_index):
    _full_size("qwen2vl2b", proj_index)


@pytest.mark.parametrize("proj_index", [0, 4])
def test_full_size_cluster_sparse_routed(proj_index):
    # the 2B layer set at T = 2048 with each routed expert on 32 channels
    _full_size("qwen2vl2b", proj_index, routed_channels=32)


# The two larger prefill layer sets at their full sizes, in the launch configuration the bench
# times (the forward picks tiles and splits from the shape alone): 256 seeded rows per projection
# against the oracle, routing on the same rows, and all weight codes bit-exact. These reach what
# the 2B set does not: 64 groups per output tile at K = 8192 and 231 at K = 29568, N = 29568 on
# 256-token tiles, and T = 8192 through the cooperative route/quantize launch.

@pytest.mark.slow
@pytest.mark.parametrize("proj_index", range(5))
def test_full_size_internvl2_8b_layer_set(proj_index):
    _full_size("internvl2_8b", proj_index, n_rows=256)


@pytest.mark.slow
@pytest.mark.parametrize("proj_index", range(7))
def test_full_size_qwen2vl72b_layer_set(proj_index):
    cfg = qi.CONFIGS["qwen2vl72b"]
    c = Case(cfg, cfg.projections[proj_index], cfg.T, proj_index=proj_index)
    Y = _sampled_check(c, 256, proj_index)
    # the bench stores bf16: that output is the checked fp32 output rounded, element by element
    assert torch.equal(c.gpu_forward(torch.bfloat16), Y.to(torch.bfloat16))


@pytest.mark.slow
@pytest.mark.parametrize("routed_channels", [0, 32])
@pytest.mark.parametrize("proj_index", range(7))
def test_full_size_qwen2vl72b_routed_rank32(proj_index, routed_channels):
    # the routed-rank-32 ablation (five adapter atoms per unit on 256-token tiles), dense and with
    # cluster-sparse routed experts on 32 channels each; three more runs must be bit-identical
    cfg = qi.CONFIGS["qwen2vl72b_rr32"]
    c = Case(cfg, cfg.projections[proj_index], cfg.T, proj_index=proj_index, routed_channels=routed_channels)
    Y = _sampled_check(c, 256, 100 + proj_index)
    for _ in range(3):
        assert torch.equal(c.gpu_forward(), Y)
    assert qe.device_error() == 0


@pytest.mark.parametrize("proj_index", range(5))
def test_full_size_qwen2vl2b_w4a8_fp16_scales(proj_index):
    # W4A8 with fp16 group scales, the 2B layer set at T = 2048
    _full_size("qwen2vl2b_w4a8_s16", proj_index)


@pytest.mark.parametrize("T", [1, 16])
@pytest.mark.parametrize("proj_index", [0, 2])
def test_full_size_decode_w4a8_fp16_scales(T, proj_index):
    cfg = qi.CONFIGS["decode72b_w4a8_s16"].with_(T=T)
    c = Case(cfg, cfg.projections[proj_index], T, proj_index=proj_index)
    _forward_check(c, with_acc=False)


@pytest.mark.parametrize("T,K,N,group,a_bits", [(16, 1024, 640, 64, 8), (300, 512, 2048, 128, 6), (3, 384, 200, 64, 6)])
def test_forward_fp16_scales_small(T, K, N, group, a_bits):
    # every accumulator bit-exact with codes computed from fp16 scales (prefill and decode kernels)
    cfg = _cfg(group=group, a_bits=a_bits, rank_shared=32, n_routed=8, rank_routed=4, x_dtype="bf16",
               spec="qwen2b" if K >= 1024 else "tiny", scale_fp16=True)
    _forward_check(Case(cfg, qi.Projection("p", K, N), T))


@pytest.mark.parametrize("cfg_name", ["qwen2vl2b_w4a16", "qwen2vl2b_w3a16"])
@pytest.mark.parametrize("proj_index", range(5))
def test_full_size_weight_only_prefill(cfg_name, proj_index):
    # W4A16 / W3A16 prefill of the 2B layer set (T = 2048): 128-token tiles
    _full_size(cfg_name, proj_index)


@pytest.mark.parametrize("cfg_name", ["decode72b_w4a8", "decode72b_w3a16"])
@pytest.mark.parametrize("T", [1, 4, 16])
@pytest.mark.parametrize("proj_index", [0, 2])
def test_full_size_decode(cfg_name, T, proj_index):
    cfg = qi.CONFIGS[cfg_name].with_(T=T)
    proj = cfg.projections[proj_index]
    c = Case(cfg, proj, T, proj_index=proj_index)
    Y, _, expert, _, _ = c.gpu_debug(with_acc=False)
    e = expert.cpu().numpy()
    _, e_ref = oracle.route(c.inp["X"], c.inp["G"])
    check_routing(c.inp["X"], c.inp["G"], e, e_ref)
    Y_ref, _ = c.oracle_forward(expert_override=e)
    err = rel_err(Y.cpu().numpy(), Y_ref)
    assert err <= Y_TOL, err


@pytest.mark.parametrize("cfg_name,proj_index,T", [("tiny", 0, 64), ("qwen2vl2b", 4, 300), ("qwen2vl2b", 0, 129)])
def test_forward_ignores_workspace_contents(cfg_name, proj_index, T):
    # The header promises that the workspace's contents on entry do not matter:
    # garbage in the scratch must give bit-identical results.
    cfg = qi.CONFIGS[cfg_name]
    c = Case(cfg, cfg.projections[proj_index], T, proj_index=proj_index)
    ws = c.layer.workspace(T)
    outs = []
    for fill in (0x00, 0xFF, 0x7F):
        ws.fill_(fill)
        Y = torch.empty((T, c.proj.d_out), dtype=torch.float32, device="cuda")
        qe.linear_forward(c.desc, c.layer.weights, c.Xd, Y, ws)
        torch.cuda.synchronize()
        assert qe.device_error() == 0
        outs.append(Y)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


@pytest.mark.parametrize("proj_index", [2, 4])
def test_forward_full_size_is_deterministic(proj_index):
    # Every output element comes from one fixed sequence of operations: repeated runs of a
    # full-size layer must be bit-identical (a race shows up as a few differing rows).
    cfg = qi.CONFIGS["qwen2vl2b"]
    c = Case(cfg, cfg.projections[proj_index], cfg.T, proj_index=proj_index)
    ys = [c.gpu_forward() for _ in range(8)]
    for y in ys[1:]:
        bad = (~(y == ys[0]).all(dim=1)).nonzero().flatten().tolist()
        assert not bad, f"rows differing between runs: {bad[:10]}"


# ---------------------------------------------------------------- fp16 range of the packed up-projections

def test_adapter_up_projection_beyond_fp16_range_is_reported():
    # The packed up-projections are fp16 (qe.h, qe_pack_adapters). A bf16 value beyond 65504 is
    # stored as 65504 and reported through the device error word (0x201); values inside the
    # range leave the word clear.
    cfg = _cfg(T=16)
    proj = cfg.projections[0]
    inp = qi.layer_inputs(cfg, proj, T=16)
    assert qe.device_error() == 0
    Case(cfg, proj, 16, inp=inp)
    assert qe.device_error() == 0
    big = dict(inp)
    B = inp["B_s"].clone()
    B[0, 5] = 1.0e5
    big["B_s"] = B
    Case(cfg, proj, 16, inp=big)
    assert qe.device_error() == 0x201
    assert qe.device_error() == 0  # reading the word cleared it


@pytest.mark.parametrize("T", [16, 300])
def test_adapter_up_projection_below_fp16_normal_range(T):
    # Up-projection entries around 2e-6 sit in fp16's subnormal range (below 2^-14), where the
    # packed values keep fewer significant bits. The forward (decode product at T = 16, the int8
    # GEMM at T = 300) still meets the output tolerance against the oracle, which uses the bf16
    # values exactly.
    cfg = _cfg(T=T)
    proj = cfg.projections[0]
    inp = qi.layer_inputs(cfg, proj, T=T)
    small = dict(inp)
    small["B_s"] = (inp["B_s"].float() * 1e-4).to(torch.bfloat16)
    small["B_r"] = (inp["B_r"].float() * 1e-4).to(torch.bfloat16)
    _forward_check(Case(cfg, proj, T, inp=small))
