"""Shared helpers of the GPU parity tests: build a layer on both sides from the
same seeded inputs, and compare with the tolerance the layer's fp outputs must meet."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import qe_inputs as qi
import quantized_gemm_moe_b200 as qe

# Final fp outputs: max relative error 2e-3 (bf16 adapters, fp32 accumulate), measured
# per element against max(|y_ref|, rms of the reference row), with fp32 outputs.
Y_TOL = 2e-3


def rel_err(y, yref) -> float:
    y = np.asarray(y, np.float64)
    yref = np.asarray(yref, np.float64)
    rms = np.sqrt((yref ** 2).mean(axis=-1, keepdims=True))
    den = np.maximum(np.abs(yref), rms)
    den = np.where(den > 0, den, 1.0)
    return float((np.abs(y - yref) / den).max())


def cuda(a, dtype=None):
    if isinstance(a, np.ndarray):
        t = torch.from_numpy(np.ascontiguousarray(a))
    else:
        t = a
    if dtype is not None:
        t = t.to(dtype)
    return t.contiguous().cuda()


def f32(a) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        return a.detach().float().cpu().numpy()
    return np.asarray(a, np.float32)


class Case:
    """One layer with its inputs on both sides (CPU oracle and GPU library)."""

    def __init__(self, cfg: qi.LayerConfig, proj: qi.Projection, T: int, proj_index: int = 0, inp=None,
                 routed_channels: int = 0, sparse_seed: int = 77):
        """routed_channels > 0: cluster-sparse routed experts (qe_inputs.sparse_routed). The oracle
        then gets the equivalent dense A_r: zero outside each expert's channels."""
        self.cfg = cfg
        self.proj = proj
        self.T = T
        self.inp = inp if inp is not None else qi.layer_inputs(cfg, proj, T=T, proj_index=proj_index)
        self.desc = qe.make_desc(proj.d_in, proj.d_out, cfg.group, cfg.w_bits, cfg.a_bits, cfg.rank_shared,
                                 cfg.n_routed, cfg.rank_routed, routed_channels, cfg.scale_fp16)
        i = self.inp
        self.Xd = cuda(i["X"])
        if routed_channels:
            ch, A_rs = qi.sparse_routed(proj.d_in, cfg.n_routed, routed_channels, cfg.rank_routed, sparse_seed)
            dense = torch.zeros((cfg.n_routed, proj.d_in, cfg.rank_routed), dtype=torch.bfloat16)
            for e in range(cfg.n_routed):
                dense[e, torch.from_numpy(ch[e]).long()] += A_rs[e]
            i["A_r"] = dense
            self.layer = qe.QELayer.from_float(self.desc, cuda(i["W"]), cuda(i["s"]), cuda(i["A_s"]), cuda(i["B_s"]),
                                               cuda(A_rs), cuda(i["B_r"]), cuda(i["G"]),
                                               channels=cuda(ch))
        else:
            self.layer = qe.QELayer.from_float(self.desc, cuda(i["W"]), cuda(i["s"]), cuda(i["A_s"]), cuda(i["B_s"]),
                                               cuda(i["A_r"]), cuda(i["B_r"]), cuda(i["G"]))
        self._ref = None

    def oracle_weights(self):
        if self._ref is None:
            self._ref = oracle.quantize_weights(self.inp["W"], self.inp["s"], self.cfg.group, self.cfg.w_bits,
                                                scale_fp16=self.cfg.scale_fp16)
        return self._ref

    def oracle_forward(self, rows=None, expert_override=None):
        codes, scales, _, _ = self.oracle_weights()
        i = self.inp
        return oracle.qe_forward(i["X"], codes, scales, oracle.smoothing_inverse(i["s"]), i["A_s"], i["B_s"], i["A_r"], i["B_r"], i["G"],
                                 self.cfg.group, self.cfg.a_bits, rows=rows, expert_override=expert_override)

    def gpu_forward(self, out_dtype=torch.float32):
        Y = self.layer.forward(self.Xd, out_dtype=out_dtype)
        torch.cuda.synchronize()
        assert qe.device_error() == 0
        return Y

    def gpu_debug(self, with_acc: bool):
        T, N, G = self.T, self.proj.d_out, self.proj.d_in // self.cfg.group
        Y = torch.empty((T, N), dtype=torch.float32, device="cuda")
        acc = torch.full((T, N, G), -(2 ** 31), dtype=torch.int32, device="cuda") if with_acc else None
        expert = torch.empty(T, dtype=torch.int32, device="cuda")
        perm = torch.empty(T, dtype=torch.int32, device="cuda")
        sa = torch.empty(T, dtype=torch.float32, device="cuda")
        qe.linear_forward_debug(self.desc, self.layer.weights, self.Xd, Y, self.layer.workspace(T), acc, expert,
                                perm, sa)
        torch.cuda.synchronize()
        assert qe.device_error() == 0
        return Y, acc, expert, perm, sa


def check_routing(X, G, gpu_expert, oracle_expert):
    """Router choices must be bit-exact except on near-ties (fp32 vs fp64 logits).
    Returns the tokens where the GPU legitimately took the other side of a near-tie."""
    gpu_expert = np.asarray(gpu_expert)
    oracle_expert = np.asarray(oracle_expert)
    diff = np.nonzero(gpu_expert != oracle_expert)[0]
    if diff.size:
        L, _ = oracle.route(np.asarray(f32(X))[diff], f32(G))
        bound = oracle.router_near_tie_bound(np.asarray(f32(X))[diff], f32(G))
        gap = L[np.arange(diff.size), gpu_expert[diff]] - L[np.arange(diff.size), oracle_expert[diff]]
        assert (gap <= bound).all(), f"router mismatch beyond the fp32 near-tie bound at tokens {diff[gap > bound]}"
    return diff
