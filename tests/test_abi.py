"""CPU checks of the C-ABI boundary: the library loads, exports every symbol
include/qe.h declares, and its host-side sizing and validation behave as the
header documents. No compute call runs here (there is no GPU)."""
import ctypes
import os
import re

import pytest

import quantized_gemm_moe_b200 as qe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "qe.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qe_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from quantized_gemm_moe_b200 import build
    build.build()
    return qe.load()


def test_library_exports_every_declared_symbol(lib):
    declared = _declared_symbols()
    assert declared, "no declarations parsed from include/qe.h"
    assert sorted(qe.EXPORTS) == declared
    for name in declared:
        assert hasattr(lib, name), name


def test_sizes_follow_documented_layout(lib):
    d = qe.make_desc(1536, 8960, 128, 4, 6, 32, 8, 4)
    assert qe.packed_weight_bytes(d) == (8960 // 128) * (1536 // 128) * 8192
    d3 = qe.make_desc(8192, 29568, 128, 3, 16, 32, 8, 4)
    assert qe.packed_weight_bytes(d3) == (29568 // 128) * (8192 // 128) * 6144
    # ragged d_out pads to whole 128-row blocks
    dr = qe.make_desc(256, 200, 64, 4, 8, 8, 4, 4)
    assert qe.packed_weight_bytes(dr) == 2 * 2 * 8192
    # adapters: A_catT [R_pad + 16][K] bf16 (down-projections + router rows) + B_catT [N][R_pad] fp16,
    # 256-byte aligned pieces; R_pad = round_up(r_s + N_r*r_r, 64) = 64 here
    R_pad, R_tot = 64, 80
    expect = 0
    for nbytes in (R_tot * 1536 * 2, 8960 * R_pad * 2):
        expect = ((expect + nbytes + 255) // 256) * 256
    assert qe.adapter_packed_bytes(d) == expect
    # a layer without adapters keeps only the router rows
    d0 = qe.make_desc(1536, 8960, 128, 4, 6, 0, 8, 0)
    assert qe.adapter_packed_bytes(d0) == ((16 * 1536 * 2 + 255) // 256) * 256
    assert qe.linear_workspace_bytes(d, 2048) > 2048 * 1536  # at least the int8 codes
    assert qe.linear_workspace_bytes(d, 0) > 0


@pytest.mark.parametrize("field,value,status", [
    ("group", 32, qe.QE_ERR_UNSUPPORTED),
    ("d_in", 100, qe.QE_ERR_INVALID_ARG),
    ("w_bits", 2, qe.QE_ERR_UNSUPPORTED),
    ("a_bits", 4, qe.QE_ERR_UNSUPPORTED),
    ("n_routed", 17, qe.QE_ERR_UNSUPPORTED),
    ("rank_shared", -1, qe.QE_ERR_INVALID_ARG),
    ("rank_routed", 200, qe.QE_ERR_UNSUPPORTED),  # 8 + 4*200 > 512
    ("routed_channels", -1, qe.QE_ERR_INVALID_ARG),
    ("routed_channels", 257, qe.QE_ERR_INVALID_ARG),   # more channels than d_in
])
def test_invalid_desc_rejected_before_launch(lib, field, value, status):
    d = qe.make_desc(256, 256, 64, 4, 8, 8, 4, 4)
    setattr(d, field, value)
    assert qe.packed_weight_bytes(d) == 0
    w = qe.LayerWeights(16, 16, 16, 16)
    rc = lib.qe_linear_forward(ctypes.byref(d), ctypes.byref(w), 16, 0, 4, 16, 0, 16, 1 << 30, None)
    assert rc == status


def test_forward_argument_checks(lib):
    d = qe.make_desc(256, 256, 64, 4, 8, 8, 4, 4)
    w = qe.LayerWeights(16, 16, 16, 16)
    f = lib.qe_linear_forward
    assert f(None, ctypes.byref(w), 16, 0, 4, 16, 0, 16, 1 << 30, None) == qe.QE_ERR_INVALID_ARG
    assert f(ctypes.byref(d), None, 16, 0, 4, 16, 0, 16, 1 << 30, None) == qe.QE_ERR_INVALID_ARG
    # T = 0 is a no-op that touches nothing
    assert f(ctypes.byref(d), ctypes.byref(w), None, 0, 0, None, 0, None, 0, None) == qe.QE_OK
    # misaligned pointer
    assert f(ctypes.byref(d), ctypes.byref(w), 18, 0, 4, 16, 0, 16, 1 << 30, None) == qe.QE_ERR_ALIGNMENT
    # workspace too small
    assert f(ctypes.byref(d), ctypes.byref(w), 16, 0, 4, 16, 0, 16, 8, None) == qe.QE_ERR_WORKSPACE
    # bad dtype
    assert f(ctypes.byref(d), ctypes.byref(w), 16, 7, 4, 16, 0, 16, 1 << 30, None) == qe.QE_ERR_INVALID_ARG


def test_other_entry_points_validate(lib):
    assert lib.qe_topk_importance(16, 1, 16, 4, 256, 0, 16, None, 0, None) == qe.QE_ERR_INVALID_ARG  # k = 0
    assert lib.qe_topk_importance(16, 1, 16, 4, 256, 129, 16, None, 0, None) == qe.QE_ERR_INVALID_ARG  # k > 128
    assert lib.qe_route(16, 1, 16, 4, 256, 0, 16, 16, 16, None, None) == qe.QE_ERR_INVALID_ARG  # n_routed = 0
    assert lib.qe_route(16, 1, 16, 4, 256, 17, 16, 16, 16, None, None) == qe.QE_ERR_INVALID_ARG
    assert lib.qe_act_quant(16, 1, 16, 4, 256, 5, 16, 16, None) == qe.QE_ERR_INVALID_ARG  # a_bits 5
    d = qe.make_desc(256, 256, 64, 4, 8, 8, 4, 4)
    assert lib.qe_quantize_weights(ctypes.byref(d), None, 0, 16, 16, 16, None, None, None, None) == \
        qe.QE_ERR_INVALID_ARG
    assert lib.qe_quantize_weights(ctypes.byref(d), 8, 0, 16, 16, 16, None, None, None, None) == qe.QE_ERR_ALIGNMENT
    # the s_inv output must be 16-byte aligned too
    assert lib.qe_quantize_weights(ctypes.byref(d), 16, 0, 16, 16, 16, None, None, 8, None) == qe.QE_ERR_ALIGNMENT
    assert lib.qe_pack_adapters(ctypes.byref(d), 16, 16, 16, 16, None, 16, None) == qe.QE_ERR_INVALID_ARG
    for s in range(7):
        assert lib.qe_status_string(s)


def test_cluster_sparse_sizes_and_checks(lib):
    # A_catT keeps the shared rows and the router (48 rows at r_s = 32), B_catT is unchanged, and the
    # packed buffer adds the channel lists (int32 [N_r][k_c]) and their weights (bf16 [N_r][k_c][r_r])
    d = qe.make_desc(1536, 8960, 128, 4, 6, 32, 8, 4, 32)
    expect = 0
    for nbytes in (48 * 1536 * 2, 8960 * 64 * 2, 8 * 32 * 4, 8 * 32 * 4 * 2):
        expect = ((expect + nbytes + 255) // 256) * 256
    assert qe.adapter_packed_bytes(d) == expect
    # no shared expert: the router alone is 16 rows; r_s = 8: 32 rows
    assert qe.adapter_packed_bytes(qe.make_desc(1536, 8960, 128, 4, 6, 0, 8, 4, 32)) > 0
    # the dense packing call refuses a sparse descriptor, and sparse routing needs routed ranks
    assert lib.qe_pack_adapters(ctypes.byref(d), 16, 16, 16, 16, 16, 16, None) == qe.QE_ERR_INVALID_ARG
    assert lib.qe_pack_adapters_sparse(ctypes.byref(d), 16, 16, None, 16, 16, 16, 16, None) == qe.QE_ERR_INVALID_ARG
    d_nr = qe.make_desc(1536, 8960, 128, 4, 6, 32, 8, 0, 32)
    assert qe.packed_weight_bytes(d_nr) == 0  # rejected: k_c > 0 without routed ranks
    d_wide = qe.make_desc(1536, 8960, 128, 4, 6, 248, 8, 4, 32)
    assert qe.packed_weight_bytes(d_wide) == 0  # r_s beyond the sparse GEMM widths


def test_binding_refuses_cpu_tensors(lib):
    import torch
    d = qe.make_desc(256, 256, 64, 4, 8, 8, 4, 4)
    with pytest.raises(qe.QEError):
        qe.quantize_weights(d, torch.zeros(256, 256), torch.ones(256), torch.zeros(10, dtype=torch.uint8),
                            torch.zeros(4, 256))


# (T, K, N, group, a_bits, w_bits, r_r) -> (tile tokens, adapter atoms): the GPU parity shapes
# that exercise the issuers' barrier rules must reach the tiles and atom counts they name
@pytest.mark.parametrize("T,K,N,group,a_bits,w_bits,rr,tile,atoms", [
    (2048, 512, 2048, 128, 8, 4, 32, 256, 5),
    (2048, 512, 2048, 64, 6, 4, 4, 256, 1),
    (2048, 512, 2048, 64, 8, 4, 32, 256, 5),
    (2048, 1536, 1536, 64, 6, 4, 32, 192, 5),
    (1000, 512, 1024, 128, 8, 4, 16, 128, 3),
    (1200, 512, 2048, 128, 16, 3, 32, 128, 5),
    (1200, 512, 2048, 64, 16, 4, 32, 128, 5),
    (48, 512, 1024, 64, 16, 4, 32, 64, 5),
    (200, 512, 1024, 128, 16, 3, 16, 64, 3),
])
def test_linear_plan_of_issuer_protocol_shapes(T, K, N, group, a_bits, w_bits, rr, tile, atoms):
    d = qe.make_desc(K, N, group, w_bits, a_bits, 32, 8, rr)
    p = qe.linear_plan(d, T)
    assert (p["product_tile_tokens"], p["adapter_atoms"]) == (tile, atoms)
    assert p["weight_only"] == (1 if a_bits == 16 else 0)


def test_linear_plan_of_the_2b_layer_set_and_72b_rank32():
    # the 2B layer set at T = 2048: q/o and down on 192-token tiles, gate/up on 256
    for K, N, tile in [(1536, 1536, 192), (1536, 8960, 256), (8960, 1536, 192)]:
        p = qe.linear_plan(qe.make_desc(K, N, 128, 4, 6, 32, 8, 4), 2048)
        assert (p["product_tile_tokens"], p["product_k_splits"], p["adapter_atoms"]) == (tile, 1, 1)
        assert (p["adapter_gemm_width"], p["adapter_gemm_tile"]) == (80, 80)
    # routed rank 32 at the 72B size: R_pad = 320 (five atoms), the router GEMM 384 wide in two tiles
    p = qe.linear_plan(qe.make_desc(8192, 29568, 128, 4, 6, 32, 8, 32), 8192)
    assert (p["product_tile_tokens"], p["adapter_atoms"], p["adapter_gemm_width"], p["adapter_gemm_tile"]) == \
        (256, 5, 384, 192)
    # fp32 inputs run the adapter GEMM twice (hi and lo), so the partial slots double
    pb = qe.linear_plan(qe.make_desc(1536, 1536, 128, 4, 8, 32, 8, 4), 300, qe.QE_BF16)
    pf = qe.linear_plan(qe.make_desc(1536, 1536, 128, 4, 8, 32, 8, 4), 300, qe.QE_F32)
    assert pf["adapter_gemm_splits"] == 2 * pb["adapter_gemm_splits"]
    with pytest.raises(qe.QEError):
        qe.linear_plan(qe.make_desc(1536, 1536, 128, 4, 8, 32, 8, 4), 0)


C_CLIENT = r"""
#include "qe.h"
#include <stdio.h>
int main(void) {
  qe_layer_desc d = {1536, 1536, 128, 4, 6, 32, 8, 4, 0, 0};
  qe_linear_plan_info p;
  qe_status s = qe_linear_plan(&d, 2048, QE_BF16, &p);
  printf("%d %s %d %d %zu %d\n", (int)s, qe_status_string(s), p.product_tile_tokens, p.adapter_atoms,
         qe_linear_workspace_bytes(&d, 2048), (int)qe_linear_kernel_launches(&d, 2048, QE_BF16));
  return s == QE_OK ? 0 : 1;
}
"""


def test_header_is_plain_c_and_links(lib, tmp_path):
    # the boundary is a C ABI: a strict C99 client compiles against include/qe.h without
    # warnings, links libqe.so and gets the same answers as the binding (host-only calls)
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src, exe = tmp_path / "client.c", tmp_path / "client"
    src.write_text(C_CLIENT)
    libdir = os.path.join(ROOT, "quantized_gemm_moe_b200")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                        str(src), "-L", libdir, "-lqe", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    st, text, tile, atoms, ws, launches = out.stdout.split()
    d = qe.make_desc(1536, 1536, 128, 4, 6, 32, 8, 4)
    assert (int(st), text) == (0, "ok")
    assert (int(tile), int(atoms)) == (192, 1)
    assert int(ws) == qe.linear_workspace_bytes(d, 2048)
    assert int(launches) == qe.linear_kernel_launches(d, 2048)
