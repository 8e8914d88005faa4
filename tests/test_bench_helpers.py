"""CPU checks of bench.py's arithmetic helpers (no GPU): the byte and
operation models the roofline fractions are built from."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from ternary_weight_selective_b200 import synthetic as S  # noqa: E402

PEAKS = {"hbm_gbs": 6531.3, "bf16_tflops": 1636.3}


def test_named_roofline_trissm_fused():
    wl = S.WORKLOADS["trissm"]
    names = ["bitssm_pre(quant_x+in_proj+x_proj)", "selective_scan_fused_dt",
             "bitssm_post(quant_y+out_proj)"]
    r = bench.named_roofline(wl, names, [0.0247, 0.0672, 0.0210], PEAKS, "measured")
    # in_proj 256x512, x_proj 512x48, out_proj 512x256; Delta-up is inside the scan
    assert r["ops_per_token"] == 2 * (256 * 512 + 512 * 48 + 512 * 256)
    expect = r["ops_per_token"] * 16384 / (0.0457e-3) / 1e12
    assert abs(r["achieved"] - round(expect, 2)) < 0.01
    assert r["peak"] == round(2 * 1636.3, 1) and r["unit"] == "TOPS"
    assert r["projections"] == [names[0], names[2]]


def test_named_roofline_a16_and_block():
    wl = S.WORKLOADS["mamba2_1p3b_a16"]
    names = ["row_rms_x", "gemm_in_proj", "gemm_x_proj", "gemm_dt_proj", "selective_scan",
             "row_rms_y", "gemm_out_proj"]
    r = bench.named_roofline(wl, names, [0.01, 0.17, 0.06, 0.09, 0.27, 0.02, 0.18], PEAKS, "measured")
    d, E, N, R = 2048, 4096, 16, 128
    assert r["ops_per_token"] == 2 * (d * E + E * (R + 2 * N) + E * d) + 2 * R * E
    assert r["unit"] == "TFLOP/s" and r["peak"] == 1636.3
    wb = S.WORKLOADS["trissm_block"]
    names_b = ["quant_rows_x", "gemm_in_proj", "gemm_z_proj", "conv_silu_quant_u", "gemm_x_proj",
               "selective_scan_fused_dt", "gate_quant_y", "gemm_out_proj"]
    rb = bench.named_roofline(wb, names_b, [0.01] * 8, PEAKS, "measured")
    assert rb["ops_per_token"] == 2 * (256 * 512 + 512 * 48 + 512 * 256) + 2 * 256 * 512
    assert len(rb["projections"]) == 4


def test_byte_models():
    wl = S.WORKLOADS["trissm"]
    # u int16 + scale, dt codes + factor, B, C, y fp32
    assert bench.scan_bytes_per_token(512, 16, 16) == 512 * 2 + 4 + 16 + 4 + 2 * 16 * 4 + 512 * 4
    assert bench.scan_bytes_per_token(512, 16, 16, u_f32=True) == 512 * 4 + 16 + 4 + 128 + 2048
    assert bench.pre_bytes_per_token(wl) == 256 * 2 + 512 * 2 + 4 + 128 + 16 + 4
    assert bench.post_bytes_per_token(wl) == 512 * 4 + 256 * 2
    assert bench.layer_bytes_per_token(S.WORKLOADS["trissm_block"]) > bench.layer_bytes_per_token(wl)
