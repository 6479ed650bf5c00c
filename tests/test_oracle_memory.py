"""Pins for the memory accounting formula against the figures the pages print."""
import pytest

import oracle
from conftest import read_golden


def test_printed_memory_figures_are_bits_of_the_byte_products():
    kv, _ = read_golden("memory_figures.txt")
    L, Hk, D, S = (int(kv[k]) for k in ("layers", "kv_heads", "head_dim", "seq"))
    fp32 = oracle.fp32_cache_bytes(L, Hk, S, D)
    assert fp32 == 32 * 2 * 4096 * 8 * 128 * 4 == 1_073_741_824
    values_only = oracle.cache_bytes(L, Hk, S, D, D, scale_bytes=0)
    assert values_only == 268_435_456
    # the printed GB figures equal 8x the byte products (bits), to 3 digits
    assert round(8 * fp32 / 1e9, 2) == float(kv["printed_fp32_gb"])
    assert round(8 * values_only / 1e9, 2) == float(kv["printed_q8_gb"])
    assert fp32 / values_only == float(kv["printed_reduction"])
    g32 = oracle.cache_bytes(L, Hk, S, D, int(kv["group"]))
    assert g32 == 301_989_888
    assert fp32 / g32 == pytest.approx(32 / 9)          # 3.556
    assert fp32 / g32 >= float(kv["printed_group32_vs_f32"])


def test_per_token_fp32_scale_overhead():
    # one fp32 scale per (token, kv head): head_dim + 4 bytes per row
    b = oracle.cache_bytes(1, 8, 1000, 128, 128)
    assert b == 2 * 8 * 1000 * (128 + 4)
    # against bf16 storage (2 bytes per value): 256 / 132 = 1.94 > 1.5
    assert (2 * 8 * 1000 * 128 * 2) / b > 1.5
