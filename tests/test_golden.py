"""Stored values: the pages' printed arithmetic, a hand-worked example, and an
oracle regression fixture written by tests/golden/make_golden.py."""
import json
import math
import os

import numpy as np
import pytest

import oracle as O
import synth
from decode_attention_lrkv_b200 import accounting as A

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def test_page_byte_arithmetic():
    g = _load("page_arithmetic.json")
    n = g["novakv_dense_cache"]
    dense = A.dense_kv_bytes_per_token(n["layers"], n["kv_heads"], n["d"], n["elem_bytes"])
    assert dense == 131072 and round(dense / 1000, 2) == n["printed_kb_per_token"]
    r = g["novakv_reduction"]
    assert round(100 * (1 - r["novakv_kb"] / r["dense_kb"]), 1) == r["printed_percent"]
    k = g["kvquant_fp16_basis"]
    fp16 = A.dense_kv_bytes_per_token(k["layers"], k["kv_heads"], k["d"], k["elem_bytes"])
    assert fp16 == k["printed_bytes_per_token"]
    assert round(fp16 * k["context"] / 1e9, 2) == k["printed_gb_at_context"]
    q = g["kvquant_nuq3"]
    exact = q["avg_bits"] / 16 * fp16
    assert exact == pytest.approx(109117.44, abs=1e-6)
    assert math.ceil(exact) == q["printed_stored_bytes"]
    assert round(fp16 / q["printed_ratio"]) == q["printed_ratio_bytes"]


def test_compressed_byte_counts():
    # Llama-3.1-8B geometry with r_k=64, r_v=96: 2*(64+96) B per token-head
    assert A.compressed_bytes_per_token_head(64, 96) == 320
    assert A.full_row_bytes(128) == 516
    # one decode call: 8 heads x 100 tokens, 3 of them full rank in head 0
    fc = [[3] + [0] * 7]
    b = A.decode_bytes(1, 32, 8, 128, 64, 96, [100], fc)
    want = (8 * 100 - 3) * 320 + 3 * 512 + 8 * 4 * 4 + 8 * 128 * 160 * 2 + 32 * 128 * 6
    assert b == want


def test_hand_worked_two_token_example():
    g = _load("hand_two_tokens.json")
    assert g["q"][0] == pytest.approx(2 * math.log(3), rel=1e-15)
    U = np.array(g["U"], float)[None]
    K = np.array(g["K"], float)[None, :, None, :]
    V = np.array(g["V"], float)[None, :, None, :]
    q = np.array(g["q"], float)[None, None, :]
    D = O.Dims(B=1, Hq=1, Hkv=1, d=4, r_k=2, r_v=2, T_cap=32, F_cap=32)
    for tau in (-1.0, 2.0):
        c = O.Cache.empty(D, U, U)
        O.compress(c, K, V, tau)
        np.testing.assert_allclose(O.decode_attn(c, q)[0, 0], g["expected_out"], atol=1e-14)


def test_tiny_workload_regression_fixture():
    from tests.golden.make_golden import tiny_workload_fixture
    want = _load("tiny_workload_seed0.json")
    got = tiny_workload_fixture(want["seed"])
    assert got["full_idx"] == want["full_idx"]
    assert got["coef_k_bits_sum"] == want["coef_k_bits_sum"]
    np.testing.assert_allclose(got["err_first8"], want["err_first8"], rtol=1e-12)
    np.testing.assert_allclose(got["out"], want["out"], rtol=1e-10, atol=1e-13)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_workload_routes_exactly_the_planted_outliers(seed):
    """The planted N(0,1) outlier rows (e ~ 0.87) are routed; signal rows (e ~ 0.15) are not."""
    w = synth.workload(0)
    L = synth.make_layer(w, 0, seed)
    f64 = lambda t: t.double().numpy()
    D = O.Dims(B=1, Hq=4, Hkv=1, d=128, r_k=32, r_v=32, T_cap=512, F_cap=512)
    c = O.Cache.empty(D, f64(L["U_k"]), f64(L["U_v"]))
    O.compress(c, f64(L["K"]), f64(L["V"]), w.tau)
    n = int(c.full_cnt[0, 0])
    assert c.full_idx[0, 0, :n].tolist() == L["outlier_pos"][0][0].tolist()
    assert n == round(0.02 * 512)
