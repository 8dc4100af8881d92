"""The float64 oracle against its pins (CPU only)."""
import json
import math
import os

import pytest

import ag_inputs
import oracle_pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(oracle_lib, pin):
    pin(oracle_lib)


def test_oracle_rejects_bad_arguments(oracle_lib):
    import numpy as np

    q = np.zeros((1, 1, 32, 4))
    k = np.zeros((1, 32, 4))
    v = np.zeros((1, 32, 4))
    bias = np.zeros((1, 2, 2))
    for cap in (0.0, -1.0, math.nan):
        with pytest.raises(ValueError):
            oracle_lib.attn_fwd(q, k, v, bias, block=16, cap=cap)
    with pytest.raises(ValueError):  # bias not [H, ceil(L/block), ...]
        oracle_lib.attn_fwd(q, k, v, np.zeros((1, 3, 3)), block=16, cap=5.0)
    with pytest.raises(ValueError):  # per-item bias for the wrong batch size
        oracle_lib.attn_fwd(q, k, v, np.zeros((2, 1, 2, 2)), block=16, cap=5.0)
    with pytest.raises(ValueError):  # row index out of range
        oracle_lib.attn_rows(q, k, v, bias, [[0, 0, 32]], block=16, cap=5.0)


def test_oracle_empty_batch(oracle_lib):
    import numpy as np

    out, lse = oracle_lib.attn_fwd(np.zeros((0, 8, 32, 4)), np.zeros((0, 32, 4)),
                                   np.zeros((0, 32, 4)), np.zeros((8, 2, 2)),
                                   block=16, cap=5.0)
    assert out.shape == (0, 8, 32, 4) and lse.shape == (0, 8, 32)


def test_page_workload_figures():
    """The workload sizes match the figures the pages print (fixture cites
    them): 8192 positions at 1,048,576 bp, a [1,8,8192,8192] fp32 logit
    tensor of 2 GiB, D = 128, a 16-position bias cell, P = 512."""
    with open(os.path.join(GOLDEN, "page_workload_figures.json")) as f:
        g = json.load(f)
    full = ag_inputs.WORKLOADS["full"]
    assert g["input_bp"] // g["bp_per_position"] == full.L == g["transformer_length"]
    assert g["input_bp"] // g["bp_per_pair_cell"] == full.P
    assert full.L // full.block == full.P and full.block == g["bias_cell_positions"]
    assert full.H == g["query_heads"] and full.D == g["qk_width"]
    dense = full.B * full.H * full.L * full.L * 4
    assert dense == g["dense_logit_bytes"]
    assert g["cap"] == full.cap


def test_nine_block_caps_are_drawn_from_the_set():
    st = ag_inputs.nine_block_stack()
    assert len(st.layers) == 9
    assert [w.seed for w in st.layers] == list(range(10, 19))
    assert all(w.cap in (5.0, 10.0, 30.0) for w in st.layers)
