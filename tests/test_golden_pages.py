"""The mixer's shapes and size accounting against the numbers the pages print
(tests/golden/page_numbers.json, each entry cited)."""
import json
import os

import pytest

import oracle
from gated_deltanet_mixer_gdn_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_numbers.json")))


def _printed(value: str) -> float:
    mult = {"K": 1e3, "M": 1e6}[value[-1]]
    return float(value[:-1]) * mult


def test_dims_match_pages():
    d = synth.MODEL
    assert d.num_k_heads == GOLD["num_k_heads"]["value"]
    assert d.num_v_heads == GOLD["num_v_heads"]["value"]
    assert d.head_dim == GOLD["head_dim"]["value"]
    assert d.conv_width == GOLD["conv_width"]["value"]
    # the fused projection carries q, k (16 heads each) and v (48 heads)
    assert d.conv_channels == GOLD["conv_channels"]["value"]
    assert d.value_width == GOLD["z_width"]["value"]
    assert d.num_v_heads == GOLD["gate_width"]["value"]


def test_parameter_accounting_pins_no_conv_bias():
    d = synth.MODEL
    H = GOLD["hidden"]["value"]
    conv = d.conv_channels * d.conv_width  # depthwise, no bias
    assert round(conv / 1e3, 1) == _printed(GOLD["conv1d_params_printed"]["value"]) / 1e3
    total = (H * d.conv_channels + H * d.value_width + 2 * H * d.num_v_heads  # in_proj qkv, z, b, a
             + d.value_width * H                                             # out_proj
             + conv + GOLD["gated_norm_params"]["value"] + sum(GOLD["linear_attn_params_printed"]["extra_vectors"]))
    assert round(total / 1e6, 1) == _printed(GOLD["linear_attn_params_printed"]["value"]) / 1e6
    # with a conv bias the total would still round the same, so also check the conv line alone
    assert round((conv + d.conv_channels) / 1e3, 1) != _printed(GOLD["conv1d_params_printed"]["value"]) / 1e3


def test_state_accounting():
    d = synth.MODEL
    per_layer = d.num_v_heads * d.head_dim * d.head_dim * 4  # f32
    total = per_layer * GOLD["gdn_layers"]["value"]
    assert abs(total / 1e6 - 150.0) / 150.0 < 0.01
    assert GOLD["state_dtype"]["value"] == "float32"


def test_eps_matches_page():
    assert oracle.EPS == GOLD["norm_eps"]["value"]
