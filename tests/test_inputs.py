"""The seeded input generator: deterministic, the shapes and distributions the
workloads state (CPU only)."""
import math

import torch

from linear_attention_recurrence_rule_b200.inputs import (WORKLOADS, make_decode, make_prefill,
                                                          varlen_lengths, workload_inputs)


def test_deterministic():
    a = make_prefill(2, 4, 16, 16, [33, 33], torch.bfloat16, seed=5)
    b = make_prefill(2, 4, 16, 16, [33, 33], torch.bfloat16, seed=5)
    for k in ("q", "k", "v", "g", "beta"):
        assert torch.equal(a[k], b[k])


def test_distributions():
    x = make_prefill(4, 8, 128, 128, [2048], torch.float32, seed=1)
    assert torch.allclose(x["q"].norm(dim=-1), torch.ones(1), atol=1e-5)
    assert torch.allclose(x["k"].norm(dim=-1), torch.ones(1), atol=1e-5)
    alpha = x["g"].exp()
    assert alpha.min() >= 0.9 - 1e-6 and alpha.max() <= 1.0
    assert x["beta"].min() > 0 and x["beta"].max() < 1
    assert abs(float(x["v"].std()) - 1.0) < 0.02
    assert x["h0"] is None and x["cu_seqlens"] is None


def test_workload_shapes():
    assert (WORKLOADS["long_prefill_64k"].T, WORKLOADS["long_prefill_64k"].HV) == (65536, 32)
    w = WORKLOADS["layer_prefill_4k"]
    assert (w.HK, w.HV, w.dk, w.dv, w.chunk) == (16, 32, 128, 128, 64)
    x = workload_inputs("tiny_fp32")
    assert x["q"].shape == (1, 128, 1, 32) and x["v"].shape == (1, 128, 2, 32)
    assert x["q"].dtype == torch.float32


def test_varlen_lengths_and_packing():
    lens = varlen_lengths()
    assert len(lens) == 8 and all(1024 <= L <= 32768 for L in lens)
    x = make_prefill(1, 2, 8, 8, [3, 0, 5], torch.bfloat16, seed=2, h0_std=0.02, packed=True)
    assert x["cu_seqlens"].tolist() == [0, 3, 3, 8]
    assert x["q"].shape == (1, 8, 1, 8) and x["h0"].shape == (3, 2, 8, 8)


def test_decode_inputs():
    x = make_decode(3, 4, 2, 4, 16, 8, torch.bfloat16, seed=1)
    assert x["q"].shape == (4, 3, 2, 16) and x["v"].shape == (4, 3, 4, 8)
    assert x["state"].shape == (3, 4, 8, 16) and x["state"].dtype == torch.float32
    assert math.isclose(float(x["state"].std()), 0.02, rel_tol=0.2)


def test_verify_inputs_are_decode_draws_sequence_major():
    from linear_attention_recurrence_rule_b200.inputs import make_verify
    x = make_decode(3, 4, 2, 4, 16, 8, torch.bfloat16, seed=1)
    y = make_verify(3, 4, 2, 4, 16, 8, torch.bfloat16, seed=1)
    for n in ("q", "k", "v", "g", "beta"):
        assert torch.equal(y[n], x[n].transpose(0, 1)) and y[n].is_contiguous()
    assert torch.equal(y["state"], x["state"])
    w = WORKLOADS["verify_256x4"]
    assert (w.kind, w.B, w.T, w.HK, w.HV, w.dk) == ("verify", 256, 4, 16, 32, 128)


def test_raw_projections_scale_rows_and_draw_logits():
    from linear_attention_recurrence_rule_b200.inputs import raw_projections
    x = make_decode(3, 4, 2, 4, 16, 8, torch.float32, seed=1)
    y = raw_projections(x, seed=5)
    ratio = y["k"].norm(dim=-1) / x["k"].norm(dim=-1)
    assert bool(((ratio >= 0.25) & (ratio <= 4.0)).all()) and float(ratio.std()) > 0.1
    cos = (y["q"] * x["q"]).sum(-1) / (y["q"].norm(dim=-1) * x["q"].norm(dim=-1))
    assert torch.allclose(cos, torch.ones_like(cos), atol=1e-6)
    assert y["g"].shape == x["g"].shape and float(y["g"].mean()) > 2.0
    assert torch.equal(y["v"], x["v"]) and torch.equal(y["state"], x["state"])


def test_layer_extras_shapes_dtypes_and_seed():
    from linear_attention_recurrence_rule_b200.inputs import layer_extras
    a = layer_extras(3, 64, 4, (3, 7, 2, 32), torch.bfloat16, seed=9)
    b = layer_extras(3, 64, 4, (3, 7, 2, 32), torch.bfloat16, seed=9)
    c = layer_extras(3, 64, 4, (3, 7, 2, 32), torch.bfloat16, seed=10)
    assert a["conv_weight"].shape == (64, 4) and a["conv_weight"].dtype == torch.float32
    assert a["conv_bias"].shape == (64,) and a["conv_bias"].dtype == torch.float32
    assert a["conv_state"].shape == (3, 3, 64) and a["conv_state"].dtype == torch.bfloat16
    assert a["z"].shape == (3, 7, 2, 32) and a["z"].dtype == torch.bfloat16
    for k in a:
        assert torch.equal(a[k], b[k]) and not torch.equal(a[k], c[k])
    big = layer_extras(1, 4096, 4, (1,), torch.float32, seed=1)
    assert abs(float(big["conv_weight"].std()) - 0.5) < 0.02      # N(0, 1/W), W = 4
    assert abs(float(big["conv_bias"].std()) - 0.1) < 0.01
