"""The seeded synthetic inputs follow the stated recipe (CPU generator, small sizes)."""
from __future__ import annotations

import dataclasses

import torch

from kimi_delta_attention_32_b200.workloads import (WORKLOADS, make_decode, make_prefill,
                                                    varlen_lengths)


def test_prefill_recipe():
    wl = dataclasses.replace(WORKLOADS["prefill_8k"], H=4)
    d = make_prefill(wl, "cpu", T=512)
    assert d["q"].dtype == torch.bfloat16 and d["q"].shape == (512, 4, 128)
    for x in (d["q"], d["k"]):
        n = x.double().norm(dim=-1)
        assert torch.all((n - 1).abs() < 1e-2)          # unit rows, then rounded to bf16
    g = d["g"]
    assert g.dtype == torch.float32 and torch.all(g <= 0)
    assert 0.9 < float(torch.exp(g).mean()) < 1.0        # u ~ N(4, 1): exp(g) mostly 0.9..1
    b = d["beta"]
    assert torch.all((b > 0) & (b < 1)) and abs(float(b.mean()) - 0.5) < 0.05
    assert d["h0"] is None and d["cu_host"] == [0, 512]
    # the same seed gives the same inputs
    assert torch.equal(make_prefill(wl, "cpu", T=512)["k"], d["k"])


def test_long_context_skew_channels():
    wl = dataclasses.replace(WORKLOADS["long_256k"], H=8)
    g = make_prefill(wl, "cpu", T=64)["g"]
    strong = torch.exp(g) < 0.5                          # [T, H, dk]
    per_channel = strong.all(dim=0)                      # every token of the channel decays fast
    assert torch.all(per_channel.sum(dim=-1) == 13)


def test_varlen_lengths_and_prologue_inputs():
    wl = WORKLOADS["varlen_prologue"]
    lens = varlen_lengths(wl)
    assert len(lens) == 64 and min(lens) >= 128 and max(lens) <= 16384
    assert sum(lens) == 527241
    small = dataclasses.replace(wl, N=3, H=2)
    d = make_prefill(small, "cpu", lengths=[5, 0, 70])
    assert d["cu_host"] == [0, 5, 5, 75]
    assert d["q_raw"].shape == (75, 2, 128) and d["w_v"].shape == (2 * 128, 4)
    assert d["h0"].shape == (3, 2, 128, 128) and abs(float(d["h0"].std()) - 0.02) < 2e-3


def test_decode_recipe():
    wl = WORKLOADS["decode_256x32"]
    d = make_decode(wl, "cpu", N=4, steps=3)
    assert d["q_raw"].shape == (3, 4, 32, 128) and d["g"].shape == (3, 4, 32, 128)
    assert d["conv_state"].shape == (4, 32 * 384, 3) and not d["conv_state"].any()
    assert torch.all(d["g"] <= 0)
