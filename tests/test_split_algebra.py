"""The prefill kernel's state-transition split (the U form), checked on the CPU against the
token-by-token oracle: exactly in fp64, then with bf16 rounding at every tensor-core operand.
Covers a ragged last chunk, an initial state, an output scale and chunks that fail the range
test (decay beyond e^-80 in half a chunk) and so take the exact path."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from chunked_ref import split_chunk_fwd
from oracle_pins import random_inputs


def _rel(x, y):
    return float(np.linalg.norm(x - y) / np.linalg.norm(y))


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).bfloat16().double().numpy()


@pytest.mark.parametrize("strong,gain", [(False, 1.0), (True, 6.0)])
def test_split_matches_oracle_fp64(strong, gain):
    q, k, v, g, beta, S0 = random_inputs(21, 150, 2, 128, 128, strong=strong)
    g = g * gain
    o_ref, S_ref = oracle.kda_fwd(q, k, v, g, beta, 0.7, S0)
    o, S, nbad = split_chunk_fwd(q, k, v, g, beta, 0.7, S0)
    assert (nbad > 0) == strong          # the strong decay takes the exact path
    assert _rel(o, o_ref) < 1e-10
    assert _rel(S, S_ref) < 1e-10


def test_split_every_chunk_exact_path():
    """half_range = 0 sends every chunk down the exact path (gamma_ref = 0)."""
    q, k, v, g, beta, S0 = random_inputs(22, 130, 1, 128, 128)
    o_ref, S_ref = oracle.kda_fwd(q, k, v, g, beta, 1.0, S0)
    o, S, nbad = split_chunk_fwd(q, k, v, g, beta, 1.0, S0, half_range=0.0)
    assert nbad == 3
    assert _rel(o, o_ref) < 1e-10
    assert _rel(S, S_ref) < 1e-10


@pytest.mark.parametrize("strong,gain", [(False, 1.0), (True, 6.0)])
def test_split_bf16_operands_meet_the_bar(strong, gain):
    """bf16 operands with fp32-like accumulation stay within the 1e-2 rel-L2 bar of the bf16
    I/O path (inputs are rounded to bf16 first, as the kernel receives them)."""
    q, k, v, g, beta, S0 = random_inputs(23, 200, 2, 128, 128, strong=strong)
    q, k, v = _bf16(q), _bf16(k), _bf16(v)
    g = g * gain
    S0 = S0 * 0.1
    o_ref, S_ref = oracle.kda_fwd(q, k, v, g, beta, 1.0, S0)
    o, S, _ = split_chunk_fwd(q, k, v, g, beta, 1.0, S0, rounding=_bf16)
    assert _rel(o, o_ref) < 1e-2
    assert _rel(S, S_ref) < 1e-2
