"""How far two correct chains of stacked layers drift apart, asserted (CPU only).

The stacked parity tests accept, at layer l > 0, routing that any logits within
STACK_TAU * l of the oracle's allow (tests/harness.py).  This test backs that bound with
the oracle alone: it runs a checked token of the 8-layer batch-64 stack (the stacked
parity test's own draws) through the oracle twice, once as the parity tests do and once
with the bf16 rounding of every layer-output element that lies within REL (relative) of a
rounding boundary flipped at random, which is what an independently rounding fp32 chain
does to the fp64 chain's outputs.  While both chains select the same experts, layer l's
logits must stay within STACK_TAU * l / 2 of each other (half the bound the parity tests
use), and with the stacked draws' boundary gap the two chains must keep the same set.
"""
import numpy as np
import pytest

import synth
from oracle.layer import LayerRef, build_case
from tests import harness as H

REL = 2e-6  # fp32 vs fp64 values of a layer output differ by ~1e-7 relative; 20x that


def _bits_to_f64(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _round_bf16(v):
    u = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def divergence(tokens=(0, 37), chains=5, n_layers=8, rel=REL, seed_rng=2024):
    """Worst |logit difference| per layer between the oracle chain and perturbed chains."""
    seed, dims = synth.config_seed(4), synth.TP16
    refs = [LayerRef(seed, dims, l) for l in range(n_layers)]
    case = build_case(seed, dims, 64, n_layers=n_layers, checked=list(tokens), refs=refs,
                      min_boundary_gap=[2 * H.stack_tau(l) for l in range(n_layers)])
    rng = np.random.default_rng(seed_rng)
    worst = np.zeros(n_layers)
    same_sets = True
    for tok in tokens:
        for _ in range(chains):
            cur = case["resid"][tok].copy()
            for l in range(n_layers):
                f = refs[l].front(case["attn"][l, tok][None], cur[None])
                per = case["layers"][l]
                if set(f["idx"][0].tolist()) != set(per["idx"][tok].tolist()):
                    same_sets = False
                    break
                worst[l] = max(worst[l], float(np.abs(f["logits64"][0] - per["logits64"][tok]).max()))
                v = np.asarray(refs[l].moe(f, 0)[0], np.float64)
                q_bits = _round_bf16(v)
                q = _bits_to_f64(q_bits)
                ulp = np.abs(_bits_to_f64(q_bits + 1) - q)
                near = np.abs(np.abs(v - q) - ulp / 2) < rel * np.abs(v)
                flip = near & (rng.random(v.shape) < 0.5)
                alt = np.where(v > q, q_bits + 1, q_bits - 1).astype(np.uint16)
                cur = np.where(flip, alt, q_bits).astype(np.uint16)
    return worst, same_sets


@pytest.mark.slow
def test_stacked_chains_stay_within_half_the_bound():
    worst, same_sets = divergence()
    assert same_sets, "a perturbed chain selected other experts despite the boundary gap"
    assert worst[0] == 0.0  # layer 0 sees identical inputs
    for l in range(1, len(worst)):
        assert worst[l] <= H.stack_tau(l) / 2, (l, worst[l], H.stack_tau(l))
