"""How far two correct chains of stacked layers drift apart (a script, not a test).

Runs the 8-layer batch-64 stack's checked tokens (the draws of the stacked parity
test) through the oracle twice: once as the
parity tests do, once with the bf16 rounding of every layer output element that lies
within REL (relative) of a rounding boundary flipped at random, which is what an fp32
chain does to the fp64 chain's outputs.  Prints, per layer, the largest logit
difference between the two chains and whether they selected the same experts in the
same order.  The stacked tolerance in tests/harness.py (STACK_TAU) is set from this.

    python tests/stack_divergence.py [REL=2e-6] [CHAINS_PER_TOKEN=10]
"""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import synth  # noqa: E402
from oracle.layer import LayerRef, build_case  # noqa: E402
from tests import harness as H  # noqa: E402


def _bits_to_f64(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _round_bf16(v):
    u = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def main(rel=2e-6, chains=10, tokens=(0, 37), n_layers=8):
    seed, dims = synth.config_seed(4), synth.TP16
    refs = [LayerRef(seed, dims, l) for l in range(n_layers)]
    # the stacked parity test's case, draws included
    case = build_case(seed, dims, 64, n_layers=n_layers, checked=list(tokens), refs=refs,
                      min_boundary_gap=[2 * H.stack_tau(l) for l in range(n_layers)])
    rng = np.random.default_rng(2024)
    worst = np.zeros(n_layers)
    for tok in tokens:
        for chain in range(chains):
            cur = case["resid"][tok].copy()
            row, diverged = [], False
            for l in range(n_layers):
                f = refs[l].front(case["attn"][l, tok][None], cur[None])
                per = case["layers"][l]
                dz = float(np.abs(f["logits64"][0] - per["logits64"][tok]).max())
                same = bool(np.array_equal(f["idx"][0], per["idx"][tok]))
                same_set = set(f["idx"][0].tolist()) == set(per["idx"][tok].tolist())
                diverged |= not same_set
                if not diverged:
                    worst[l] = max(worst[l], dz)
                v = np.asarray(refs[l].moe(f, 0)[0], np.float64)
                q_bits = _round_bf16(v)
                q = _bits_to_f64(q_bits)
                ulp = np.abs(_bits_to_f64(q_bits + 1) - q)
                near = np.abs(np.abs(v - q) - ulp / 2) < rel * np.abs(v)
                flip = near & (rng.random(v.shape) < 0.5)
                alt = np.where(v > q, q_bits + 1, q_bits - 1).astype(np.uint16)
                cur = np.where(flip, alt, q_bits).astype(np.uint16)
                row.append(f"L{l}:{dz:.1e}{'' if same else ('~' if same_set else '!')}")
            print(f"token {tok} chain {chain}: " + " ".join(row), flush=True)
    print("worst |dz| per layer while the selected sets agree:", " ".join(f"{w:.1e}" for w in worst))
    print("worst |dz| / layer:", " ".join(f"{w / max(l, 1):.1e}" for l, w in enumerate(worst)))


if __name__ == "__main__":
    main(float(sys.argv[1]) if len(sys.argv) > 1 else 2e-6, int(sys.argv[2]) if len(sys.argv) > 2 else 10)
