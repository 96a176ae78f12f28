"""Host-side logic with no GPU: the stacked-layer routing check, the bench's byte model and
its kernel-code hash, and the oracle-side draw rule for stacked layers."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from oracle.layer import boundary_gap, top_gap  # noqa: E402
from tests import harness as H  # noqa: E402


def _route(z, k):
    idx = np.argsort(-np.asarray(z), kind="stable")[:k]
    v = np.asarray(z)[idx]
    g = np.exp(v - v[0])
    return idx.astype(np.int32), g / g.sum()


def test_stacked_route_check_accepts_the_oracle_itself():
    rng = np.random.default_rng(0)
    z = rng.normal(size=64)
    idx, gate = _route(z, 8)
    H.check_route_stacked(idx, gate, idx, gate, z, tau=1e-3)


def test_stacked_route_check_accepts_a_near_tie_swap_and_rejects_a_far_one():
    z = np.linspace(1.0, 0.0, 32)
    z[3] = z[2] - 1e-3  # experts 2 and 3 nearly tie
    idx, gate = _route(z, 6)
    sw = idx.copy()
    sw[[2, 3]] = sw[[3, 2]]
    g_sw = gate.copy()
    g_sw[[2, 3]] = g_sw[[3, 2]]
    H.check_route_stacked(sw, g_sw, idx, gate, z, tau=1e-3)  # 1e-3 apart: within 2 tau
    far = idx.copy()
    far[[0, 1]] = far[[1, 0]]  # 1/31 apart
    g_far = gate.copy()
    g_far[[0, 1]] = g_far[[1, 0]]
    with pytest.raises(AssertionError):
        H.check_route_stacked(far, g_far, idx, gate, z, tau=1e-3)


def test_stacked_route_check_rejects_another_set_and_wrong_gates():
    rng = np.random.default_rng(1)
    z = rng.normal(size=40)
    idx, gate = _route(z, 5)
    other = idx.copy()
    other[-1] = np.argsort(-z, kind="stable")[5]  # the sixth expert instead of the fifth
    with pytest.raises(AssertionError):
        H.check_route_stacked(other, gate, idx, gate, z, tau=1.0)
    with pytest.raises(AssertionError):
        H.check_route_stacked(idx, gate + 1e-2, idx, gate, z, tau=1e-3)  # > tau / 2


def test_stack_tolerance_grows_with_depth():
    assert H.stack_tau(0) == 0.0
    assert H.stack_tau(7) == pytest.approx(7 * H.STACK_TAU)


def test_gap_helpers():
    z = np.array([5.0, 4.0, 3.5, 3.4, 1.0])
    assert top_gap(z, 3) == pytest.approx(0.1)
    assert boundary_gap(z, 3) == pytest.approx(0.1)
    assert boundary_gap(z, 2) == pytest.approx(0.5)
    assert boundary_gap(z, 5) == np.inf


def test_kernel_hash_ignores_comments(tmp_path):
    import bench
    a, b = tmp_path / "a", tmp_path / "b"
    a.mkdir()
    b.mkdir()
    code = 'int f() { return 1; }  // one\n/* block\n comment */\nconst char* s = "http://x"; // two\n'
    (a / "k.cu").write_text(code)
    (b / "k.cu").write_text("// header\n" + code.replace("// one", "// changed") + "\n\n")
    assert bench.kernels_sha(str(a)) == bench.kernels_sha(str(b))
    (b / "k.cu").write_text(code.replace("return 1", "return 2"))
    assert bench.kernels_sha(str(a)) != bench.kernels_sha(str(b))
    assert 'const char* s = "http://x";' in bench.code_only(code)


def test_fused_kernel_bytes_are_every_weight_once():
    import bench
    D = synth.TP16
    ab = bench.algorithmic_bytes(D, 1, 16)
    weights = D.d * D.d_o * 2 + D.E * D.d * 2 + D.d * 2 + 16 * 3 * D.I * D.d * 2
    assert ab["layer_fused_small_m"] == weights + D.d_o * 2 + D.d * 4
    assert bench.weight_bytes(D, [16]) == weights


@pytest.mark.slow
@pytest.mark.parametrize("B,core", [(2, 8), (4, 12), (8, 12)])
def test_bench_constructed_sets_route_as_built(B, core):
    """The benchmark's constructed inputs (attn_out = 0, residual steered towards chosen expert
    sets sharing `core` experts) select exactly those sets in the oracle."""
    import bench
    from oracle.layer import LayerRef
    D = synth.TP16
    seed_w = bench.seed_of("TP16", 1) + 1000  # the second weight copy of the rotation
    attn, resid = bench.constructed_sets(seed_w, D, B, core)
    assert attn.shape == (1, B, D.d_o) and not attn.any()
    f = LayerRef(seed_w, D, 0).front(attn[0], resid)
    sets = [set(f["idx"][b].tolist()) for b in range(B)]
    common = set.intersection(*sets)
    assert all(len(x) == D.k for x in sets) and len(common) == core
    assert len(set.union(*sets)) == core + B * (D.k - core)
