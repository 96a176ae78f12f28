"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Every case uses seeded synthetic inputs; indices and their order must match
exactly (in a stack's later layers: any order the oracle's logits allow within
the chains' divergence), gates and intermediates within fp32-vs-fp64 tolerances,
the bf16 output within the layer's bar (tests/harness.py).
"""
import gc

import numpy as np
import pytest

import synth
from oracle.layer import LayerRef, build_case
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_decode_layer_02_b200 as md
    md.load()
    synth.build_device_fill()
    yield
    gc.collect()
    torch.cuda.empty_cache()


def check_case(stack: H.GpuStack, case: dict, sampled=None, check_intermediates=True):
    """Runs the step and compares every checked token (outputs for `sampled`)."""
    out, idx, gate = stack.step(case["attn"], case["resid"])
    L = len(case["layers"])
    B = case["attn"].shape[1]
    for l, per in enumerate(case["layers"]):
        for b in per["idx"]:
            if l == 0:
                assert np.array_equal(idx[l, b], per["idx"][b]), (l, b, idx[l, b], per["idx"][b])
                H.note("gate_abs", np.abs(gate[l, b] - per["gate"][b]).max())
                assert np.allclose(gate[l, b], per["gate"][b], atol=H.GATE_ATOL, rtol=0), (l, b)
            else:
                H.check_route_stacked(idx[l, b], gate[l, b], per["idx"][b], per["gate"][b],
                                      per["logits64"][b], H.stack_tau(l), where=(l, b))
    last = case["layers"][-1]
    toks = sorted(last["out_ref"]) if sampled is None else sampled
    res = []
    for b in toks:
        extra = sum(H.ulp_bf16(case["layers"][l]["out_ref"][b]) for l in range(L - 1)) if L > 1 else 0.0
        res.append(H.check_out(out[b], last["out_ref"][b], extra))
    if check_intermediates and L == 1:
        D = stack.dims
        hg = stack.intermediate(0, B).reshape(B, D.d)
        rs = stack.intermediate(1, B)
        xg = stack.intermediate(2, B).reshape(B, D.d)
        lg = stack.intermediate(3, B).reshape(B, D.E)
        for b in last["h"]:
            assert np.allclose(hg[b], last["h"][b], atol=1e-4, rtol=1e-5)
            assert abs(rs[b] - last["rstd"][b]) <= 1e-5 * last["rstd"][b]
            assert np.allclose(xg[b], last["x"][b], atol=1e-5, rtol=1e-5)
            H.note("logit_abs", np.abs(lg[b] - last["logits64"][b]).max())
            assert np.allclose(lg[b], last["logits64"][b], atol=1e-4, rtol=0)
    return out, idx, gate, res


# --- tiny layer (d=256, d_o=256, E=16, k=2, I=128), batch 1 -----------------------------
def test_tiny_b1():
    seed = synth.config_seed(0)
    st = H.GpuStack(seed, synth.TINY, max_batch=1)
    try:
        case = build_case(seed, synth.TINY, 1)
        check_case(st, case)
    finally:
        st.close()


@pytest.mark.parametrize("B", [1, 2, 3, 5, 16, 64])
@pytest.mark.parametrize("variant", [0, 1, 2, 3])
def test_tiny_batches_and_variants(B, variant):
    seed = synth.config_seed(0) + 100 * B
    st = H.GpuStack(seed, synth.TINY, max_batch=64, force_variant=variant)
    try:
        case = build_case(seed, synth.TINY, B)
        check_case(st, case)
    finally:
        st.close()


def test_synth_device_matches_host():
    import torch
    seed = 12345
    for kind, n, start in [(synth.W_O, 1000, 0), (synth.W_GU, 777, 13), (synth.ATTN, 64, 5)]:
        x = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        synth.device_fill(x, seed, kind, layer=3, start=start)
        got = x.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, synth.gen_bf16(seed, kind, n, layer=3, start=start))


# --- ragged shapes: d not a multiple of 256 (no split-K), odd d_o/E/k/I ----------------------
@pytest.mark.parametrize("B", [1, 2, 3, 7])
def test_ragged_shapes(B):
    dims = synth.Dims(320, 192, 40, 5, 96)
    seed = synth.config_seed(9) + B
    st = H.GpuStack(seed, dims, max_batch=8)
    try:
        check_case(st, build_case(seed, dims, B))
    finally:
        st.close()


# --- max_batch equal to the batch, not a multiple of 8: the workspace is sized for max_batch
#     while the split-K router pads the batch to 8 per expert --------------------------------
@pytest.mark.parametrize("B", [3, 5])
def test_ragged_max_batch_equals_batch(B):
    dims = synth.Dims(320, 192, 40, 5, 96)
    seed = synth.config_seed(10) + B
    st = H.GpuStack(seed, dims, max_batch=B)
    try:
        check_case(st, build_case(seed, dims, B))
    finally:
        st.close()


# --- the largest shapes the library accepts, one dimension at a time -----------------------
#   d = d_o = 8192 with k = 32 and I = 512 (64 experts keep the weights at ~1.2 GB), and
#   E = 1024 with k = 32 on d = 1024 (large enough a logit spread for gapped draws).  Batch 1
#   (the fused kernel, or the large-batch kernels where its shared memory does not fit), 2
#   and 64; every token is checked.
@pytest.mark.slow
@pytest.mark.parametrize("B", [1, 2, 64])
@pytest.mark.parametrize("dims", [synth.Dims(8192, 8192, 64, 32, 512), synth.Dims(1024, 256, 1024, 32, 32)],
                         ids=["d8192_k32_I512", "E1024_k32"])
def test_maximum_sizes(dims, B):
    seed = synth.config_seed(13) + B + dims.E
    st = H.GpuStack(seed, dims, max_batch=64)
    try:
        check_case(st, build_case(seed, dims, B))
    finally:
        st.close()


# --- ties: the selection order is (logit descending, expert index ascending) ---------------
#   x = 0 makes every logit exactly 0 (every candidate ties: the routing falls back to k
#   rounds of arg-max), and a router whose rows come in identical pairs makes pairs of
#   logits bitwise equal (the lower index must come first).  TP16 shapes, at batch 1
#   (fused kernel), 2 (small-batch expert kernel) and 16 (router's routing tables).
@pytest.fixture(scope="module")
def tp16_tied():
    import torch
    seed = synth.config_seed(5)
    w = H.device_weights(seed, synth.TP16, 1)
    wr = w[0][2].view(synth.TP16.E, synth.TP16.d)
    wr[1::2] = wr[0::2]  # rows 2m and 2m + 1 identical
    torch.cuda.synchronize()
    ref = LayerRef(seed, synth.TP16, 0)
    wr_h = ref.W_r.reshape(synth.TP16.E, synth.TP16.d).copy()
    wr_h[1::2] = wr_h[0::2]
    ref.W_r = wr_h.reshape(-1)
    st = H.GpuStack(seed, synth.TP16, max_batch=16, weights=w)
    yield seed, st, ref
    st.close()


@pytest.mark.slow
@pytest.mark.parametrize("B", [1, 2, 4, 16])
def test_ties_all_logits_zero(tp16_tied, B):
    seed, st, ref = tp16_tied
    D = synth.TP16
    attn = np.zeros((1, B, D.d_o), np.uint16)
    resid = np.zeros((B, D.d), np.uint16)
    out, idx, gate = st.step(attn, resid)
    f = ref.front(attn[0], resid)
    assert np.all(f["logits32"] == 0) and np.array_equal(f["idx"], np.tile(np.arange(D.k), (B, 1)))
    for b in range(B):
        assert np.array_equal(idx[0, b], np.arange(D.k)), idx[0, b]
        assert np.allclose(gate[0, b], 1.0 / D.k, atol=H.GATE_ATOL, rtol=0)
    assert np.all(synth.bf16_bits_to_f32(out) == 0.0)


@pytest.mark.slow
@pytest.mark.parametrize("B", [1, 2, 4, 16])
def test_ties_duplicated_router_rows(tp16_tied, B):
    from oracle.layer import top_gap_distinct
    seed, st, ref = tp16_tied
    case = build_case(seed + B, synth.TP16, B, refs=[ref], gap_fn=top_gap_distinct)
    out, idx, gate, _ = check_case(st, case)
    for b in range(B):  # every selected pair of tied experts comes lower index first
        sel = idx[0, b].tolist()
        assert sum(1 for e in sel if e % 2 == 0 and e + 1 in sel) >= 1
        for e in sel:
            if e % 2 == 1 and e - 1 in sel:
                assert sel.index(e - 1) == sel.index(e) - 1, sel


@pytest.mark.parametrize("B", [1, 3])
def test_degenerate_k_equals_e_and_k1(B):
    for dims in (synth.Dims(128, 64, 4, 4, 32), synth.Dims(128, 128, 8, 1, 64)):
        seed = synth.config_seed(11) + dims.k + B
        st = H.GpuStack(seed, dims, max_batch=4)
        try:
            check_case(st, build_case(seed, dims, B))
        finally:
            st.close()


@pytest.mark.parametrize("B", [1, 2, 4, 16])
def test_determinism_replay(B):
    """Replays give the same bits on every kernel path: the fused kernel (its o_proj units
    taken from a counter in a different order every launch; at d = 256 all of them are), the
    small-batch kernels for two and four tokens, and the large-batch kernels."""
    seed = synth.config_seed(0) + 7 + B
    st = H.GpuStack(seed, synth.TINY, max_batch=16)
    try:
        case = build_case(seed, synth.TINY, B)
        o1, i1, g1 = st.step(case["attn"], case["resid"])
        o2, i2, g2 = st.step(case["attn"], case["resid"], reps=3)
        assert np.array_equal(o1, o2) and np.array_equal(i1, i2) and np.array_equal(g1, g2)
    finally:
        st.close()


# --- full-size layer (one GPU's 1/16 tensor-parallel shard), batch 1 --------------------------
@pytest.fixture(scope="module")
def tp16():
    seed = synth.config_seed(1)
    st = H.GpuStack(seed, synth.TP16, max_batch=64)
    ref = LayerRef(seed, synth.TP16, 0)
    yield seed, st, ref
    st.close()


@pytest.mark.slow
def test_tp16_b1_replay_bits(tp16):
    """Full-size batch 1: two launches of the fused kernel give the same output bits."""
    seed, st, ref = tp16
    case = build_case(seed + 11, synth.TP16, 1, refs=[ref])
    o1, i1, g1 = st.step(case["attn"], case["resid"])
    o2, i2, g2 = st.step(case["attn"], case["resid"], reps=2)
    assert np.array_equal(o1, o2) and np.array_equal(i1, i2) and np.array_equal(g1, g2)


@pytest.mark.slow
def test_tp16_b1(tp16):
    seed, st, ref = tp16
    check_case(st, build_case(seed, synth.TP16, 1, refs=[ref]))


@pytest.mark.slow
def test_tp16_b1_counter_ordered_kernel(tp16):
    seed, _, ref = tp16
    st = H.GpuStack(seed, synth.TP16, max_batch=2, force_variant=3, weights=H.device_weights(seed, synth.TP16, 1))
    try:
        check_case(st, build_case(seed, synth.TP16, 1, refs=[ref]))
        attn0, resid0, _ = H.constructed_b2(seed, synth.TP16, 8, ref=ref)
        check_case(st, build_case(seed, synth.TP16, 2, attn0=attn0, resid0=resid0, refs=[ref]))
    finally:
        st.close()


@pytest.mark.slow
@pytest.mark.parametrize("overlap", [16, 8, 0])
def test_tp16_b2_overlap(tp16, overlap):
    seed, st, ref = tp16
    attn0, resid0, (S0, S1) = H.constructed_b2(seed, synth.TP16, overlap, ref=ref)
    case = build_case(seed, synth.TP16, 2, attn0=attn0, resid0=resid0, refs=[ref])
    out, idx, gate, _ = check_case(st, case)
    assert len(set(idx[0, 0]) & set(idx[0, 1])) == overlap


# --- speculative verification: 1 sequence x (3 or 7 drafts + 1) tokens sharing 12 experts ------
@pytest.mark.slow
@pytest.mark.parametrize("B", [4, 8])
def test_tp16_speculative_shapes(tp16, B):
    seed, st, ref = tp16
    attn0, resid0, sets = H.constructed_shared(seed, synth.TP16, B, core=12, ref=ref)
    case = build_case(seed, synth.TP16, B, attn0=attn0, resid0=resid0, refs=[ref])
    out, idx, gate, _ = check_case(st, case)  # every token
    assert len(set(idx[0].ravel().tolist())) == 12 + B * (synth.TP16.k - 12)


@pytest.mark.slow
@pytest.mark.parametrize("B", [5, 6])
def test_tp16_speculative_split_halves(tp16, B):
    """5 or 6 draft tokens sharing 12 experts: the expert phase runs as a four-token launch
    and a one- or two-token launch (the union, 12 + 4 B experts, is under half the 16 B
    entries); every token is checked."""
    seed, st, ref = tp16
    attn0, resid0, _ = H.constructed_shared(seed, synth.TP16, B, core=12, ref=ref)
    case = build_case(seed, synth.TP16, B, attn0=attn0, resid0=resid0, refs=[ref])
    out, idx, gate, _ = check_case(st, case)
    assert len(set(idx[0].ravel().tolist())) == 12 + B * (synth.TP16.k - 12)


@pytest.mark.slow
def test_tp16_speculative_max_batch_4(tp16):
    """The speculative shape on a handle whose max_batch is the batch (4), as a verifier that
    sizes its handle exactly would create it."""
    seed, st0, ref = tp16
    st = H.GpuStack(seed, synth.TP16, max_batch=4, weights=st0.weights)
    try:
        attn0, resid0, _ = H.constructed_shared(seed, synth.TP16, 4, core=12, ref=ref)
        check_case(st, build_case(seed, synth.TP16, 4, attn0=attn0, resid0=resid0, refs=[ref]))
    finally:
        st.close()


# --- the small-batch kernels up to four tokens: they take a batch while its (token, expert)
#     entries fit the per-CTA routing's 64, else the large-batch kernels run ------------------
def kernels_run(st, B):
    """Names of the kernels one eager step of this batch launches."""
    import torch
    D = st.dims
    attn = torch.zeros((1, B, D.d_o), dtype=torch.bfloat16, device="cuda")
    resid = torch.zeros((B, D.d), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((B, D.d), dtype=torch.bfloat16, device="cuda")
    return [n for n, _ in st.md.moe_decode_profile_step(st.h, B, attn, resid, out)]


@pytest.mark.parametrize("B,k,small", [(3, 20, True), (4, 16, True), (4, 20, False)])
def test_small_path_entry_limit(B, k, small):
    dims = synth.Dims(256, 256, 64, k, 128)
    seed = synth.config_seed(12) + 10 * B + k
    st = H.GpuStack(seed, dims, max_batch=4)
    try:
        names = kernels_run(st, B)
        assert ("experts_small_m" in names) == small, names
        check_case(st, build_case(seed, dims, B))
    finally:
        st.close()


@pytest.mark.slow
def test_tp16_b4_independent(tp16):
    """Four independent tokens: the largest union (64 experts) the four-token kernels hold."""
    seed, st, ref = tp16
    case = build_case(seed + 4, synth.TP16, 4, refs=[ref])
    out, idx, gate, _ = check_case(st, case)  # every token
    assert "experts_small_m" in kernels_run(st, 4)


# --- full-size layer (1/8 shard, I=256), batch 16 and 64 -------------------------------------
@pytest.fixture(scope="module")
def tp8():
    seed = synth.config_seed(3)
    st = H.GpuStack(seed, synth.TP8, max_batch=64)
    ref = LayerRef(seed, synth.TP8, 0)
    yield seed, st, ref
    st.close()


@pytest.mark.slow
@pytest.mark.parametrize("B", [16, 64])
def test_tp8_batches(tp8, B):
    seed, st, ref = tp8
    check_case(st, build_case(seed, synth.TP8, B, refs=[ref]))  # every token


# --- stack of 8 full-size layers, batch 1 and 64, prefetch on and off -----------------------------
@pytest.fixture(scope="module")
def stack8():
    seed = synth.config_seed(4)
    w = H.device_weights(seed, synth.TP16, 8)
    refs = [LayerRef(seed, synth.TP16, l) for l in range(8)]
    yield seed, w, refs, {}
    del w


@pytest.mark.slow
@pytest.mark.parametrize("prefetch", [0, 1])
@pytest.mark.parametrize("B", [1, 64])
def test_stack8(stack8, B, prefetch):
    seed, w, refs, cases = stack8
    st = H.GpuStack(seed, synth.TP16, n_layers=8, max_batch=64, prefetch=prefetch, weights=w)
    try:
        if B not in cases:  # every token, every layer
            cases[B] = build_case(seed, synth.TP16, B, n_layers=8, refs=refs,
                                  min_boundary_gap=[2 * H.stack_tau(l) for l in range(8)])
        check_case(st, cases[B])
    finally:
        st.close()
