"""Shared helpers of the parity tests: seeded device weights, oracle cases, tolerances.

Tolerances (floating point), from the layer's stated acceptance bar:
  * selected expert indices and their order: exact;
  * bf16 output, per element: |gpu - ref| <= 2e-2 + ulp_bf16(ref) / 2, where ref is
    the oracle's fp64 value before rounding (a perfectly rounded bf16 output can be
    half an ulp away, and half an ulp exceeds 2e-2 once |ref| >= 8);
  * bf16 output, relative L2: ||gpu - ref|| / ||ref|| <= 5e-3;
  * in a stack, each earlier layer boundary adds one bf16 ulp of that layer's output
    per element (the two chains round independently; a different rounding is
    carried unchanged by the residual path), and layers after the first are checked
    with check_route_stacked (below).
Intermediates are checked more tightly than the output (fp32 vs fp64 arithmetic).
"""
from __future__ import annotations

import numpy as np

import synth
from oracle.layer import LayerRef, build_case, token_attn, top_gap  # noqa: F401

MAX_ABS = 2e-2
REL_L2 = 5e-3
# A gate moves by at most the largest logit error: the sum over j of |d gate_i / d logit_j|
# is 2 g_i (1 - g_i) <= 1/2, applied to logit differences of at most twice the logit error;
# fp32 rounding of the softmax itself adds ~1e-7.  The logits differ from the fp64 oracle's
# by the fp32 rounding of o_proj (d_o = 8192 products, on the tensor cores above batch 2),
# RMSNorm and the router (d = 7168 products): up to 6.6e-6 measured at full size, every token
# checked.  So gates are held to 1e-5.
GATE_ATOL = 1e-5

# Worst errors seen by the parity checks of this session (reported by conftest at the end).
WORST = {"gate_abs": 0.0, "logit_abs": 0.0, "out_excess": -1.0, "out_rel_l2": 0.0}


def note(key: str, value: float) -> None:
    WORST[key] = max(WORST[key], float(value))
# Later layers of a stack see inputs that differ between the two chains: each rounds its
# layer outputs to bf16 on its own, and elements whose fp32 and fp64 values straddle a
# rounding boundary come out one ulp apart.  Such a difference does not stay small: it
# moves the next layer's logits, hence its gates, hence every element of its output, and
# more elements round differently there.  Running the oracle twice, the second time with
# the roundings of elements within 2e-6 (relative) of a boundary flipped at random, moves
# layer l's logits by up to 1e-3 * l (20 chains of the 8-layer batch-64 stack, worst 6.8e-3
# at layer 7; tests/test_stack_divergence.py asserts half the bound below on a sample) as long as both chains select the same
# experts, and by ~2e-2 once a near tie at the k-th / (k+1)-th boundary selects a
# different one.  So for layer l > 0 the bound on |logit difference| is STACK_TAU * l
# (twice the worst seen), the stacked draws keep the selection boundary at least twice
# that apart (build_case's min_boundary_gap), and check_route_stacked accepts any order
# that the oracle's logits allow within the bound.
STACK_TAU = 2e-3


def stack_tau(layer: int) -> float:
    return STACK_TAU * layer


def check_route_stacked(idx: np.ndarray, gate: np.ndarray, ref_idx: np.ndarray, ref_gate: np.ndarray,
                        ref_logits: np.ndarray, tau: float, where=None) -> None:
    """One stacked layer's routing of one token against the oracle chain's.

    With logits within tau of the oracle's: the selected set is the oracle's (the draws
    keep the selection boundary 2 tau wide); any two experts whose oracle logits are more
    than 2 tau apart keep the oracle's order, closer ones may come in either order; each
    gate moves by at most tau / 2 (sum over j of |d gate_i / d logit_j| = 2 g_i (1 - g_i)).
    """
    idx = np.asarray(idx)
    assert set(idx.tolist()) == set(np.asarray(ref_idx).tolist()), (where, idx, ref_idx)
    z = np.asarray(ref_logits, np.float64)[idx]
    for j in range(len(idx)):
        assert np.all(z[j] >= z[j + 1:] - 2 * tau), (where, j, idx, ref_idx)
    pos = {int(e): j for j, e in enumerate(ref_idx)}
    g_ref = np.array([ref_gate[pos[int(e)]] for e in idx])
    assert np.allclose(gate, g_ref, atol=tau / 2, rtol=0), (where, np.abs(gate - g_ref).max())


def ulp_bf16(v: np.ndarray) -> np.ndarray:
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 7).astype(np.int64))


def check_out(gpu_bits: np.ndarray, ref: np.ndarray, extra_tol: np.ndarray | float = 0.0) -> dict:
    g = synth.bf16_bits_to_f32(gpu_bits).astype(np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(g - ref)
    tol = MAX_ABS + 0.5 * ulp_bf16(ref) + extra_tol
    rel = float(np.linalg.norm(g - ref) / np.linalg.norm(ref))
    res = {"max_abs": float(err.max()), "worst_excess": float((err - tol).max()), "rel_l2": rel,
           "n_bad": int((err > tol).sum())}
    note("out_excess", res["worst_excess"])
    note("out_rel_l2", rel)
    assert res["n_bad"] == 0, res
    assert rel <= REL_L2, res
    return res


# --- device side -------------------------------------------------------------------------
def device_weights(seed: int, dims: synth.Dims, n_layers: int, device="cuda"):
    import torch
    sz = dims.sizes()
    layers = []
    for l in range(n_layers):
        t = {}
        for kind in (synth.W_O, synth.GAMMA, synth.W_R, synth.W_GU, synth.W_DOWN):
            x = torch.empty(sz[kind], dtype=torch.bfloat16, device=device)
            synth.device_fill(x, seed, kind, layer=l)
            t[kind] = x
        layers.append((t[synth.W_O], t[synth.GAMMA], t[synth.W_R], t[synth.W_GU], t[synth.W_DOWN]))
    torch.cuda.synchronize()
    return layers


class GpuStack:
    """A handle over seeded device weights, plus a step with numpy in/out."""

    def __init__(self, seed, dims, n_layers=1, max_batch=1, prefetch=0, force_variant=0, weights=None):
        import torch
        import moe_decode_layer_02_b200 as md
        self.md, self.torch = md, torch
        self.dims, self.L, self.maxB = dims, n_layers, max_batch
        self.weights = weights or device_weights(seed, dims, n_layers)
        cfg = md.config(dims.d, dims.d_o, dims.E, dims.k, dims.I, max_batch, n_layers,
                        enable_prefetch=prefetch, force_variant=force_variant)
        self.h = md.moe_decode_create(cfg, self.weights, torch.cuda.current_stream())

    def step(self, attn_bits: np.ndarray, resid_bits: np.ndarray, reps: int = 1):
        torch, md, D = self.torch, self.md, self.dims
        L, B = attn_bits.shape[0], attn_bits.shape[1]
        dev = "cuda"
        attn = torch.from_numpy(attn_bits.view(np.int16).copy()).to(dev).view(torch.bfloat16)
        resid = torch.from_numpy(resid_bits.view(np.int16).copy()).to(dev).view(torch.bfloat16)
        out = torch.empty((B, D.d), dtype=torch.bfloat16, device=dev)
        idx = torch.full((L, B, D.k), -1, dtype=torch.int32, device=dev)
        gate = torch.full((L, B, D.k), -1.0, dtype=torch.float32, device=dev)
        s = torch.cuda.current_stream()
        for _ in range(reps):
            md.moe_decode_step(self.h, B, attn, resid, out, idx, gate, s)
        rc = md.moe_decode_sync_status(self.h, s)
        assert rc == 0, md.strerror(rc)
        return (out.view(torch.int16).cpu().numpy().view(np.uint16), idx.cpu().numpy(), gate.cpu().numpy())

    def intermediate(self, which: int, B: int):
        torch, D = self.torch, self.dims
        n = {0: B * D.d, 1: B, 2: B * D.d, 3: B * D.E}[which]
        buf = torch.empty(n, dtype=torch.float32, device="cuda")
        self.md.moe_decode_get_intermediate(self.h, which, buf, n * 4, torch.cuda.current_stream())
        torch.cuda.synchronize()
        return buf.cpu().numpy()

    def close(self):
        if self.h:
            self.md.moe_decode_destroy(self.h)
            self.h = 0


# --- constructed batch-2 overlaps ---------------------------------------------------------------
def constructed_b2(seed: int, dims: synth.Dims, overlap: int, lift: float = 15.0, ref: LayerRef | None = None):
    """Batch-2 inputs whose two top-k sets share exactly `overlap` experts.

    Token b's normalised activation is steered towards a chosen set S_b:
    x* = z + lift * sum_{e in S_b} W_r[e] / |W_r[e]|^2 with z ~ N(0, 1) from the seeded
    generator, h* = x* / gamma, and residual_in = bf16(h* - W_o . attn_out).  The oracle
    then confirms top-k(x) = S_b and the gap rule; otherwise z is redrawn.
    """
    from oracle import get as get_oracle
    o = get_oracle()
    ref = ref or LayerRef(seed, dims, 0)
    E, k, d = dims.E, dims.k, dims.d
    rng = np.random.default_rng(seed * 1000 + overlap)
    S0 = rng.choice(E, k, replace=False)
    rest = np.setdiff1d(np.arange(E), S0)
    S1 = np.concatenate([S0[:overlap], rng.choice(rest, k - overlap, replace=False)])
    Wr = synth.bf16_bits_to_f32(ref.W_r).astype(np.float64).reshape(E, d)
    gam = synth.bf16_bits_to_f32(ref.gamma).astype(np.float64)
    attn0, resid0 = [], []
    for b, S in enumerate((S0, S1)):
        for att in range(50):
            attn = token_attn(seed, dims, 0, b, att)
            z = synth.bf16_bits_to_f32(synth.host_token(seed, synth.LIFT_Z, d, token=b, attempt=att)).astype(np.float64)
            xs = z + lift * (Wr[S] / (Wr[S] ** 2).sum(1, keepdims=True)).sum(0)
            hs = xs / gam
            wo_attn = o.oproj_residual(ref.W_o, attn, np.zeros(d, np.uint16), 1, d, dims.d_o)[0]
            resid = synth.f64_to_bf16_bits(hs - wo_attn)
            f = ref.front(attn[None], resid[None])
            if set(f["idx"][0].tolist()) == set(S.tolist()) and top_gap(f["logits64"][0], k) >= 1e-3:
                break
        else:
            raise RuntimeError("construction failed")
        attn0.append(attn)
        resid0.append(resid)
    return np.stack(attn0), np.stack(resid0), (S0, S1)


# --- speculative-verification batches: B tokens sharing a core of experts -------------------------
def constructed_shared(seed: int, dims: synth.Dims, B: int, core: int, lift: float = 15.0,
                       ref: LayerRef | None = None):
    """B tokens whose top-k sets share `core` experts (a draft-verification step: one sequence's
    next tokens mostly route alike); each token adds k - core experts of its own.

    Same construction as constructed_b2: x* = z + lift * sum_{e in S_b} W_r[e] / |W_r[e]|^2,
    h* = x* / gamma, residual_in = bf16(h* - W_o . attn_out); the oracle confirms each token's
    set and the gap rule, else z is redrawn."""
    from oracle import get as get_oracle
    o = get_oracle()
    ref = ref or LayerRef(seed, dims, 0)
    E, k, d = dims.E, dims.k, dims.d
    rng = np.random.default_rng(seed * 7919 + 131 * B + core)
    C = rng.choice(E, core, replace=False)
    rest = rng.permutation(np.setdiff1d(np.arange(E), C))
    priv = rest[:B * (k - core)].reshape(B, k - core)
    Wr = synth.bf16_bits_to_f32(ref.W_r).astype(np.float64).reshape(E, d)
    gam = synth.bf16_bits_to_f32(ref.gamma).astype(np.float64)
    attn0, resid0, sets = [], [], []
    for b in range(B):
        S = np.concatenate([C, priv[b]])
        for att in range(50):
            attn = token_attn(seed, dims, 0, b, att)
            z = synth.bf16_bits_to_f32(synth.host_token(seed, synth.LIFT_Z, d, token=b, attempt=att)).astype(np.float64)
            xs = z + lift * (Wr[S] / (Wr[S] ** 2).sum(1, keepdims=True)).sum(0)
            wo_attn = o.oproj_residual(ref.W_o, attn, np.zeros(d, np.uint16), 1, d, dims.d_o)[0]
            resid = synth.f64_to_bf16_bits(xs / gam - wo_attn)
            f = ref.front(attn[None], resid[None])
            if set(f["idx"][0].tolist()) == set(S.tolist()) and top_gap(f["logits64"][0], k) >= 1e-3:
                break
        else:
            raise RuntimeError("construction failed")
        attn0.append(attn)
        resid0.append(resid)
        sets.append(S)
    return np.stack(attn0), np.stack(resid0), sets
