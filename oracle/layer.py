"""Oracle runs of whole layers and layer stacks on seeded inputs.

TEST INFRASTRUCTURE ONLY (tests, smoke check, the benchmark's CPU-baseline
leg).  Weights are regenerated on the host from the seeded generator; an
expert's weights are materialised only when a checked token selects it, and for a
whole batch they are taken one expert at a time (``LayerRef.moe_many``).

Gap rule.  The selected expert indices must match the CUDA path exactly, so
inputs are drawn such that, for every checked token and layer, every adjacent
gap among the k+1 largest oracle logits is at least ``min_gap`` (1e-3); this
covers the k-th/(k+1)-th gap that decides the set and the gaps that decide
the order.  A token whose draw fails is redrawn with the next attempt number
of its own counter stream (layer 0: its attn_out and residual_in; later
layers of a stack: its attn_out), so other tokens are unaffected.
"""
from __future__ import annotations

import numpy as np

import synth

from . import get as _get_oracle


def top_gap(logits_row: np.ndarray, k: int) -> float:
    """Smallest adjacent gap among the k+1 largest values of one row."""
    s = np.sort(np.asarray(logits_row, np.float64))[::-1][: k + 1]
    return float(np.min(s[:-1] - s[1:])) if s.size > 1 else np.inf


def top_gap_distinct(logits_row: np.ndarray, k: int) -> float:
    """Smallest gap between adjacent DISTINCT values among the k+1 largest of one row, and
    0 when the k-th and (k+1)-th largest are equal (the selected set is then not unique)."""
    s = np.sort(np.asarray(logits_row, np.float64))[::-1][: k + 1]
    if s.size > k and s[k - 1] == s[k]:
        return 0.0
    u = np.unique(s)
    return float(np.min(np.diff(u))) if u.size > 1 else np.inf


def boundary_gap(logits_row: np.ndarray, k: int) -> float:
    """Gap between the k-th and (k+1)-th largest values of one row (inf when k = E)."""
    s = np.sort(np.asarray(logits_row, np.float64))[::-1][: k + 1]
    return float(s[k - 1] - s[k]) if s.size > k else np.inf


class LayerRef:
    """One layer's seeded weights on the host plus oracle calls over them."""

    def __init__(self, seed: int, dims: synth.Dims, layer: int = 0, eps: float = 1e-6, oracle=None):
        self.seed, self.dims, self.layer, self.eps = seed, dims, layer, eps
        self.o = oracle or _get_oracle()
        w = synth.host_weights(seed, dims, layer)
        self.W_o, self.gamma, self.W_r = w[synth.W_O], w[synth.GAMMA], w[synth.W_R]
        self._experts: dict[int, tuple[np.ndarray, np.ndarray]] = {}

    def expert(self, e: int):
        if e not in self._experts:
            self._experts[e] = synth.host_expert(self.seed, self.dims, int(e), self.layer)
        return self._experts[e]

    def front(self, attn: np.ndarray, resid: np.ndarray) -> dict:
        D = self.dims
        B = attn.shape[0]
        return self.o.front(self.W_o, self.gamma, self.W_r, attn, resid, B=B, d=D.d, d_o=D.d_o,
                            E=D.E, k=D.k, eps=self.eps)

    def moe(self, f: dict, b: int):
        sel = f["idx"][b]
        gus, dns = zip(*[self.expert(e) for e in sel])
        return self.o.moe_token(list(gus), list(dns), f["x"][b], f["h"][b], f["gate"][b], self.dims.I)

    def moe_many(self, fronts: dict) -> dict:
        """Steps 5-6 for many tokens, expert by expert.

        ``fronts`` maps a token to its one-token front result.  Each selected expert's
        weights are generated once, applied to every token that selected it and dropped,
        so host memory stays bounded at any batch.  The arithmetic is the oracle's own
        per-token path (oracle_expert for each selected slot, then oracle_combine over the
        slots in ascending order), only the loop that materialises the weights differs.
        Returns token -> (out_ref, out_bf16, a [k][I])."""
        D = self.dims
        users: dict[int, list] = {}
        for b, f in fronts.items():
            for j, e in enumerate(f["idx"][0]):
                users.setdefault(int(e), []).append((b, j))
        ys = {b: [None] * D.k for b in fronts}
        acts = {b: np.empty((D.k, D.I)) for b in fronts}
        for e in sorted(users):
            gu, dn = self._experts.get(e) or synth.host_expert(self.seed, D, e, self.layer)
            for b, j in users[e]:
                a, y = self.o.expert(gu, dn, fronts[b]["x"][0], D.I)
                ys[b][j] = y
                acts[b][j] = a
        out = {}
        for b, f in fronts.items():
            ref, ob = self.o.combine(f["h"][0], f["gate"][0], ys[b])
            out[b] = (ref, ob, acts[b])
        return out


def token_attn(seed, dims, layer, b, attempt):
    return synth.host_token(seed, synth.ATTN, dims.d_o, layer=layer, token=b, attempt=attempt)


def token_resid(seed, dims, b, attempt):
    return synth.host_token(seed, synth.RESID, dims.d, layer=0, token=b, attempt=attempt)


def build_case(seed: int, dims: synth.Dims, B: int, n_layers: int = 1, checked=None,
               min_gap: float = 1e-3, max_attempts: int = 200, resid0=None, attn0=None,
               refs=None, moe_tokens=None, min_boundary_gap=None, gap_fn=None) -> dict:
    """Seeded inputs for a B-token, n_layers-deep step and the oracle's answers.

    ``checked`` lists the tokens the oracle follows through every layer (all
    of them by default); those tokens satisfy the gap rule at every layer.
    Unchecked tokens keep attempt 0.  ``resid0`` ([B][d] bf16 bits) replaces
    the drawn layer-0 residual and ``attn0`` ([B][d_o]) the drawn layer-0 attention
    output (used by constructed batch-2 cases); fixed inputs are never redrawn.
    ``moe_tokens`` (one-layer cases only) limits the expert half of the oracle to a
    subset of the checked tokens; the others get indices and gates only.
    ``min_boundary_gap`` (one value per layer) also asks of each checked token's draw
    that the k-th and (k+1)-th largest logits lie that far apart, so that an input
    perturbed within half of it still selects the same experts.  ``gap_fn`` replaces
    ``top_gap`` as the gap rule (e.g. ``top_gap_distinct`` for routers with tied rows).

    Returns attn [L][B][d_o] and resid [B][d] (bf16 bits), the attempts used,
    and per layer the oracle's front results and outputs for checked tokens.
    """
    checked = list(range(B)) if checked is None else list(checked)
    if moe_tokens is not None and n_layers != 1:
        raise ValueError("moe_tokens needs a one-layer case")
    moe_set = set(checked if moe_tokens is None else moe_tokens)
    refs = refs or [LayerRef(seed, dims, l) for l in range(n_layers)]
    attn = np.stack([np.stack([token_attn(seed, dims, l, b, 0) for b in range(B)])
                     for l in range(n_layers)])
    fixed0 = resid0 is not None or attn0 is not None
    if attn0 is not None:
        attn[0] = np.array(attn0, np.uint16).reshape(B, dims.d_o)
    if resid0 is None:
        resid = np.stack([token_resid(seed, dims, b, 0) for b in range(B)])
    else:
        resid = np.array(resid0, np.uint16).reshape(B, dims.d)
    attempts = np.zeros((n_layers, B), np.int32)
    layers = []
    cur = {b: resid[b] for b in checked}
    for l in range(n_layers):
        ref = refs[l]
        per = {"idx": {}, "gate": {}, "out_ref": {}, "out_bf16": {}, "h": {}, "x": {},
               "logits32": {}, "logits64": {}, "rstd": {}, "a": {}}
        fronts = {}
        for b in checked:
            for att in range(max_attempts):
                if att:
                    attn[l, b] = token_attn(seed, dims, l, b, att)
                    if l == 0:
                        cur[b] = token_resid(seed, dims, b, att)
                        resid[b] = cur[b]
                f = ref.front(attn[l, b][None], cur[b][None])
                ok = (gap_fn or top_gap)(f["logits64"][0], dims.k) >= min_gap
                if ok and min_boundary_gap is not None:
                    ok = boundary_gap(f["logits64"][0], dims.k) >= min_boundary_gap[l]
                if ok:
                    break
                if fixed0 and l == 0:
                    raise RuntimeError("fixed layer-0 inputs violate the gap rule")
            else:
                raise RuntimeError(f"no gapped draw for token {b} layer {l}")
            attempts[l, b] = att
            for key in ("idx", "gate", "h", "x", "logits32", "logits64", "rstd"):
                per[key][b] = f[key][0]
            if b in moe_set:
                fronts[b] = f
        for b, (out_ref, out_bf16, a) in ref.moe_many(fronts).items():
            per["out_ref"][b], per["out_bf16"][b], per["a"][b] = out_ref, out_bf16, a
            cur[b] = out_bf16
        layers.append(per)
    return {"attn": attn, "resid": resid, "attempts": attempts, "layers": layers,
            "checked": checked, "refs": refs}
