"""ctypes wrapper of the CPU oracle (oracle/oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may use this package; the CUDA library never does.  It is
built from plain C with gcc (no fast-math, no FP contraction) and computes in
double precision; see the header of oracle.c for the definition it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "oracle.c")
LIB = os.path.join(_HERE, "liboracle.so")

_P = ctypes.c_void_p
_I = ctypes.c_int


def build(out: str = LIB, mutant: int = 0, force: bool = False) -> str:
    """Compile the oracle with gcc; ``mutant`` selects a deliberately wrong variant."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-o", out, SRC, "-lm"]
        if mutant:
            cmd.insert(1, f"-DORACLE_MUTANT={int(mutant)}")
        subprocess.check_call(cmd)
    return out


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_P)


def _u16(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.uint16)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


class Oracle:
    """One loaded build of the oracle (the reference build, or a test mutant)."""

    def __init__(self, path: str | None = None):
        path = path or build()
        self.path = path
        lib = ctypes.CDLL(path)
        for name, argt in {
            "oracle_oproj_residual": [_I, _I, _I, _P, _P, _P, _P],
            "oracle_rmsnorm": [_I, _I, _P, _P, ctypes.c_double, _P, _P],
            "oracle_router": [_I, _I, _I, _P, _P, _P],
            "oracle_topk_gates": [_I, _I, _I, _P, _P, _P],
            "oracle_expert": [_I, _I, _P, _P, _P, _P, _P],
            "oracle_combine": [_I, _I, _P, _P, _P, _P, _P],
            "oracle_front": [_I, _I, _I, _I, _I, ctypes.c_double] + [_P] * 12,
            "oracle_moe_token": [_I, _I, _I] + [_P] * 8,
            "oracle_set_threads": [_I],
        }.items():
            f = getattr(lib, name)
            f.argtypes = argt
            f.restype = _I if name != "oracle_set_threads" else None
        lib.oracle_bf16_rne.argtypes = [ctypes.c_double]
        lib.oracle_bf16_rne.restype = ctypes.c_uint16
        lib.oracle_mutant.restype = _I
        lib.oracle_threads.restype = _I
        self.lib = lib

    # -- plumbing ---------------------------------------------------------------
    @property
    def mutant(self) -> int:
        return self.lib.oracle_mutant()

    def threads(self) -> int:
        return self.lib.oracle_threads()

    def set_threads(self, n: int) -> None:
        self.lib.oracle_set_threads(int(n))

    @staticmethod
    def _check(rc: int, name: str):
        if rc != 0:
            raise ValueError(f"{name} rejected its arguments ({rc})")

    # -- steps ------------------------------------------------------------------
    def bf16_rne(self, v: float) -> int:
        return int(self.lib.oracle_bf16_rne(float(v)))

    def oproj_residual(self, W_o, attn, resid, B: int, d: int, d_o: int) -> np.ndarray:
        W_o, attn, resid = _u16(W_o), _u16(attn), _u16(resid)
        assert W_o.size == d * d_o and attn.size == B * d_o and resid.size == B * d
        h = np.empty((B, d), np.float64)
        self._check(self.lib.oracle_oproj_residual(B, d, d_o, _ptr(W_o), _ptr(attn), _ptr(resid),
                                                   _ptr(h)), "oproj_residual")
        return h

    def rmsnorm(self, h, gamma, eps: float = 1e-6):
        h, gamma = _f64(h), _u16(gamma)
        B, d = h.shape
        rstd = np.empty(B, np.float64)
        x = np.empty((B, d), np.float64)
        self._check(self.lib.oracle_rmsnorm(B, d, _ptr(h), _ptr(gamma), eps, _ptr(rstd), _ptr(x)),
                    "rmsnorm")
        return rstd, x

    def router(self, W_r, x, E: int) -> np.ndarray:
        W_r, x = _u16(W_r), _f64(x)
        B, d = x.shape
        assert W_r.size == E * d
        lg = np.empty((B, E), np.float64)
        self._check(self.lib.oracle_router(B, d, E, _ptr(W_r), _ptr(x), _ptr(lg)), "router")
        return lg

    def topk_gates(self, logits32, k: int):
        lg = np.ascontiguousarray(logits32, dtype=np.float32)
        B, E = lg.shape
        idx = np.empty((B, k), np.int32)
        gate = np.empty((B, k), np.float64)
        self._check(self.lib.oracle_topk_gates(B, E, k, _ptr(lg), _ptr(idx), _ptr(gate)), "topk")
        return idx, gate

    def expert(self, W_gu, W_down, x, I: int):
        W_gu, W_down, x = _u16(W_gu), _u16(W_down), _f64(x)
        d = x.size
        assert W_gu.size == 2 * I * d and W_down.size == d * I
        a = np.empty(I, np.float64)
        y = np.empty(d, np.float64)
        self._check(self.lib.oracle_expert(d, I, _ptr(W_gu), _ptr(W_down), _ptr(x), _ptr(a),
                                           _ptr(y)), "expert")
        return a, y

    def combine(self, h, gate, ys):
        h, gate = _f64(h), _f64(gate)
        ys = [_f64(y) for y in ys]
        d, k = h.size, gate.size
        arr = (_P * k)(*[y.ctypes.data for y in ys])
        out = np.empty(d, np.float64)
        ob = np.empty(d, np.uint16)
        self._check(self.lib.oracle_combine(d, k, _ptr(h), _ptr(gate), arr, _ptr(out), _ptr(ob)),
                    "combine")
        return out, ob

    def front(self, W_o, gamma, W_r, attn, resid, *, B, d, d_o, E, k, eps=1e-6):
        """Steps 1-4 for B tokens: dict of h, rstd, x, logits64, logits32, idx, gate."""
        W_o, gamma, W_r, attn, resid = map(_u16, (W_o, gamma, W_r, attn, resid))
        assert W_o.size == d * d_o and gamma.size == d and W_r.size == E * d
        assert attn.size == B * d_o and resid.size == B * d
        r = {"h": np.empty((B, d)), "rstd": np.empty(B), "x": np.empty((B, d)),
             "logits64": np.empty((B, E)), "logits32": np.empty((B, E), np.float32),
             "idx": np.empty((B, k), np.int32), "gate": np.empty((B, k))}
        self._check(self.lib.oracle_front(
            B, d, d_o, E, k, eps, _ptr(W_o), _ptr(gamma), _ptr(W_r), _ptr(attn), _ptr(resid),
            _ptr(r["h"]), _ptr(r["rstd"]), _ptr(r["x"]), _ptr(r["logits64"]),
            _ptr(r["logits32"]), _ptr(r["idx"]), _ptr(r["gate"])), "front")
        return r

    def moe_token(self, W_gu_sel, W_down_sel, x, h, gate, I: int):
        """Steps 5-6 for one token: (out_ref fp64, out bf16 bits, a [k][I])."""
        x, h, gate = _f64(x), _f64(h), _f64(gate)
        k, d = gate.size, x.size
        gus = [_u16(w) for w in W_gu_sel]
        dns = [_u16(w) for w in W_down_sel]
        assert len(gus) == k and len(dns) == k
        agu = (_P * k)(*[w.ctypes.data for w in gus])
        adn = (_P * k)(*[w.ctypes.data for w in dns])
        a = np.empty((k, I))
        out = np.empty(d)
        ob = np.empty(d, np.uint16)
        self._check(self.lib.oracle_moe_token(d, I, k, agu, adn, _ptr(x), _ptr(h), _ptr(gate),
                                              _ptr(a), _ptr(out), _ptr(ob)), "moe_token")
        return out, ob, a


_default: Oracle | None = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
