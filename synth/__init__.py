"""Seeded synthetic inputs for the MoE decode-layer step.

This module is shared by the tests, the benchmark and the smoke check. It
holds random-number generation and bf16 format handling only: none of the
layer's arithmetic lives here, and it imports neither the oracle nor the
CUDA library.

Generator
---------
Every value is addressed by a counter, so any slice of any tensor can be
regenerated on its own (the oracle side regenerates only the experts a token
selected) and the host and device produce identical bits:

* Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as
  easy as 1, 2, 3", SC'11) maps a 128-bit counter and a 64-bit key to four
  32-bit words; each word gives two 16-bit draws (low half first).
* A 16-bit draw ``u`` picks entry ``u`` of a 65536-entry bf16 table holding
  the quantiles ``q(k) = F^-1((k + 0.5) / 65536)`` of the target
  distribution, rounded to bf16.  The table is built once here in float64
  and uploaded unchanged to the device fill kernel, so the only arithmetic
  on either side is integer.

Distributions (the workload statement of the decode layer):
  weights ``N(0, 0.02)``; RMSNorm scale ``1 + N(0, 0.02)``; activations
  ``N(0, 1)``.  The quantile table truncates the normal at about 4.3 sigma
  and resolves it far below bf16 precision in the body.

Counter layout for element ``n`` of a stream:
  ``c0, c1`` = low / high 32 bits of ``n // 8``; ``c2`` = stream id
  ``(kind << 24) | (layer << 16) | token``; ``c3`` = attempt;
  key = (seed low 32 bits, seed high 32 bits).  Element ``n`` takes 16-bit
  half ``n % 8`` of the block (word ``(n % 8) // 2``, low half when even).
"""
from __future__ import annotations

import functools
import os

import numpy as np

# --- stream kinds --------------------------------------------------------------
W_O, GAMMA, W_R, W_GU, W_DOWN, ATTN, RESID, LIFT_Z = 1, 2, 3, 4, 5, 6, 7, 8

SEED_BASE = 0x5EED

PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85

_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr: np.ndarray, key: tuple[int, int]) -> np.ndarray:
    """Philox4x32 with 10 rounds on an ``[N, 4]`` uint32 counter array."""
    c = [ctr[:, i].astype(np.uint64) for i in range(4)]
    k0, k1 = int(key[0]) & 0xFFFFFFFF, int(key[1]) & 0xFFFFFFFF
    m0, m1 = np.uint64(PHILOX_M0), np.uint64(PHILOX_M1)
    for r in range(10):
        if r:
            k0 = (k0 + PHILOX_W0) & 0xFFFFFFFF
            k1 = (k1 + PHILOX_W1) & 0xFFFFFFFF
        p0 = m0 * c[0]
        p1 = m1 * c[2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c = [hi1 ^ c[1] ^ np.uint64(k0), lo1, hi0 ^ c[3] ^ np.uint64(k1), lo0]
    return np.stack([x.astype(np.uint32) for x in c], axis=1)


def stream_id(kind: int, layer: int = 0, token: int = 0) -> int:
    if not (0 <= kind < 256 and 0 <= layer < 256 and 0 <= token < 65536):
        raise ValueError("stream id field out of range")
    return (kind << 24) | (layer << 16) | token


def draws_u16(seed: int, sid: int, attempt: int, start: int, count: int) -> np.ndarray:
    """16-bit draws ``start .. start+count-1`` of stream ``sid``."""
    if count <= 0:
        return np.zeros(0, np.uint16)
    b0 = start // 8
    b1 = (start + count + 7) // 8
    blk = np.arange(b0, b1, dtype=np.uint64)
    ctr = np.empty((blk.size, 4), np.uint32)
    ctr[:, 0] = (blk & _MASK32).astype(np.uint32)
    ctr[:, 1] = (blk >> np.uint64(32)).astype(np.uint32)
    ctr[:, 2] = sid & 0xFFFFFFFF
    ctr[:, 3] = attempt & 0xFFFFFFFF
    out = philox4x32_10(ctr, (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF))
    halves = np.empty((blk.size, 8), np.uint16)
    halves[:, 0::2] = (out & 0xFFFF).astype(np.uint16)
    halves[:, 1::2] = (out >> 16).astype(np.uint16)
    flat = halves.reshape(-1)
    off = start - b0 * 8
    return flat[off:off + count].copy()


# --- bf16 format handling -------------------------------------------------------
def bf16_bits_to_f32(u16: np.ndarray) -> np.ndarray:
    return (np.asarray(u16, np.uint16).astype(np.uint32) << 16).view(np.float32)


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even), finite inputs."""
    v = np.asarray(v, np.float64)
    out = np.zeros(v.shape, np.uint16)
    nz = v != 0
    a = np.abs(v[nz])
    _, ex = np.frexp(a)                     # a = f * 2**ex, f in [0.5, 1)
    ulp = np.ldexp(1.0, np.maximum(ex - 8, -133))
    r = np.rint(a / ulp) * ulp              # rint: ties to even
    f32 = (np.sign(v[nz]) * r).astype(np.float32)  # exact: r has <= 8 significant bits
    out[nz] = (f32.view(np.uint32) >> 16).astype(np.uint16)
    neg0 = (~nz) & np.signbit(v)
    out[neg0] = 0x8000
    return out


# --- quantile tables ------------------------------------------------------------
@functools.lru_cache(maxsize=None)
def table(dist: str) -> np.ndarray:
    """65536-entry bf16 quantile table for ``dist`` in {'w', 'gamma', 'act'}."""
    from scipy.special import ndtri
    p = (np.arange(65536, dtype=np.float64) + 0.5) / 65536.0
    z = ndtri(p)
    if dist == "w":
        v = 0.02 * z
    elif dist == "gamma":
        v = 1.0 + 0.02 * z
    elif dist == "act":
        v = z
    else:
        raise ValueError(dist)
    t = f64_to_bf16_bits(v)
    t.setflags(write=False)
    return t


KIND_DIST = {W_O: "w", GAMMA: "gamma", W_R: "w", W_GU: "w", W_DOWN: "w",
             ATTN: "act", RESID: "act", LIFT_Z: "act"}


def gen_bf16_numpy(seed: int, kind: int, count: int, *, layer: int = 0, token: int = 0,
                   attempt: int = 0, start: int = 0) -> np.ndarray:
    """bf16 bits of elements ``start .. start+count-1`` of one seeded stream (numpy)."""
    u = draws_u16(seed, stream_id(kind, layer, token), attempt, start, count)
    return table(KIND_DIST[kind])[u]


def gen_bf16(seed: int, kind: int, count: int, *, layer: int = 0, token: int = 0,
             attempt: int = 0, start: int = 0) -> np.ndarray:
    """bf16 bits of elements ``start .. start+count-1`` of one seeded stream.

    Uses the C fill (synth_host.c, same bits) once it is built, else numpy."""
    lib = _host_lib()
    if lib is None or count <= 0:
        return gen_bf16_numpy(seed, kind, count, layer=layer, token=token, attempt=attempt, start=start)
    tab = table(KIND_DIST[kind])
    out = np.empty(count, np.uint16)
    rc = lib.synth_host_fill_bf16(out.ctypes.data, count, start, seed & 0xFFFFFFFFFFFFFFFF,
                                  stream_id(kind, layer, token), attempt & 0xFFFFFFFF, tab.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"synth_host_fill_bf16 failed ({rc})")
    return out


def config_seed(config_id: int) -> int:
    return SEED_BASE + int(config_id)


# --- layer inputs ---------------------------------------------------------------
class Dims:
    """Shapes of one decode layer (weights row-major ``[out][in]``)."""

    def __init__(self, d, d_o, n_experts, top_k, inter):
        self.d, self.d_o, self.E, self.k, self.I = int(d), int(d_o), int(n_experts), int(top_k), int(inter)

    def sizes(self):
        d, d_o, E, I = self.d, self.d_o, self.E, self.I
        return {W_O: d * d_o, GAMMA: d, W_R: E * d, W_GU: E * 2 * I * d, W_DOWN: E * d * I}

    def __repr__(self):
        return f"Dims(d={self.d}, d_o={self.d_o}, E={self.E}, k={self.k}, I={self.I})"


TINY = Dims(256, 256, 16, 2, 128)
TP16 = Dims(7168, 8192, 896, 16, 128)
TP8 = Dims(7168, 8192, 896, 16, 256)


def host_weights(seed: int, dims: Dims, layer: int = 0, kinds=(W_O, GAMMA, W_R)) -> dict:
    """Whole weight tensors on the host (for the dense ones, or tiny shapes)."""
    sz = dims.sizes()
    return {k: gen_bf16(seed, k, sz[k], layer=layer) for k in kinds}


def host_expert(seed: int, dims: Dims, e: int, layer: int = 0):
    """``(W_gu[e] [2I][d], W_down[e] [d][I])`` bf16 bits of one expert."""
    d, I = dims.d, dims.I
    ngu, ndn = 2 * I * d, d * I
    gu = gen_bf16(seed, W_GU, ngu, layer=layer, start=e * ngu).reshape(2 * I, d)
    dn = gen_bf16(seed, W_DOWN, ndn, layer=layer, start=e * ndn).reshape(d, I)
    return gu, dn


def host_token(seed: int, kind: int, n: int, *, layer: int = 0, token: int = 0, attempt: int = 0):
    return gen_bf16(seed, kind, n, layer=layer, token=token, attempt=attempt)


# --- host fill (C, OpenMP) ------------------------------------------------------------
_HERE = os.path.dirname(os.path.abspath(__file__))
SYNTH_HOST_SO = os.path.join(_HERE, "libsynth_host.so")
_host = None


def build_host_fill(force: bool = False) -> str:
    """Compile the host fill (plain C, gcc, OpenMP) next to this file."""
    import subprocess
    src = os.path.join(_HERE, "synth_host.c")
    if force or not os.path.exists(SYNTH_HOST_SO) or os.path.getmtime(SYNTH_HOST_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o",
                               SYNTH_HOST_SO, src])
    return SYNTH_HOST_SO


def _host_lib():
    global _host
    if _host is None and os.path.exists(SYNTH_HOST_SO):
        import ctypes
        lib = ctypes.CDLL(SYNTH_HOST_SO)
        lib.synth_host_fill_bf16.restype = ctypes.c_int
        lib.synth_host_fill_bf16.argtypes = [ctypes.c_void_p, ctypes.c_ulonglong, ctypes.c_ulonglong,
                                             ctypes.c_ulonglong, ctypes.c_uint, ctypes.c_uint,
                                             ctypes.c_void_p]
        _host = lib
    return _host


# --- device fill (optional CUDA helper) -------------------------------------------
SYNTH_SO = os.path.join(_HERE, "libsynth.so")


def build_device_fill(force: bool = False) -> str:
    """Compile the device fill kernel (sm_100a) next to this file."""
    import subprocess
    src = os.path.join(_HERE, "synth_fill.cu")
    if force or not os.path.exists(SYNTH_SO) or os.path.getmtime(SYNTH_SO) < os.path.getmtime(src):
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                               "-lineinfo", "-shared", "-Xcompiler", "-fPIC", "-o", SYNTH_SO, src])
    return SYNTH_SO


_lib = None
_dev_tables: dict = {}


def _synth_lib():
    global _lib
    if _lib is None:
        import ctypes
        if not os.path.exists(SYNTH_SO):
            raise RuntimeError(f"{SYNTH_SO} is not built; run build_device_fill()")
        lib = ctypes.CDLL(SYNTH_SO)
        lib.synth_fill_bf16.restype = ctypes.c_int
        lib.synth_fill_bf16.argtypes = [ctypes.c_void_p, ctypes.c_ulonglong, ctypes.c_ulonglong,
                                        ctypes.c_ulonglong, ctypes.c_uint, ctypes.c_uint,
                                        ctypes.c_void_p, ctypes.c_void_p]
        _lib = lib
    return _lib


def device_fill(t, seed: int, kind: int, *, layer: int = 0, token: int = 0, attempt: int = 0,
                start: int = 0, stream=None):
    """Fill the contiguous bf16 CUDA tensor ``t`` with elements ``start..`` of a stream."""
    import torch
    assert t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
    dev = t.device.index
    key = (dev, KIND_DIST[kind])
    if key not in _dev_tables:
        tab = torch.from_numpy(table(KIND_DIST[kind]).view(np.int16).copy()).to(t.device)
        _dev_tables[key] = tab
    tab = _dev_tables[key]
    s = stream if stream is not None else torch.cuda.current_stream(t.device).cuda_stream
    rc = _synth_lib().synth_fill_bf16(t.data_ptr(), t.numel(), start, seed,
                                      stream_id(kind, layer, token), attempt, tab.data_ptr(), s)
    if rc != 0:
        raise RuntimeError(f"synth_fill_bf16 failed ({rc})")
    return t
