"""The C ABI: the library loads and exports every declared entry point (CPU), and
create/step reject what the header says they reject (GPU)."""
import ctypes
import glob
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for hdr in sorted(glob.glob(os.path.join(ROOT, "include", "*.h"))):
        text = open(hdr).read()
        names += re.findall(r"MOE_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return names


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("moe_decode_create", "moe_decode_step", "moe_decode_destroy", "moe_decode_strerror"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from moe_decode_layer_02_b200 import build as b
    lib_path = b.build()
    lib = ctypes.CDLL(lib_path)  # loads without a GPU: no device call at load time
    for n in declared_functions():
        assert hasattr(lib, n), n
    import moe_decode_layer_02_b200 as md
    assert set(md.EXPORTED) <= set(declared_functions())
    assert md.strerror(md.MOE_ERR_ALIGNMENT) == "pointer not 16-byte aligned"


def test_binding_has_no_cpu_fallback(tmp_path):
    import moe_decode_layer_02_b200 as md
    saved = md._lib
    md._lib = None
    try:
        with pytest.raises(RuntimeError):
            md.load(str(tmp_path / "missing.so"))
    finally:
        md._lib = saved


def test_create_rejects_bad_config_without_touching_the_gpu():
    import moe_decode_layer_02_b200 as md
    md.load()
    bad = [md.config(100, 256, 16, 2, 128, 1),     # d not a multiple of 64
           md.config(256, 256, 16, 40, 128, 1),    # top_k > 32
           md.config(256, 256, 2048, 2, 128, 1),   # too many experts
           md.config(256, 256, 16, 2, 100, 1),     # inter not a multiple of 32
           md.config(256, 256, 16, 2, 128, 65),    # batch above 64
           md.config(256, 256, 16, 2, 128, 1, rms_eps=0.0)]
    w = [(16, 16, 16, 16, 16)]
    for cfg in bad:
        with pytest.raises(md.MoeError) as ei:
            md.moe_decode_create(cfg, w)
        assert ei.value.code == md.MOE_ERR_UNSUPPORTED_CONFIG
    with pytest.raises(md.MoeError) as ei:
        md.moe_decode_create(md.config(256, 256, 16, 2, 128, 1), [(0, 16, 16, 16, 16)])
    assert ei.value.code == md.MOE_ERR_INVALID_ARG
    with pytest.raises(md.MoeError) as ei:
        md.moe_decode_create(md.config(256, 256, 16, 2, 128, 1), [(16, 18, 16, 16, 16)])
    assert ei.value.code == md.MOE_ERR_ALIGNMENT
    assert md.moe_decode_destroy(0) == 0
    assert md.moe_decode_destroy(0xDEAD0) == md.MOE_ERR_INVALID_ARG


@pytest.mark.gpu
def test_step_argument_checks():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_decode_layer_02_b200 as md
    import synth
    from tests.harness import device_weights
    synth.build_device_fill()
    dims = synth.TINY
    w = device_weights(1, dims, 1)
    h = md.moe_decode_create(md.config(dims.d, dims.d_o, dims.E, dims.k, dims.I, 4), w)
    try:
        attn = torch.zeros((4, dims.d_o), dtype=torch.bfloat16, device="cuda")
        res = torch.zeros((4, dims.d), dtype=torch.bfloat16, device="cuda")
        out = torch.zeros((4, dims.d), dtype=torch.bfloat16, device="cuda")
        for B in (0, 5, -1):
            with pytest.raises(md.MoeError) as ei:
                md.moe_decode_step(h, B, attn, res, out)
            assert ei.value.code == md.MOE_ERR_INVALID_ARG
        with pytest.raises(md.MoeError) as ei:
            md.moe_decode_step(h, 1, attn.data_ptr() + 2, res, out)
        assert ei.value.code == md.MOE_ERR_ALIGNMENT
        with pytest.raises(md.MoeError):
            md.moe_decode_get_intermediate(h, 9, out, 16)
        md.moe_decode_step(h, 2, attn, res, out)
        assert md.moe_decode_sync_status(h) == 0
        assert md.moe_decode_kernels_per_step(h, 1) == 1  # batch 1: one layer kernel
        assert md.moe_decode_kernels_per_step(h, 2) == 3  # batch 2: o_proj, router, small-M experts
        assert md.moe_decode_kernels_per_step(h, 4) == 3  # up to batch 4 the same three kernels
    finally:
        assert md.moe_decode_destroy(h) == 0
    assert md.moe_decode_destroy(h) == md.MOE_ERR_INVALID_ARG  # destroyed twice: rejected
    for variant, per_b in ((1, 3), (2, 4), (3, 1)):  # unfused small-batch; large-batch; counter-ordered
        h = md.moe_decode_create(md.config(dims.d, dims.d_o, dims.E, dims.k, dims.I, 4,
                                           force_variant=variant), w)
        try:
            assert md.moe_decode_kernels_per_step(h, 1) == per_b
            assert md.moe_decode_kernels_per_step(h, 2) == per_b
        finally:
            assert md.moe_decode_destroy(h) == 0


@pytest.mark.gpu
def test_host_buffer_step_matches_device_step():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import synth
    from oracle.layer import build_case
    from tests.harness import GpuStack
    synth.build_device_fill()
    seed = synth.config_seed(0) + 55
    st = GpuStack(seed, synth.TINY, max_batch=8)
    try:
        case = build_case(seed, synth.TINY, 3, checked=[0])
        out_d, idx_d, gate_d = st.step(case["attn"], case["resid"])
        out_h = np.zeros((3, synth.TINY.d), np.uint16)
        idx_h = np.zeros((1, 3, synth.TINY.k), np.int32)
        gate_h = np.zeros((1, 3, synth.TINY.k), np.float32)
        st.md.moe_decode_step_host(st.h, 3, np.ascontiguousarray(case["attn"]), np.ascontiguousarray(case["resid"]),
                                   out_h, idx_h, gate_h)
        assert np.array_equal(out_h, out_d) and np.array_equal(idx_h, idx_d) and np.array_equal(gate_h, gate_d)
        # another batch, outputs only (no top-k buffers), into unpinned numpy memory
        case1 = build_case(seed + 1, synth.TINY, 1, checked=[0])
        out1_d, _, _ = st.step(case1["attn"], case1["resid"])
        out1_h = np.zeros((1, synth.TINY.d), np.uint16)
        st.md.moe_decode_step_host(st.h, 1, np.ascontiguousarray(case1["attn"]),
                                   np.ascontiguousarray(case1["resid"]), out1_h)
        assert np.array_equal(out1_h, out1_d)
        # the same batch again (the cached graph with its staging copies), new inputs
        case2 = build_case(seed + 2, synth.TINY, 3, checked=[0])
        out2_d, idx2_d, gate2_d = st.step(case2["attn"], case2["resid"])
        st.md.moe_decode_step_host(st.h, 3, np.ascontiguousarray(case2["attn"]),
                                   np.ascontiguousarray(case2["resid"]), out_h, idx_h, gate_h)
        assert np.array_equal(out_h, out2_d) and np.array_equal(idx_h, idx2_d) and np.array_equal(gate_h, gate2_d)
    finally:
        st.close()


@pytest.mark.gpu
def test_host_buffer_step_pinned_caller_buffers():
    """Pinned host buffers of the caller (torch pin_memory) and a mix with pageable outputs:
    results equal the device step's, on a new graph and on its replay."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import synth
    from oracle.layer import build_case
    from tests.harness import GpuStack
    synth.build_device_fill()
    dims = synth.Dims(256, 256, 16, 4, 128)  # top_k * 4 bytes per token: whole 16-byte words
    seed = synth.config_seed(0) + 91
    st = GpuStack(seed, dims, max_batch=4)
    try:
        for B in (1, 3, 3):
            case = build_case(seed + B, dims, B, checked=[0])
            out_d, idx_d, gate_d = st.step(case["attn"], case["resid"])
            pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
            attn_p = pin(case["attn"].view(np.int16))
            resid_p = pin(case["resid"].view(np.int16))
            out_p = torch.zeros((B, dims.d), dtype=torch.int16).pin_memory()
            idx_p = torch.zeros((1, B, dims.k), dtype=torch.int32).pin_memory()
            gate_p = torch.zeros((1, B, dims.k), dtype=torch.float32).pin_memory()
            st.md.moe_decode_step_host(st.h, B, attn_p, resid_p, out_p, idx_p, gate_p)
            assert np.array_equal(out_p.numpy().view(np.uint16), out_d)
            assert np.array_equal(idx_p.numpy(), idx_d) and np.array_equal(gate_p.numpy(), gate_d)
            out_h = np.zeros((B, dims.d), np.uint16)
            st.md.moe_decode_step_host(st.h, B, attn_p, resid_p, out_h)
            assert np.array_equal(out_h, out_d)
    finally:
        st.close()


@pytest.mark.gpu
@pytest.mark.parametrize("B", [1, 2, 5])
def test_host_buffer_step_two_layer_stack(B):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import synth
    from oracle.layer import build_case
    from tests.harness import GpuStack
    synth.build_device_fill()
    seed = synth.config_seed(0) + 77 + B
    st = GpuStack(seed, synth.TINY, n_layers=2, max_batch=8)
    try:
        case = build_case(seed, synth.TINY, B, n_layers=2, checked=[0])
        out_d, idx_d, gate_d = st.step(case["attn"], case["resid"])
        out_h = np.zeros((B, synth.TINY.d), np.uint16)
        idx_h = np.zeros((2, B, synth.TINY.k), np.int32)
        gate_h = np.zeros((2, B, synth.TINY.k), np.float32)
        for _ in range(2):
            st.md.moe_decode_step_host(st.h, B, np.ascontiguousarray(case["attn"]),
                                       np.ascontiguousarray(case["resid"]), out_h, idx_h, gate_h)
            assert np.array_equal(out_h, out_d) and np.array_equal(idx_h, idx_d) and np.array_equal(gate_h, gate_d)
    finally:
        st.close()
