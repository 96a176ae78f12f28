"""The device error path through the C ABI: bounded waits that run out and an index check
that fires are reported by moe_decode_sync_status, cleared by it, and the next step is
correct.  No fault: the probe's waits give up after 1 ms (a flag nothing sets)."""
import numpy as np
import pytest

import synth
from oracle.layer import build_case
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


@pytest.mark.parametrize("B", [1, 2, 5])
@pytest.mark.parametrize("what,code", [(1, "MOE_ERR_DEVICE_TIMEOUT"), (2, "MOE_ERR_DEVICE_BOUNDS")])
def test_error_recorded_cleared_and_next_step_green(what, code, B):
    import torch
    import moe_decode_layer_02_b200 as md
    seed = synth.config_seed(0) + 31 * B
    st = H.GpuStack(seed, synth.TINY, max_batch=8)
    s = torch.cuda.current_stream()
    try:
        case = build_case(seed, synth.TINY, B)
        o1, i1, g1 = st.step(case["attn"], case["resid"])  # green before
        md.moe_decode_check_error_path(st.h, what, 1_000_000, s)
        assert md.moe_decode_sync_status(st.h, s) == getattr(md, code)
        assert md.moe_decode_sync_status(st.h, s) == md.MOE_OK  # the record was cleared
        o2, i2, g2 = st.step(case["attn"], case["resid"])  # asserts a clean status itself
        assert np.array_equal(o1, o2) and np.array_equal(i1, i2) and np.array_equal(g1, g2)
        ref = case["layers"][0]
        for b in range(B):
            assert np.array_equal(i2[0, b], ref["idx"][b])
            H.check_out(o2[b], ref["out_ref"][b])
    finally:
        st.close()


def test_error_probe_rejects_bad_arguments():
    import torch
    import moe_decode_layer_02_b200 as md
    st = H.GpuStack(synth.config_seed(0), synth.TINY, max_batch=1)
    try:
        for what, lim in [(0, 1000), (3, 1000), (1, 0), (1, 10_000_001)]:
            with pytest.raises(md.MoeError) as ei:
                md.moe_decode_check_error_path(st.h, what, lim, torch.cuda.current_stream())
            assert ei.value.code == md.MOE_ERR_INVALID_ARG
    finally:
        st.close()
