"""moe_decode_step_static (no device allocation; scratch in the library's static array)
against moe_decode_step on the same seeded inputs.  Collected last (file name); it must
pass both after the other tests and alone in a fresh process."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

RAGGED = synth.Dims(320, 192, 40, 5, 96)


def _torch():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _inputs(torch, seed, dims, B):
    attn = np.stack([synth.host_token(seed, synth.ATTN, dims.d_o, token=b) for b in range(B)])
    resid = np.stack([synth.host_token(seed, synth.RESID, dims.d, token=b) for b in range(B)])
    to_dev = lambda a: torch.from_numpy(a.view(np.int16).copy()).cuda().view(torch.bfloat16)
    return to_dev(attn), to_dev(resid)


# Both entry points launch the same deterministic kernels on the same inputs, so their
# outputs, indices and gates must agree bit for bit; force_variant 1 at batch 1 selects the
# three small-batch kernels in both.
@pytest.mark.parametrize("dims,B,variant", [(synth.TINY, 1, 0), (synth.TINY, 2, 0), (RAGGED, 1, 0),
                                            (RAGGED, 2, 0), (synth.TINY, 1, 1), (RAGGED, 1, 1),
                                            (synth.TINY, 1, 3), (RAGGED, 2, 3),
                                            (synth.TP16, 1, 0), (synth.TP16, 2, 0), (synth.TP16, 1, 3),
                                            (synth.TP16, 2, 3)])
def test_static_step_matches_step_twice(dims, B, variant):
    torch = _torch()
    import moe_decode_layer_02_b200 as md
    from tests.harness import device_weights
    synth.build_device_fill()
    seed = 41
    w = device_weights(seed, dims, 1)[0]
    cfg = md.config(dims.d, dims.d_o, dims.E, dims.k, dims.I, 2, force_variant=variant)
    s = torch.cuda.current_stream()
    attn, resid = _inputs(torch, seed, dims, B)
    h = md.moe_decode_create(cfg, [w], s)
    try:
        out_ref = torch.empty((B, dims.d), dtype=torch.bfloat16, device="cuda")
        idx_ref = torch.full((B, dims.k), -1, dtype=torch.int32, device="cuda")
        gate_ref = torch.full((B, dims.k), -1.0, dtype=torch.float32, device="cuda")
        md.moe_decode_step(h, B, attn, resid, out_ref, idx_ref, gate_ref, s)
        assert md.moe_decode_sync_status(h, s) == 0
    finally:
        assert md.moe_decode_destroy(h) == 0
    outs, idxs, gates, errs = [], [], [], []
    for _ in range(2):  # two calls in a row on one stream, no synchronisation between them
        outs.append(torch.full((B, dims.d), float("nan"), dtype=torch.bfloat16, device="cuda"))
        idxs.append(torch.full((B, dims.k), -1, dtype=torch.int32, device="cuda"))
        gates.append(torch.full((B, dims.k), -1.0, dtype=torch.float32, device="cuda"))
        errs.append(torch.full((4,), 0x7F7F7F7F, dtype=torch.int32, device="cuda"))
        md.moe_decode_step_static(cfg, w, B, attn, resid, outs[-1], idxs[-1], gates[-1], errs[-1], s)
    torch.cuda.synchronize()
    for out, idx, gate, err in zip(outs, idxs, gates, errs):
        assert int(err[0]) == 0
        assert torch.equal(idx, idx_ref)
        assert torch.equal(gate, gate_ref)
        assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))


def test_static_step_rejects_what_it_cannot_run():
    torch = _torch()
    import moe_decode_layer_02_b200 as md
    s = torch.cuda.current_stream()
    # force_variant 3, n_experts = 1024, batch 2: the split-K router's partial sums
    # (SMs x 1024 x 2 floats) and the rest need about 1.7 MB on a 148-SM part, more than
    # MOE_STATIC_SCRATCH_BYTES.
    # The size checks run before anything is launched or read, so small dummy buffers stand
    # in for the weights and activations.
    d, d_o, E, k, I = 8192, 64, 1024, 32, 512
    z = lambda n: torch.zeros(n, dtype=torch.bfloat16, device="cuda")
    w = tuple(z(64) for _ in range(5))
    attn, resid, out = z(64), z(64), z(64)
    cfg = md.config(d, d_o, E, k, I, 2, force_variant=3)
    with pytest.raises(md.MoeError) as ei:
        md.moe_decode_step_static(cfg, w, 2, attn, resid, out, stream=s)
    assert ei.value.code == md.MOE_ERR_SCRATCH_LIMIT
    assert md.strerror(md.MOE_ERR_SCRATCH_LIMIT) == "scratch need exceeds the static array"
    tiny = synth.TINY
    cfg = md.config(tiny.d, tiny.d_o, tiny.E, tiny.k, tiny.I, 2)
    for B in (0, 3):
        with pytest.raises(md.MoeError) as ei:
            md.moe_decode_step_static(cfg, w, B, attn, resid, out, stream=s)
        assert ei.value.code == md.MOE_ERR_INVALID_ARG
    for bad in (md.config(tiny.d, tiny.d_o, tiny.E, tiny.k, tiny.I, 2, n_layers=2),
                md.config(tiny.d, tiny.d_o, tiny.E, tiny.k, tiny.I, 2, force_variant=2)):
        with pytest.raises(md.MoeError) as ei:
            md.moe_decode_step_static(bad, w, 1, attn, resid, out, stream=s)
        assert ei.value.code == md.MOE_ERR_UNSUPPORTED_CONFIG
    with pytest.raises(md.MoeError) as ei:
        md.moe_decode_step_static(cfg, w, 1, attn.data_ptr() + 2, resid, out, stream=s)
    assert ei.value.code == md.MOE_ERR_ALIGNMENT
    torch.cuda.synchronize()
