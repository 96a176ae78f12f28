"""Tensor-parallel partitioning of the layer, checked on the CPU with two gloo ranks.

The pages' deployment shards the layer over 8-16 GPUs: the attention output projection is
fused with its all-reduce and the residual step, and the routing work is split across the
GPUs and combined ("vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300 with agent-assisted
kernels", section "How the specialised decode path works").  The partition taken here, for
N ranks (rank r):
  o_proj    W_o's input columns (d_o) split: rank r forms W_o[:, slice_r] . attn[slice_r],
            rank 0 adds the residual; an all-reduce (sum) gives h on every rank;
  RMSNorm   on the full h, on every rank;
  router    the experts split: rank r computes the logits of its E / N experts; an
            all-gather gives every rank all logits, and every rank selects the same top-k;
  experts   each expert's intermediate size I split: rank r holds gate/up rows and W_down
            columns of its I / N slice, forms its slice of every selected expert's down
            projection and the gate-weighted sum of those; an all-reduce (sum) plus h
            gives the output.
This test runs that partition with the oracle's own functions on each rank's slice of the
seeded weights and checks it against the unsplit oracle: the logits agree exactly (each
expert's dot product is computed whole on one rank), so do the selected experts, and h and
the output agree to fp64 rounding (only the order of the sums changes)."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DIMS = (256, 256, 16, 2, 128)  # d, d_o, E, k, I (the tiny layer)
B = 2


def _inputs():
    sys.path.insert(0, ROOT)
    import synth
    dims = synth.Dims(*DIMS)
    seed = synth.config_seed(0) + 901
    w = synth.host_weights(seed, dims, 0)
    attn = np.stack([synth.host_token(seed, synth.ATTN, dims.d_o, token=b) for b in range(B)])
    resid = np.stack([synth.host_token(seed, synth.RESID, dims.d, token=b) for b in range(B)])
    return seed, dims, w, attn, resid


def _rank(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        o = oracle.get()
        seed, D, w, attn, resid = _inputs()
        W_o = w[synth.W_O].reshape(D.d, D.d_o)
        W_r = w[synth.W_R].reshape(D.E, D.d)
        ko, ke, ki = D.d_o // world, D.E // world, D.I // world
        so, se, si = slice(rank * ko, (rank + 1) * ko), slice(rank * ke, (rank + 1) * ke), slice(rank * ki, (rank + 1) * ki)
        # o_proj partial (rank 0 adds the residual), all-reduce
        res_r = resid if rank == 0 else np.zeros_like(resid)
        h_r = o.oproj_residual(np.ascontiguousarray(W_o[:, so]), np.ascontiguousarray(attn[:, so]), res_r, B, D.d, ko)
        h = torch.from_numpy(h_r.copy())
        dist.all_reduce(h)
        h = h.numpy()
        rstd, x = o.rmsnorm(h, w[synth.GAMMA])
        # router over this rank's experts, all-gather
        lg_r = torch.from_numpy(o.router(np.ascontiguousarray(W_r[se]), x, ke))
        parts = [torch.empty_like(lg_r) for _ in range(world)]
        dist.all_gather(parts, lg_r)
        logits = torch.cat(parts, dim=1).numpy()
        idx, gate = o.topk_gates(logits.astype(np.float32), D.k)
        # experts over this rank's slice of I, gate-weighted, all-reduce
        comb = np.zeros((B, D.d))
        for b in range(B):
            ys = []
            for e in idx[b]:
                gu, dn = synth.host_expert(seed, D, int(e), 0)
                gu_r = np.concatenate([gu[si], gu[D.I:][si]])          # gate rows, then up rows
                dn_r = np.ascontiguousarray(dn[:, si])                  # [d][I / N]
                ys.append(o.expert(gu_r, dn_r, x[b], ki)[1])
            comb[b] = o.combine(np.zeros(D.d), gate[b], ys)[0]
        ct = torch.from_numpy(comb)
        dist.all_reduce(ct)
        out = h + ct.numpy()
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), h=h, logits=logits, idx=idx, gate=gate, out=out)
    finally:
        dist.destroy_process_group()


def test_tensor_parallel_split_matches_unsplit_oracle(tmp_path):
    pytest.importorskip("torch")
    import socket

    import torch.multiprocessing as mp

    import oracle
    from oracle.layer import LayerRef
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    mp.start_processes(_rank, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    seed, D, w, attn, resid = _inputs()
    ref = LayerRef(seed, D, 0, oracle=oracle.get())
    f = ref.front(attn, resid)
    outs = ref.moe_many({b: {k: v[b:b + 1] for k, v in f.items()} for b in range(B)})
    for r in range(2):
        got = np.load(tmp_path / f"r{r}.npz")
        assert np.allclose(got["h"], f["h"], rtol=0, atol=1e-12)
        assert np.array_equal(got["logits"], f["logits64"])            # whole dot products on one rank
        assert np.array_equal(got["idx"], f["idx"]) and np.allclose(got["gate"], f["gate"], rtol=0, atol=1e-15)
        for b in range(B):
            assert np.allclose(got["out"][b], outs[b][0], rtol=0, atol=1e-11)
