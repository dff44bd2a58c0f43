"""Sequence-parallel attention schedules (ring and Ulysses) on CPU gloo ranks.

Each rank holds a contiguous shard of the tokens.  The local attention and
the log-sum-exp merge are the oracle's, so these tests check the host-side
schedules -- who sends what to whom, in which order, and how the hops are
merged -- against attention over the whole sequence.  The CUDA kernels behind
the default local operations are checked in test_gpu_kernels.py."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(S, H, seed=7):
    r = np.random.default_rng(seed)
    return [r.standard_normal((S, H * 128)) for _ in range(3)]


def _rank(rank, world, port, S, H, out):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from oracle import dit_oracle as O
    from diffusion_transformer_block_flux_b200 import sequence_parallel as sp

    def o_attn(q, k, v, o, lse, h):
        qn, kn, vn = q.numpy(), k.numpy(), v.numpy()
        o.copy_(torch.from_numpy(O.attention(qn, kn, vn, h)))
        if lse is not None:
            lse.copy_(torch.from_numpy(O.attention_lse(qn, kn, h)))

    def o_merge(parts, lses, o, lse, h):
        m, l = O.attention_merge([p.numpy() for p in parts], [x.double().numpy() for x in lses])
        o.copy_(torch.from_numpy(m))
        lse.copy_(torch.from_numpy(l))

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v = _inputs(S, H)
        n = S // world
        sl = slice(rank * n, (rank + 1) * n)
        ref = O.attention(q, k, v, H)[sl]
        ref_lse = O.attention_lse(q, k, H)[:, sl]
        qs, ks, vs = (torch.from_numpy(np.ascontiguousarray(t[sl])) for t in (q, k, v))
        o_ring = torch.empty_like(qs)
        lse = sp.ring_attention(qs, ks, vs, o_ring, H, attn=o_attn, merge=o_merge)
        o_uly = torch.empty_like(qs)
        sp.ulysses_attention(qs, ks, vs, o_uly, H, attn=o_attn)
        out[rank] = (float(np.abs(o_ring.numpy() - ref).max()),
                     float(np.abs(lse.double().numpy() - ref_lse).max() / np.abs(ref_lse).max()),
                     float(np.abs(o_uly.numpy() - ref).max()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ring_and_ulysses_schedules_equal_full_attention(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    S, H = 24, 4
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, S, H, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    for r in range(world):
        ring_err, lse_err, uly_err = out[r]
        # the ring's merge takes the running lse in fp32 (the CUDA contract)
        assert ring_err < 1e-6, (r, ring_err)
        assert lse_err < 1e-6, (r, lse_err)
        assert uly_err < 1e-12, (r, uly_err)
