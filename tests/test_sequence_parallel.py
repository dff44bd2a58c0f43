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
        # the plans hold lse as [1, H, S] (the CUDA layout [B, H, S])
        m, l = O.attention_merge([p.numpy() for p in parts], [x.double().numpy().reshape(h, -1) for x in lses])
        o.copy_(torch.from_numpy(m))
        lse.copy_(torch.from_numpy(l).reshape(lse.shape))

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v = _inputs(S, H)
        n = S // world
        sl = slice(rank * n, (rank + 1) * n)
        ref = O.attention(q, k, v, H)[sl]
        ref_lse = O.attention_lse(q, k, H)[:, sl]
        qs, ks, vs = (torch.from_numpy(np.ascontiguousarray(t[sl])) for t in (q, k, v))
        ring = []
        for g in range(1, world + 1):  # shards per attention step: 1 (the ring) .. N (gather all)
            o_ring = torch.empty_like(qs)
            lse = sp.ring_attention(qs, ks, vs, o_ring, H, attn=o_attn, merge=o_merge, shards_per_step=g)
            ring.append((float(np.abs(o_ring.numpy() - ref).max()),
                         float(np.abs(lse.double().numpy() - ref_lse).max() / np.abs(ref_lse).max())))
        o_uly = torch.empty_like(qs)
        sp.ulysses_attention(qs, ks, vs, o_uly, H, attn=o_attn)
        out[rank] = (ring, float(np.abs(o_uly.numpy() - ref).max()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
def test_ring_and_ulysses_schedules_equal_full_attention(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    S, H = 24, (6 if world == 3 else 4)
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, S, H, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    for r in range(world):
        ring, uly_err = out[r]
        # the ring's merge takes the running lse in fp32 (the CUDA contract)
        for g, (ring_err, lse_err) in enumerate(ring, 1):
            assert ring_err < 1e-6, (r, g, ring_err)
            assert lse_err < 1e-6, (r, g, lse_err)
        assert uly_err < 1e-12, (r, uly_err)


def _oracle_ops(O, torch, D, H, M, eps=1e-6):
    """The block's per-token steps as oracle functions on float64 CPU tensors,
    with the contracts of sequence_parallel.CudaBlockOps (the RoPE argument is
    this shard's rows of the angle table)."""

    class Ops:
        def adaln(self, w, vec, mod):
            mod[0] = torch.from_numpy(O.linear(O.silu(vec[0].numpy()), w["W_mod"], w["b_mod"]))

        def modulate_norm(self, x, mod, y):
            m = mod[0].numpy()
            y.copy_(torch.from_numpy(O.modulate(O.layer_norm(x.numpy(), eps), m[:D], m[D:2 * D])))

        def qkv_mlp(self, w, y, phi, qkv, cat):
            h = O.linear(y.numpy(), w["W1"], w["b1"])
            q = O.apply_rope(O.rms_norm_heads(h[:, :D], w["q_scale"], H, eps), phi, H)
            k = O.apply_rope(O.rms_norm_heads(h[:, D:2 * D], w["k_scale"], H, eps), phi, H)
            qkv.copy_(torch.from_numpy(np.concatenate([q, k, h[:, 2 * D:3 * D]], axis=1)))
            cat[:, D:] = torch.from_numpy(O.gelu_tanh(h[:, 3 * D:]))

        def out_proj(self, w, cat, x, mod, out):
            g = mod[0, 2 * D:].numpy()
            out.copy_(torch.from_numpy(x.numpy() + g * O.linear(cat.numpy(), w["W2"], w["b2"])))

    return Ops()


def _sp_block_rank(rank, world, port, mode, out):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from oracle import dit_oracle as O
    from diffusion_transformer_block_flux_b200 import sequence_parallel as sp
    from diffusion_transformer_block_flux_b200 import synth

    def o_attn(q, k, v, o, lse, h):
        qn, kn, vn = q.numpy(), k.numpy(), v.numpy()
        o.copy_(torch.from_numpy(O.attention(qn, kn, vn, h)))
        if lse is not None:
            lse.copy_(torch.from_numpy(O.attention_lse(qn, kn, h)).reshape(lse.shape))

    def o_merge(parts, lses, o, lse, h):
        m, l = O.attention_merge([p.numpy() for p in parts], [x.double().numpy().reshape(h, -1) for x in lses])
        o.copy_(torch.from_numpy(m))
        lse.copy_(torch.from_numpy(l).reshape(lse.shape))

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        shape = synth.BlockShape("sp", 4, 4, 3, 512, 4, 256)  # S = 16 tokens, 4 heads
        wb = synth.single_block_weights(shape, bias_std=0.1, norm_scale_std=0.1)
        ab = synth.block_activations(shape)
        w = synth.to_f64(wb)
        f = synth.to_f64(ab)
        S, D, H, M = shape.S, shape.D, shape.H, shape.M
        n = S // world
        sl = slice(rank * n, (rank + 1) * n)
        ref = O.single_block(f["x"], f["vec"], f["ids"], w, H)[sl]
        phi = O.rope_angles(f["ids"], (16, 56, 56))[sl]
        blk = sp.SequenceParallelSingleBlock(n, D, H, M, "cpu", mode=mode, ops=_oracle_ops(O, torch, D, H, M),
                                             attn=o_attn, merge=None if mode == "ulysses" else o_merge,
                                             dtype=torch.float64)
        x = torch.from_numpy(np.ascontiguousarray(f["x"][sl]))
        vec = torch.from_numpy(f["vec"]).reshape(1, -1)
        y = torch.empty_like(x)
        blk.forward(w, x, vec, phi, y)
        first = y.clone()
        blk.forward(w, x, vec, phi, y)  # the plan's buffers are reused: same result again
        out[rank] = (float(np.abs(y.numpy() - ref).max() / np.abs(ref).max()),
                     bool(torch.equal(first, y)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,mode", [(2, "ring"), (4, "ring"), (2, "ulysses"), (4, "ulysses")])
def test_sequence_parallel_single_block_equals_the_block(world, mode):
    """The whole single-stream block with its tokens sharded over 2 or 4 gloo
    ranks (per-token steps on the local shard with that shard's RoPE rows,
    attention by the ring or by Ulysses) equals the oracle's block over the
    whole sequence on every rank's rows.  The ring carries its running lse in
    fp32 (the CUDA contract), hence the 1e-6 relative bound."""
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_sp_block_rank, args=(r, world, port, mode, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    for r in range(world):
        err, same = out[r]
        assert err < (1e-6 if mode == "ring" else 1e-12), (r, err)
        assert same, r
