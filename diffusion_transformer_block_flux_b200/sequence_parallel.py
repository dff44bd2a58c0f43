"""Sequence-parallel attention and the sequence-parallel single-stream block
over the ranks of a torch.distributed group.

Page: "compile_graph" (chenyy20.com) §5 and §6.  The sequence is split evenly
over the GPUs and every per-token step stays local; only attention needs the
whole sequence.  Two ways to assemble it:
  - Ring: K and V travel around the ranks by point-to-point transfers, one hop
    per rank; every hop computes attention of the local queries against the
    shard in hand and merges it into the running result by log-sum-exp.
  - Ulysses: an all-to-all trades tokens for heads, so each rank holds the
    whole sequence for H/N heads; local attention; an all-to-all trades back.
§6 captures the whole step, transfers included, as one CUDA graph: that needs
fixed buffers and no allocation inside the step, so every plan below owns its
buffers, allocated once, and a call only launches work on the current stream.

Each rank holds a contiguous shard of S/N tokens: rank r owns tokens
[r S/N, (r+1) S/N).  Tensors are [S/N, H*128] row views (head h at columns
h*128, any row stride), as the block entry points lay them out.  The local
operations default to this library's CUDA kernels (dit_attention with its
log-sum-exp, dit_attention_merge, and the block's kernels); `ops` (or
`attn` / `merge`) can be replaced by objects with the same contracts, which
the multi-process CPU tests use to check the schedules themselves.
"""
from __future__ import annotations


def _cuda_attn(q, k, v, o, lse, H):
    from . import dit_attention
    dit_attention(q, k, v, o, 1, q.shape[0], k.shape[0], H, lse=lse)


def _cuda_merge(o_parts, lse_parts, o, lse, H):
    from . import dit_attention_merge
    dit_attention_merge(o_parts, lse_parts, o, lse, 1, o.shape[0], H)


def _peer(group, r):
    import torch.distributed as dist
    return r if group is None else dist.get_global_rank(group, r)


def _cuda_attn_acc(q, k, v, o, lse, H):
    from . import dit_attention_accumulate
    dit_attention_accumulate(q, k, v, o, lse, 1, q.shape[0], k.shape[0], H)


def auto_key_splits(S_loc, H, device):
    """Key splits for the local attention of S_loc queries: the attention
    kernel runs one CTA per 256 queries and head, so a short local sequence
    leaves SMs idle (576 queries x 24 heads: 72 CTAs on 148 SMs); splitting the
    keys into parts merged by log-sum-exp (dit_attention_split) fills them."""
    import torch
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    ctas = -(-S_loc // 256) * H
    return max(1, min(4, sms // max(1, ctas)))


class RingAttention:
    """One rank's ring attention with buffers owned by the plan.

    Call: out = attention(q, K, V) where K and V are the concatenation of every
    rank's k and v shards.  Shards travel one per hop: at hop h this rank sends
    the shard it received last (its own at hop 0) to rank r+1 and receives the
    next one from rank r-1, N - 1 hops in all, each hop's send and receive
    posted as one batch.  Received shards land in consecutive rows of a
    staging ring, and every `shards_per_step` shards (G) one attention launch
    covers them: the first writes `out` and the running log-sum-exp, the
    later ones merge into both in their epilogue (dit_attention_accumulate),
    while the next G shards are still arriving.  G = 1 is the ring of the
    compile_graph page (§5); larger G trades overlap for longer launches
    (G = N gathers every shard before one launch).  Returns the fp32
    log-sum-exp [1, H, S/N] of the local queries over all keys (a buffer of
    the plan).

    With `attn` and `merge` given (the CPU tests' oracle operations), a later
    step writes its own result to a partial buffer and `merge` folds it in.

    key_splits (CUDA operations only): each step's keys are cut into that many
    parts computed side by side and merged by log-sum-exp
    (dit_attention_split), for local query counts too small to fill the GPU;
    None picks it from the SM count (auto_key_splits)."""

    def __init__(self, S_loc, H, device, dtype=None, group=None, attn=None, merge=None, shards_per_step=1,
                 key_splits=None):
        import torch
        import torch.distributed as dist
        dtype = dtype or torch.bfloat16
        self.H, self.S_loc, self.group = H, S_loc, group
        self.N = dist.get_world_size(group)
        self.r = dist.get_rank(group)
        self.G = max(1, min(int(shards_per_step), self.N))
        custom = attn is not None or merge is not None
        self.attn = attn or _cuda_attn
        self.merge = merge or _cuda_merge
        self.acc = None if custom else _cuda_attn_acc
        D = H * 128
        self.splits = 1
        if not custom:
            from . import dit_attention_split_workspace
            self.splits = int(key_splits) if key_splits is not None else auto_key_splits(S_loc, H, device)
            if self.splits > 1:
                self.ws = torch.empty(dit_attention_split_workspace(1, S_loc, H, self.splits), dtype=torch.uint8,
                                      device=device)
        slots = 2 * self.G if self.N > self.G else self.G  # two stages in flight while more shards follow
        self.slots = slots
        self.k = torch.empty((slots * S_loc, D), dtype=dtype, device=device)
        self.v = torch.empty_like(self.k)
        self.lse = torch.empty((1, H, S_loc), dtype=torch.float32, device=device)
        if self.acc is None:
            self.part = torch.empty((S_loc, D), dtype=dtype, device=device)
            self.lse_part = torch.empty_like(self.lse)
        self.nxt = _peer(group, (self.r + 1) % self.N)
        self.prv = _peer(group, (self.r - 1) % self.N)

    def _rows(self, slot, n=1):
        a = slot * self.S_loc
        return slice(a, a + n * self.S_loc)

    def _step(self, q, first_slot, n, out, first):
        H = self.H
        kk, vv = self.k[self._rows(first_slot, n)], self.v[self._rows(first_slot, n)]
        if self.splits > 1:
            from . import dit_attention_split
            dit_attention_split(q, kk, vv, out, 1, q.shape[0], kk.shape[0], H, self.splits, self.ws, lse=self.lse,
                                accumulate=not first)
        elif first:
            self.attn(q, kk, vv, out, self.lse, H)
        elif self.acc is not None:
            self.acc(q, kk, vv, out, self.lse, H)
        else:
            self.attn(q, kk, vv, self.part, self.lse_part, H)
            self.merge([out, self.part], [self.lse, self.lse_part], out, self.lse, H)

    def __call__(self, q, k, v, out):
        import torch.distributed as dist
        D, N, G, S = self.H * 128, self.N, self.G, self.slots
        self.k[self._rows(0)].copy_(k[:, :D])
        self.v[self._rows(0)].copy_(v[:, :D])
        step_first = 0  # slot of the current step's first shard
        for h in range(N):  # shard h (received at hop h - 1, or the local one) sits in slot h % S
            reqs = []
            if h < N - 1:
                # one group for the sends and the receives: with NCCL, separate calls
                # would queue every rank's send ahead of its receive and wait in a cycle
                cur, nxt = self._rows(h % S), self._rows((h + 1) % S)
                reqs = dist.batch_isend_irecv([
                    dist.P2POp(dist.isend, self.k[cur], self.nxt, self.group),
                    dist.P2POp(dist.isend, self.v[cur], self.nxt, self.group),
                    dist.P2POp(dist.irecv, self.k[nxt], self.prv, self.group),
                    dist.P2POp(dist.irecv, self.v[nxt], self.prv, self.group)])
            if (h + 1) % G == 0 or h == N - 1:  # the step's last shard is in hand
                n = h - (h // G) * G + 1
                self._step(q, step_first, n, out, h < G)
                step_first = (h + 1) % S
            for req in reqs:
                req.wait()
        return self.lse


class UlyssesAttention:
    """One rank's Ulysses attention with buffers owned by the plan.

    Call: out = attention(q, K, V) over the whole sequence with heads split
    across ranks: an all-to-all gives rank r all tokens of heads
    [r H/N, (r+1) H/N), attention runs there, and a second all-to-all returns
    every rank its own tokens.  H must be a multiple of the group size."""

    def __init__(self, S_loc, H, device, dtype=None, group=None, attn=None):
        import torch
        import torch.distributed as dist
        dtype = dtype or torch.bfloat16
        self.N = dist.get_world_size(group)
        if H % self.N:
            raise ValueError(f"{H} heads do not split over {self.N} ranks")
        self.H, self.S_loc, self.group = H, S_loc, group
        self.attn = attn or _cuda_attn
        self.Hl = H // self.N
        w = self.Hl * 128
        # q, k, v; chunk i of the token shard goes to rank i / comes from rank i
        self.send = torch.empty((3, self.N, S_loc, w), dtype=dtype, device=device)
        self.recv = torch.empty_like(self.send)
        self.o_heads = torch.empty((self.N * S_loc, w), dtype=dtype, device=device)
        self.o_back = torch.empty((self.N, S_loc, w), dtype=dtype, device=device)

    def __call__(self, q, k, v, out):
        import torch.distributed as dist
        N, S_loc, Hl = self.N, self.S_loc, self.Hl
        w = Hl * 128
        for i, t in enumerate((q, k, v)):  # [S_loc, H*128] -> [N, S_loc, w]: head group i -> rank i
            self.send[i].copy_(t[:, :N * w].reshape(S_loc, N, w).transpose(0, 1))
        for i in range(3):
            dist.all_to_all_single(self.recv[i], self.send[i], group=self.group)
        # rank i's tokens in rank order: the whole sequence for this rank's heads
        qh, kh, vh = (self.recv[i].view(N * S_loc, w) for i in range(3))
        self.attn(qh, kh, vh, self.o_heads, None, Hl)
        dist.all_to_all_single(self.o_back, self.o_heads.view(N, S_loc, w), group=self.group)
        out[:, :N * w].copy_(self.o_back.transpose(0, 1).reshape(S_loc, N * w))  # head group i came from rank i
        return out


def ring_attention(q, k, v, out, H, group=None, attn=None, merge=None, shards_per_step=1, key_splits=None):
    """One-off ring attention (a plan built for this call); see RingAttention."""
    plan = RingAttention(q.shape[0], H, q.device, q.dtype, group, attn, merge, shards_per_step, key_splits)
    lse = plan(q, k, v, out)
    return lse[0]


def ulysses_attention(q, k, v, out, H, group=None, attn=None):
    """One-off Ulysses attention (a plan built for this call); see UlyssesAttention."""
    return UlyssesAttention(q.shape[0], H, q.device, q.dtype, group, attn)(q, k, v, out)


class CudaBlockOps:
    """The per-token steps of the single-stream block as this library's
    kernels (the same calls dit_single_block_fwd makes)."""

    def __init__(self, D, H, M, eps=1e-6):
        self.D, self.H, self.M, self.eps = D, H, M, eps

    def adaln(self, w, vec, mod):
        from . import dit_adaln_modulation
        dit_adaln_modulation(vec, w["W_mod"], w["b_mod"], mod)

    def modulate_norm(self, x, mod, y):
        from . import dit_modulate_norm
        D = self.D
        dit_modulate_norm(x, mod[0, :D], mod[0, D:2 * D], y, 1, x.shape[0], self.eps)

    def qkv_mlp(self, w, y, rope, qkv, cat):
        from . import dit_gemm_epilogue, DIT_EPI_BIAS_GELU_COLS
        D = self.D
        dit_gemm_epilogue(y, w["W1"], qkv, epi=DIT_EPI_BIAS_GELU_COLS, bias=w["b1"], C2=cat[:, D:],
                          split_col=3 * D, gelu_col_begin=3 * D, qk_cols=2 * D, qk_norm=1, qk_eps=self.eps,
                          q_scale=w["q_scale"], k_scale=w["k_scale"], rope=rope, rope_rows=y.shape[0])

    def out_proj(self, w, cat, x, mod, out):
        from . import dit_gemm_epilogue, DIT_EPI_BIAS_GATED_RESIDUAL
        D = self.D
        dit_gemm_epilogue(cat, w["W2"], out, epi=DIT_EPI_BIAS_GATED_RESIDUAL, bias=w["b2"],
                          gate=mod[0, 2 * D:], gate_stride=0, resid=x, rows_per_batch=x.shape[0])


class SequenceParallelSingleBlock:
    """Flux single-stream block over a sequence sharded across the ranks of a
    group ("compile_graph" §5-§6): adaLN, LayerNorm + modulate, the fused
    QKV|MLP-in GEMM (QK RMSNorm + RoPE with this shard's rows of the RoPE
    table, GELU on the MLP columns) and the output GEMM with the gated residual
    run on the local S/N tokens; attention assembles the whole sequence by the
    ring or by Ulysses.  Every buffer is allocated here, once, so a forward
    launches work only and can be captured, transfers included, into a CUDA
    graph.

    forward(w, x, vec, rope, out): x, out [S/N, D] bf16 (out may be x); vec
    [1, D] bf16; rope: this shard's rows of the RoPE table [S/N, 64, 2] fp32."""

    def __init__(self, S_loc, D, H, M, device, group=None, mode="ring", ops=None, attn=None, merge=None,
                 dtype=None, eps=1e-6, shards_per_step=1, key_splits=None):
        import torch
        dtype = dtype or torch.bfloat16
        if mode not in ("ring", "ulysses"):
            raise ValueError(f"mode {mode!r}")
        self.D, self.M, self.S_loc = D, M, S_loc
        self.ops = ops or CudaBlockOps(D, H, M, eps)
        self.mod = torch.empty((1, 3 * D), dtype=torch.float32 if dtype == torch.bfloat16 else dtype, device=device)
        self.y = torch.empty((S_loc, D), dtype=dtype, device=device)
        self.qkv = torch.empty((S_loc, 3 * D), dtype=dtype, device=device)
        self.cat = torch.empty((S_loc, D + M), dtype=dtype, device=device)
        if mode == "ring":
            self.attention = RingAttention(S_loc, H, device, dtype, group, attn, merge, shards_per_step, key_splits)
        else:
            self.attention = UlyssesAttention(S_loc, H, device, dtype, group, attn)

    def forward(self, w, x, vec, rope, out):
        D = self.D
        self.ops.adaln(w, vec, self.mod)
        self.ops.modulate_norm(x, self.mod, self.y)
        self.ops.qkv_mlp(w, self.y, rope, self.qkv, self.cat)
        self.attention(self.qkv[:, :D], self.qkv[:, D:2 * D], self.qkv[:, 2 * D:], self.cat[:, :D])
        self.ops.out_proj(w, self.cat, x, self.mod, out)
        return out
