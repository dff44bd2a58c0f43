"""Plain fp64 CPU oracle for the Flux-style DiT block forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only the tests, the smoke check and the benchmark's CPU
baseline leg use it.  It shares no code with the CUDA library.

Every function takes float64 numpy arrays (the exact bf16 input values, widened)
and returns float64 arrays.  There is no intermediate rounding.  Matrix
products use numpy's float64 matmul as a library primitive; nothing is blocked,
fused or reordered beyond what each definition states.

Sources (web pages, cited by title and section):
  [CG]  "compile_graph" write-up on ChituDiffusion / Flux.1-dev (chenyy20.com).
        §1.1 names the fused tail: LayerNorm, GELU and the adaLN modulation
        (1+scale)*x+shift.  §2 gives the single-stream block shape
        (S=4608, dim 3072, 24 heads x 128, bf16) and the 57-block model.
        §3.1 names RoPE as complex arithmetic computed from position ids, and
        the two block lists (double-stream "transformer_blocks" and
        single-stream "single_transformer_blocks").  §6.3 fixes the attention
        layout (B, S, H, D).  §2 and §8 give the flowmatch-euler 50-step loop.
        §5 merges the partial results of ring attention by log-sum-exp; §7
        skips model steps (MeanCache) with a finite-difference prediction.
  [WAN] Wan2.1 local-acceleration page (mhpq.cn), §1.1: video DiT blocks are
        dominated by self-attention over long (t, h, w) token sequences.
  [SDXL] SDXL inference-optimisation guide (javey-q.github.io), §3.3:
        classifier-free guidance, noise_u + scale (noise_c - noise_u) as batch 2,
        switched off for the late steps.
Where the pages leave a step open, the reading taken is stated at the function
and collected in the design notes (readings s1-s15).

Parity status: every function below is pinned by tests in tests/test_oracle_*.py
against invariants, closed forms or brute force; none is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

# --------------------------------------------------------------------------
# Elementwise maps
# --------------------------------------------------------------------------


def silu(z):
    """SiLU z * sigmoid(z).  Applied to the conditioning vector before the
    adaLN linear (reading s1)."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def gelu_tanh(u):
    """GELU, tanh approximation: 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3))).
    [CG] §1.1 names GELU in the fused tail; the tanh variant is reading s8."""
    u = np.asarray(u, dtype=np.float64)
    c = math.sqrt(2.0 / math.pi)
    return 0.5 * u * (1.0 + np.tanh(c * (u + 0.044715 * u * u * u)))


# --------------------------------------------------------------------------
# Normalisations and modulation ([CG] §1.1)
# --------------------------------------------------------------------------


def layer_norm(x, eps=1e-6):
    """Row LayerNorm without affine: (x - mean) / sqrt(biased var + eps) over
    the last axis (reading s2)."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def modulate(n, shift, scale):
    """adaLN modulation (1 + scale) * n + shift, [CG] §1.1."""
    return (1.0 + scale) * n + shift


def linear(x, W, b=None):
    """nn.Linear: x W^T + b, with W stored [out, in]."""
    y = np.asarray(x, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T
    if b is not None:
        y = y + b
    return y


def adaln_modulation(vec, W, b, n_chunks):
    """m = W silu(vec) + b, split into n_chunks equal vectors.

    Single-stream block: (shift, scale, gate).  Double-stream block, per
    stream, and the video block: (shift1, scale1, gate1, shift2, scale2, gate2).
    Final layer: (shift, scale).  Reading s1 (SiLU first, with bias)."""
    m = linear(silu(vec), W, b)
    return np.split(m, n_chunks, axis=-1)


def rms_norm_heads(x, scale, n_heads, eps=1e-6):
    """Per (token, head) RMSNorm over head_dim: x / sqrt(mean(x^2) + eps) * scale.
    x is [S, H*d] (heads concatenated); scale is [d]."""
    S = x.shape[0]
    xh = x.reshape(S, n_heads, -1)
    ms = (xh * xh).mean(axis=-1, keepdims=True)
    return (xh / np.sqrt(ms + eps) * scale).reshape(S, -1)


# --------------------------------------------------------------------------
# 3-axis rotary position embedding ([CG] §3.1: complex RoPE from ids)
# --------------------------------------------------------------------------


def rope_angles(ids, axes_dim, theta=10000.0):
    """Rotation angle of every (token, pair).

    ids: [S, n_axes] integer positions.  axes_dim: per-axis head-dim share
    (Flux (16, 56, 56); video (44, 42, 42)), summing to head_dim.  Pair p of the
    head vector is (2p, 2p+1).  Pairs are assigned to axes in order; pair j of
    axis a (j counted from that axis's first pair) turns by
    pos_a * theta^(-2j / axes_dim[a]).  Readings s4, s5."""
    ids = np.asarray(ids, dtype=np.float64)
    cols = []
    for a, da in enumerate(axes_dim):
        j = np.arange(da // 2, dtype=np.float64)
        omega = theta ** (-2.0 * j / da)
        cols.append(ids[:, a:a + 1] * omega[None, :])
    return np.concatenate(cols, axis=1)  # [S, head_dim/2]


def apply_rope(x, phi, n_heads):
    """Rotate each pair (x0, x1) of every head by its angle phi:
    (x0 cos - x1 sin, x0 sin + x1 cos), i.e. multiply x0 + i x1 by e^{i phi}.
    x is [S, H*d]; phi is [S, d/2]."""
    S = x.shape[0]
    xh = x.reshape(S, n_heads, -1, 2)
    c = np.cos(phi)[:, None, :]
    s = np.sin(phi)[:, None, :]
    x0 = xh[..., 0]
    x1 = xh[..., 1]
    out = np.stack([x0 * c - x1 * s, x0 * s + x1 * c], axis=-1)
    return out.reshape(S, -1)


# --------------------------------------------------------------------------
# Attention ([CG] §2: full joint attention, 24 heads x 128; §6.3: (B, S, H, D))
# --------------------------------------------------------------------------


def attention(q, k, v, n_heads, scale=None, rows=None):
    """softmax(q k^T * scale) v per head, no mask (reading s7).

    q: [Sq, H*d], k, v: [Skv, H*d].  Returns [Sq, H*d] with heads
    concatenated (o[t, h*d + i]).  rows: optional query-row subset; the result
    then has one row per entry of rows."""
    Sq = q.shape[0]
    d = q.shape[1] // n_heads
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if rows is not None:
        q = q[rows]
        Sq = q.shape[0]
    out = np.empty((Sq, n_heads * d), dtype=np.float64)
    for h in range(n_heads):
        sl = slice(h * d, (h + 1) * d)
        logits = (q[:, sl] @ k[:, sl].T) * scale
        logits = logits - logits.max(axis=1, keepdims=True)
        p = np.exp(logits)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, sl] = p @ v[:, sl]
    return out


def attention_lse(q, k, n_heads, scale=None):
    """Natural-log sum-exp of the scaled logits per (head, query): [H, Sq]."""
    d = q.shape[1] // n_heads
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    res = np.empty((n_heads, q.shape[0]))
    for h in range(n_heads):
        sl = slice(h * d, (h + 1) * d)
        logits = (q[:, sl] @ k[:, sl].T) * scale
        mx = logits.max(axis=1)
        res[h] = mx + np.log(np.exp(logits - mx[:, None]).sum(axis=1))
    return res


def attention_merge(outs, lses):
    """Combine attention results over disjoint key sets ([CG] §5: sequence-
    parallel ring attention merges each hop's partial result by its
    log-sum-exp).  With key set j giving o_j (softmax over that set alone)
    and lse_j, the attention over the union is
        lse = log sum_j exp(lse_j),  o = sum_j exp(lse_j - lse) o_j.
    outs: list of [Sq, H*d]; lses: list of [H, Sq] (natural log).
    Returns (o [Sq, H*d], lse [H, Sq]).

    A part over an empty key set has lse = log 0 = -inf and weight 0.  When
    every part of a row is empty the union is empty too: lse = -inf and, by
    the convention of the empty sum, o = 0."""
    n_heads = lses[0].shape[0]
    L = np.stack(lses)                      # [n, H, Sq]
    m = L.max(axis=0)
    empty = np.isneginf(m)
    ms = np.where(empty, 0.0, m)            # any finite shift: every term is exp(-inf) = 0 there
    tot = np.exp(L - ms).sum(axis=0)
    lse = np.where(empty, -np.inf, ms + np.log(np.where(empty, 1.0, tot)))
    Sq = outs[0].shape[0]
    d = outs[0].shape[1] // n_heads
    o = np.zeros((Sq, n_heads, d))
    for oj, lj in zip(outs, lses):
        wj = np.where(empty, 0.0, np.exp(lj - np.where(empty, 0.0, lse)))
        o += wj.T[:, :, None] * oj.reshape(Sq, n_heads, d)
    return o.reshape(Sq, n_heads * d), lse


# --------------------------------------------------------------------------
# Blocks
# --------------------------------------------------------------------------


def single_block(x, vec, ids, w, n_heads, axes_dim=(16, 56, 56), theta=10000.0,
                 eps=1e-6, rows=None):
    """Flux single-stream block ([CG] §2 shape, §1.1 tail ops, §3.1 RoPE).

    x: [S, D] tokens, text first then image (reading s6).  vec: [D] condition.
    w: dict with W_mod [3D, D], b_mod [3D], W1 [3D+M, D], b1 [3D+M],
       q_scale [d], k_scale [d], W2 [D, D+M], b2 [D].
    Steps:
      1. (shift, scale, gate) = W_mod silu(vec) + b_mod
      2. y = (1 + scale) LN(x) + shift
      3. h = y W1^T + b1 = [q | k | v | mlp]
      4. q, k <- RMSNorm per head (x q_scale / k_scale); then RoPE from ids
      5. o = softmax(q k^T / sqrt(d)) v; a = gelu_tanh(mlp)
      6. out = x + gate * ([o | a] W2^T + b2)
    rows: optional subset of output rows (all keys/values are still computed
    from every token)."""
    D = x.shape[1]
    shift, scale, gate = adaln_modulation(vec, w["W_mod"], w["b_mod"], 3)
    y = modulate(layer_norm(x, eps), shift, scale)
    W1, b1 = w["W1"], w["b1"]
    phi = rope_angles(ids, axes_dim, theta)
    k = linear(y, W1[D:2 * D], b1[D:2 * D])
    v = linear(y, W1[2 * D:3 * D], b1[2 * D:3 * D])
    k = apply_rope(rms_norm_heads(k, w["k_scale"], n_heads, eps), phi, n_heads)
    sel = slice(None) if rows is None else rows
    yr = y[sel]
    q = linear(yr, W1[0:D], b1[0:D])
    q = apply_rope(rms_norm_heads(q, w["q_scale"], n_heads, eps), phi[sel], n_heads)
    mlp = gelu_tanh(linear(yr, W1[3 * D:], b1[3 * D:]))
    o = attention(q, k, v, n_heads)
    cat = np.concatenate([o, mlp], axis=1)
    return x[sel] + gate * linear(cat, w["W2"], w["b2"])


def double_block(img, txt, vec, ids, w, n_heads, axes_dim=(16, 56, 56),
                 theta=10000.0, eps=1e-6, rows_img=None, rows_txt=None):
    """Flux double-stream block ([CG] §3.1 "transformer_blocks").

    Each stream s in (txt, img) has its own adaLN (6 chunks), QKV linear,
    QK RMSNorm scales, output projection and MLP (weights w["txt"], w["img"]:
    W_mod [6D, D], b_mod, W_qkv [3D, D], b_qkv, q_scale, k_scale,
    W_proj [D, D], b_proj, W_mlp1 [M, D], b_mlp1, W_mlp2 [D, M], b_mlp2).
    Attention is joint over the concatenation txt | img (reading s6), with
    RoPE from ids (ids rows: text first).  Then per stream
      x += gate1 * (o W_proj^T + b_proj)
      x += gate2 * MLP((1 + scale2) LN(x) + shift2),  MLP = W_mlp2 gelu(W_mlp1 . + b) + b.
    Returns (img', txt').  rows_img / rows_txt: optional output-row subsets
    (given together; every key and value is still computed from all tokens)."""
    streams = {"txt": txt, "img": img}
    D = img.shape[1]
    mods, qs, ks, vs = {}, {}, {}, {}
    for s in ("txt", "img"):
        ws = w[s]
        mods[s] = adaln_modulation(vec, ws["W_mod"], ws["b_mod"], 6)
        shift1, scale1 = mods[s][0], mods[s][1]
        y = modulate(layer_norm(streams[s], eps), shift1, scale1)
        qkv = linear(y, ws["W_qkv"], ws["b_qkv"])
        qs[s] = rms_norm_heads(qkv[:, 0:D], ws["q_scale"], n_heads, eps)
        ks[s] = rms_norm_heads(qkv[:, D:2 * D], ws["k_scale"], n_heads, eps)
        vs[s] = qkv[:, 2 * D:3 * D]
    phi = rope_angles(ids, axes_dim, theta)
    q = apply_rope(np.concatenate([qs["txt"], qs["img"]]), phi, n_heads)
    k = apply_rope(np.concatenate([ks["txt"], ks["img"]]), phi, n_heads)
    v = np.concatenate([vs["txt"], vs["img"]])
    n_txt = txt.shape[0]
    if rows_img is None:
        sel = {"txt": np.arange(n_txt), "img": np.arange(img.shape[0])}
    else:
        sel = {"txt": np.asarray(rows_txt), "img": np.asarray(rows_img)}
    joint_rows = np.concatenate([sel["txt"], n_txt + sel["img"]])
    o = attention(q, k, v, n_heads, rows=joint_rows)
    n_sel_txt = len(sel["txt"])
    outs = {"txt": o[:n_sel_txt], "img": o[n_sel_txt:]}
    res = {}
    for s in ("txt", "img"):
        ws = w[s]
        _, _, gate1, shift2, scale2, gate2 = mods[s]
        x = streams[s][sel[s]] + gate1 * linear(outs[s], ws["W_proj"], ws["b_proj"])
        y = modulate(layer_norm(x, eps), shift2, scale2)
        hmid = gelu_tanh(linear(y, ws["W_mlp1"], ws["b_mlp1"]))
        res[s] = x + gate2 * linear(hmid, ws["W_mlp2"], ws["b_mlp2"])
    return res["img"], res["txt"]


def video_block(x, ctx, vec, ids, w, n_heads, axes_dim=(44, 42, 42),
                theta=10000.0, eps=1e-6, rows=None):
    """Wan-style video DiT block ([WAN] §1.1; reading s10).

    x: [S, D] video tokens with (t, h, w) ids; ctx: [Sc, D] text context
    (already projected to D).  Weights: W_mod [6D, D], b_mod, W_qkv [3D, D],
    b_qkv, W_o [D, D], b_o, W_cq [D, D], b_cq, W_ckv [2D, D], b_ckv,
    W_co [D, D], b_co, W_f1 [M, D], b_f1, W_f2 [D, M], b_f2.
      x += gate1 * SelfAttn(RoPE(q), RoPE(k), v) W_o^T   on (1+scale1) LN(x) + shift1
      x += CrossAttn(q = LN(x) W_cq^T, k|v = ctx W_ckv^T) W_co^T   (no gate, no RoPE)
      x += gate2 * FFN((1+scale2) LN(x) + shift2),  FFN = W_f2 gelu(W_f1 . + b) + b
    No QK RMSNorm.  rows: optional output-row subset (keys/values of the self
    attention are computed from every token; the residual stream after the
    self-attention is only needed at the selected rows)."""
    D = x.shape[1]
    shift1, scale1, gate1, shift2, scale2, gate2 = adaln_modulation(
        vec, w["W_mod"], w["b_mod"], 6)
    y = modulate(layer_norm(x, eps), shift1, scale1)
    phi = rope_angles(ids, axes_dim, theta)
    W, b = w["W_qkv"], w["b_qkv"]
    k = apply_rope(linear(y, W[D:2 * D], b[D:2 * D]), phi, n_heads)
    v = linear(y, W[2 * D:3 * D], b[2 * D:3 * D])
    sel = slice(None) if rows is None else rows
    q = apply_rope(linear(y[sel], W[0:D], b[0:D]), phi[sel], n_heads)
    o = attention(q, k, v, n_heads)
    xr = x[sel] + gate1 * linear(o, w["W_o"], w["b_o"])
    cq = linear(layer_norm(xr, eps), w["W_cq"], w["b_cq"])
    ckv = linear(ctx, w["W_ckv"], w["b_ckv"])
    co = attention(cq, ckv[:, :D], ckv[:, D:], n_heads)
    xr = xr + linear(co, w["W_co"], w["b_co"])
    y2 = modulate(layer_norm(xr, eps), shift2, scale2)
    f = linear(gelu_tanh(linear(y2, w["W_f1"], w["b_f1"])), w["W_f2"], w["b_f2"])
    return xr + gate2 * f


# --------------------------------------------------------------------------
# Whole model and sampler ([CG] §2, §7, §8: Flux.1-dev, flowmatch-euler)
# --------------------------------------------------------------------------


def timestep_embedding(t, dim=256, max_period=10000.0, time_factor=1000.0):
    """[cos(1000 t f_k), sin(1000 t f_k)], f_k = max_period^(-k/(dim/2)),
    k = 0 .. dim/2 - 1 (reading s9)."""
    half = dim // 2
    f = max_period ** (-np.arange(half, dtype=np.float64) / half)
    args = time_factor * float(t) * f
    return np.concatenate([np.cos(args), np.sin(args)])


def patchify(latent, p=2):
    """[C, 2Hg, 2Wg] -> [Hg*Wg, C*p*p]; token (h, w) row-major, feature
    index c*p*p + ph*p + pw (reading s9)."""
    C, Hh, Ww = latent.shape
    Hg, Wg = Hh // p, Ww // p
    t = latent.reshape(C, Hg, p, Wg, p).transpose(1, 3, 0, 2, 4)
    return t.reshape(Hg * Wg, C * p * p)


def unpatchify(tokens, C, Hg, Wg, p=2):
    """Inverse of patchify."""
    t = tokens.reshape(Hg, Wg, C, p, p).transpose(2, 0, 3, 1, 4)
    return t.reshape(C, Hg * p, Wg * p)


def flux_velocity(img_tok, txt_raw, t, ids, model, n_heads, axes_dim=(16, 56, 56),
                  theta=10000.0, eps=1e-6):
    """One model forward: velocity for the patchified latent img_tok at time t.

    model: img_in (W, b), txt_in (W, b), time_in (W1, b1, W2, b2),
    double (list of double_block weight dicts), single (list of single_block
    weight dicts), final (W_mod [2D, D], b_mod, W_out [C*4, D], b_out)."""
    img = linear(img_tok, model["W_img_in"], model["b_img_in"])
    txt = linear(txt_raw, model["W_txt_in"], model["b_txt_in"])
    temb = timestep_embedding(t)
    vec = linear(silu(linear(temb, model["W_t1"], model["b_t1"])),
                 model["W_t2"], model["b_t2"])
    for wd in model["double"]:
        img, txt = double_block(img, txt, vec, ids, wd, n_heads, axes_dim, theta, eps)
    x = np.concatenate([txt, img])
    for ws in model["single"]:
        x = single_block(x, vec, ids, ws, n_heads, axes_dim, theta, eps)
    img = x[txt.shape[0]:]
    shift, scale = adaln_modulation(vec, model["W_fmod"], model["b_fmod"], 2)
    y = modulate(layer_norm(img, eps), shift, scale)
    return linear(y, model["W_out"], model["b_out"])


def euler_sample(latent, txt_raw, ids, model, n_heads, steps, axes_dim=(16, 56, 56),
                 theta=10000.0, eps=1e-6, fresh=None, cache_order=1, txt_uncond=None, guidance=1.0,
                 cfg_steps=None):
    """Flow-match Euler over the linear schedule t_i = 1 - i/steps:
    x <- x + (t_{i+1} - t_i) v(x, t_i).  Returns the final latent [C, H, W]
    (reading s9: no resolution shift, no guidance embedding).

    Model-level step cache ([CG] §7): fresh[i] = 1 runs the model at step i;
    fresh[i] = 0 predicts the velocity from the model velocities of earlier
    fresh steps.  cache_order 0 reuses the last one; 1 extrapolates linearly
    in t from the last two (a finite-difference estimate of dv/dt), using the
    last one alone while only one exists.

    Classifier-free guidance (the SDXL inference-optimisation guide
    (javey-q.github.io) §3.3, read for the flow-matching velocity): with
    txt_uncond, a model step evaluates the velocity for both texts and uses
    v = v_u + guidance (v_c - v_u).  cfg_steps limits guidance to the first
    cfg_steps steps (the guide's late-step cut-off); later steps use v_c
    alone.  Cached steps predict from the guided velocities."""
    C, Hh, Ww = latent.shape
    x = patchify(np.asarray(latent, dtype=np.float64))
    hist = []  # (t, v) of fresh steps, newest last
    for i in range(steps):
        t0 = 1.0 - i / steps
        t1 = 1.0 - (i + 1) / steps
        if fresh is None or fresh[i]:
            v = flux_velocity(x, txt_raw, t0, ids, model, n_heads, axes_dim, theta, eps)
            if txt_uncond is not None and (cfg_steps is None or i < cfg_steps):
                vu = flux_velocity(x, txt_uncond, t0, ids, model, n_heads, axes_dim, theta, eps)
                v = vu + guidance * (v - vu)
            hist.append((t0, v))
        else:
            ta, va = hist[-1]
            if cache_order == 1 and len(hist) >= 2:
                tb, vb = hist[-2]
                v = va + (t0 - ta) * (va - vb) / (ta - tb)
            else:
                v = va
        x = x + (t1 - t0) * v
    return unpatchify(x, C, Hh // 2, Ww // 2)


# --------------------------------------------------------------------------
# Work model (used to express measured times as FLOP/s)
# --------------------------------------------------------------------------


def single_block_flops(S, D, M, H, d=128, B=1):
    """Algorithmic FLOPs of one single-stream block: 2MNK per linear plus
    4 S^2 H d for attention (two contractions)."""
    gemm = 2.0 * S * D * (3 * D + M) + 2.0 * S * (D + M) * D
    attn = 4.0 * S * S * H * d
    mod = 2.0 * D * 3 * D
    return B * (gemm + attn + mod)
